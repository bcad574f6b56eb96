"""Host-side logic: the block allocator and the seeded decode-step builder."""
import numpy as np
import pytest

import oracle
import workloads as wl
from workloads import (BlockAllocator, PoolExhausted, Sequence, allocate_tokens,
                       append_token, check_invariants, free_sequence)


def test_append_fills_slots_in_order():
    """A logical block fills its slots in order and a new block starts when
    the last one is full ("啃透vLLM源码", §2.2, append_tokens)."""
    a = BlockAllocator(8, 4, order=[5, 2, 7, 0, 1, 3, 4, 6])
    s = Sequence()
    slots = [append_token(a, s)[0] for _ in range(10)]
    assert s.block_table == [5, 2, 7]
    assert slots == [20, 21, 22, 23, 8, 9, 10, 11, 28, 29]
    assert s.num_tokens == 10
    check_invariants(a, [s])


def test_copy_on_write_on_shared_block():
    """Two holders of a partly filled block: the one that appends gets a copy
    ("vLLM基础", §2.3)."""
    a = BlockAllocator(6, 4)
    s1 = Sequence()
    allocate_tokens(a, s1, 6)            # blocks 0 (full), 1 (2 of 4 slots)
    s2 = Sequence(block_table=[a.fork(b) for b in s1.block_table], num_tokens=6)
    check_invariants(a, [s1, s2])
    slot, pair = append_token(a, s2)
    assert pair == (1, 2) and s2.block_table == [0, 2] and slot == 2 * 4 + 2
    assert a.ref_count[1] == 1 and a.ref_count[0] == 2
    check_invariants(a, [s1, s2])
    slot, pair = append_token(a, s1)     # s1 is now the only holder: no copy
    assert pair is None and slot == 1 * 4 + 2
    free_sequence(a, s1)
    free_sequence(a, s2)
    assert a.num_free == 6
    check_invariants(a, [])


def test_pool_exhausted():
    a = BlockAllocator(2, 16)
    s = Sequence()
    allocate_tokens(a, s, 32)
    assert not a.can_allocate(1)
    with pytest.raises(PoolExhausted):
        append_token(a, s)


@pytest.mark.parametrize("maker,kw", [
    (wl.tiny, {}),
    (wl.llama_layer, {"num_seqs": 12}),
    (wl.long_context, {"num_seqs": 2, "ctx_range": (3000, 5000), "num_blocks": 800}),
    (wl.prefix_cow, {}),
    (wl.full_step, {"num_seqs": 40, "num_layers": 2, "block_size": 8}),
])
def test_step_invariants(maker, kw):
    st = maker(**kw)
    m = st.meta
    check_invariants(m["allocator"], m["seqs"], m["phantom_holders"])
    bs = st.block_size
    for s in range(st.num_seqs):
        n = int(st.context_lens[s])
        nblk = -(-n // bs)
        assert np.all(st.block_tables[s, :nblk] >= 0)
        assert np.all(st.block_tables[s, nblk:] == -1)
        slot = int(st.slot_mapping[s])
        assert slot // bs == st.block_tables[s, (n - 1) // bs]
        assert slot % bs == (n - 1) % bs
    # Every referenced block has pre-step content for the slots before the
    # new token; free blocks have none.
    for b in m["allocator"].free_blocks():
        assert st.valid_slots[b] == 0


def test_config_sizes():
    t = wl.tiny()
    assert list(t.context_lens) == [1, 17, 33, 100] and t.num_blocks == 64
    l = wl.llama_layer()
    assert l.num_seqs == 96 and l.num_blocks == 8192 and l.num_heads == 32
    assert l.context_lens.min() >= 128 and l.context_lens.max() <= 2048
    assert np.isclose(l.scale, np.float32(1 / np.sqrt(128)))


def test_prefix_cow_reading():
    st = wl.prefix_cow()
    bs = st.block_size
    prefix = st.block_tables[0, :1024 // bs]
    for s in range(st.num_seqs):
        assert np.array_equal(st.block_tables[s, :1024 // bs], prefix)
    assert np.all(st.ref_count[prefix] == st.num_seqs)
    suffix = st.context_lens - 1 - 1024
    assert len(st.copy_pairs) == int(np.sum(suffix % bs != 0))
    assert not set(st.copy_pairs[:, 0].tolist()) & set(prefix.tolist())
    # The source block stays with the forked sibling only.
    assert np.all(st.ref_count[st.copy_pairs[:, 0]] == 1)
    assert np.all(st.ref_count[st.copy_pairs[:, 1]] == 1)


def test_host_pools_poison():
    st = wl.tiny()
    k, v = wl.host_pools(st)
    nan = wl.nan_bits("f16")
    for b in range(st.num_blocks):
        n = st.valid_slots[b]
        assert np.all(k[b, :, n:, :] == nan) and np.all(v[b, :, n:, :] == nan)
        assert not np.any(k[b, :, :n, :] == nan)


def test_subset_matches_full_step():
    """The sub-step built for a few sequences gives those sequences the same
    oracle outputs as the full step."""
    st = wl.prefix_cow(num_seqs=10, suffix_range=(1, 60), num_heads=2, head_dim=64)
    full, _, _ = oracle.run_step(st)
    ids = [7, 0, 3]
    sub = wl.subset(st, ids)
    part, _, _ = oracle.run_step(sub)
    assert np.array_equal(part, full[ids])


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32) * 100
    ref = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wl.to_storage_bits(x, "bf16"), ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "fp8"])
def test_large_pool_tiles_are_distinct(monkeypatch, dtype):
    """Pools with more tiles than the bank give every tile its own code (bank
    row, sign mask): no two tiles hold the same values, each tile is its bank
    row with whole token rows negated (fp8: the code bytes' sign bit; the row
    scales untouched), and the device-side assembly gives the same bytes."""
    import torch
    import workloads.steps as steps
    from workloads.device import device_pools
    monkeypatch.setattr(steps, "MAX_BANK_ROWS", 64)
    st = wl.tiny(seed=3, dtype=dtype)
    R = st.base.shape[0]
    assert R == 64
    k, v = wl.host_pools(st)
    L = st.layers[0]
    NB, H, bs = st.num_blocks, st.num_kv_heads, st.block_size
    tiles, codes = [], []
    for pool, rows in ((k, L.tile_rows_k), (v, L.tile_rows_v)):
        flat = pool.reshape(NB * H, -1)
        live = (rows >= 0).reshape(-1)
        tiles.append(flat[live])
        codes.append(rows.reshape(-1)[live])
    tiles, codes = np.concatenate(tiles), np.concatenate(codes)
    assert len(tiles) > R                                   # the bank is reused...
    assert len(np.unique(codes)) == len(codes)              # ...under distinct codes
    assert len(np.unique(tiles, axis=0)) == len(tiles)      # and distinct contents
    bank_row, flips = steps.tile_parts(codes, R, bs)
    D = st.head_dim
    for t in range(len(tiles)):
        base = st.base[bank_row[t]]
        got = tiles[t]
        if dtype == "fp8":
            c_got, c_base = got[: bs * D].reshape(bs, D), base[: bs * D].reshape(bs, D)
            s_got, s_base = got[bs * D:].reshape(bs, 4), base[bs * D:].reshape(bs, 4)
            signs = (c_got ^ c_base) == 0x80
            nan = steps.E4M3_NAN
        else:
            c_got, c_base = got.reshape(bs, D), base.reshape(bs, D)
            signs = (c_got ^ c_base) == 0x8000
            nan = steps.nan_bits(dtype)
        same = c_got == c_base
        # Slots past a block's last token are NaN-filled: only live rows count.
        for r in np.nonzero(~np.all(c_got == nan, axis=1))[0]:
            assert signs[r].all() if flips[t, r] else same[r].all()
            if dtype == "fp8":
                assert np.array_equal(s_got[r], s_base[r])            # scales kept
    if dtype != "fp8":
        dk, dv = device_pools(st, 0, "cpu")
        assert np.array_equal(dk.view(torch.int16).numpy().view(np.uint16), k)
        assert np.array_equal(dv.view(torch.int16).numpy().view(np.uint16), v)
