"""pa_swap_blocks between a GPU pool and a pool in pinned host memory:
bit-exact against the oracle's block copy, round trips, and a decode after
swap-in that matches the decode before swap-out bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_417_b200 as pk
import workloads as wl
from tests.gpu_harness import to_bits
from workloads.device import device_step

pytestmark = pytest.mark.gpu


def _bits_tensor(a, device):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16)
    return t.to(device) if device == "cuda" else t.pin_memory()


@pytest.mark.parametrize("bs,D", [(16, 128), (8, 64), (32, 128)])
def test_swap_out_and_in_bit_exact(bs, D):
    rng = np.random.default_rng(bs + D)
    L, H = 3, 4
    gk = [rng.integers(0, 1 << 16, size=(40, H, bs, D), dtype=np.uint16) for _ in range(L)]
    gv = [rng.integers(0, 1 << 16, size=(40, H, bs, D), dtype=np.uint16) for _ in range(L)]
    hk = [rng.integers(0, 1 << 16, size=(9, H, bs, D), dtype=np.uint16) for _ in range(L)]
    hv = [rng.integers(0, 1 << 16, size=(9, H, bs, D), dtype=np.uint16) for _ in range(L)]
    dgk = [_bits_tensor(x, "cuda") for x in gk]
    dgv = [_bits_tensor(x, "cuda") for x in gv]
    dhk = [_bits_tensor(x, "host") for x in hk]
    dhv = [_bits_tensor(x, "host") for x in hv]
    out_map = np.array([[7, 0], [31, 8], [2, 3], [39, 5]], dtype=np.int64)
    pk.swap_blocks(dgk, dgv, dhk, dhv, torch.from_numpy(out_map).cuda())
    torch.cuda.synchronize()
    oracle.swap_blocks(gk, gv, hk, hv, out_map)
    for l in range(L):
        assert np.array_equal(to_bits(dhk[l]), hk[l]) and np.array_equal(to_bits(dhv[l]), hv[l])
    # Swap in to other device blocks, with the mapping table in pinned memory.
    in_map = np.array([[0, 11], [8, 12], [3, 13], [5, 14]], dtype=np.int64)
    pk.swap_blocks(dhk, dhv, dgk, dgv, torch.from_numpy(in_map).pin_memory())
    torch.cuda.synchronize()
    oracle.swap_blocks(hk, hv, gk, gv, in_map)
    for l in range(L):
        assert np.array_equal(to_bits(dgk[l]), gk[l]) and np.array_equal(to_bits(dgv[l]), gv[l])


def test_pageable_host_memory_is_refused():
    k = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    pageable = torch.zeros(4, 2, 16, 64, dtype=torch.float16)  # not pinned
    m = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(pk.PagedKVError) as e:
        pk.swap_blocks([k], [k], [pageable], [pageable], m)
    assert e.value.status == pk.PA_ERR_INVALID_ARG
    with pytest.raises(pk.PagedKVError):
        pk.swap_blocks([k], [k], [k], [k], torch.tensor([[0, 1]], dtype=torch.int64))


def test_bad_pair_is_flagged():
    k = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    h = torch.ones(2, 2, 16, 64, dtype=torch.float16).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    m = torch.tensor([[0, 2], [1, 0]], dtype=torch.int64, device="cuda")  # 2 outside host pool
    pk.swap_blocks([k], [k], [h], [h], m, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVERR_COPY_PAIR
    assert bool((h[1] == 1).all()) and bool((h[0] == 0).all())


def test_decode_after_swap_in_matches_before_swap_out():
    st = wl.llama_layer(num_seqs=10, num_blocks=1024)
    d = device_step(st, "cuda")
    kc, vc = d["key_caches"][0], d["value_caches"][0]
    pk.write_kv(d["new_key"][0], d["new_value"][0], d["slot_mapping"], kc, vc)
    before = torch.empty_like(d["query"][0])
    pk.decode(before, d["query"][0], kc, vc, d["block_tables"], d["context_lens"],
              st.max_context_len, float(st.scale))
    # Swap sequences 2 and 7 out, clobber their GPU blocks, swap them back in.
    blocks = sorted({int(b) for s in (2, 7) for b in st.block_tables[s] if b >= 0})
    hk = torch.empty((len(blocks),) + tuple(kc.shape[1:]), dtype=kc.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_map = torch.tensor([[b, i] for i, b in enumerate(blocks)], dtype=torch.int64).cuda()
    pk.swap_blocks([kc], [vc], [hk], [hv], out_map)
    idx = torch.tensor(blocks, device="cuda")
    kc[idx] = float("nan")
    vc[idx] = float("nan")
    pk.swap_blocks([hk], [hv], [kc], [vc], out_map[:, [1, 0]].contiguous())
    after = torch.empty_like(before)
    pk.decode(after, d["query"][0], kc, vc, d["block_tables"], d["context_lens"],
              st.max_context_len, float(st.scale))
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
