"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bit-exact for pa_write_kv and pa_copy_blocks (whole pools compared);
max |gpu - oracle| <= 2e-3 for pa_decode with fp16 output (fp32
accumulation). Every workload, at reduced and at full size, is compared
element by element over all of its outputs (the full step on its first and
last layers), with both pools byte for byte; failures report the maximum and
mean error and the worst (sequence, head, dim).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests import paged_cases as pc
from tests.gpu_harness import (TOL, check_outputs_and_pools, decode_case, max_err, run_step,
                               to_bits, to_f64)

pytestmark = pytest.mark.gpu
import paged_kv_cache_417_b200 as pk  # noqa: E402


def check_full(step, partition_size=0, out_dtype=None, tol=TOL):
    outs, d, err = run_step(step, partition_size=partition_size, out_dtype=out_dtype)
    assert err == 0, f"dev_err {err}"
    for li in range(step.num_layers):
        ref, kref, vref = oracle.run_step(step, li)
        e = max_err(outs[li], ref)
        assert e <= tol, f"{step.name} layer {li}: max err {e}"
        assert np.array_equal(to_bits(d["key_caches"][li]), kref), "key pool differs"
        assert np.array_equal(to_bits(d["value_caches"][li]), vref), "value pool differs"
    return outs


# --------------------------------------------------------------------- configs

@pytest.mark.parametrize("partition", [0, 32, 64])
def test_tiny(partition):
    check_full(wl.tiny(), partition_size=partition)


def test_tiny_bf16():
    st = wl.tiny(dtype="bf16")
    check_full(st, out_dtype=torch.float32)
    outs, _, _ = run_step(st)
    ref, _, _ = oracle.run_step(st)
    got = to_f64(outs[0])
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-3)


@pytest.mark.parametrize("partition", [0, 256, 2048])
def test_llama_layer_reduced(partition):
    st = wl.llama_layer(num_seqs=12, num_blocks=1024)
    check_full(st, partition_size=partition)


def test_llama_layer_full_size():
    """All 96 sequences x 32 heads, every output element, both pools."""
    st = wl.llama_layer()
    outs, d, err = run_step(st)
    assert err == 0
    check_outputs_and_pools(st, outs, d, [0])


@pytest.mark.parametrize("partition", [0, 128])
def test_long_context_reduced(partition):
    st = wl.long_context(num_seqs=3, ctx_range=(3000, 6000), num_blocks=1500)
    check_full(st, partition_size=partition)


def test_long_context_full_size():
    """8 sequences of 16k-32k tokens (split partitions), every element."""
    st = wl.long_context()
    outs, d, err = run_step(st)
    assert err == 0
    check_outputs_and_pools(st, outs, d, [0])


def test_prefix_cow_full_size():
    st = wl.prefix_cow()
    assert st.copy_pairs.shape[0] > 0
    check_full(st)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_full_step_reduced(bs):
    st = wl.full_step(block_size=bs, num_seqs=24, num_layers=3)
    check_full(st)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_full_step_full_size(bs):
    """32 layers x 256 sequences: every output element and both pools of the
    first and last layers; every layer finite."""
    st = wl.full_step(block_size=bs)
    outs, d, err = run_step(st)
    assert err == 0
    check_outputs_and_pools(st, outs, d, [0, st.num_layers - 1])
    for li in range(st.num_layers):
        assert bool(torch.isfinite(outs[li]).all())
    del d


# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("D,bs", [(64, 8), (64, 16), (64, 32), (128, 8), (128, 32)])
@pytest.mark.parametrize("partition", [0, 32])
def test_shapes_and_ragged_tails(D, bs, partition):
    rng = np.random.default_rng(D * 100 + bs)
    ctxs = [1, bs - 1, bs, bs + 1, 2 * bs + 3, 63, 64, 65, 300, 777]
    c = pc.paged_case(rng, ctxs, 3, D, bs)
    out, err = decode_case(c, partition_size=partition)
    assert err == 0
    ref = orc_decode(c)
    assert max_err(out, ref) <= TOL


def orc_decode(c):
    return oracle.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"],
                         c["dtype"])


def test_context_zero_and_one():
    rng = np.random.default_rng(31)
    c = pc.paged_case(rng, [0, 1, 16, 17, 0], 2, 128, 16)
    for partition in (0, 32):
        out, err = decode_case(c, partition_size=partition)
        assert err == 0
        got = to_f64(out)
        assert np.all(got[0] == 0) and np.all(got[4] == 0)
        v0 = pc.widen_bits(c["V"][1][0], "f16")
        assert np.array_equal(got[1], v0), "ctx = 1 must return v0 exactly"
        assert max_err(out, orc_decode(c)) <= TOL


def test_split_matches_single_and_oracle():
    rng = np.random.default_rng(32)
    c = pc.paged_case(rng, [5000, 8000, 33, 4097], 2, 128, 16)
    ref = orc_decode(c)
    single, _ = decode_case(c, partition_size=8192, out_dtype=torch.float32)
    for partition in (32, 128, 512, 0):
        split, err = decode_case(c, partition_size=partition, out_dtype=torch.float32)
        assert err == 0
        assert max_err(split, ref) <= TOL
        assert float((split - single).abs().max()) <= TOL
    assert max_err(single, ref) <= TOL


def test_max_context_len_larger_than_needed():
    rng = np.random.default_rng(33)
    c = pc.paged_case(rng, [40, 200], 2, 128, 16)
    out, err = decode_case(c, partition_size=64, max_context_len=4000)
    assert err == 0 and max_err(out, orc_decode(c)) <= TOL


def test_block_permutation_is_bit_exact():
    rng = np.random.default_rng(34)
    c = pc.paged_case(rng, [70, 513, 1000], 2, 128, 16, num_blocks=200)
    a, _ = decode_case(c)
    pi = rng.permutation(c["kpool"].shape[0])
    c2 = dict(c)
    c2["kpool"] = np.empty_like(c["kpool"])
    c2["vpool"] = np.empty_like(c["vpool"])
    c2["kpool"][pi] = c["kpool"]
    c2["vpool"][pi] = c["vpool"]
    c2["bt"] = np.where(c["bt"] >= 0, pi[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    b, _ = decode_case(c2)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_same_content_different_blocks_same_output():
    rng = np.random.default_rng(35)
    c = pc.paged_case(rng, [300, 300], 2, 128, 16)
    # Make sequence 1 a copy of sequence 0 through its own blocks.
    bs = 16
    j = np.arange(300)
    c["kpool"][c["bt"][1][j // bs], :, j % bs] = c["K"][0]
    c["vpool"][c["bt"][1][j // bs], :, j % bs] = c["V"][0]
    c["q"][1] = c["q"][0]
    out, _ = decode_case(c)
    assert torch.equal(out[0].view(torch.int16), out[1].view(torch.int16))


def test_bf16_cache():
    rng = np.random.default_rng(36)
    c = pc.paged_case(rng, [1, 31, 500, 1500], 4, 128, 16, dtype="bf16")
    out, err = decode_case(c, out_dtype=torch.float32)
    assert err == 0 and max_err(out, orc_decode(c)) <= TOL


def test_bad_block_id_sets_flag_and_nan():
    rng = np.random.default_rng(37)
    c = pc.paged_case(rng, [100, 100], 2, 64, 16)
    c["bt"][0, 2] = c["kpool"].shape[0] + 5
    for partition in (0, 32):
        out, err = decode_case(c, partition_size=partition)
        assert err & pk.PA_DEVERR_BLOCK_ID
        assert bool(torch.isnan(out[0]).all())
        ref = orc_decode({**c, "bt": c["bt"][1:], "q": c["q"][1:], "ctx": c["ctx"][1:]})
        assert max_err(out[1:], ref) <= TOL


def test_context_longer_than_max_is_flagged():
    rng = np.random.default_rng(38)
    c = pc.paged_case(rng, [100, 50], 2, 64, 16)
    _, err = decode_case(c, max_context_len=64)
    assert err & pk.PA_DEVERR_CONTEXT_LEN


def test_bad_slot_and_copy_pair_are_flagged():
    H, bs, D, NB = 2, 16, 64, 8
    kc = torch.zeros(NB, H, bs, D, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    key = torch.ones(2, H, D, dtype=torch.float16, device="cuda")
    slots = torch.tensor([NB * bs, -1], dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.write_kv(key, key, slots, kc, vc, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVERR_SLOT
    assert not bool(kc.any()) and not bool(vc.any())
    err.zero_()
    pairs = torch.tensor([[0, NB], [1, 2]], dtype=torch.int64, device="cuda")
    kc[1] = 1.0
    pk.copy_blocks([kc], [vc], pairs, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pk.PA_DEVERR_COPY_PAIR
    assert bool((kc[2] == 1.0).all())


def test_copy_blocks_many_layers_bit_exact():
    rng = np.random.default_rng(39)
    L, NB, H, bs, D = 5, 12, 3, 8, 128
    ks = [rng.integers(0, 1 << 16, size=(NB, H, bs, D), dtype=np.uint16) for _ in range(L)]
    vs = [rng.integers(0, 1 << 16, size=(NB, H, bs, D), dtype=np.uint16) for _ in range(L)]
    pairs = np.array([[3, 9], [0, 11], [7, 1]], dtype=np.int64)
    dk = [torch.from_numpy(k.view(np.int16)).view(torch.float16).cuda() for k in ks]
    dv = [torch.from_numpy(v.view(np.int16)).view(torch.float16).cuda() for v in vs]
    pk.copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(ks, vs, pairs)
    for l in range(L):
        assert np.array_equal(to_bits(dk[l]), ks[l]) and np.array_equal(to_bits(dv[l]), vs[l])


def test_empty_inputs():
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    q = torch.zeros(0, 2, 64, dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    bt = torch.zeros(0, 1, dtype=torch.int32, device="cuda")
    ctx = torch.zeros(0, dtype=torch.int32, device="cuda")
    pk.decode(out, q, kc, kc, bt, ctx, 0, 0.125)
    pk.write_kv(q, q, torch.zeros(0, dtype=torch.int64, device="cuda"), kc, kc)
    pk.copy_blocks([kc], [kc], torch.zeros(0, 2, dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()


def test_maximum_partition_and_many_partitions():
    rng = np.random.default_rng(40)
    c = pc.paged_case(rng, [8000, 8192, 1], 1, 128, 32)
    ref = orc_decode(c)
    for partition in (8192, 32):
        out, err = decode_case(c, partition_size=partition)
        assert err == 0 and max_err(out, ref) <= TOL


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait that nothing completes gives up after its limit, reports
    PA_DEVERR_TIMEOUT, and the next decode on the same context is correct."""
    assert pk.selftest_wait_timeout(2000) & pk.PA_DEVERR_TIMEOUT
    rng = np.random.default_rng(41)
    c = pc.paged_case(rng, [30, 300], 2, 128, 16)
    out, err = decode_case(c)
    assert err == 0 and max_err(out, orc_decode(c)) <= TOL
