"""Grouped query heads (num_heads = G * num_kv_heads; query head h reads K/V
head h // G) on the CUDA path against the oracle; the fused append writes
each K/V head's new row once per group."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.gpu_harness import TOL, max_err, run_step, run_step_fused, to_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv_heads", [8, 4, 1])
@pytest.mark.parametrize("dtype", ["f16", "fp8"])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("partition", [0, 64])
def test_grouped_heads_match_oracle(kv_heads, dtype, fused, partition):
    st = wl.llama_layer(num_seqs=8, num_blocks=1000, num_kv_heads=kv_heads, dtype=dtype)
    run = run_step_fused if fused else run_step
    outs, d, err = run(st, partition_size=partition)
    assert err == 0
    ref, kref, vref = oracle.run_step(st, 0)
    assert max_err(outs[0], ref) <= TOL
    assert np.array_equal(to_bits(d["key_caches"][0]), kref)
    assert np.array_equal(to_bits(d["value_caches"][0]), vref)


def test_grouped_heads_fused_equals_separate():
    st = wl.full_step(num_seqs=16, num_layers=1, num_kv_heads=8)
    a, da, _ = run_step(st)
    b, db, _ = run_step_fused(st)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(da["key_caches"][0].view(torch.int16), db["key_caches"][0].view(torch.int16))


def test_grouped_heads_d64_bs8():
    st = wl.llama_layer(num_seqs=5, num_blocks=1500, num_heads=12, num_kv_heads=3, head_dim=64,
                        block_size=8)
    outs, d, err = run_step_fused(st)
    ref, kref, _ = oracle.run_step(st, 0)
    assert err == 0 and max_err(outs[0], ref) <= TOL
    assert np.array_equal(to_bits(d["key_caches"][0]), kref)


# ------------------------------------------------- grouped kernel, edge cases
# 16-bit caches with 2 <= G <= 16 take decode_group_kernel (one CTA per K/V
# head for the whole group, TMA-staged tiles, warp MMAs); fp8 and G > 16
# keep the per-query-head kernel.

from tests import paged_cases as pc  # noqa: E402
from tests.gpu_harness import decode_case, to_f64  # noqa: E402
from workloads.steps import to_storage_bits  # noqa: E402

import paged_kv_cache_417_b200 as pk  # noqa: E402


def gqa_case(rng, ctx_list, G, Hkv, D, bs, dtype="f16", num_blocks=None):
    """A paged case with Hkv K/V heads and G * Hkv query heads."""
    c = pc.paged_case(rng, ctx_list, Hkv, D, bs, num_blocks=num_blocks, dtype=dtype)
    S = len(ctx_list)
    c["q"] = to_storage_bits(rng.standard_normal((S, G * Hkv, D), dtype=np.float32), dtype)
    return c


def orc(c):
    return oracle.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"],
                         c["dtype"])


@pytest.mark.parametrize("G", [2, 3, 4, 8, 12, 16])
@pytest.mark.parametrize("D,bs", [(128, 16), (64, 8), (128, 32), (128, 8), (64, 32)])
@pytest.mark.parametrize("partition", [0, 32])
def test_group_kernel_shapes_and_ragged_tails(G, D, bs, partition):
    rng = np.random.default_rng(1000 * G + 10 * D + bs)
    ctxs = [1, bs - 1, bs, bs + 1, 15, 16, 17, 63, 64, 65, 300, 777]
    c = gqa_case(rng, ctxs, G, 2, D, bs)
    out, err = decode_case(c, partition_size=partition)
    assert err == 0
    assert max_err(out, orc(c)) <= TOL


@pytest.mark.parametrize("G", [4, 16])
def test_group_kernel_bf16(G):
    rng = np.random.default_rng(50 + G)
    c = gqa_case(rng, [1, 17, 200, 1000, 3000], G, 2, 128, 16, dtype="bf16")
    ref = orc(c)
    for partition in (0, 64):
        out32, err = decode_case(c, partition_size=partition, out_dtype=torch.float32)
        assert err == 0 and max_err(out32, ref) <= TOL
        out, _ = decode_case(c, partition_size=partition)
        got = to_f64(out)
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-3)


def test_group_kernel_context_zero_and_one():
    rng = np.random.default_rng(60)
    c = gqa_case(rng, [0, 1, 16, 0, 33], 4, 2, 128, 16)
    for partition in (0, 32):
        out, err = decode_case(c, partition_size=partition)
        assert err == 0
        got = to_f64(out)
        assert np.all(got[0] == 0) and np.all(got[3] == 0)
        # ctx = 1: every query head of the group returns v0 of its K/V head.
        v0 = pc.widen_bits(c["V"][1][0], "f16")  # [Hkv, D]
        assert np.array_equal(got[1], np.repeat(v0, 4, axis=0))
        assert max_err(out, orc(c)) <= TOL


def test_group_kernel_split_matches_single():
    rng = np.random.default_rng(61)
    c = gqa_case(rng, [5000, 8000, 33, 4097], 8, 2, 128, 16)
    ref = orc(c)
    single, _ = decode_case(c, partition_size=8192, out_dtype=torch.float32)
    assert max_err(single, ref) <= TOL
    for partition in (32, 512, 0):
        split, err = decode_case(c, partition_size=partition, out_dtype=torch.float32)
        assert err == 0 and max_err(split, ref) <= TOL
        assert float((split - single).abs().max()) <= TOL


def test_group_kernel_block_permutation_is_bit_exact():
    rng = np.random.default_rng(62)
    c = gqa_case(rng, [70, 513, 1000], 4, 2, 128, 16, num_blocks=200)
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


def test_group_kernel_bad_block_id_sets_flag_and_nan():
    rng = np.random.default_rng(63)
    c = gqa_case(rng, [100, 100], 4, 2, 64, 16)
    c["bt"][0, 2] = c["kpool"].shape[0] + 5
    for partition in (0, 32):
        out, err = decode_case(c, partition_size=partition)
        assert err & pk.PA_DEVERR_BLOCK_ID
        assert bool(torch.isnan(out[0]).all())
        ref = orc({**c, "bt": c["bt"][1:], "q": c["q"][1:], "ctx": c["ctx"][1:]})
        assert max_err(out[1:], ref) <= TOL


def test_group_kernel_max_context_len_larger_than_needed():
    rng = np.random.default_rng(64)
    c = gqa_case(rng, [40, 200], 8, 1, 128, 16)
    out, err = decode_case(c, partition_size=64, max_context_len=4000)
    assert err == 0 and max_err(out, orc(c)) <= TOL


@pytest.mark.parametrize("G", [2, 16])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_group_kernel_fused_equals_separate(G, dtype):
    st = wl.llama_layer(num_seqs=10, num_blocks=800, num_heads=4 * G, num_kv_heads=4,
                        dtype=dtype)
    for partition in (0, 64):
        a, da, ea = run_step(st, partition_size=partition)
        b, db, eb = run_step_fused(st, partition_size=partition)
        assert ea == 0 and eb == 0
        assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
        for key in ("key_caches", "value_caches"):
            assert torch.equal(da[key][0].view(torch.int16), db[key][0].view(torch.int16))
    ref, kref, vref = oracle.run_step(st, 0)
    if dtype == "f16":
        assert max_err(b[0], ref) <= TOL
    assert np.array_equal(to_bits(db["key_caches"][0]), kref)
    assert np.array_equal(to_bits(db["value_caches"][0]), vref)


def test_group_kernel_full_size_sampled():
    st = wl.llama_layer(num_kv_heads=8)
    outs, d, err = run_step_fused(st)
    assert err == 0
    ctx = st.context_lens
    rng = np.random.default_rng(65)
    ids = sorted(set([int(np.argmin(ctx)), int(np.argmax(ctx))] +
                     rng.choice(st.num_seqs, 5, replace=False).tolist()))
    sub = wl.subset(st, ids)
    ref, _, _ = oracle.run_step(sub, 0)
    assert max_err(outs[0][torch.as_tensor(ids, device="cuda")], ref) <= TOL


# ------------------------------------------- fp8 cache on the grouped kernel
# fp8 (e4m3 + row scales) caches with f16 rows and head_dim 128 and
# 2 <= G <= 16 take the grouped tensor-core kernel (K codes widened into the
# B fragments, V tiles transposed in registers, V scales folded into P).

@pytest.mark.parametrize("G,bs", [(2, 16), (3, 8), (4, 32), (8, 8), (12, 16), (16, 32)])
@pytest.mark.parametrize("partition", [0, 64])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_group_kernel_fp8_matches_oracle(G, bs, partition, fused):
    st = wl.llama_layer(num_seqs=6, num_blocks=1500, num_heads=2 * G, num_kv_heads=2,
                        block_size=bs, dtype="fp8", ctx_range=(1, 700))
    run = run_step_fused if fused else run_step
    outs, d, err = run(st, partition_size=partition)
    assert err == 0
    ref, kref, vref = oracle.run_step(st, 0)
    assert max_err(outs[0], ref) <= TOL
    assert np.array_equal(to_bits(d["key_caches"][0]), kref)
    assert np.array_equal(to_bits(d["value_caches"][0]), vref)


def test_group_kernel_fp8_fused_equals_separate_and_split_matches_single():
    st = wl.llama_layer(num_seqs=8, num_blocks=2000, num_heads=32, num_kv_heads=4,
                        dtype="fp8", ctx_range=(900, 3000))
    a, da, _ = run_step(st)
    b, db, _ = run_step_fused(st)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(da["key_caches"][0].data, db["key_caches"][0].data)
    ref, _, _ = oracle.run_step(st, 0)
    single, _, e1 = run_step(st, partition_size=4096, out_dtype=torch.float32)
    split, _, e2 = run_step(st, partition_size=256, out_dtype=torch.float32)
    assert e1 == 0 and e2 == 0
    assert max_err(single[0], ref) <= TOL and max_err(split[0], ref) <= TOL
    assert float((split[0] - single[0]).abs().max()) <= TOL


def test_group_kernel_fp8_full_size_sampled():
    st = wl.llama_layer(num_kv_heads=8, dtype="fp8")
    outs, d, err = run_step_fused(st)
    assert err == 0
    ctx = st.context_lens
    rng = np.random.default_rng(66)
    ids = sorted(set([int(np.argmin(ctx)), int(np.argmax(ctx))] +
                     rng.choice(st.num_seqs, 4, replace=False).tolist()))
    ref, _, _ = oracle.run_step(wl.subset(st, ids), 0)
    assert max_err(outs[0][torch.as_tensor(ids, device="cuda")], ref) <= TOL
