"""Grouped query heads on decode_group_kernel (one CTA per K/V head and
partition): shapes at the edges of its launch logic, against the fp64 oracle.

Many tiny units (512 sequences x 32 K/V heads), tiny inputs with empty
sequences, one long unit split into many partitions, batches on both sides of
the longest-first ordering limit, a workspace too small (refused before any
launch), repeated calls and CUDA-graph replays (bit-identical outputs,
arrival counters back at zero), a bad block id inside a split sequence, and
the benchmark's grouped layers at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_417_b200 as pk
import workloads as wl
from tests import paged_cases as pc
from tests.gpu_harness import (TOL, check_outputs_and_pools, decode_case, err_report,
                               run_step, run_step_fused)
from workloads.steps import to_storage_bits

pytestmark = pytest.mark.gpu


def gqa_case(rng, ctx_list, G, Hkv, D, bs, dtype="f16", num_blocks=None):
    c = pc.paged_case(rng, ctx_list, Hkv, D, bs, num_blocks=num_blocks, dtype=dtype)
    c["q"] = to_storage_bits(
        rng.standard_normal((len(ctx_list), G * Hkv, D), dtype=np.float32), dtype)
    return c


def orc(c):
    return oracle.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"],
                         c["dtype"])


def check(out, ref, what=""):
    mx, mean, worst = err_report(out, ref)
    assert mx <= TOL, f"{what}: max err {mx:.3e} at {worst}, mean {mean:.3e}"


def test_many_tiny_units():
    """512 sequences x 32 K/V heads of 1-20 tokens: 16,384 single-chunk
    units in natural order."""
    rng = np.random.default_rng(70)
    ctxs = rng.integers(1, 21, size=512).tolist()
    c = gqa_case(rng, ctxs, 2, 32, 64, 8)
    out, err = decode_case(c)
    assert err == 0
    check(out, orc(c), "tiny units")


def test_tiny_inputs_with_empty_sequences():
    rng = np.random.default_rng(71)
    for ctxs in ([5], [1, 2], [17, 0, 3]):
        c = gqa_case(rng, ctxs, 4, 2, 128, 16)
        out, err = decode_case(c)
        assert err == 0
        check(out, orc(c), f"ctx {ctxs}")


@pytest.mark.parametrize("G", [4, 16])
def test_one_long_unit_in_many_partitions(G):
    """A single 33000-token unit: the automatic partition splits it into
    many CTAs; the last to finish merges them all."""
    rng = np.random.default_rng(72 + G)
    c = gqa_case(rng, [33000], G, 1, 128, 16)
    out, err = decode_case(c, out_dtype=torch.float32)
    assert err == 0
    check(out, orc(c), "one long unit")


@pytest.mark.parametrize("S", [128, 129, 513])
def test_large_batches(S):
    """128 sequences are handed out longest first, 129 and 513 in natural
    order; all match the oracle, fused and separate."""
    st = wl.llama_layer(seed=73, num_seqs=S, ctx_range=(1, 300), num_blocks=S * 20 + 64,
                        num_heads=16, num_kv_heads=4, head_dim=64)
    for runner in (run_step, run_step_fused):
        outs, d, err = runner(st)
        assert err == 0
        check_outputs_and_pools(st, outs, d, [0])


def test_workspace_too_small_is_refused():
    """A split decode with a workspace smaller than
    pa_decode_workspace_size is refused before any launch; with the full
    size it matches the oracle."""
    rng = np.random.default_rng(74)
    c = gqa_case(rng, [3000, 40, 2600, 900], 8, 2, 128, 16)
    dt = torch.float16
    up = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(dt).cuda()  # noqa: E731
    q, kc, vc = up(c["q"]), up(c["kpool"]), up(c["vpool"])
    bt, ctx = torch.from_numpy(c["bt"]).cuda(), torch.from_numpy(c["ctx"]).cuda()
    S, H, D = q.shape
    mcl = int(c["ctx"].max())
    out = torch.empty_like(q)
    pk.decode(out, q, kc, vc, bt, ctx, mcl, float(c["scale"]),
              workspace=pk.alloc_workspace(S, H, D, mcl))
    torch.cuda.synchronize()
    check(out, orc(c), "full workspace")
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pk.PagedKVError) as e:
        pk.decode(torch.empty_like(q), q, kc, vc, bt, ctx, mcl, float(c["scale"]),
                  partition_size=256, workspace=small)
    assert e.value.status == pk.PA_ERR_WORKSPACE


def test_repeated_calls_and_graph_replays_are_bit_identical():
    st = wl.llama_layer(seed=75, num_kv_heads=4)
    outs, d, err = run_step_fused(st)
    assert err == 0
    first = outs[0].clone()
    S, H, D = d["query"][0].shape
    ws = pk.alloc_workspace(S, H, D, st.max_context_len)
    out = torch.empty_like(first)

    def step():
        pk.write_kv_decode(out, d["query"][0], d["new_key"][0], d["new_value"][0],
                           d["key_caches"][0], d["value_caches"][0], d["block_tables"],
                           d["context_lens"], st.max_context_len, float(st.scale),
                           workspace=ws)

    step()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    counters = ws[:256 * 1024].view(torch.int32)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert not bool(counters.any())
        assert torch.equal(out.view(torch.int16), first.view(torch.int16))
    check_outputs_and_pools(st, [out], d, [0])


def test_bad_block_id_inside_a_split_unit():
    """A bad id in a long unit (split across CTAs) makes that sequence NaN
    and sets the flag; the other sequences are unaffected."""
    rng = np.random.default_rng(76)
    c = gqa_case(rng, [20000, 300, 150], 8, 1, 128, 16)
    c["bt"][0, 700] = c["kpool"].shape[0] + 3
    out, err = decode_case(c)
    assert err & pk.PA_DEVERR_BLOCK_ID
    assert bool(torch.isnan(out[0]).all())
    ref = orc({**c, "bt": c["bt"][1:], "q": c["q"][1:], "ctx": c["ctx"][1:]})
    check(out[1:], ref, "other sequences")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "fp8"])
@pytest.mark.parametrize("kv_heads", [8, 4, 2])
def test_llama_layer_grouped_full_size(dtype, kv_heads):
    """The benchmark's grouped-heads workloads: 96 sequences, 32 query heads
    over 8, 4 or 2 K/V heads; every output element and both pools."""
    st = wl.llama_layer(num_kv_heads=kv_heads, dtype=dtype)
    out_dtype = torch.float32 if dtype == "bf16" else None
    outs, d, err = run_step_fused(st, out_dtype=out_dtype)
    assert err == 0
    check_outputs_and_pools(st, outs, d, [0])
