"""pa_write_kv_decode (the new token's K/V write fused into decode) against
the oracle's separate write-then-decode, and against the library's own
separate pa_write_kv + pa_decode calls (bit-identical: same bytes, same
arithmetic order)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.gpu_harness import (TOL, check_outputs_and_pools, max_err, run_step,
                               run_step_fused, to_bits, to_f64)

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", lambda: wl.tiny()),
    ("llama_reduced", lambda: wl.llama_layer(num_seqs=12, num_blocks=1024)),
    ("long_reduced", lambda: wl.long_context(num_seqs=3, ctx_range=(3000, 6000),
                                             num_blocks=1500)),
    ("prefix_cow", lambda: wl.prefix_cow()),
    ("full_bs8", lambda: wl.full_step(block_size=8, num_seqs=24, num_layers=2)),
    ("full_bs16", lambda: wl.full_step(block_size=16, num_seqs=24, num_layers=2)),
    ("full_bs32", lambda: wl.full_step(block_size=32, num_seqs=24, num_layers=2)),
    ("tiny_bf16", lambda: wl.tiny(dtype="bf16")),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("partition", [0, 64])
def test_fused_matches_oracle(name, make, partition):
    st = make()
    out_dtype = torch.float32 if st.dtype == "bf16" else None
    outs, d, err = run_step_fused(st, partition_size=partition, out_dtype=out_dtype)
    assert err == 0
    for li in range(st.num_layers):
        ref, kref, vref = oracle.run_step(st, li)
        assert max_err(outs[li], ref) <= TOL
        assert np.array_equal(to_bits(d["key_caches"][li]), kref)
        assert np.array_equal(to_bits(d["value_caches"][li]), vref)


@pytest.mark.parametrize("partition", [0, 32, 512])
def test_fused_bit_identical_to_separate_calls(partition):
    st = wl.llama_layer(num_seqs=16, num_blocks=2048)
    a, da, _ = run_step(st, partition_size=partition)
    b, db, _ = run_step_fused(st, partition_size=partition)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(da["key_caches"][0].view(torch.int16), db["key_caches"][0].view(torch.int16))
    assert torch.equal(da["value_caches"][0].view(torch.int16),
                       db["value_caches"][0].view(torch.int16))


def test_fused_full_size():
    """The benchmark's workload through the fused call: all 96 sequences,
    every output element, both pools byte for byte."""
    st = wl.llama_layer()
    outs, d, err = run_step_fused(st)
    assert err == 0
    check_outputs_and_pools(st, outs, d, [0])


def test_fused_context_one_and_zero():
    """ctx = 1: the output is the new value row itself; ctx = 0: nothing is
    appended and the output is zero."""
    st = wl.tiny(context_lens=(1, 1, 19, 1))
    outs, d, err = run_step_fused(st)
    assert err == 0
    got = to_f64(outs[0])
    nv = st.layers[0].new_value.view(np.float16).astype(np.float64)
    for s in (0, 1, 3):
        assert np.array_equal(got[s], nv[s])
    import paged_kv_cache_417_b200 as pk
    d2 = {k: v for k, v in d.items()}
    ctx0 = torch.zeros_like(d2["context_lens"])
    kc_before = d2["key_caches"][0].clone()
    out = torch.empty_like(d2["query"][0])
    pk.write_kv_decode(out, d2["query"][0], d2["new_key"][0], d2["new_value"][0],
                       d2["key_caches"][0], d2["value_caches"][0], d2["block_tables"], ctx0,
                       st.max_context_len, float(st.scale))
    torch.cuda.synchronize()
    assert not bool(out.any())
    assert torch.equal(kc_before.view(torch.int16), d2["key_caches"][0].view(torch.int16))
