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
