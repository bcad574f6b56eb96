"""The separate merge kernel (reduce_kernel) against the fp64 oracle.

Split partitions are normally merged by the last CTA of each sequence. Two
shapes take a second kernel instead: more (sequence, head) slots than a
workspace has arrival counters (num_seqs * num_heads > 65536), and more
merge weights per CTA than its shared-memory buffer holds (heads per CTA x
partitions > 8192). Each case runs through pa_write_kv + pa_decode and
through the fused pa_write_kv_decode, and is compared element by element
with the oracle, both pools byte for byte.
"""
import pytest

import paged_kv_cache_417_b200 as pk
import workloads as wl
from tests.gpu_harness import check_outputs_and_pools, run_step, run_step_fused

pytestmark = pytest.mark.gpu


def _check_both_paths(step, partition):
    for runner in (run_step, run_step_fused):
        outs, d, err = runner(step, partition_size=partition)
        assert err == 0, f"dev_err {err}"
        check_outputs_and_pools(step, outs, d, [0])
        del d


def test_reduce_kernel_more_slots_than_counters():
    """2100 sequences x 32 heads = 67200 (sequence, head) slots > 65536, every
    context split into 2 partitions of 32 tokens."""
    st = wl.llama_layer(seed=11, num_seqs=2100, ctx_range=(33, 48), num_blocks=6600,
                        num_heads=32, head_dim=64)
    assert st.num_seqs * st.num_heads > 65536
    assert pk.decode_partition_size(st.num_seqs, st.num_heads,
                                    pk.CacheDesc(st.num_blocks, 16, 32, 64, pk.PA_F16,
                                                 pk.PA_F16),
                                    st.max_context_len, 32) == 32
    _check_both_paths(st, 32)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "fp8"])
def test_reduce_kernel_grouped_heads_many_partitions(dtype):
    """16 query heads on one K/V head (the grouped kernel), 17k-token
    contexts in partitions of 32 tokens: 16 x ~550 merge weights > 8192."""
    st = wl.llama_layer(seed=12, num_seqs=2, ctx_range=(17000, 17600), num_blocks=2300,
                        num_heads=16, num_kv_heads=1, head_dim=128, dtype=dtype)
    assert 16 * -(-st.max_context_len // 32) > 8192
    if dtype == "bf16":
        import torch
        from tests.gpu_harness import TOL
        for runner in (run_step, run_step_fused):
            outs, d, err = runner(st, partition_size=32, out_dtype=torch.float32)
            assert err == 0
            check_outputs_and_pools(st, outs, d, [0], tol=TOL)
        return
    _check_both_paths(st, 32)


def test_reduce_kernel_one_head_many_partitions():
    """One head, 263,000 tokens in partitions of 32: 8219 partitions, more
    merge weights than the merging CTA holds, on the per-head kernel."""
    st = wl.llama_layer(seed=13, num_seqs=1, ctx_range=(263000, 263000), num_blocks=16500,
                        num_heads=1, head_dim=64)
    assert -(-st.max_context_len // 32) > 8192
    _check_both_paths(st, 32)
