"""Decode steps whose integer inputs come from the library's C++ block manager.

The benchmark builds each step's block tables, context lengths, slots and
copy-on-write pairs with pa_bm_prepare_decode (the bookkeeping of
"啃透vLLM源码", §2.2-§3, and "vLLM基础", §2.3). Here every workload runs
pa_copy_blocks -> pa_write_kv_decode (and the separate calls) from those
inputs; the oracle runs on the Python allocator's inputs for the same seed.
The two input sets must be identical, the GPU outputs from them bit-identical
to the GPU outputs from the Python inputs, within the tolerance of the
oracle's, and both pools byte-exact with the oracle's.
"""
import numpy as np
import pytest
import torch

import bench
import workloads as wl
from tests.gpu_harness import check_outputs_and_pools

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)

CASES = [
    ("tiny", lambda: wl.tiny()),
    ("llama7b_layer", lambda: wl.llama_layer()),
    ("long_context_reduced", lambda: wl.long_context(num_seqs=3, ctx_range=(3000, 6000),
                                                     num_blocks=1500)),
    ("prefix_cow", lambda: wl.prefix_cow()),
    ("full_step_bs8", lambda: wl.full_step(block_size=8, num_seqs=64, num_layers=2)),
    ("full_step_bs16", lambda: wl.full_step(block_size=16, num_seqs=64, num_layers=2)),
    ("full_step_bs32", lambda: wl.full_step(block_size=32, num_seqs=64, num_layers=2)),
]


def _run(step, integer_inputs, fused):
    d = bench.upload_step(step, DEV, integer_inputs)
    lch = bench.StepLauncher(step, d, DEV, fused=fused)
    lch.one_step()
    torch.cuda.synchronize()
    return lch.outs, d


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
def test_step_from_native_block_manager(name, make, fused):
    st = make()
    native = bench.native_inputs(st)
    for k in bench.INTEGER_INPUTS:
        assert np.array_equal(native[k], getattr(st, k)), k
    outs, d = _run(st, native, fused)
    layers = [0] if st.num_layers == 1 else [0, st.num_layers - 1]
    check_outputs_and_pools(st, outs, d, layers)
    del d
    py_outs, _ = _run(st, None, fused)
    for a, b in zip(outs, py_outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
