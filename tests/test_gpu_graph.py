"""The benchmarked path under parity: the decode step captured in a CUDA graph
and replayed, exactly as ``bench.py`` builds and runs it (its own
``StepLauncher`` and ``E2EPipeline``), against the fp64 oracle.

The pages put the decode step of the worker in a CUDA graph
("啃透vLLM源码", §4, the model runner's graph capture); the benchmark's
numbers come from such replays (the fused K/V write + decode per layer), and
its end-to-end figure from two more graphs captured over separate input and
output buffers fed by pinned-host copies on their own streams. Each replay
rewrites the new tokens into the same slots and recomputes the same
outputs, so after any number of replays every output element must match the
oracle's step and both pools must equal the oracle's post-step pools byte for
byte. On the split (long-context) workload each replay also runs the
partition merge, whose arrival counters must be back at zero after every
replay for the next one to merge correctly.
"""
import numpy as np
import pytest
import torch

import bench
from tests.gpu_harness import TOL, check_outputs_and_pools, err_report, to_bits

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _launcher(config, **kw):
    step = bench.make_step(config, 0, **kw)
    d = bench.upload_step(step, DEV)
    return step, d, bench.StepLauncher(step, d, DEV, fused=True, partition=0)


def _last_layers(step):
    return [0] if step.num_layers == 1 else [0, step.num_layers - 1]


def test_graph_step_llama_layer_matches_oracle():
    """96 sequences x 32 heads, fused write + decode replayed from one graph:
    every output element and both pools after the 1st and the 5th replay."""
    step, d, lch = _launcher("llama7b_layer")
    g = lch.capture()
    g.replay()
    torch.cuda.synchronize()
    check_outputs_and_pools(step, lch.outs, d, [0])
    first = lch.outs[0].clone()
    for _ in range(4):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(lch.outs[0].view(torch.int16), first.view(torch.int16)), \
        "replays disagree"
    check_outputs_and_pools(step, lch.outs, d, [0])


def test_e2e_pipeline_graphs_match_oracle():
    """The end-to-end leg: two graphs over their own input/output buffers,
    inputs uploaded with non-blocking copies from pinned memory on an upload
    stream, outputs downloaded on another; what arrives in host memory for
    both buffer sets equals the oracle's outputs, and the pools are exact."""
    step, d, lch = _launcher("llama7b_layer")
    pipe = bench.E2EPipeline(lch, graph=True)
    pipe.run(5)
    torch.cuda.synchronize()
    import oracle
    ref, kref, vref = oracle.run_step(step, 0)
    for b in range(2):
        out = pipe.host_outputs(b)[0]
        mx, mean, worst = err_report(out, ref)
        assert mx <= TOL, f"buffer set {b}: max err {mx:.3e} at {worst}, mean {mean:.3e}"
    assert np.array_equal(to_bits(d["key_caches"][0]), kref)
    assert np.array_equal(to_bits(d["value_caches"][0]), vref)
    # The first replays of a buffer set and the device-resident step agree.
    g = lch.capture()
    g.replay()
    torch.cuda.synchronize()
    for b in range(2):
        assert torch.equal(pipe.host_outputs(b)[0].to(DEV).view(torch.int16),
                           lch.outs[0].view(torch.int16))


def test_graph_step_long_context_split_replays():
    """8 sequences of 16k-32k tokens: split into partitions merged by the
    last CTA of each sequence. Four replays; the outputs match the oracle
    after the first and the last, and the arrival counters (the first 256 KiB
    of the workspace) are zero after each replay."""
    step, d, lch = _launcher("long_context")
    assert lch.split, "the long-context workload must take the split path"
    g = lch.capture()
    counters = lch.ws[:256 * 1024].view(torch.int32)
    for k in range(4):
        g.replay()
        torch.cuda.synchronize()
        assert not bool(counters.any()), f"arrival counters not reset after replay {k}"
        if k in (0, 3):
            check_outputs_and_pools(step, lch.outs, d, [0])


def test_graph_step_prefix_cow_matches_oracle():
    """Copy-on-write block copies inside the graph, then fused write +
    decode: outputs and pools (copied blocks included) after three
    replays."""
    step, d, lch = _launcher("prefix_cow")
    assert lch.has_copy
    g = lch.capture()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    check_outputs_and_pools(step, lch.outs, d, [0])


def test_graph_step_full_step_matches_oracle():
    """All 32 layers x 256 sequences (block size 16) replayed from one graph
    twice: every output element and both pools of layers 0 and 31."""
    step, d, lch = _launcher("full_step_bs16")
    g = lch.capture()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    check_outputs_and_pools(step, lch.outs, d, _last_layers(step))
