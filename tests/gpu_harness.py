"""Run decode steps through the CUDA library for the parity tests."""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_417_b200 as pk
from workloads.device import device_step

TOL = 2e-3  # max |gpu - oracle| for fp16 output, fp32 accumulation


def to_bits(t) -> np.ndarray:
    """Raw storage of a cache or tensor: uint16 patterns, or bytes for fp8."""
    if isinstance(t, pk.Fp8Cache):
        return t.data.detach().cpu().numpy()
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def wrap_caches(step, d):
    """fp8 pools come from device_step as uint8 tensors: wrap them."""
    if step.dtype == "fp8":
        for key in ("key_caches", "value_caches"):
            d[key] = [pk.Fp8Cache(t, step.block_size, step.head_dim, torch.float16)
                      for t in d[key]]
    return d


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def run_step(step, layers=None, partition_size=0, out_dtype=None):
    """copy_blocks (all layers) -> per layer write_kv, decode. Returns
    (outs list, device dict, dev_err int)."""
    layers = list(range(step.num_layers)) if layers is None else list(layers)
    d = wrap_caches(step, device_step(step, "cuda", layers))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if step.copy_pairs.shape[0]:
        pk.copy_blocks(d["key_caches"], d["value_caches"], d["copy_pairs"], dev_err=err)
    outs = []
    for i, _ in enumerate(layers):
        kc, vc = d["key_caches"][i], d["value_caches"][i]
        pk.write_kv(d["new_key"][i], d["new_value"][i], d["slot_mapping"], kc, vc, dev_err=err)
        q = d["query"][i]
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device="cuda")
        pk.decode(out, q, kc, vc, d["block_tables"], d["context_lens"], step.max_context_len,
                  float(step.scale), partition_size=partition_size, dev_err=err)
        outs.append(out)
    torch.cuda.synchronize()
    return outs, d, int(err.item())


def err_report(gpu_out: torch.Tensor, ref: np.ndarray):
    """(max |gpu - ref|, mean |gpu - ref|, worst index) over every element."""
    got = to_f64(gpu_out)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite output"
    if not ref.size:
        return 0.0, 0.0, ()
    err = np.abs(got - ref)
    k = int(np.argmax(err))
    return float(err.flat[k]), float(err.mean()), tuple(int(i) for i in
                                                         np.unravel_index(k, err.shape))


def check_outputs_and_pools(step, outs, d, layers, tol=TOL, out_index=None):
    """Every output element of ``layers`` against the oracle's full step
    (copy-on-write, write, decode) on the same inputs, and both pools of
    those layers byte for byte. ``out_index(li)`` gives the position of layer
    ``li`` in ``outs`` and ``d`` (default: li)."""
    import oracle
    for li in layers:
        i = li if out_index is None else out_index(li)
        ref, kref, vref = oracle.run_step(step, li)
        mx, mean, worst = err_report(outs[i], ref)
        assert mx <= tol, (f"{step.name} layer {li}: max err {mx:.3e} at (s, h, d) = {worst}, "
                           f"mean {mean:.3e}")
        for pool, want in ((d["key_caches"][i], kref), (d["value_caches"][i], vref)):
            got = to_bits(pool)
            if not np.array_equal(got, want):
                bad = np.argwhere(got != want)
                raise AssertionError(f"{step.name} layer {li}: pool differs at {bad[:3].tolist()} "
                                     f"({len(bad)} elements)")


def max_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    got = to_f64(gpu_out)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite output"
    return float(np.max(np.abs(got - ref))) if ref.size else 0.0


def decode_case(c, partition_size=0, out_dtype=None, max_context_len=None):
    """Decode a tests.paged_cases case on the GPU."""
    dt = torch.float16 if c["dtype"] == "f16" else torch.bfloat16

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).cuda()

    q, kc, vc = up(c["q"]), up(c["kpool"]), up(c["vpool"])
    bt = torch.from_numpy(c["bt"]).cuda()
    ctx = torch.from_numpy(c["ctx"]).cuda()
    out = torch.empty(q.shape, dtype=out_dtype or dt, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mcl = int(c["ctx"].max()) if max_context_len is None else max_context_len
    pk.decode(out, q, kc, vc, bt, ctx, mcl, float(c["scale"]), partition_size=partition_size,
              dev_err=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def run_step_fused(step, layers=None, partition_size=0, out_dtype=None):
    """copy_blocks (all layers) -> per layer write_kv_decode (one launch)."""
    layers = list(range(step.num_layers)) if layers is None else list(layers)
    d = wrap_caches(step, device_step(step, "cuda", layers))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if step.copy_pairs.shape[0]:
        pk.copy_blocks(d["key_caches"], d["value_caches"], d["copy_pairs"], dev_err=err)
    outs = []
    for i, _ in enumerate(layers):
        q = d["query"][i]
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device="cuda")
        pk.write_kv_decode(out, q, d["new_key"][i], d["new_value"][i], d["key_caches"][i],
                           d["value_caches"][i], d["block_tables"], d["context_lens"],
                           step.max_context_len, float(step.scale),
                           partition_size=partition_size, dev_err=err)
        outs.append(out)
    torch.cuda.synchronize()
    return outs, d, int(err.item())
