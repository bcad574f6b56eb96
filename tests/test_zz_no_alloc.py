"""pa_decode_noalloc: decode for callers that cannot allocate device memory
while they decode (an engine whose KV block pool took almost all device
memory, or a runtime that forbids cudaMalloc after start-up because it may
synchronise the device). It must give the same output as pa_decode with a
caller workspace, call after call, although every call reuses the same
built-in scratch array.

This file is collected last on purpose, so a run that stops at its first
failure has run every other test before this one."""
import ctypes

import numpy as np
import pytest
import torch

from tests import paged_cases as pc
from tests.gpu_harness import TOL

pytestmark = pytest.mark.gpu


def _upload(c):
    dt = torch.float16 if c["dtype"] == "f16" else torch.bfloat16

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).cuda()

    return dict(q=up(c["q"]), kc=up(c["kpool"]), vc=up(c["vpool"]),
                bt=torch.from_numpy(c["bt"]).cuda(), ctx=torch.from_numpy(c["ctx"]).cuda())


def _call(pk, fn_name, t, c, partition, workspace=None):
    """One decode through the C ABI; returns (output, dev_err)."""
    L = pk._lib
    out = torch.empty(t["q"].shape, dtype=t["q"].dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = pk.cache_desc(t["kc"])
    S, H, _ = t["q"].shape
    stream = torch.cuda.current_stream().cuda_stream
    args = [out.data_ptr(), pk._DTYPE[out.dtype], t["q"].data_ptr(), S, H, t["kc"].data_ptr(),
            t["vc"].data_ptr(), ctypes.byref(desc), t["bt"].data_ptr(), t["bt"].shape[1],
            t["ctx"].data_ptr(), int(c["ctx"].max()), float(c["scale"]), partition]
    if fn_name == "pa_decode":
        args += [workspace.data_ptr(), workspace.numel(), err.data_ptr(), stream]
    else:
        args += [err.data_ptr(), stream]
    status = getattr(L, fn_name)(*args)
    assert status == pk.PA_OK, L.pa_last_error().decode()
    return out, err


def _grouped_case(rng, ctxs, kv_heads, group, D, bs):
    """A paged case with ``group`` query heads per K/V head."""
    c = pc.paged_case(rng, ctxs, kv_heads, D, bs)
    c["q"] = pc.to_storage_bits(
        rng.standard_normal((len(ctxs), kv_heads * group, D), dtype=np.float32), "f16")
    return c


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_noalloc_matches_decode_on_consecutive_calls():
    """Two calls in a row per case (and cases back to back on the same
    array): each output is bit-identical to pa_decode's with a caller
    workspace, since both run the same kernel with the same partitions and
    merge them in the same order."""
    import paged_kv_cache_417_b200 as pk
    rng = np.random.default_rng(77)
    cases = [  # split contexts (partials go through the scratch), then other batches
        (pc.paged_case(rng, [3000, 17, 1500, 4096, 1], 4, 128, 16), 256),
        (pc.paged_case(rng, [700, 2048, 33, 999], 8, 64, 32), 0),
        (_grouped_case(rng, [5000, 40, 2600], 2, 4, 128, 16), 512),
    ]
    for c, partition in cases:
        t = _upload(c)
        S, H, D = c["q"].shape
        ws = pk.alloc_workspace(S, H, D, int(c["ctx"].max()), partition)
        ref, err_ref = _call(pk, "pa_decode", t, c, partition, ws)
        first, err1 = _call(pk, "pa_decode_noalloc", t, c, partition)
        second, err2 = _call(pk, "pa_decode_noalloc", t, c, partition)
        torch.cuda.synchronize()
        assert int(err_ref.item()) == 0 and int(err1.item()) == 0 and int(err2.item()) == 0
        assert bool(torch.isfinite(first).all())
        assert _same_bits(first, ref), "first call differs from pa_decode"
        assert _same_bits(second, ref), "second call differs from pa_decode"
        assert float((first.float() - ref.float()).abs().max()) <= TOL


def test_noalloc_separate_merge_kernel_path():
    """Grouped heads whose merge weights exceed the merging CTA's buffer
    (8 heads x 1032 partitions of 32 tokens) take the separate merge kernel;
    both calls match pa_decode bit for bit and the oracle within the
    tolerance."""
    import oracle
    import paged_kv_cache_417_b200 as pk
    rng = np.random.default_rng(78)
    c = _grouped_case(rng, [33000, 700], 1, 8, 128, 16)
    t = _upload(c)
    S, H, D = c["q"].shape
    ws = pk.alloc_workspace(S, H, D, int(c["ctx"].max()), 32)
    assert ws.numel() <= pk.NOALLOC_SCRATCH_BYTES
    ref, err_ref = _call(pk, "pa_decode", t, c, 32, ws)
    got1, err1 = _call(pk, "pa_decode_noalloc", t, c, 32)
    got2, err2 = _call(pk, "pa_decode_noalloc", t, c, 32)
    torch.cuda.synchronize()
    assert int(err_ref.item()) == 0 and int(err1.item()) == 0 and int(err2.item()) == 0
    assert _same_bits(got1, ref) and _same_bits(got2, ref)
    want = oracle.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"])
    assert float(np.max(np.abs(got1.double().cpu().numpy() - want))) <= TOL


def test_noalloc_rejects_work_beyond_its_scratch():
    import paged_kv_cache_417_b200 as pk
    # 2048 sequences x 32 heads split into 64 partitions of 128 tokens need
    # far more than 32 MiB of partial results: refused before any launch.
    need = pk.decode_workspace_size(2048, 32, 128, 8192, 128)
    assert need > pk.NOALLOC_SCRATCH_BYTES
    kc = torch.zeros(4, 32, 16, 128, dtype=torch.float16, device="cuda")
    q = torch.zeros(2048, 32, 128, dtype=torch.float16, device="cuda")
    bt = torch.zeros(2048, 512, dtype=torch.int32, device="cuda")
    ctx = torch.ones(2048, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedKVError) as e:
        pk.decode_noalloc(torch.empty_like(q), q, kc, kc, bt, ctx, 8192, 0.1,
                          partition_size=128)
    assert e.value.status == pk.PA_ERR_WORKSPACE
