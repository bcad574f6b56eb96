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


def test_noalloc_matches_decode_on_consecutive_calls():
    import paged_kv_cache_417_b200 as pk
    rng = np.random.default_rng(77)
    cases = [  # split contexts (partials go through the scratch), then a second batch
        (pc.paged_case(rng, [3000, 17, 1500, 4096, 1], 4, 128, 16), 256),
        (pc.paged_case(rng, [700, 2048, 33, 999], 8, 64, 32), 0),
    ]
    for c, partition in cases:
        t = _upload(c)
        S, H, D = c["q"].shape
        ws = pk.alloc_workspace(S, H, D, int(c["ctx"].max()), partition)
        ref, err_ref = _call(pk, "pa_decode", t, c, partition, ws)
        got, err_got = _call(pk, "pa_decode_noalloc", t, c, partition)
        torch.cuda.synchronize()
        assert int(err_ref.item()) == 0 and int(err_got.item()) == 0
        assert bool(torch.isfinite(got).all())
        assert float((got.float() - ref.float()).abs().max()) <= TOL


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
