"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import paged_kv_cache_417_b200 as pk
    return pk


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \t\*]*?\b(pa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["pa_write_kv", "pa_decode", "pa_copy_blocks", "pa_decode_workspace_size",
              "pa_write_kv_decode", "pa_status_string", "pa_last_error", "pa_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in declared_functions():
        assert hasattr(so, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    for s in range(5):
        assert lib._lib.pa_status_string(s)
    assert lib.version() >= 100


def _desc(lib, nb=16, bs=16, h=2, d=64, dt=0):
    return lib.CacheDesc(nb, bs, h, d, dt)


def test_decode_rejects_bad_arguments_on_host(lib):
    L = lib._lib
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: checks fail first
    cases = [
        (_desc(lib, d=96), lib.PA_ERR_UNSUPPORTED),        # head_dim
        (_desc(lib, bs=64), lib.PA_ERR_UNSUPPORTED),       # block_size
        (_desc(lib, dt=2), lib.PA_ERR_UNSUPPORTED),        # fp32 cache
        (_desc(lib, h=3), lib.PA_ERR_UNSUPPORTED),         # num_heads != kv heads
    ]
    for desc, want in cases:
        st = L.pa_decode(fake, 0, fake, 1, 2, fake, fake, ctypes.byref(desc), fake, 1, fake,
                         16, 0.125, 0, None, 0, None, None)
        assert st == want, (desc.head_dim, desc.block_size, st)
        assert L.pa_last_error()
    desc = _desc(lib)
    # unaligned query
    st = L.pa_decode(fake, 0, ctypes.c_void_p(0x1002), 1, 2, fake, fake, ctypes.byref(desc),
                     fake, 1, fake, 16, 0.125, 0, None, 0, None, None)
    assert st == lib.PA_ERR_INVALID_ARG
    # bad partition size
    st = L.pa_decode(fake, 0, fake, 1, 2, fake, fake, ctypes.byref(desc), fake, 1, fake, 16,
                     0.125, 48, None, 0, None, None)
    assert st == lib.PA_ERR_INVALID_ARG
    # null pointers
    st = L.pa_decode(None, 0, fake, 1, 2, fake, fake, ctypes.byref(desc), fake, 1, fake, 16,
                     0.125, 0, None, 0, None, None)
    assert st == lib.PA_ERR_INVALID_ARG
    # zero sequences: nothing to do, no launch
    st = L.pa_decode(None, 0, None, 0, 2, None, None, ctypes.byref(desc), None, 0, None, 0,
                     0.125, 0, None, 0, None, None)
    assert st == lib.PA_OK
    # split needed but no workspace (32 partitions of 32 tokens)
    st = L.pa_decode(fake, 0, fake, 1, 2, fake, fake, ctypes.byref(desc), fake, 64, fake,
                     1024, 0.125, 32, None, 0, None, None)
    assert st == lib.PA_ERR_WORKSPACE


def test_write_and_copy_reject_bad_arguments(lib):
    L = lib._lib
    fake = ctypes.c_void_p(0x1000)
    desc = _desc(lib)
    assert L.pa_write_kv(fake, fake, -1, 2, fake, fake, fake, ctypes.byref(desc), None,
                         None) == lib.PA_ERR_INVALID_ARG
    assert L.pa_write_kv(fake, fake, 0, 2, fake, fake, fake, ctypes.byref(desc), None,
                         None) == lib.PA_OK
    assert L.pa_write_kv(None, fake, 3, 2, fake, fake, fake, ctypes.byref(desc), None,
                         None) == lib.PA_ERR_INVALID_ARG
    assert L.pa_write_kv(fake, fake, 3, 2, fake, fake, fake, None, None,
                         None) == lib.PA_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 1)(0x1000)
    assert L.pa_copy_blocks(arr, arr, 0, fake, 1, ctypes.byref(desc), None,
                            None) == lib.PA_ERR_INVALID_ARG
    assert L.pa_copy_blocks(arr, arr, 1, fake, 0, ctypes.byref(desc), None, None) == lib.PA_OK
    bad = (ctypes.c_void_p * 1)(0x1004)
    assert L.pa_copy_blocks(bad, bad, 1, fake, 1, ctypes.byref(desc), None,
                            None) == lib.PA_ERR_INVALID_ARG


def test_workspace_and_partition_sizes(lib):
    # single pass: no workspace
    assert lib.decode_workspace_size(4, 4, 64, 100, 0) == 0
    assert lib.decode_workspace_size(4, 4, 64, 512, 512) == 0
    # explicit partitions: 65536 int32 arrival counters, acc [S,H,P,D] fp32
    # padded to 256 B, then (m, l) pairs
    S, H, D, ctx, P = 3, 5, 128, 1000, 256
    parts = -(-ctx // P)
    acc = S * H * parts * D * 4
    want = 65536 * 4 + -(-acc // 256) * 256 + S * H * parts * 2 * 4
    assert lib.decode_workspace_size(S, H, D, ctx, P) == want
    # automatic: a bound that covers the smallest automatic partition (128)
    assert lib.decode_workspace_size(S, H, D, ctx, 0) >= lib.decode_workspace_size(S, H, D, ctx,
                                                                                   128)
    with pytest.raises(ValueError):
        lib.decode_workspace_size(S, H, D, ctx, 40)
    def desc(hkv, dtype=lib.PA_F16, nb=8192, d=128, bs=16, io=lib.PA_F16):
        return lib.CacheDesc(nb, bs, hkv, d, dtype, dtype if dtype != lib.PA_FP8_E4M3 else io)

    assert lib.decode_partition_size(S, H, desc(H, d=D), 100, 0) == 128  # single, rounded to 32
    assert lib.decode_partition_size(96, 32, desc(32), 2048, 0) == 2048  # single pass
    assert lib.decode_partition_size(8, 32, desc(32), 32768, 0) == 2048
    assert lib.decode_partition_size(1, 32, desc(32), 32768, 0) == 1024  # 32 x 32 CTAs
    # 8 sequences x 32 heads, contexts up to ~600 tokens (the small-batch
    # step): halved until the grid has 4 CTAs per SM (256 x 3 >= 4 x 148)
    assert lib.decode_partition_size(8, 32, desc(32), 600, 0) == 256
    assert lib.decode_partition_size(96, 32, desc(32), 2048, 1024) == 1024
    assert lib.decode_partition_size(1, 1, desc(1), 30000, 0) == 128
    # Grouped heads (2 <= G <= 16) on a 16-bit cache, or on an fp8 cache with
    # f16 rows and head_dim 128: the tensor-core kernel, one CTA row per K/V
    # head. Batches of up to 128 sequences (handed out longest first):
    # 2048-token partitions halved while the grid has fewer than 2 CTAs per
    # SM; larger batches: 1024 halved while it has fewer CTAs than SMs.
    # fp8 without grouping, with bf16 rows or head_dim 64 stays on one CTA
    # row per query head.
    assert lib.decode_partition_size(96, 32, desc(8), 2048, 0) == 2048  # single pass
    assert lib.decode_partition_size(96, 32, desc(8, lib.PA_BF16), 4096, 0) == 2048
    assert lib.decode_partition_size(96, 32, desc(2), 2048, 0) == 1024  # 192 x 2 CTAs
    assert lib.decode_partition_size(96, 32, desc(8), 1000, 0) == 1024  # single pass
    assert lib.decode_partition_size(1, 32, desc(8), 32768, 0) == 512  # 8 x 64 CTAs
    assert lib.decode_partition_size(1, 32, desc(8), 4096, 0) == 256  # 8 x 16 CTAs
    assert lib.decode_partition_size(256, 32, desc(8), 2048, 0) == 1024  # natural order
    assert lib.decode_partition_size(96, 32, desc(8, lib.PA_FP8_E4M3), 4096, 0) == 2048
    assert lib.decode_partition_size(96, 32, desc(32, lib.PA_FP8_E4M3), 2048, 0) == 2048
    assert lib.decode_partition_size(96, 32, desc(8, lib.PA_FP8_E4M3, io=lib.PA_BF16),
                                      2048, 0) == 2048
    assert lib.decode_partition_size(96, 32, desc(32, lib.PA_FP8_E4M3, d=64), 2048, 0) == 2048
    with pytest.raises(ValueError):
        lib.decode_partition_size(96, 32, desc(7), 2048, 0)  # 32 % 7 != 0
    assert lib.decode_partition_size(96, 32, desc(1), 2048, 0) == 2048  # G = 32 > 16


def test_newer_entry_points_reject_bad_arguments_on_host(lib):
    """Checks that return before any CUDA call (fake pointers are never
    dereferenced)."""
    L = lib._lib
    fake = ctypes.c_void_p(0x1000)
    # An empty pool with a positive max_context_len cannot be decoded.
    empty = _desc(lib, nb=0)
    st = L.pa_decode(fake, 0, fake, 1, 2, fake, fake, ctypes.byref(empty), fake, 1, fake, 16,
                     0.125, 0, None, 0, None, None)
    assert st == lib.PA_ERR_INVALID_ARG and b"empty pool" in L.pa_last_error()
    # The fused call needs both new rows.
    desc = _desc(lib)
    st = L.pa_write_kv_decode(fake, 0, fake, None, fake, 1, 2, fake, fake, ctypes.byref(desc),
                              fake, 1, fake, 16, 0.125, 0, None, 0, None, None)
    assert st == lib.PA_ERR_INVALID_ARG
    # pa_decode_noalloc refuses work whose partials exceed its built-in
    # scratch (64 sequences x 64 heads x 256 partitions of 32 tokens).
    big = _desc(lib, h=64, d=128)
    st = L.pa_decode_noalloc(fake, 0, fake, 64, 64, fake, fake, ctypes.byref(big), fake, 256,
                             fake, 8192, 0.125, 32, None, None)
    assert st == lib.PA_ERR_WORKSPACE and b"scratch" in L.pa_last_error()
    # Self-test of the bounded wait: device flag required, limit in (0, 1 s].
    assert L.pa_selftest_wait_timeout(None, 10, None) == lib.PA_ERR_INVALID_ARG
    assert L.pa_selftest_wait_timeout(fake, 0, None) == lib.PA_ERR_INVALID_ARG
    assert L.pa_selftest_wait_timeout(fake, 1000001, None) == lib.PA_ERR_INVALID_ARG


def test_noalloc_checks_arguments_like_decode(lib):
    """pa_decode_noalloc runs pa_decode's argument checks in the same order:
    for arguments that fail before the workspace matters, both calls return
    the same status (fake pointers are never dereferenced)."""
    L = lib._lib
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)  # not 16-byte aligned
    ok = _desc(lib, h=2)
    # (num_seqs, num_heads, desc, max_blocks, max_ctx, partition, out_dtype, query, scale)
    cases = [
        (0, 3, ok, 1, 16, 0, 0, fake, 0.1),          # heads not a multiple, empty batch
        (4, 3, ok, 1, 16, 0, 0, fake, 0.1),          # heads not a multiple
        (0, 2, _desc(lib, d=96), 1, 16, 0, 0, fake, 0.1),
        (0, 2, ok, 1, 16, 0, 7, fake, 0.1),          # out_dtype
        (0, 2, ok, 1, 16, 48, 0, fake, 0.1),         # partition not a multiple of 32
        (2, 2, ok, -1, 16, 0, 0, fake, 0.1),         # negative max_blocks_per_seq
        (2, 2, ok, 1, -5, 0, 0, fake, 0.1),          # negative max_context_len
        (70000, 2, ok, 1, 16, 0, 0, fake, 0.1),      # too many sequences
        (2, 2, ok, 1, 16, 0, 0, None, 0.1),          # NULL query
        (2, 2, ok, 1, 16, 0, 0, odd, 0.1),           # misaligned query
        (2, 2, ok, 1, 16, 0, 0, fake, float("nan")),  # NaN scale
        (2, 2, _desc(lib, nb=0), 1, 16, 0, 0, fake, 0.1),  # empty pool
        (0, 2, ok, 1, 16, 0, 0, fake, 0.1),          # valid, empty batch: PA_OK
    ]
    for S, H, desc, mb, mcl, part, odt, q, scale in cases:
        a = L.pa_decode(fake, odt, q, S, H, fake, fake, ctypes.byref(desc), fake, mb, fake, mcl,
                        scale, part, None, 0, None, None)
        b = L.pa_decode_noalloc(fake, odt, q, S, H, fake, fake, ctypes.byref(desc), fake, mb,
                                fake, mcl, scale, part, None, None)
        assert a == b, (S, H, mb, mcl, part, odt, a, b)
    assert L.pa_decode(fake, 0, fake, 0, 3, fake, fake, ctypes.byref(ok), fake, 1, fake, 16,
                       0.1, 0, None, 0, None, None) == lib.PA_ERR_UNSUPPORTED


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="would launch on fake pointers where a GPU exists")
def test_grouped_decode_without_a_gpu_fails_cleanly(lib):
    """With no GPU, a call that passes the host checks reports a CUDA error
    (no CPU fallback computes anything)."""
    L = lib._lib
    fake = ctypes.c_void_p(0x1000)
    for dt in (0, 3):  # f16, and fp8 with f16 rows (both take the grouped kernel)
        desc = lib.CacheDesc(16, 16, 2, 128, dt, 0)
        st = L.pa_decode(fake, 0, fake, 1, 8, fake, fake, ctypes.byref(desc), fake, 1, fake,
                         16, 0.125, 0, None, 0, None, None)
        assert st == lib.PA_ERR_CUDA, L.pa_last_error()
