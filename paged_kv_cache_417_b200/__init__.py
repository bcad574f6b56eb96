"""Python binding of libpagedkv (include/pagedkv.h): paged decode attention
and its cache-maintenance calls on B200 (sm_100a).

Argument marshalling only: tensors are passed to the C ABI as raw device
pointers with the current CUDA stream; every step of the computation runs in
the library's kernels. There is no fallback: importing this module fails if
the library has not been built (``python paged_kv_cache_417_b200/build.py``).

Cache tensors are [num_blocks, num_heads, block_size, head_dim] fp16/bf16
(see the header for the full contract).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python paged_kv_cache_417_b200/build.py` "
        "(nvcc, sm_100a). There is no non-CUDA fallback.")

_lib = ctypes.CDLL(LIB_PATH)

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA = range(5)
PA_F16, PA_BF16, PA_F32, PA_FP8_E4M3 = 0, 1, 2, 3
PA_DEVERR_BLOCK_ID = 1
PA_DEVERR_CONTEXT_LEN = 2
PA_DEVERR_SLOT = 4
PA_DEVERR_TIMEOUT = 8
PA_DEVERR_COPY_PAIR = 16
PA_MAX_LAYERS = 256

_DTYPE = {torch.float16: PA_F16, torch.bfloat16: PA_BF16, torch.float32: PA_F32}


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int), ("io_dtype", ctypes.c_int)]


class Fp8Cache:
    """An fp8 (e4m3) K or V cache: a uint8 tensor [num_blocks, num_heads,
    block_size*head_dim + 4*block_size] whose (block, head) tiles hold
    block_size rows of head_dim codes and then one fp32 scale per row.
    ``io_dtype`` is the dtype of the query/key/value rows used with it."""

    def __init__(self, data, block_size, head_dim, io_dtype=torch.float16):
        if data.dtype != torch.uint8 or data.dim() != 3:
            raise ValueError("fp8 cache data must be uint8 [num_blocks, heads, tile bytes]")
        if data.shape[2] != block_size * head_dim + 4 * block_size:
            raise ValueError("tile bytes must be block_size*head_dim + 4*block_size")
        if io_dtype not in (torch.float16, torch.bfloat16):
            raise ValueError("io_dtype must be float16 or bfloat16")
        self.data, self.block_size, self.head_dim, self.io_dtype = data, block_size, head_dim, \
            io_dtype

    @classmethod
    def empty(cls, num_blocks, num_heads, block_size, head_dim, io_dtype=torch.float16,
              device="cuda"):
        data = torch.empty(num_blocks, num_heads, block_size * head_dim + 4 * block_size,
                           dtype=torch.uint8, device=device)
        return cls(data, block_size, head_dim, io_dtype)

    def data_ptr(self):
        return self.data.data_ptr()

    def is_contiguous(self):
        return self.data.is_contiguous()

    def is_pinned(self):
        return self.data.is_pinned()

    @property
    def is_cuda(self):
        return self.data.is_cuda

    @property
    def device(self):
        return self.data.device

    @property
    def shape(self):
        return self.data.shape


_P = ctypes.c_void_p
_i32 = ctypes.c_int32
_lib.pa_write_kv.restype = ctypes.c_int
_lib.pa_write_kv.argtypes = [_P, _P, _i32, _i32, _P, _P, _P, ctypes.POINTER(CacheDesc), _P, _P]
_lib.pa_decode_workspace_size.restype = ctypes.c_size_t
_lib.pa_decode_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _i32]
_lib.pa_decode_partition_size.restype = _i32
_lib.pa_decode_partition_size.argtypes = [_i32, _i32, ctypes.POINTER(CacheDesc), _i32, _i32]
_lib.pa_decode.restype = ctypes.c_int
_lib.pa_decode.argtypes = [_P, ctypes.c_int, _P, _i32, _i32, _P, _P, ctypes.POINTER(CacheDesc),
                           _P, _i32, _P, _i32, ctypes.c_float, _i32, _P, ctypes.c_size_t, _P, _P]
_lib.pa_write_kv_decode.restype = ctypes.c_int
_lib.pa_write_kv_decode.argtypes = [_P, ctypes.c_int, _P, _P, _P, _i32, _i32, _P, _P,
                                    ctypes.POINTER(CacheDesc), _P, _i32, _P, _i32,
                                    ctypes.c_float, _i32, _P, ctypes.c_size_t, _P, _P]
_lib.pa_decode_noalloc.restype = ctypes.c_int
_lib.pa_decode_noalloc.argtypes = [_P, ctypes.c_int, _P, _i32, _i32, _P, _P,
                                   ctypes.POINTER(CacheDesc), _P, _i32, _P, _i32,
                                   ctypes.c_float, _i32, _P, _P]
_lib.pa_copy_blocks.restype = ctypes.c_int
_lib.pa_copy_blocks.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(_P), _i32, _P, _i32,
                                ctypes.POINTER(CacheDesc), _P, _P]
_lib.pa_swap_blocks.restype = ctypes.c_int
_lib.pa_swap_blocks.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(CacheDesc),
                                ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(CacheDesc),
                                _i32, _P, _i32, _P, _P]
_lib.pa_selftest_wait_timeout.restype = ctypes.c_int
_lib.pa_selftest_wait_timeout.argtypes = [_P, ctypes.c_uint32, _P]
_lib.pa_status_string.restype = ctypes.c_char_p
_lib.pa_status_string.argtypes = [ctypes.c_int]
_lib.pa_last_error.restype = ctypes.c_char_p
_lib.pa_last_error.argtypes = []
_lib.pa_version.restype = _i32
_lib.pa_version.argtypes = []

SIZE_MAX = ctypes.c_size_t(-1).value


class PagedKVError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_lib.pa_status_string(status).decode()}: {detail}")


def _check(status: int) -> None:
    if status != PA_OK:
        raise PagedKVError(status, _lib.pa_last_error().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def cache_desc(key_cache) -> CacheDesc:
    if isinstance(key_cache, Fp8Cache):
        nb, h, _ = key_cache.data.shape
        return CacheDesc(nb, key_cache.block_size, h, key_cache.head_dim, PA_FP8_E4M3,
                         _DTYPE[key_cache.io_dtype])
    if key_cache.dim() != 4:
        raise ValueError("cache must be [num_blocks, num_heads, block_size, head_dim]")
    nb, h, bs, d = key_cache.shape
    if key_cache.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("cache dtype must be float16 or bfloat16")
    return CacheDesc(nb, bs, h, d, _DTYPE[key_cache.dtype], _DTYPE[key_cache.dtype])


def io_dtype(cache) -> torch.dtype:
    """dtype of the query/key/value rows used with a cache."""
    return cache.io_dtype if isinstance(cache, Fp8Cache) else cache.dtype


def _need(t, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _need_cache(c, name: str, like=None):
    if isinstance(c, Fp8Cache):
        _need(c.data, name)
        if like is not None and (not isinstance(like, Fp8Cache) or c.shape != like.shape):
            raise ValueError(f"{name} does not match the other cache")
        return
    _need(c, name)
    if like is not None and (isinstance(like, Fp8Cache) or c.dtype != like.dtype or
                             c.shape != like.shape):
        raise ValueError(f"{name} does not match the other cache")


def version() -> int:
    return int(_lib.pa_version())


def write_kv(key, value, slot_mapping, key_cache, value_cache, dev_err=None):
    """Store new tokens' K/V ([T, H, D]) at ``slot_mapping`` (int64 [T]) in
    the caches; negative slots are skipped."""
    _need_cache(key_cache, "key_cache")
    _need_cache(value_cache, "value_cache", key_cache)
    for t, n in ((key, "key"), (value, "value")):
        _need(t, n, io_dtype(key_cache))
    _need(slot_mapping, "slot_mapping", torch.int64)
    if key.shape != value.shape:
        raise ValueError("shape mismatch")
    desc = cache_desc(key_cache)
    _check(_lib.pa_write_kv(_ptr(key), _ptr(value), key.shape[0], key.shape[1],
                            _ptr(slot_mapping), _ptr(key_cache), _ptr(value_cache),
                            ctypes.byref(desc), _ptr(dev_err), _stream(key_cache)))


def decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len, partition_size=0):
    n = _lib.pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len,
                                      partition_size)
    if n == SIZE_MAX:
        raise ValueError("invalid arguments to decode_workspace_size")
    return int(n)


def decode_partition_size(num_seqs, num_heads, cache, max_context_len, partition_size=0):
    """``cache``: a key cache (tensor or Fp8Cache) or a CacheDesc."""
    desc = cache if isinstance(cache, CacheDesc) else cache_desc(cache)
    n = _lib.pa_decode_partition_size(num_seqs, num_heads, ctypes.byref(desc),
                                      max_context_len, partition_size)
    if n < 0:
        raise ValueError("invalid arguments to decode_partition_size")
    return int(n)


def alloc_workspace(num_seqs, num_heads, head_dim, max_context_len, partition_size=0,
                    device="cuda"):
    """A decode workspace, zero-filled (its counter region must start at
    zero; every call leaves it so)."""
    n = decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len, partition_size)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def decode(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len,
           scale, partition_size=0, workspace=None, dev_err=None):
    """out[s,h,:] = softmax(scale * q K^T) V over each sequence's cached
    tokens. ``out`` may be fp16, bf16 or fp32; ``workspace`` is allocated
    here when not given."""
    _need_cache(key_cache, "key_cache")
    _need_cache(value_cache, "value_cache", key_cache)
    _need(query, "query", io_dtype(key_cache))
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need(out, "out")
    if out.dtype not in _DTYPE:
        raise ValueError("out dtype must be float16, bfloat16 or float32")
    if out.shape != query.shape:
        raise ValueError("shape mismatch")
    desc = cache_desc(key_cache)
    S, H, D = query.shape
    if workspace is None:
        workspace = alloc_workspace(S, H, D, int(max_context_len), partition_size,
                                    query.device)
    mb = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(_lib.pa_decode(_ptr(out), _DTYPE[out.dtype], _ptr(query), S, H, _ptr(key_cache),
                          _ptr(value_cache), ctypes.byref(desc), _ptr(block_tables), mb,
                          _ptr(context_lens), int(max_context_len), float(scale),
                          int(partition_size), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(dev_err),
                          _stream(query)))
    return out


def write_kv_decode(out, query, key, value, key_cache, value_cache, block_tables,
                    context_lens, max_context_len, scale, partition_size=0, workspace=None,
                    dev_err=None):
    """:func:`write_kv` + :func:`decode` in one launch for a batch where
    every sequence appends one token: ``key``/``value`` [S, H, D] are the new
    rows, stored at position ``context_lens[s] - 1`` of each sequence (the
    slot its block table gives), and attention covers every token including
    them."""
    _need_cache(key_cache, "key_cache")
    _need_cache(value_cache, "value_cache", key_cache)
    _need(query, "query", io_dtype(key_cache))
    _need(key, "key", io_dtype(key_cache))
    _need(value, "value", io_dtype(key_cache))
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need(out, "out")
    if out.dtype not in _DTYPE:
        raise ValueError("out dtype must be float16, bfloat16 or float32")
    if out.shape != query.shape or key.shape != value.shape or key.shape[0] != query.shape[0] \
            or key.shape[2] != query.shape[2]:
        raise ValueError("shape mismatch")
    desc = cache_desc(key_cache)
    S, H, D = query.shape
    if workspace is None:
        workspace = alloc_workspace(S, H, D, int(max_context_len), partition_size,
                                    query.device)
    mb = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(_lib.pa_write_kv_decode(_ptr(out), _DTYPE[out.dtype], _ptr(query), _ptr(key),
                                   _ptr(value), S, H, _ptr(key_cache), _ptr(value_cache),
                                   ctypes.byref(desc), _ptr(block_tables), mb,
                                   _ptr(context_lens), int(max_context_len), float(scale),
                                   int(partition_size), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(),
                                   _ptr(dev_err), _stream(query)))
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def decode_noalloc(out, query, key_cache, value_cache, block_tables, context_lens,
                   max_context_len, scale, partition_size=0, dev_err=None):
    """Like :func:`decode`, for callers that must not allocate device memory
    while decoding (for example an engine that has handed almost all device
    memory to its KV block pool): partial results of split contexts go to a
    fixed 32 MiB array inside the library instead of a workspace. A split
    call first clears the array's arrival counters on the current stream.
    Calls that overlap on the GPU share the array and race (their outputs are
    wrong, with no error); serialised calls are unaffected. The first call on
    a device looks up the array's address and should come before any stream
    capture."""
    _need_cache(key_cache, "key_cache")
    _need_cache(value_cache, "value_cache", key_cache)
    _need(query, "query", io_dtype(key_cache))
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    _need(out, "out")
    if out.dtype not in _DTYPE:
        raise ValueError("out dtype must be float16, bfloat16 or float32")
    if out.shape != query.shape:
        raise ValueError("shape mismatch")
    desc = cache_desc(key_cache)
    S, H, D = query.shape
    mb = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(_lib.pa_decode_noalloc(_ptr(out), _DTYPE[out.dtype], _ptr(query), S, H,
                                  _ptr(key_cache), _ptr(value_cache), ctypes.byref(desc),
                                  _ptr(block_tables), mb, _ptr(context_lens),
                                  int(max_context_len), float(scale), int(partition_size),
                                  _ptr(dev_err), _stream(query)))
    return out


def copy_blocks(key_caches, value_caches, block_mapping, dev_err=None):
    """Copy whole blocks (src, dst) = block_mapping[i] in every layer's K
    and V cache (copy-on-write)."""
    if len(key_caches) != len(value_caches) or not key_caches:
        raise ValueError("need the same, non-zero number of K and V caches")
    _need(block_mapping, "block_mapping", torch.int64)
    for c in list(key_caches) + list(value_caches):
        _need_cache(c, "cache", key_caches[0])
    desc = cache_desc(key_caches[0])
    L = len(key_caches)
    kp = (_P * L)(*[c.data_ptr() for c in key_caches])
    vp = (_P * L)(*[c.data_ptr() for c in value_caches])
    n = block_mapping.shape[0] if block_mapping.numel() else 0
    _check(_lib.pa_copy_blocks(kp, vp, L, _ptr(block_mapping), n, ctypes.byref(desc),
                               _ptr(dev_err), _stream(key_caches[0])))


def swap_blocks(src_key_caches, src_value_caches, dst_key_caches, dst_value_caches,
                block_mapping, dev_err=None):
    """Copy block ``block_mapping[i][0]`` of every source layer's K/V cache to
    block ``block_mapping[i][1]`` of the destination caches. Pools may be CUDA
    tensors or pinned CPU tensors (swap out / swap in); pageable CPU memory
    is refused. Runs on the current CUDA stream."""
    L = len(src_key_caches)
    groups = (src_key_caches, src_value_caches, dst_key_caches, dst_value_caches)
    if L == 0 or any(len(g) != L for g in groups):
        raise ValueError("need the same, non-zero number of caches in every list")
    for g in groups:
        for c in g:
            if not c.is_contiguous():
                raise ValueError("caches must be contiguous")
    if block_mapping.dtype != torch.int64 or not block_mapping.is_contiguous():
        raise ValueError("block_mapping must be a contiguous int64 tensor")
    sd, dd = cache_desc(src_key_caches[0]), cache_desc(dst_key_caches[0])
    arr = lambda cs: (_P * L)(*[c.data_ptr() for c in cs])  # noqa: E731
    n = block_mapping.shape[0] if block_mapping.numel() else 0
    dev = next((c.device for g in groups for c in g if c.is_cuda), None)
    stream = torch.cuda.current_stream(dev).cuda_stream
    _check(_lib.pa_swap_blocks(arr(src_key_caches), arr(src_value_caches), ctypes.byref(sd),
                               arr(dst_key_caches), arr(dst_value_caches), ctypes.byref(dd),
                               L, _ptr(block_mapping), n, _ptr(dev_err), stream))


def selftest_wait_timeout(limit_us: int = 1000, device="cuda") -> int:
    """Run the bounded-wait self-test and return the device error bits it
    produced (PA_DEVERR_TIMEOUT expected)."""
    err = torch.zeros(1, dtype=torch.int32, device=device)
    _check(_lib.pa_selftest_wait_timeout(_ptr(err), int(limit_us),
                                         torch.cuda.current_stream(err.device).cuda_stream))
    torch.cuda.synchronize(err.device)
    return int(err.item())
