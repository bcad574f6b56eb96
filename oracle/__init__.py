"""CPU oracle for one decode step of paged attention (fp64, plain C).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline use it; the product path never imports it. It shares no code with
the CUDA library; the two meet only in the seeded inputs of :mod:`workloads`.

Functions and the passages they follow:

* :func:`write_kv` - each new token's K/V go to the slot the block table
  assigns ("vLLM基础", §2.2 steps 4-6; "啃透vLLM源码", §2.2 append_tokens).
* :func:`copy_blocks` - copy-on-write duplication of shared blocks
  ("vLLM基础", §2.3).
* :func:`swap_blocks` - blocks moved between a GPU pool and a host pool
  ("啃透vLLM源码", §3, swap out / swap in).
* :func:`decode` - attention over the cache reached through physical block
  indices ("VLLM源码解析", core technology: paged_attention_forward); exact
  attention, gathered then evaluated with the textbook softmax in fp64.
* :func:`kv_cache_bytes` - the per-sequence K/V sizing ("vLLM基础", §2.3).
* :func:`write_kv_fp8`, :func:`decode_fp8` - the same write and decode on an
  fp8 (e4m3) cache with one fp32 scale per row (KV-cache quantisation, named
  by "vLLM基础", §2.5 as further tuning; the format is a reading).

Pinned by ``tests/test_oracle_pins.py`` (closed forms, brute force in 50-digit
decimal arithmetic, dense attention through scipy's softmax on the unpaged
copy, permutation invariance, the pages' worked sizing figures and
block-table sketch).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_DT = {"f16": 0, "bf16": 1}


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected raw 16-bit patterns (uint16)")
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes front end of one build of oracle.c (the default build, or a
    copy with a planted mistake in the tests)."""

    def __init__(self, path):
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_decode.restype = ctypes.c_int
        L.oracle_decode.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.c_int32, P, P, ctypes.c_int64, ctypes.c_int32,
                                    ctypes.c_int, P, ctypes.c_int32, P, ctypes.c_double,
                                    ctypes.c_int]
        L.oracle_write_kv.restype = ctypes.c_int
        L.oracle_write_kv.argtypes = [P, P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                      P, P, P, ctypes.c_int64, ctypes.c_int32]
        L.oracle_copy_blocks.restype = ctypes.c_int
        L.oracle_copy_blocks.argtypes = [ctypes.POINTER(P), ctypes.POINTER(P), ctypes.c_int32,
                                         P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_swap_blocks.restype = ctypes.c_int
        L.oracle_swap_blocks.argtypes = [ctypes.POINTER(P), ctypes.POINTER(P), ctypes.c_int64,
                                         ctypes.POINTER(P), ctypes.POINTER(P), ctypes.c_int64,
                                         ctypes.c_int32, P, ctypes.c_int64, ctypes.c_int64]
        L.oracle_write_kv_fp8.restype = ctypes.c_int
        L.oracle_write_kv_fp8.argtypes = [P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int32,
                                          ctypes.c_int32, P, P, P, ctypes.c_int64,
                                          ctypes.c_int32]
        L.oracle_decode_fp8.restype = ctypes.c_int
        L.oracle_decode_fp8.argtypes = [P, P, ctypes.c_int, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_int64,
                                        ctypes.c_int32, P, ctypes.c_int32, P, ctypes.c_double,
                                        ctypes.c_int]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_kv_cache_bytes.restype = ctypes.c_int64
        L.oracle_kv_cache_bytes.argtypes = [ctypes.c_int64] * 5
        L.oracle_widen.restype = ctypes.c_double
        L.oracle_widen.argtypes = [ctypes.c_uint16, ctypes.c_int]
        L.oracle_num_threads.restype = ctypes.c_int
        self.lib = L
        self.path = path

    def widen(self, bits: int, dtype: str = "f16") -> float:
        return self.lib.oracle_widen(int(bits), _DT[dtype])

    def kv_cache_bytes(self, layers, tokens, heads, head_dim, elem_bytes) -> int:
        return int(self.lib.oracle_kv_cache_bytes(layers, tokens, heads, head_dim,
                                                  elem_bytes))

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def write_kv(self, key, value, slot_mapping, key_cache, value_cache, block_size):
        """In place on ``key_cache``/``value_cache`` (uint16 [NB, H, bs, D])."""
        key, value = _u16(key), _u16(value)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        T, H, D = key.shape
        assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
        assert key_cache.dtype == np.uint16 and value_cache.dtype == np.uint16
        rc = self.lib.oracle_write_kv(_ptr(key), _ptr(value), T, H, D, _ptr(slots),
                                      _ptr(key_cache), _ptr(value_cache),
                                      key_cache.shape[0], block_size)
        if rc:
            raise ValueError("oracle_write_kv: slot outside the pool")

    def copy_blocks(self, key_caches, value_caches, mapping):
        """In place on every layer's pools; mapping int64 [N, 2] = (src, dst)."""
        mapping = np.ascontiguousarray(mapping, dtype=np.int64).reshape(-1, 2)
        L = len(key_caches)
        if L == 0:
            return
        nb = key_caches[0].shape[0]
        elems = int(np.prod(key_caches[0].shape[1:]))
        for c in list(key_caches) + list(value_caches):
            assert c.flags.c_contiguous and c.dtype == np.uint16 and c.shape[0] == nb
        kp = (ctypes.c_void_p * L)(*[c.ctypes.data for c in key_caches])
        vp = (ctypes.c_void_p * L)(*[c.ctypes.data for c in value_caches])
        rc = self.lib.oracle_copy_blocks(kp, vp, L, _ptr(mapping), mapping.shape[0], nb,
                                         elems)
        if rc:
            raise ValueError("oracle_copy_blocks: block id outside the pool")

    def swap_blocks(self, src_keys, src_values, dst_keys, dst_values, mapping):
        """In place on the destination pools; mapping int64 [N, 2] =
        (source block, destination block)."""
        mapping = np.ascontiguousarray(mapping, dtype=np.int64).reshape(-1, 2)
        L = len(src_keys)
        if L == 0:
            return
        elems = int(np.prod(src_keys[0].shape[1:]))
        for c in list(src_keys) + list(src_values) + list(dst_keys) + list(dst_values):
            assert c.flags.c_contiguous and c.dtype == np.uint16
            assert int(np.prod(c.shape[1:])) == elems
        arr = lambda cs: (ctypes.c_void_p * L)(*[c.ctypes.data for c in cs])  # noqa: E731
        rc = self.lib.oracle_swap_blocks(arr(src_keys), arr(src_values), src_keys[0].shape[0],
                                         arr(dst_keys), arr(dst_values), dst_keys[0].shape[0],
                                         L, _ptr(mapping), mapping.shape[0], elems)
        if rc:
            raise ValueError("oracle_swap_blocks: block id outside its pool")

    def e4m3_decode(self, code: int) -> float:
        return self.lib.oracle_e4m3_decode(int(code))

    def e4m3_encode(self, x: float) -> int:
        return int(self.lib.oracle_e4m3_encode(float(x)))

    def write_kv_fp8(self, key, value, slot_mapping, key_cache, value_cache, block_size,
                     io_dtype="f16"):
        """Quantise new tokens into fp8 pools (uint8 [NB, H, bs*D + 4*bs])."""
        key, value = _u16(key), _u16(value)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        T, H, D = key.shape
        for c in (key_cache, value_cache):
            assert c.flags.c_contiguous and c.dtype == np.uint8
            assert c.shape[1:] == (H, block_size * D + 4 * block_size)
        rc = self.lib.oracle_write_kv_fp8(_ptr(key), _ptr(value), _DT[io_dtype], T, H, D,
                                          _ptr(slots), _ptr(key_cache), _ptr(value_cache),
                                          key_cache.shape[0], block_size)
        if rc:
            raise ValueError("oracle_write_kv_fp8: slot outside the pool")

    def decode_fp8(self, query, key_cache, value_cache, block_tables, context_lens, scale,
                   block_size, io_dtype="f16", threads=0):
        query = _u16(query)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = query.shape
        Hk = key_cache.shape[1]
        assert key_cache.dtype == np.uint8 and value_cache.shape == key_cache.shape
        assert key_cache.shape[2] == block_size * D + 4 * block_size and H % Hk == 0
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self.lib.oracle_decode_fp8(_ptr(out), _ptr(query), _DT[io_dtype], S, H, Hk, D,
                                        _ptr(np.ascontiguousarray(key_cache)),
                                        _ptr(np.ascontiguousarray(value_cache)),
                                        key_cache.shape[0], block_size, _ptr(bt), bt.shape[1],
                                        _ptr(ctx), float(scale), int(threads))
        if rc:
            raise ValueError("oracle_decode_fp8: block id or context length outside the pool")
        return out

    def decode(self, query, key_cache, value_cache, block_tables, context_lens, scale,
               dtype="f16", threads=0):
        """fp64 [S, H, D] attention output."""
        query = _u16(query)
        key_cache, value_cache = _u16(key_cache), _u16(value_cache)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, H, D = query.shape
        NB, Hk, bs, Dc = key_cache.shape
        assert Dc == D and H % Hk == 0 and value_cache.shape == key_cache.shape
        assert bt.ndim == 2 and bt.shape[0] == S and ctx.shape == (S,)
        out = np.zeros((S, H, D), dtype=np.float64)
        rc = self.lib.oracle_decode(_ptr(out), _ptr(query), S, H, Hk, D, _ptr(key_cache),
                                    _ptr(value_cache), NB, bs, _DT[dtype], _ptr(bt),
                                    bt.shape[1], _ptr(ctx), float(scale), int(threads))
        if rc:
            raise ValueError("oracle_decode: block id or context length outside the pool")
        return out

    def step_on_pools(self, step, layer, kc, vc, threads=0):
        """Copy-on-write, write the new tokens, decode: one layer of a
        :class:`workloads.DecodeStep` on the given host pools (in place).
        Returns the fp64 output [S, H, D]."""
        L = step.layers[layer]
        if step.dtype == "fp8":
            # Whole-block copies are byte copies: view the pools as 16-bit.
            k16 = kc.reshape(kc.shape[0], -1).view(np.uint16)
            v16 = vc.reshape(vc.shape[0], -1).view(np.uint16)
            self.copy_blocks([k16], [v16], step.copy_pairs)
            self.write_kv_fp8(L.new_key, L.new_value, step.slot_mapping, kc, vc,
                              step.block_size, step.io_dtype)
            return self.decode_fp8(L.query, kc, vc, step.block_tables, step.context_lens,
                                   float(step.scale), step.block_size, step.io_dtype, threads)
        self.copy_blocks([kc], [vc], step.copy_pairs)
        self.write_kv(L.new_key, L.new_value, step.slot_mapping, kc, vc, step.block_size)
        return self.decode(L.query, kc, vc, step.block_tables, step.context_lens,
                           float(step.scale), step.dtype, threads)

    def run_step(self, step, layer=0, threads=0):
        """The whole step on the host for one layer of a
        :class:`workloads.DecodeStep`: copy-on-write, write the new tokens,
        then decode. Returns (out fp64 [S,H,D], key_pool, value_pool), the
        pools in their post-step state."""
        from workloads import host_pools
        kc, vc = host_pools(step, layer)
        out = self.step_on_pools(step, layer, kc, vc, threads)
        return out, kc, vc


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def widen(bits, dtype="f16"):
    return default().widen(bits, dtype)


def kv_cache_bytes(layers, tokens, heads, head_dim, elem_bytes):
    return default().kv_cache_bytes(layers, tokens, heads, head_dim, elem_bytes)


def num_threads():
    return default().num_threads()


def write_kv(*a, **k):
    return default().write_kv(*a, **k)


def copy_blocks(*a, **k):
    return default().copy_blocks(*a, **k)


def decode(*a, **k):
    return default().decode(*a, **k)


def swap_blocks(*a, **k):
    return default().swap_blocks(*a, **k)


def write_kv_fp8(*a, **k):
    return default().write_kv_fp8(*a, **k)


def decode_fp8(*a, **k):
    return default().decode_fp8(*a, **k)


def run_step(*a, **k):
    return default().run_step(*a, **k)
