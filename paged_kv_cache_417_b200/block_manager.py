"""Python binding of the host block manager (include/pagedkv_block_manager.h).

Marshalling only: the free list, reference counts, block tables and
copy-on-write decisions live in the C++ library.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import PA_OK, PagedKVError, _lib

_P = ctypes.c_void_p
_i32, _i64 = ctypes.c_int32, ctypes.c_int64
_lib.pa_bm_create.restype = _P
_lib.pa_bm_create.argtypes = [_i32, _i32, _P]
_lib.pa_bm_destroy.restype = None
_lib.pa_bm_destroy.argtypes = [_P]
for _n, _a in [("pa_bm_num_free", [_P]), ("pa_bm_can_allocate", [_P, _i32]),
               ("pa_bm_ref_count", [_P, _i32]), ("pa_bm_num_tokens", [_P, _i64]),
               ("pa_bm_block_table", [_P, _i64, _P, _i32])]:
    getattr(_lib, _n).restype = _i32
    getattr(_lib, _n).argtypes = _a
for _n, _a in [("pa_bm_add_sequence", [_P, _i64]), ("pa_bm_allocate_tokens", [_P, _i64, _i32]),
               ("pa_bm_fork", [_P, _i64, _i64]), ("pa_bm_append_token", [_P, _i64, _P, _P, _P]),
               ("pa_bm_free_sequence", [_P, _i64]),
               ("pa_bm_prepare_decode", [_P, _P, _i32, _i32, _P, _P, _P, _P, _P])]:
    getattr(_lib, _n).restype = ctypes.c_int
    getattr(_lib, _n).argtypes = _a


def _check(status):
    if status != PA_OK:
        raise PagedKVError(status, _lib.pa_last_error().decode())


class BlockManager:
    """Free list + reference counts + per-sequence block tables over a pool
    of ``num_blocks`` blocks of ``block_size`` tokens."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.shape != (num_blocks,):
                raise ValueError("free_order must list every block once")
        self._h = _lib.pa_bm_create(num_blocks, block_size,
                                    None if order is None else order.ctypes.data)
        if not self._h:
            raise ValueError("bad pool arguments (or free_order is not a permutation)")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            _lib.pa_bm_destroy(h)
            self._h = None

    @property
    def num_free(self) -> int:
        return _lib.pa_bm_num_free(self._h)

    def can_allocate(self, n: int) -> bool:
        return bool(_lib.pa_bm_can_allocate(self._h, n))

    def ref_count(self, block: int) -> int:
        return _lib.pa_bm_ref_count(self._h, block)

    def ref_counts(self) -> np.ndarray:
        return np.array([self.ref_count(b) for b in range(self.num_blocks)], dtype=np.int64)

    def add_sequence(self, seq: int) -> None:
        _check(_lib.pa_bm_add_sequence(self._h, seq))

    def allocate_tokens(self, seq: int, n: int) -> None:
        _check(_lib.pa_bm_allocate_tokens(self._h, seq, n))

    def fork(self, parent: int, child: int) -> None:
        _check(_lib.pa_bm_fork(self._h, parent, child))

    def append_token(self, seq: int):
        """Returns (slot, (src, dst) or None)."""
        slot, src, dst = _i64(), _i64(), _i64()
        _check(_lib.pa_bm_append_token(self._h, seq, ctypes.byref(slot), ctypes.byref(src),
                                       ctypes.byref(dst)))
        return slot.value, (None if src.value < 0 else (src.value, dst.value))

    def free_sequence(self, seq: int) -> None:
        _check(_lib.pa_bm_free_sequence(self._h, seq))

    def num_tokens(self, seq: int) -> int:
        return _lib.pa_bm_num_tokens(self._h, seq)

    def block_table(self, seq: int) -> list:
        n = _lib.pa_bm_block_table(self._h, seq, None, 0)
        if n < 0:
            raise KeyError(seq)
        out = np.zeros(max(n, 1), dtype=np.int32)
        _lib.pa_bm_block_table(self._h, seq, out.ctypes.data, n)
        return out[:n].tolist()

    def prepare_decode(self, seqs, max_blocks_per_seq: int) -> dict:
        """Append one token to each of ``seqs`` and return the decode step's
        inputs: block_tables, context_lens, slot_mapping, copy_pairs."""
        ids = np.ascontiguousarray(seqs, dtype=np.int64)
        n = ids.shape[0]
        bt = np.empty((n, max_blocks_per_seq), dtype=np.int32)
        ctx = np.empty(n, dtype=np.int32)
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        npairs = _i32()
        _check(_lib.pa_bm_prepare_decode(self._h, ids.ctypes.data, n, max_blocks_per_seq,
                                         bt.ctypes.data, ctx.ctypes.data, slots.ctypes.data,
                                         pairs.ctypes.data, ctypes.byref(npairs)))
        return {"block_tables": bt, "context_lens": ctx, "slot_mapping": slots,
                "copy_pairs": pairs[:npairs.value].copy()}
