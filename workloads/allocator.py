"""Host-side block allocator used to build decode-step inputs.

This is the bookkeeping half of PagedAttention as the pages describe it:

* The KV cache is cut into fixed-size physical blocks (default 16 tokens)
  that may sit anywhere in the pool ("啃透vLLM源码", §2.2; "vLLM基础", §2.3).
* A physical block carries a reference count so that several sequences can
  share it ("啃透vLLM源码", §2.2, the ``PhysicalTokenBlock`` sketch).
* Each sequence owns a block table that maps logical block ``i`` to a
  physical block id ("vLLM基础", §2.3, the block-table sketch).
* A logical block fills its slots in order, ``num_tokens`` advancing by the
  number of tokens appended ("啃透vLLM源码", §2.2, ``append_tokens``).
* Blocks come from a free list and go back to it when a sequence finishes
  ("vLLM基础", §2.3; "啃透vLLM源码", §3, ``schedule``).
* Copy-on-write: sequences that share a prefix share its physical blocks until
  one of them must write a different token into a shared block; that block is
  then copied ("vLLM基础", §2.3).

The allocator does no attention arithmetic. It only produces the integer
inputs of a decode step: block tables, the slot of each new token and the
(src, dst) pairs that the copy-on-write step must duplicate.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


class PoolExhausted(RuntimeError):
    """Raised when the free list is empty (admission control: the scheduler
    stops admitting work when blocks run out, "啃透vLLM源码", §3)."""


class BlockAllocator:
    """Free list + reference counts over ``num_blocks`` physical blocks.

    ``order`` fixes the order in which free blocks are handed out; the
    workloads pass a seeded permutation so that every sequence's blocks are
    scattered across the pool.
    """

    def __init__(self, num_blocks: int, block_size: int, order=None):
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("num_blocks must be >= 0 and block_size > 0")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if order is None:
            order = np.arange(num_blocks)
        order = np.asarray(order, dtype=np.int64)
        if sorted(order.tolist()) != list(range(num_blocks)):
            raise ValueError("order must be a permutation of range(num_blocks)")
        # Pop from the front: reverse so list.pop() returns order[0] first.
        self._free = [int(b) for b in order[::-1]]
        self.ref_count = np.zeros(num_blocks, dtype=np.int64)

    # -- free list -------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def can_allocate(self, n: int) -> bool:
        return n <= len(self._free)

    def allocate(self) -> int:
        if not self._free:
            raise PoolExhausted("no free physical block left")
        b = self._free.pop()
        assert self.ref_count[b] == 0
        self.ref_count[b] = 1
        return b

    def fork(self, block: int) -> int:
        """Add one more holder of ``block`` (prefix sharing)."""
        if self.ref_count[block] <= 0:
            raise ValueError(f"fork of free block {block}")
        self.ref_count[block] += 1
        return block

    def release(self, block: int) -> None:
        if self.ref_count[block] <= 0:
            raise ValueError(f"release of free block {block}")
        self.ref_count[block] -= 1
        if self.ref_count[block] == 0:
            self._free.append(int(block))

    def free_blocks(self) -> set:
        return set(self._free)


@dataclass
class Sequence:
    """One sequence's block table and token count."""

    block_table: list = field(default_factory=list)
    num_tokens: int = 0


def allocate_tokens(alloc: BlockAllocator, seq: Sequence, n: int) -> None:
    """Reserve room for ``n`` more tokens of ``seq`` (a prompt or a suffix).

    Fills the last logical block first, then takes fresh blocks. Writing into
    a shared block is not allowed here; use :func:`append_token` for that.
    """
    bs = alloc.block_size
    for _ in range(n):
        if seq.num_tokens % bs == 0:
            seq.block_table.append(alloc.allocate())
        else:
            last = seq.block_table[-1]
            if alloc.ref_count[last] > 1:
                raise ValueError("allocate_tokens into a shared block")
        seq.num_tokens += 1


def append_token(alloc: BlockAllocator, seq: Sequence):
    """Append one decode token to ``seq``.

    Returns ``(slot, cow_pair)``: ``slot = block * block_size + offset`` is
    where the new token's K/V go; ``cow_pair`` is ``(src, dst)`` when the
    target block was shared and had to be copied first, else ``None``.
    """
    bs = alloc.block_size
    offset = seq.num_tokens % bs
    pair = None
    if offset == 0:
        seq.block_table.append(alloc.allocate())
    else:
        last = seq.block_table[-1]
        if alloc.ref_count[last] > 1:
            dst = alloc.allocate()
            alloc.release(last)
            seq.block_table[-1] = dst
            pair = (last, dst)
    block = seq.block_table[-1]
    seq.num_tokens += 1
    return block * bs + offset, pair


def free_sequence(alloc: BlockAllocator, seq: Sequence) -> None:
    """Return every block of a finished sequence."""
    for b in seq.block_table:
        alloc.release(b)
    seq.block_table = []
    seq.num_tokens = 0


def check_invariants(alloc: BlockAllocator, seqs, extra_holders=()) -> None:
    """Reference counts equal the number of table references (plus any
    holders outside ``seqs``); the free list and the used blocks are
    disjoint and together cover the pool."""
    counts = np.zeros(alloc.num_blocks, dtype=np.int64)
    for s in seqs:
        for b in s.block_table:
            counts[b] += 1
    for b in extra_holders:
        counts[b] += 1
    if not np.array_equal(counts, alloc.ref_count):
        raise AssertionError("ref_count differs from the number of holders")
    free = alloc.free_blocks()
    used = set(np.nonzero(alloc.ref_count)[0].tolist())
    if free & used:
        raise AssertionError("a block is both free and in use")
    if free | used != set(range(alloc.num_blocks)):
        raise AssertionError("free and used blocks do not cover the pool")
    if len(free) != alloc.num_free:
        raise AssertionError("duplicate entry in the free list")
