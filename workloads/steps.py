"""Seeded synthetic decode-step inputs.

A *decode step* is what one iteration of the engine does to the KV cache of a
batch of running sequences ("vLLM基础", §2.2, steps 4-6): every sequence gets
one new token, whose K/V are written into the slot its block table assigns,
after copy-on-write has duplicated any shared block that the write would touch
("vLLM基础", §2.3); then attention runs for one query token per sequence over
all of its context, the new token included.

This module only draws numbers and builds integer tables. It holds none of the
attention arithmetic, so it can feed both the CUDA path and the CPU oracle.

Cache contents are stored compactly: every (block, head) tile of a pool is a
row of a bank ``base`` of N(0,1) tiles (drawn in fp32, rounded to the storage
type), named by a tile code. Small pools get a distinct bank row per tile.
Large pools use a 32768-row bank, which keeps generation fast, and give every
tile a distinct code (bank row, sign mask): the tile is the bank row with the
sign of its token row r flipped where bit r of the mask is set (fp8: the code
bytes' sign bit; the row scales stay). A sign flip is exact in every storage
format and keeps every element an N(0,1) draw, and no two tiles of a pool hold
the same values, so a kernel that reads the wrong tile cannot land on equal
contents. Unused blocks, and slots past the last token of a partly filled
block, hold NaN so that any read of them shows up.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

from .allocator import BlockAllocator, Sequence, allocate_tokens, append_token

F16_NAN = np.uint16(0x7E00)
BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)
F32_NAN_BYTES = np.array([np.nan], dtype=np.float32).view(np.uint8)
MAX_BANK_ROWS = 32768


MASK_BITS = 16  # token rows of a tile whose sign a tile code can flip


def tile_parts(codes: np.ndarray, bank_rows: int, block_size: int):
    """Split tile codes (>= 0) into bank rows and per-token-row sign flips:
    code = mask * bank_rows + row; flips[..., r] = bit r of mask."""
    codes = np.asarray(codes, dtype=np.int64)
    rows = codes % bank_rows
    mask = codes // bank_rows
    flips = (mask[..., None] >> np.arange(block_size, dtype=np.int64)) & 1
    return rows, flips.astype(bool)


def _distinct_codes(rng, n: int, bank_rows: int, block_size: int) -> np.ndarray:
    """n distinct tile codes: bank rows with sign masks, drawn uniformly."""
    space = bank_rows << min(block_size, MASK_BITS)
    codes = rng.integers(0, space, size=n)
    while True:
        uniq, first = np.unique(codes, return_index=True)
        if len(uniq) == n:
            return codes
        dup = np.ones(n, dtype=bool)
        dup[first] = False
        codes[dup] = rng.integers(0, space, size=int(dup.sum()))


def fp8_tile_bytes(block_size: int, head_dim: int) -> int:
    """Bytes of one (block, head) tile of an fp8 pool: block_size rows of
    head_dim e4m3 codes, then block_size fp32 row scales."""
    return block_size * head_dim + 4 * block_size


def to_storage_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to fp16 or bf16 (round to nearest even) and return
    the raw 16-bit patterns as uint16."""
    x = np.asarray(x, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        u = x.view(np.uint32).astype(np.uint64)
        u = u + 0x7FFF + ((u >> 16) & 1)
        out = (u >> 16).astype(np.uint16)
        out[np.isnan(x)] = BF16_NAN
        return out
    raise ValueError(f"unknown dtype {dtype!r}")


def nan_bits(dtype: str) -> np.uint16:
    return F16_NAN if dtype == "f16" else BF16_NAN


def io_dtype_of(dtype: str) -> str:
    """The dtype of query/key/value rows: the cache's own for 16-bit caches,
    fp16 for fp8 caches."""
    return "f16" if dtype == "fp8" else dtype


@dataclass
class LayerInputs:
    query: np.ndarray       # uint16 [S, H, D]
    new_key: np.ndarray     # uint16 [S, H, D]
    new_value: np.ndarray   # uint16 [S, H, D]
    tile_rows_k: np.ndarray  # int64 [NB, Hkv], tile code (see tile_parts) or -1 (NaN tile)
    tile_rows_v: np.ndarray  # int64 [NB, Hkv]


@dataclass
class DecodeStep:
    name: str
    num_seqs: int
    num_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str
    scale: np.float32
    context_lens: np.ndarray   # int32 [S], after the new token is appended
    block_tables: np.ndarray   # int32 [S, MB], -1 past each table's end
    slot_mapping: np.ndarray   # int64 [S], slot of each new token
    copy_pairs: np.ndarray     # int64 [N, 2], (src, dst) to copy before writing
    valid_slots: np.ndarray    # int32 [NB], filled slots per block before the step
    base: np.ndarray           # uint16 [R, bs*D] tile bank (fp8: uint8 [R, tile bytes])
    layers: list = field(default_factory=list)
    ref_count: np.ndarray = None  # int64 [NB], after the step
    meta: dict = field(default_factory=dict)
    num_kv_heads: int = 0      # K/V heads (0: same as num_heads)

    def __post_init__(self):
        if not self.num_kv_heads:
            self.num_kv_heads = self.num_heads

    @property
    def num_layers(self) -> int:
        return len(self.layers)

    @property
    def io_dtype(self) -> str:
        return io_dtype_of(self.dtype)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0


def _draw_bits(rng, shape, dtype):
    return to_storage_bits(rng.standard_normal(shape, dtype=np.float32), dtype)


def _draw_fp8_tiles(rng, rows, block_size, head_dim):
    """fp8 tiles: codes uniform over the finite e4m3 codes (0x7F and 0xFF
    are NaN), then one positive fp32 scale per row."""
    codes = rng.integers(0, 254, size=(rows, block_size * head_dim), dtype=np.uint16)
    codes = np.where(codes >= 0x7F, codes + 1, codes).astype(np.uint8)   # skip 0x7F
    scales = rng.uniform(0.002, 0.008, size=(rows, block_size)).astype(np.float32)
    return np.concatenate([codes, scales.view(np.uint8)], axis=1)


def build_step(rng, name, *, num_blocks, block_size, num_heads, head_dim,
               pre_tokens, num_layers=1, scale=None, dtype="f16",
               prefix_tokens=0, fork_partial_tail=False, order=None, num_kv_heads=None):
    """Build one decode step.

    ``pre_tokens[s]`` tokens of sequence ``s`` are in the cache before the
    step; the step appends one. With ``prefix_tokens > 0`` every sequence
    starts with the same ``prefix_tokens`` tokens held in shared blocks (one
    physical copy, ref_count = number of sequences) and ``pre_tokens`` counts
    the private suffix. ``fork_partial_tail`` gives each sequence's partly
    filled last block a second holder (a forked sibling that is not decoded),
    so appending into it triggers copy-on-write.
    """
    if dtype not in ("f16", "bf16", "fp8"):
        raise ValueError(dtype)
    bs, H, D = int(block_size), int(num_heads), int(head_dim)
    Hk = int(num_kv_heads or num_heads)
    if H % Hk:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    S = len(pre_tokens)
    if order is None:
        order = rng.permutation(num_blocks)
    alloc = BlockAllocator(num_blocks, bs, order)
    seqs = [Sequence() for _ in range(S)]
    if prefix_tokens:
        if prefix_tokens % bs:
            raise ValueError("prefix_tokens must fill whole blocks")
        if S:
            allocate_tokens(alloc, seqs[0], prefix_tokens)
            for s in seqs[1:]:
                s.block_table = [alloc.fork(b) for b in seqs[0].block_table]
                s.num_tokens = prefix_tokens
    for s, n in zip(seqs, pre_tokens):
        allocate_tokens(alloc, s, int(n))
    phantom = []
    if fork_partial_tail:
        for s in seqs:
            if s.num_tokens % bs:
                phantom.append(alloc.fork(s.block_table[-1]))
    # Filled slots per block before the step.
    valid = np.zeros(num_blocks, dtype=np.int32)
    for s in seqs:
        for i, b in enumerate(s.block_table):
            valid[b] = min(bs, s.num_tokens - i * bs)
    slots, pairs = [], []
    for s in seqs:
        slot, pair = append_token(alloc, s)
        slots.append(slot)
        if pair is not None:
            pairs.append(pair)

    ctx = np.array([s.num_tokens for s in seqs], dtype=np.int32)
    mb = max(1, max((len(s.block_table) for s in seqs), default=1))
    bt = np.full((S, mb), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        bt[i, : len(s.block_table)] = s.block_table

    # Tile bank: a distinct row per filled tile when that fits the bank,
    # else rows drawn with replacement.
    filled = np.nonzero(valid > 0)[0]
    n_tiles = 2 * len(filled) * Hk
    rows = max(1, min(n_tiles, MAX_BANK_ROWS))
    if dtype == "fp8":
        base = _draw_fp8_tiles(rng, rows, bs, D)
    else:
        base = _draw_bits(rng, (rows, bs * D), dtype)
    io = io_dtype_of(dtype)
    layers = []
    for _ in range(num_layers):
        if n_tiles <= rows:
            pick = rng.permutation(rows)[:n_tiles] if n_tiles else np.zeros(0, np.int64)
        else:
            pick = _distinct_codes(rng, n_tiles, rows, bs)
        pick = pick.astype(np.int64).reshape(2, len(filled), Hk) if n_tiles else \
            np.zeros((2, 0, Hk), np.int64)
        tk = np.full((num_blocks, Hk), -1, dtype=np.int64)
        tv = np.full((num_blocks, Hk), -1, dtype=np.int64)
        tk[filled] = pick[0]
        tv[filled] = pick[1]
        layers.append(LayerInputs(
            query=_draw_bits(rng, (S, H, D), io),
            new_key=_draw_bits(rng, (S, Hk, D), io),
            new_value=_draw_bits(rng, (S, Hk, D), io),
            tile_rows_k=tk, tile_rows_v=tv))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    step = DecodeStep(
        name=name, num_seqs=S, num_heads=H, head_dim=D, block_size=bs,
        num_blocks=num_blocks, dtype=dtype, scale=np.float32(scale),
        context_lens=ctx, block_tables=bt,
        slot_mapping=np.array(slots, dtype=np.int64),
        copy_pairs=np.array(pairs, dtype=np.int64).reshape(-1, 2),
        valid_slots=valid, base=base, layers=layers,
        ref_count=alloc.ref_count.copy(),
        meta={"allocator": alloc, "seqs": seqs, "phantom_holders": phantom,
              "prefix_tokens": prefix_tokens,
              # The allocation history, for replaying the same step on
              # another block manager: free order, cached tokens per
              # sequence (the suffix when there is a shared prefix), and
              # whether each partly filled last block has a second holder.
              "free_order": np.asarray(order, dtype=np.int64).copy(),
              "pre_tokens": np.asarray(pre_tokens, dtype=np.int64).copy(),
              "fork_partial_tail": bool(fork_partial_tail)}, num_kv_heads=Hk)
    return step


# ---------------------------------------------------------------------------
# The five workloads. Each takes its sizes as keyword arguments so that the
# parity tests can run the same recipe at sizes the oracle finishes quickly.
# ---------------------------------------------------------------------------

def tiny(seed=0, dtype="f16", context_lens=(1, 17, 33, 100)):
    """1 layer, 4 sequences, 4 heads, head_dim 64, block_size 16, pool of 64
    blocks, scale 1/sqrt(64)."""
    rng = np.random.default_rng(seed)
    pre = [c - 1 for c in context_lens]
    return build_step(rng, "tiny", num_blocks=64, block_size=16, num_heads=4,
                      head_dim=64, pre_tokens=pre, scale=0.125, dtype=dtype)


def llama_layer(seed=1, dtype="f16", num_seqs=96, ctx_range=(128, 2048),
                num_blocks=8192, num_heads=32, head_dim=128, block_size=16, num_kv_heads=None):
    """Llama-7B-shaped single-layer decode: 96 sequences, 32 heads,
    head_dim 128, block_size 16, context_lens uniform in [128, 2048], block
    ids from a seeded shuffle of an 8192-block pool."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(ctx_range[0], ctx_range[1] + 1, size=num_seqs)
    return build_step(rng, "llama7b_layer_b%d" % num_seqs, num_blocks=num_blocks,
                      block_size=block_size, num_heads=num_heads, head_dim=head_dim,
                      pre_tokens=ctx - 1, dtype=dtype, num_kv_heads=num_kv_heads)


def long_context(seed=2, dtype="f16", num_seqs=8, ctx_range=(16384, 32768),
                 num_blocks=20000, num_heads=32, head_dim=128, block_size=16):
    """8 sequences with 16k-32k tokens of context scattered over a 20000-block
    pool: the split-context path."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(ctx_range[0], ctx_range[1] + 1, size=num_seqs)
    return build_step(rng, "long_context_s%d" % num_seqs, num_blocks=num_blocks,
                      block_size=block_size, num_heads=num_heads, head_dim=head_dim,
                      pre_tokens=ctx - 1, dtype=dtype)


def prefix_cow(seed=3, dtype="f16", num_seqs=64, prefix_tokens=1024,
               suffix_range=(1, 512), num_heads=32, head_dim=128, block_size=16,
               num_blocks=None):
    """64 sequences sharing a 1024-token prefix (64 physical blocks,
    ref_count 64) plus private suffixes of 1-512 tokens. Each partly filled
    suffix block is also held by a forked sibling, so appending one token
    copies it first (copy-on-write)."""
    rng = np.random.default_rng(seed)
    suffix = rng.integers(suffix_range[0], suffix_range[1] + 1, size=num_seqs)
    if num_blocks is None:
        need = prefix_tokens // block_size + int(np.sum(-(-suffix // block_size))) \
            + 2 * num_seqs
        num_blocks = int(math.ceil(need * 1.25))
    return build_step(rng, "prefix_cow_s%d" % num_seqs, num_blocks=num_blocks,
                      block_size=block_size, num_heads=num_heads, head_dim=head_dim,
                      pre_tokens=suffix, prefix_tokens=prefix_tokens,
                      fork_partial_tail=True, dtype=dtype)


def full_step(seed=4, dtype="f16", block_size=16, num_seqs=256, num_layers=32,
              mean_ctx=300, max_ctx=4096, num_heads=32, head_dim=128, num_kv_heads=None):
    """All layers of a Llama-7B-shaped cache for 256 sequences whose
    context_lens are geometric with mean 300, capped at 4096. The block
    tables are shared by all layers; each layer has its own pool."""
    rng = np.random.default_rng(seed)
    ctx = np.minimum(rng.geometric(1.0 / mean_ctx, size=num_seqs), max_ctx)
    need = int(np.sum(-(-ctx // block_size)))
    num_blocks = int(math.ceil(need * 1.25)) + 1
    return build_step(rng, "full_step_bs%d" % block_size, num_blocks=num_blocks,
                      block_size=block_size, num_heads=num_heads, head_dim=head_dim,
                      pre_tokens=ctx - 1, num_layers=num_layers, dtype=dtype,
                      num_kv_heads=num_kv_heads)


CONFIGS = {
    "tiny": tiny,
    "llama7b_layer": llama_layer,
    "long_context": long_context,
    "prefix_cow": prefix_cow,
    "full_step": full_step,
}


# ---------------------------------------------------------------------------
# Materialising pools on the host and taking sub-batches.
# ---------------------------------------------------------------------------

def host_pools(step: DecodeStep, layer: int = 0):
    """Return the pre-step (key_pool, value_pool) of one layer as uint16
    arrays [NB, H, bs, D] (fp8: uint8 [NB, H, bs*D + 4*bs])."""
    bs, H, D = step.block_size, step.num_kv_heads, step.head_dim
    L = step.layers[layer]
    if step.dtype == "fp8":
        return _host_pools_fp8(step, L)
    nan = nan_bits(step.dtype)
    R = step.base.shape[0]
    pools = []
    for rows in (L.tile_rows_k, L.tile_rows_v):
        bank_row, flips = tile_parts(np.maximum(rows, 0), R, bs)
        p = step.base[bank_row.reshape(-1)].reshape(step.num_blocks, H, bs, D).copy()
        p ^= np.where(flips, np.uint16(0x8000), np.uint16(0))[..., None]
        p[rows < 0] = nan
        mask = np.arange(bs)[None, :] >= step.valid_slots[:, None]
        p.transpose(0, 2, 1, 3)[mask] = nan
        pools.append(p)
    return pools[0], pools[1]


def _host_pools_fp8(step, L):
    bs, H, D = step.block_size, step.num_kv_heads, step.head_dim
    tb = fp8_tile_bytes(bs, D)
    dead = np.arange(bs)[None, :] >= step.valid_slots[:, None]          # [NB, bs]
    R = step.base.shape[0]
    pools = []
    for rows in (L.tile_rows_k, L.tile_rows_v):
        bank_row, flips = tile_parts(np.maximum(rows, 0), R, bs)
        p = step.base[bank_row.reshape(-1)].reshape(step.num_blocks, H, tb).copy()
        codes = p[:, :, : bs * D].reshape(step.num_blocks, H, bs, D)
        codes ^= np.where(flips, np.uint8(0x80), np.uint8(0))[..., None]
        p[rows < 0] = E4M3_NAN
        scales = p[:, :, bs * D:].reshape(step.num_blocks, H, bs, 4)
        codes.transpose(0, 2, 1, 3)[dead] = E4M3_NAN
        scales.transpose(0, 2, 1, 3)[dead] = F32_NAN_BYTES
        for b in np.nonzero((rows < 0).any(axis=1))[0]:
            scales[b][rows[b] < 0] = F32_NAN_BYTES
        pools.append(p)
    return pools[0], pools[1]


def subset(step: DecodeStep, seq_ids) -> DecodeStep:
    """A smaller step with only ``seq_ids``: the blocks they reference (and the
    sources of their copy-on-write pairs) renumbered 0..n-1, same contents.
    The outputs of the sub-step for sequence ``k`` equal the outputs of the
    full step for ``seq_ids[k]``."""
    seq_ids = np.asarray(seq_ids, dtype=np.int64)
    bs = step.block_size
    bt = step.block_tables[seq_ids]
    ref = set(int(b) for b in bt.reshape(-1) if b >= 0)
    pairs = [tuple(p) for p in step.copy_pairs.tolist() if p[1] in ref]
    blocks = sorted(ref | {p[0] for p in pairs})
    remap = np.full(step.num_blocks, -1, dtype=np.int64)
    remap[blocks] = np.arange(len(blocks))
    new_bt = np.where(bt >= 0, remap[np.maximum(bt, 0)], -1).astype(np.int32)
    used_cols = max(1, int(np.max(np.sum(new_bt >= 0, axis=1), initial=1)))
    new_bt = new_bt[:, :used_cols]
    slots = step.slot_mapping[seq_ids]
    new_slots = np.where(slots >= 0, remap[slots // bs] * bs + slots % bs, slots)
    new_pairs = np.array([(remap[a], remap[b]) for a, b in pairs],
                         dtype=np.int64).reshape(-1, 2)
    layers = [LayerInputs(query=L.query[seq_ids], new_key=L.new_key[seq_ids],
                          new_value=L.new_value[seq_ids],
                          tile_rows_k=L.tile_rows_k[blocks],
                          tile_rows_v=L.tile_rows_v[blocks]) for L in step.layers]
    return DecodeStep(
        name=step.name + "_subset", num_seqs=len(seq_ids), num_heads=step.num_heads,
        head_dim=step.head_dim, block_size=bs, num_blocks=len(blocks),
        dtype=step.dtype, scale=step.scale,
        context_lens=step.context_lens[seq_ids].copy(), block_tables=new_bt,
        slot_mapping=new_slots.astype(np.int64), copy_pairs=new_pairs,
        valid_slots=step.valid_slots[blocks].copy(), base=step.base, layers=layers,
        ref_count=None, meta={"parent": step.name, "seq_ids": seq_ids},
        num_kv_heads=step.num_kv_heads)


def kv_bytes_read(step: DecodeStep) -> int:
    """K/V bytes one decode over every sequence of one layer must read:
    context_len tokens x heads x 2 (K and V) x the bytes of a row (head_dim
    x 2 for 16-bit caches; head_dim codes + a 4-byte scale for fp8)."""
    per_row = step.head_dim + 4 if step.dtype == "fp8" else step.head_dim * 2
    return int(np.sum(step.context_lens.astype(np.int64))) * step.num_kv_heads * per_row * 2
