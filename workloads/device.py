"""Upload a :class:`~workloads.steps.DecodeStep` to a torch device.

Plumbing only: the pools are assembled from the tile bank with torch indexing,
the tile codes' sign flips and NaN fills, exactly as
:func:`workloads.steps.host_pools` does on the host, so both sides see the same
bytes.
"""
from __future__ import annotations

import numpy as np
import torch

from .steps import DecodeStep, nan_bits

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


def _bits_to_tensor(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(TORCH_DTYPE[dtype]).to(device)


def device_pools(step: DecodeStep, layer: int, device, base_dev=None):
    """Pre-step (key_cache, value_cache) of one layer, [NB, H, bs, D]
    (fp8: uint8 [NB, H, bs*D + 4*bs], built on the host)."""
    bs, H, D = step.block_size, step.num_kv_heads, step.head_dim
    if step.dtype == "fp8":
        from .steps import host_pools
        k, v = host_pools(step, layer)
        return torch.from_numpy(k).to(device), torch.from_numpy(v).to(device)
    if base_dev is None:
        base_dev = _bits_to_tensor(step.base, step.dtype, device)
    L = step.layers[layer]
    nan = torch.tensor([int(nan_bits(step.dtype))], dtype=torch.int32).to(torch.int16)
    nan = nan.view(TORCH_DTYPE[step.dtype]).item()
    valid = torch.from_numpy(step.valid_slots).to(device)
    slot_dead = torch.arange(bs, device=device)[None, :] >= valid[:, None]  # [NB, bs]
    R = step.base.shape[0]
    shifts = torch.arange(bs, device=device, dtype=torch.int64)
    pools = []
    for rows in (L.tile_rows_k, L.tile_rows_v):
        r = torch.from_numpy(rows).to(device)
        code = r.clamp(min=0)
        p = base_dev.index_select(0, (code % R).reshape(-1)).view(step.num_blocks, H, bs, D)
        # Sign flips of the tile code's mask (workloads.steps.tile_parts).
        flips = (((code // R)[..., None] >> shifts) & 1).to(torch.int16) * -32768
        p = (p.view(torch.int16) ^ flips[..., None]).view(p.dtype)
        p.masked_fill_((r < 0)[:, :, None, None], nan)
        p.masked_fill_(slot_dead[:, None, :, None], nan)
        pools.append(p)
    return pools[0], pools[1]


def device_step(step: DecodeStep, device, layers=None):
    """All inputs of a step on ``device`` as a dict of tensors."""
    layers = range(step.num_layers) if layers is None else layers
    base_dev = None if step.dtype == "fp8" else _bits_to_tensor(step.base, step.dtype, device)
    out = {
        "context_lens": torch.from_numpy(step.context_lens).to(device),
        "block_tables": torch.from_numpy(step.block_tables).to(device),
        "slot_mapping": torch.from_numpy(step.slot_mapping).to(device),
        "copy_pairs": torch.from_numpy(step.copy_pairs).to(device),
        "key_caches": [], "value_caches": [], "query": [], "new_key": [],
        "new_value": [],
    }
    for li in layers:
        kc, vc = device_pools(step, li, device, base_dev)
        L = step.layers[li]
        out["key_caches"].append(kc)
        out["value_caches"].append(vc)
        out["query"].append(_bits_to_tensor(L.query, step.io_dtype, device))
        out["new_key"].append(_bits_to_tensor(L.new_key, step.io_dtype, device))
        out["new_value"].append(_bits_to_tensor(L.new_value, step.io_dtype, device))
    del base_dev
    return out
