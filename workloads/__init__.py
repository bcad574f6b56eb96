"""Seeded synthetic inputs for paged decode attention.

Shared by the CUDA path's tests and bench and by the CPU oracle; holds no
attention arithmetic (see :mod:`workloads.steps`).
"""
from .allocator import (BlockAllocator, PoolExhausted, Sequence, allocate_tokens,
                        append_token, check_invariants, free_sequence)
from .steps import (CONFIGS, DecodeStep, LayerInputs, build_step, full_step,
                    fp8_tile_bytes, host_pools, io_dtype_of, kv_bytes_read, llama_layer,
                    long_context, nan_bits, prefix_cow, subset, tiny, to_storage_bits)
