// cache_ops.cuh - the two cache-maintenance kernels of a decode step.
//
// write_kv_kernel: store each new token's K and V in the slot its block table
// gives it ("vLLM基础", §2.2 steps 4-6; the in-order slot fill of
// "啃透vLLM源码", §2.2 append_tokens). One CTA per token; every head's row
// is head_dim * 2 bytes, moved as 16-byte vectors.
//
// swap_blocks_kernel: whole blocks between two pool sets of one block shape,
// typically a GPU pool and a pool in pinned host memory that the GPU reaches
// over PCIe ("啃透vLLM源码", §3: blocks go to CPU memory when GPU memory
// runs short and come back when needed). One CTA per (pair, layer, K-or-V),
// eight 16-byte loads in flight per thread to cover the longer latency of
// host memory.
//
// copy_blocks_kernel: copy-on-write duplication of whole shared blocks
// ("vLLM基础", §2.3). One CTA per (pair, layer, K-or-V) copies one
// num_heads * block_size * head_dim block with 16-byte vectors, four loads in
// flight per thread before the stores.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "pagedkv.h"
#include "ptx.cuh"


namespace pagedkv {


struct WriteParams {
    const uint4 *key;   // [T][H][D] as 16-byte vectors
    const uint4 *value;
    const int64_t *slot_mapping;
    uint4 *key_cache;   // [NB][H][BS][D]
    uint4 *value_cache;
    int32_t *dev_err;
    int64_t num_slots;  // num_blocks * block_size
    int32_t num_heads, vecs_per_row, block_size;
};

__global__ void __launch_bounds__(128) write_kv_kernel(const __grid_constant__ WriteParams p)
{
    pdl_launch_dependents();
    pdl_wait_prior_grid(); // inputs may come from the previous kernel
    const int t = blockIdx.x;
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0)
        return; // padding
    if (slot >= p.num_slots) {
        if (threadIdx.x == 0)
            report(p.dev_err, PA_DEVERR_SLOT);
        return;
    }
    const int64_t blk = slot / p.block_size, off = slot % p.block_size;
    const int per_token = p.num_heads * p.vecs_per_row;
    const uint4 *k = p.key + (size_t)t * per_token;
    const uint4 *v = p.value + (size_t)t * per_token;
    // All loads of a round before its stores: the stores may alias nothing
    // the loads read, but the compiler cannot know that.
    constexpr int U = 4;
    for (int base = threadIdx.x; base < per_token; base += blockDim.x * U) {
        uint4 kr[U], vr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            if (i < per_token) {
                kr[u] = k[i];
                vr[u] = v[i];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            if (i < per_token) {
                const int h = i / p.vecs_per_row, e = i - h * p.vecs_per_row;
                const size_t dst =
                    (((size_t)blk * p.num_heads + h) * p.block_size + off) * p.vecs_per_row + e;
                p.key_cache[dst] = kr[u];
                p.value_cache[dst] = vr[u];
            }
        }
    }
}

// write_kv_fp8_kernel: the same write into an fp8 cache. A warp quantises
// one (token, head) row of K and one of V: amax over the row, scale =
// amax / 448, codes = e4m3(x * (448 / amax)) with round-to-nearest-even and
// saturation; lane l stores codes [l*D/32, (l+1)*D/32), lane 0 the scale.
// One CTA (4 warps) per token, warps striding over the heads.
struct WriteFp8Params {
    const void *key; // [T][H][D] of QT
    const void *value;
    const int64_t *slot_mapping;
    uint8_t *key_cache; // [NB][H][BS*D codes + BS fp32 scales]
    uint8_t *value_cache;
    int32_t *dev_err;
    int64_t num_slots;
    int32_t num_heads, head_dim, block_size;
};

template <typename QT, int D>
__device__ __forceinline__ void quantize_row_to(const QT *x, uint8_t *codes, float *scale,
                                                int lane)
{
    constexpr int EPL = D / 32; // elements per lane
    float v[EPL];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        v[e] = static_cast<float>(x[lane * EPL + e]);
        amax = fmaxf(amax, fabsf(v[e]));
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float inv = amax > 0.f ? 448.f / amax : 0.f;
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
        const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(
            make_float2(v[e] * inv, v[e + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        packed |= (uint32_t)c2 << (8 * e);
    }
    if constexpr (EPL == 4)
        reinterpret_cast<uint32_t *>(codes)[lane] = packed;
    else
        reinterpret_cast<uint16_t *>(codes)[lane] = (uint16_t)packed;
    if (lane == 0)
        *scale = amax / 448.f;
}

template <typename QT, int D>
__global__ void __launch_bounds__(128) write_kv_fp8_kernel(const __grid_constant__ WriteFp8Params p)
{
    pdl_launch_dependents();
    pdl_wait_prior_grid();
    const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0)
        return;
    if (slot >= p.num_slots) {
        if (threadIdx.x == 0)
            report(p.dev_err, PA_DEVERR_SLOT);
        return;
    }
    const int64_t blk = slot / p.block_size, off = slot % p.block_size;
    const size_t tile_bytes = (size_t)p.block_size * D + 4 * (size_t)p.block_size;
    for (int h = warp; h < p.num_heads; h += blockDim.x >> 5) {
        const size_t row = ((size_t)t * p.num_heads + h) * D;
        const size_t tile = ((size_t)blk * p.num_heads + h) * tile_bytes;
        quantize_row_to<QT, D>(static_cast<const QT *>(p.key) + row,
                               p.key_cache + tile + (size_t)off * D,
                               reinterpret_cast<float *>(p.key_cache + tile +
                                                         (size_t)p.block_size * D) + off,
                               lane);
        quantize_row_to<QT, D>(static_cast<const QT *>(p.value) + row,
                               p.value_cache + tile + (size_t)off * D,
                               reinterpret_cast<float *>(p.value_cache + tile +
                                                         (size_t)p.block_size * D) + off,
                               lane);
    }
}

struct CopyParams {
    uint4 *key_caches[PA_MAX_LAYERS];
    uint4 *value_caches[PA_MAX_LAYERS];
    const int64_t *block_mapping; // [N][2] = (src, dst)
    int32_t *dev_err;
    int64_t block_vecs;           // 16-byte vectors per block
    int64_t num_blocks;
};

__global__ void __launch_bounds__(256) copy_blocks_kernel(const __grid_constant__ CopyParams p)
{
    pdl_launch_dependents();
    pdl_wait_prior_grid();
    const int pair = blockIdx.x, layer = blockIdx.y, which = blockIdx.z;
    const int64_t src = p.block_mapping[2 * pair], dst = p.block_mapping[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
        if (threadIdx.x == 0 && layer == 0 && which == 0)
            report(p.dev_err, PA_DEVERR_COPY_PAIR);
        return;
    }
    uint4 *base = which ? p.value_caches[layer] : p.key_caches[layer];
    const uint4 *from = base + src * p.block_vecs;
    uint4 *to = base + dst * p.block_vecs;
    constexpr int U = 4;
    const int64_t stride = (int64_t)blockDim.x * U;
    int64_t i = threadIdx.x;
    for (; i + (U - 1) * blockDim.x < p.block_vecs; i += stride) {
        uint4 r[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            r[u] = from[i + u * blockDim.x];
#pragma unroll
        for (int u = 0; u < U; ++u)
            to[i + u * blockDim.x] = r[u];
    }
    for (; i < p.block_vecs; i += blockDim.x)
        to[i] = from[i];
}

struct SwapParams {
    const uint4 *src_k[PA_MAX_LAYERS];
    const uint4 *src_v[PA_MAX_LAYERS];
    uint4 *dst_k[PA_MAX_LAYERS];
    uint4 *dst_v[PA_MAX_LAYERS];
    const int64_t *block_mapping; // [N][2] = (source block, destination block)
    int32_t *dev_err;
    int64_t block_vecs;
    int64_t src_blocks, dst_blocks;
};

__global__ void __launch_bounds__(256) swap_blocks_kernel(const __grid_constant__ SwapParams p)
{
    pdl_launch_dependents();
    pdl_wait_prior_grid();
    const int pair = blockIdx.x, layer = blockIdx.y, which = blockIdx.z;
    const int64_t a = p.block_mapping[2 * pair], b = p.block_mapping[2 * pair + 1];
    if (a < 0 || a >= p.src_blocks || b < 0 || b >= p.dst_blocks) {
        if (threadIdx.x == 0 && layer == 0 && which == 0)
            report(p.dev_err, PA_DEVERR_COPY_PAIR);
        return;
    }
    const uint4 *from = (which ? p.src_v[layer] : p.src_k[layer]) + a * p.block_vecs;
    uint4 *to = (which ? p.dst_v[layer] : p.dst_k[layer]) + b * p.block_vecs;
    constexpr int U = 8;
    const int64_t stride = (int64_t)blockDim.x * U;
    int64_t i = threadIdx.x;
    for (; i + (U - 1) * blockDim.x < p.block_vecs; i += stride) {
        uint4 r[U];
#pragma unroll
        for (int u = 0; u < U; ++u)
            r[u] = from[i + u * blockDim.x];
#pragma unroll
        for (int u = 0; u < U; ++u)
            to[i + u * blockDim.x] = r[u];
    }
    for (; i < p.block_vecs; i += blockDim.x)
        to[i] = from[i];
}

} // namespace pagedkv
