// pagedkv.cu - the C ABI (include/pagedkv.h): host-side argument checks,
// launch-shape choices and kernel launches. Nothing here allocates memory or
// synchronises.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "pagedkv.h"

#include "cache_ops.cuh"
#include "last_error.h"
#include "decode.cuh"
#include "decode_group.cuh"

using namespace pagedkv;

namespace {

// Decode launch shape: 4 warps x 2 bulk-copy stages of 8 KiB per warp =
// 64 KiB of rings per CTA, 3 CTAs per SM. The macros only exist so that
// tuning sweeps can build variants.
#ifndef PA_SPLIT_WARPS
#define PA_SPLIT_WARPS 4
#endif
#ifndef PA_SPLIT_STAGES
#define PA_SPLIT_STAGES 2
#endif
constexpr int kSplitWarps = PA_SPLIT_WARPS;
constexpr int kSplitStages = PA_SPLIT_STAGES;
// Grouped-heads decode: 4 warps x 2 TMA stages of 16 tokens (8 KiB at
// head_dim 128) per warp, 3 CTAs per SM. PA_GROUP_KERNEL=0 builds a variant
// that sends grouped heads to decode_split_kernel, for comparisons.
#ifndef PA_GROUP_KERNEL
#define PA_GROUP_KERNEL 1
#endif
#ifndef PA_GROUP_WARPS
#define PA_GROUP_WARPS 4
#endif
#ifndef PA_GROUP_STAGES
#define PA_GROUP_STAGES 2
#endif
constexpr int kGroupWarps = PA_GROUP_WARPS;
constexpr int kGroupStages = PA_GROUP_STAGES;
// Automatic partition of decode_split_kernel: halve 2048 while the grid
// (sequences x heads x partitions at max_context_len) has fewer CTAs than
// this many per SM, about 1.3 waves of 3 resident CTAs. B200, 8 sequences x
// 32 layers (contexts of a few hundred tokens): 19.1 us per layer at 128
// tokens (the floor, reached with 12 per SM), 15.1 us at 256 (this target),
// 16.9 at 512; launches with more units are unaffected (2048).
constexpr int kTargetCtasPerSm = 4;
constexpr int kMinAutoPartition = 128;
constexpr int kAutoPartition = 2048;
// The grouped kernel streams best in long partitions. When it hands out the
// longest sequences first (batches of up to kRankMaxSeqs), its automatic
// choice is 2048 tokens, halved (down to 256) while the grid would have
// fewer than 2 CTAs per SM (B200, Llama-7B layer: 8 K/V heads 73 us at 2048
// vs 81 us at 1024; 4 K/V heads 49 us at either; 2 K/V heads 37 us at 1024
// vs 43 us at 2048). In natural order (larger batches) long last units drain
// slowly, so it starts from 1024 and halves while there are fewer CTAs than
// SMs (256 sequences x 32 layers: 74 us per layer at 1024, single pass
// slower).
constexpr int kGroupMinAutoPartition = 256;
constexpr int kPartitionQuantum = 32;
constexpr int kMaxDevices = 64;

pa_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count_of_current_device()
{
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 148;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0)
        return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

pa_status check_cache(const pa_cache_desc *c)
{
    if (!c)
        return fail(PA_ERR_INVALID_ARG, "cache descriptor is NULL");
    if (c->num_blocks < 0 || c->block_size <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0)
        return fail(PA_ERR_INVALID_ARG, "cache descriptor has a non-positive size");
    if (c->dtype != PA_F16 && c->dtype != PA_BF16 && c->dtype != PA_FP8_E4M3)
        return fail(PA_ERR_UNSUPPORTED, "cache dtype %d (need PA_F16, PA_BF16 or PA_FP8_E4M3)",
                    (int)c->dtype);
    if (c->dtype == PA_FP8_E4M3 && c->io_dtype != PA_F16 && c->io_dtype != PA_BF16)
        return fail(PA_ERR_UNSUPPORTED, "fp8 cache io_dtype %d (need PA_F16 or PA_BF16)",
                    (int)c->io_dtype);
    if (c->head_dim != 64 && c->head_dim != 128)
        return fail(PA_ERR_UNSUPPORTED, "head_dim %d (built: 64, 128)", c->head_dim);
    if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d (built: 8, 16, 32)", c->block_size);
    return PA_OK;
}

// Bytes of one (block, head) tile and of one block (all heads).
size_t tile_bytes(const pa_cache_desc *c)
{
    const size_t rows = (size_t)c->block_size;
    return c->dtype == PA_FP8_E4M3 ? rows * c->head_dim + 4 * rows : rows * c->head_dim * 2;
}

size_t block_bytes(const pa_cache_desc *c) { return tile_bytes(c) * (size_t)c->num_kv_heads; }

// decode_group_kernel (one CTA per K/V head and group, tensor-core tiles)
// takes 2 <= G <= 16 for 16-bit caches and for fp8 caches with f16 rows and
// head_dim 128, for pools whose rows (num_blocks * num_kv_heads *
// block_size) index as int32 tensor-map coordinates. Everything else goes to
// decode_split_kernel (one CTA per query head). At G = 1 the tile rows are
// 15/16 padding: B200, fp8 Llama-7B layer, 265 us on the tiles against
// 182 us on decode_split_kernel's FMAs.
#ifndef PA_FP8_GROUP_KERNEL
#define PA_FP8_GROUP_KERNEL 1
#endif
bool use_group_kernel(const pa_cache_desc *c, int32_t num_heads)
{
    if (!PA_GROUP_KERNEL || c->num_kv_heads <= 0 || num_heads % c->num_kv_heads != 0)
        return false;
    const int G = num_heads / c->num_kv_heads;
    const int64_t rows = (int64_t)c->num_blocks * c->num_kv_heads * c->block_size;
    if (rows <= 0 || rows > INT32_MAX || G > kGroupMaxHeads)
        return false;
    if (c->dtype == PA_FP8_E4M3)
        return PA_FP8_GROUP_KERNEL && G >= 2 && c->io_dtype == PA_F16 && c->head_dim == 128;
    return G >= 2;
}

// Whether a launch hands out its sequences longest first (ranked_sequence).
// Each CTA pays a dependent round trip for it, so it is worth it only when
// the drain of long last units dominates: the grouped kernel for batches of
// up to kRankMaxSeqs; decode_split_kernel only for grids of at least six
// waves of units of at least 1024 tokens (B200: Llama-7B layer 256.7 ->
// 252.0 us, fp8 183.3 -> 174.4 us; with shorter or fewer units - the
// prefix-sharing batch, 8-sequence batches - it was 8-12 % slower).
constexpr int kRankMinWaves = 6;
constexpr int kRankMinPartition = 1024;
constexpr int kResidentCtasPerSm = 3;
bool rank_sequences(int32_t num_seqs, int32_t num_heads, const pa_cache_desc *c, int P,
                    int64_t parts)
{
    if (num_seqs > kRankMaxSeqs)
        return false;
    if (use_group_kernel(c, num_heads))
        return true;
    const int64_t ctas = (int64_t)num_seqs * num_heads * parts;
    return P >= kRankMinPartition &&
           ctas >= (int64_t)kRankMinWaves * kResidentCtasPerSm * sm_count_of_current_device();
}

// Partition (tokens per work unit) for a decode; >= max_context_len means a
// single pass. Automatic choice for decode_split_kernel (one CTA row per
// (sequence, query head)): 2048 tokens, halved (down to 128) while the grid
// would give fewer than kTargetCtasPerSm CTAs per SM. For
// decode_group_kernel (one CTA row per (sequence, K/V head)): 2048, halved
// (down to 256) while the grid has fewer than 2 CTAs per SM.
int choose_partition(int32_t num_seqs, int32_t num_heads, const pa_cache_desc *c,
                     int32_t max_ctx, int32_t requested, int sm_count)
{
    int P = requested;
    if (P == 0) {
        const bool grouped = use_group_kernel(c, num_heads);
        const bool ranked = grouped && num_seqs <= kRankMaxSeqs;
        const int64_t units = (int64_t)num_seqs * (grouped ? c->num_kv_heads : num_heads);
        const int floor_p = grouped ? kGroupMinAutoPartition : kMinAutoPartition;
        const int64_t target =
            (int64_t)(!grouped ? kTargetCtasPerSm : ranked ? 2 : 1) * sm_count;
        P = !grouped ? kAutoPartition : ranked ? 2048 : 1024;
        while (P > floor_p && units * ((max_ctx + P - 1) / P) < target)
            P /= 2;
    }
    if (max_ctx <= P) {
        const int single = ((max_ctx > 0 ? max_ctx : 1) + kPartitionQuantum - 1) /
                           kPartitionQuantum * kPartitionQuantum;
        return single;
    }
    return P;
}

pa_status check_partition_request(int32_t partition_size)
{
    if (partition_size < 0 || partition_size % kPartitionQuantum != 0 ||
        partition_size > kMaxPartition)
        return fail(PA_ERR_INVALID_ARG,
                    "partition_size %d: need 0 or a multiple of %d up to %d", partition_size,
                    kPartitionQuantum, kMaxPartition);
    return PA_OK;
}

// Split workspace: [arrival counters, kSplitCounters int32][partial sums
// acc, units*parts*D fp32, padded to 256 B][(max, sum) pairs]. The counter
// region comes first and is used for nothing else, so it stays zero from
// call to call whatever the shapes; it must be zero before the first call.
constexpr size_t kCounterBytes = (size_t)kSplitCounters * sizeof(int32_t);
// Floats of shared memory the merging CTA may use for weights: the smallest
// ring area of any decode instantiation (fp8, head_dim 64: 8704 floats;
// grouped, head_dim 64: 8192).
constexpr int64_t kMergeWeights = 8192;

size_t workspace_bytes_for(int64_t units, int64_t num_parts, int head_dim)
{
    const size_t acc = (size_t)(units * num_parts * head_dim) * sizeof(float);
    const size_t acc_padded = (acc + 255) / 256 * 256;
    return kCounterBytes + acc_padded + (size_t)(units * num_parts * 2) * sizeof(float);
}

// Raise a kernel's dynamic shared-memory limit once per device. `done` must
// be distinct for every kernel (one static per template instantiation of the
// caller), since the attribute belongs to the function.
template <typename Kernel>
cudaError_t allow_smem(Kernel k, size_t bytes, std::atomic<size_t> (&done)[kMaxDevices])
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_relaxed) >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess)
        return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < kMaxDevices)
        done[dev].store(bytes, std::memory_order_relaxed);
    return cudaSuccess;
}

// Every kernel of the library is launched with programmatic stream
// serialisation: it may be scheduled while the previous kernel of the stream
// drains, and it waits (griddepcontrol.wait) for that kernel before reading
// or writing anything, in every CTA, so stream order holds for all data.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T, typename QT, int D, int BS>
pa_status launch_decode(const DecodeParams &p, cudaStream_t stream)
{
    using Cfg = SplitCfg<T, D, BS, kSplitWarps, kSplitStages>;
    auto kernel = decode_split_kernel<T, QT, D, BS, kSplitWarps, kSplitStages>;
    static std::atomic<size_t> smem_set[kMaxDevices];
    cudaError_t e = allow_smem(kernel, Cfg::smem_bytes(kMaxPartition), smem_set);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    e = launch_pdl(kernel, dim3(p.num_heads, p.num_seqs, p.num_parts), dim3(kSplitWarps * 32),
                   Cfg::smem_bytes(p.partition_size), stream, p);
    if (e != cudaSuccess)
        return cuda_fail(e, "decode launch");
    if (p.num_parts > 1 && !p.ws_count) {
        e = launch_pdl(reduce_kernel<D>, dim3(p.num_heads, p.num_seqs, 1), dim3(D), 0, stream, p,
                       (int)BS);
        if (e != cudaSuccess)
            return cuda_fail(e, "reduce launch");
    }
    return ok();
}

template <typename T, typename QT, int D>
pa_status dispatch_bs(const DecodeParams &p, int bs, cudaStream_t st)
{
    switch (bs) {
    case 8: return launch_decode<T, QT, D, 8>(p, st);
    case 16: return launch_decode<T, QT, D, 16>(p, st);
    case 32: return launch_decode<T, QT, D, 32>(p, st);
    }
    return fail(PA_ERR_UNSUPPORTED, "block_size %d", bs);
}

// The row view of a 16-bit pool that decode_group_kernel copies from: dims
// (64 elements, head_dim/64 128-byte units, rows), boxes of min(block_size,
// 16) whole rows, 128-byte swizzle. The encoder is the driver's, looked up
// once.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder()
{
    static std::atomic<EncodeTiledFn> cached{nullptr};
    EncodeTiledFn f = cached.load(std::memory_order_acquire);
    if (f)
        return f;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return nullptr;
    }
    f = reinterpret_cast<EncodeTiledFn>(fn);
    cached.store(f, std::memory_order_release);
    return f;
}

pa_status encode_pool_rows(CUtensorMap *map, const void *pool, const pa_cache_desc *c)
{
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc)
        return fail(PA_ERR_CUDA, "the driver has no cuTensorMapEncodeTiled");
    if (c->dtype == PA_FP8_E4M3) {
        // Codes of each (block, head) tile: dims (head_dim bytes, block_size
        // rows, tiles), the tile stride stepping over its row scales.
        const cuuint64_t dims[3] = {(cuuint64_t)c->head_dim, (cuuint64_t)c->block_size,
                                    (cuuint64_t)c->num_blocks * c->num_kv_heads};
        const cuuint64_t strides[2] = {(cuuint64_t)c->head_dim, tile_bytes(c)};
        const cuuint32_t box[3] = {(cuuint32_t)c->head_dim,
                                   (cuuint32_t)std::min<int32_t>(c->block_size, 16), 1};
        const cuuint32_t elem_strides[3] = {1, 1, 1};
        const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(pool),
                               dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
        return PA_OK;
    }
    const cuuint32_t units = (cuuint32_t)c->head_dim / 64;
    const cuuint64_t dims[3] = {64, units,
                                (cuuint64_t)c->num_blocks * c->num_kv_heads * c->block_size};
    const cuuint64_t strides[2] = {128, (cuuint64_t)c->head_dim * 2};
    const cuuint32_t box[3] = {64, units, (cuuint32_t)std::min<int32_t>(c->block_size, 16)};
    const cuuint32_t elem_strides[3] = {1, 1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(pool), dims,
                           strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return PA_OK;
}

template <typename T, int D, int BS, bool TWO>
pa_status launch_group(const GroupParams &gp, cudaStream_t stream)
{
    using Cfg = GroupCfg<T, D, BS, kGroupWarps, kGroupStages>;
    auto kernel = decode_group_kernel<T, D, BS, kGroupWarps, kGroupStages, TWO>;
    static std::atomic<size_t> smem_set[kMaxDevices];
    const DecodeParams &p = gp.p;
    cudaError_t e = allow_smem(kernel, Cfg::smem_bytes(kMaxPartition), smem_set);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(group decode)");
    e = launch_pdl(kernel, dim3(p.num_kv_heads, p.num_seqs, p.num_parts),
                   dim3(kGroupWarps * 32), Cfg::smem_bytes(p.partition_size), stream, gp);
    if (e != cudaSuccess)
        return cuda_fail(e, "group decode launch");
    if (p.num_parts > 1 && !p.ws_count) {
        e = launch_pdl(reduce_kernel<D>, dim3(p.num_heads, p.num_seqs, 1), dim3(D), 0, stream, p,
                       (int)BS);
        if (e != cudaSuccess)
            return cuda_fail(e, "reduce launch");
    }
    return ok();
}

template <typename T, int D, int BS>
pa_status group_rows(const GroupParams &gp, cudaStream_t st)
{
    if (gp.p.num_heads / gp.p.num_kv_heads > 8)
        return launch_group<T, D, BS, true>(gp, st);
    return launch_group<T, D, BS, false>(gp, st);
}

template <typename T, int D>
pa_status group_bs(const GroupParams &gp, int bs, cudaStream_t st)
{
    switch (bs) {
    case 8: return group_rows<T, D, 8>(gp, st);
    case 16: return group_rows<T, D, 16>(gp, st);
    case 32: return group_rows<T, D, 32>(gp, st);
    }
    return fail(PA_ERR_UNSUPPORTED, "block_size %d", bs);
}

pa_status dispatch_group(const DecodeParams &p, const pa_cache_desc *c, cudaStream_t st)
{
    GroupParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.p = p;
    pa_status s = encode_pool_rows(&gp.tk, p.key_cache, c);
    if (s == PA_OK)
        s = encode_pool_rows(&gp.tv, p.value_cache, c);
    if (s != PA_OK)
        return s;
    if (c->dtype == PA_FP8_E4M3) // f16 rows, head_dim 128 (use_group_kernel)
        return group_bs<E4M3, 128>(gp, c->block_size, st);
    const bool bf = c->dtype == PA_BF16;
    if (c->head_dim == 64)
        return bf ? group_bs<__nv_bfloat16, 64>(gp, c->block_size, st)
                  : group_bs<__half, 64>(gp, c->block_size, st);
    return bf ? group_bs<__nv_bfloat16, 128>(gp, c->block_size, st)
              : group_bs<__half, 128>(gp, c->block_size, st);
}

template <typename T, typename QT>
pa_status dispatch_d(const DecodeParams &p, int d, int bs, cudaStream_t st)
{
    if (d == 64)
        return dispatch_bs<T, QT, 64>(p, bs, st);
    return dispatch_bs<T, QT, 128>(p, bs, st);
}

pa_status dispatch_decode(const DecodeParams &p, const pa_cache_desc *c, cudaStream_t st)
{
    if (use_group_kernel(c, p.num_heads))
        return dispatch_group(p, c, st);
    if (c->dtype == PA_F16)
        return dispatch_d<__half, __half>(p, c->head_dim, c->block_size, st);
    if (c->dtype == PA_BF16)
        return dispatch_d<__nv_bfloat16, __nv_bfloat16>(p, c->head_dim, c->block_size, st);
    if (c->io_dtype == PA_F16)
        return dispatch_d<E4M3, __half>(p, c->head_dim, c->block_size, st);
    return dispatch_d<E4M3, __nv_bfloat16>(p, c->head_dim, c->block_size, st);
}

} // namespace

extern "C" {

const char *pa_status_string(pa_status s)
{
    switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int32_t pa_version(void) { return 100; }

pa_status pa_write_kv(const void *key, const void *value, int32_t num_tokens, int32_t num_heads,
                      const int64_t *slot_mapping, void *key_cache, void *value_cache,
                      const pa_cache_desc *cache, int32_t *dev_err, void *stream)
{
    pa_status s = check_cache(cache);
    if (s != PA_OK)
        return s;
    if (num_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "num_tokens %d < 0", num_tokens);
    if (num_heads != cache->num_kv_heads)
        return fail(PA_ERR_UNSUPPORTED, "num_heads %d != num_kv_heads %d", num_heads,
                    cache->num_kv_heads);
    if (num_tokens == 0)
        return ok();
    if (!key || !value || !slot_mapping || !key_cache || !value_cache)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID_ARG, "key, value and caches must be 16-byte aligned");
    if (cache->dtype == PA_FP8_E4M3) {
        WriteFp8Params q;
        q.key = key;
        q.value = value;
        q.slot_mapping = slot_mapping;
        q.key_cache = static_cast<uint8_t *>(key_cache);
        q.value_cache = static_cast<uint8_t *>(value_cache);
        q.dev_err = dev_err;
        q.num_slots = (int64_t)cache->num_blocks * cache->block_size;
        q.num_heads = num_heads;
        q.head_dim = cache->head_dim;
        q.block_size = cache->block_size;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        const bool f16 = cache->io_dtype == PA_F16;
        cudaError_t e;
        if (cache->head_dim == 64)
            e = f16 ? launch_pdl(write_kv_fp8_kernel<__half, 64>, dim3(num_tokens), dim3(128), 0, st, q)
                    : launch_pdl(write_kv_fp8_kernel<__nv_bfloat16, 64>, dim3(num_tokens), dim3(128), 0, st, q);
        else
            e = f16 ? launch_pdl(write_kv_fp8_kernel<__half, 128>, dim3(num_tokens), dim3(128), 0, st, q)
                    : launch_pdl(write_kv_fp8_kernel<__nv_bfloat16, 128>, dim3(num_tokens), dim3(128), 0, st, q);
        if (e != cudaSuccess)
            return cuda_fail(e, "write_kv launch");
        return ok();
    }
    WriteParams p;
    p.key = static_cast<const uint4 *>(key);
    p.value = static_cast<const uint4 *>(value);
    p.slot_mapping = slot_mapping;
    p.key_cache = static_cast<uint4 *>(key_cache);
    p.value_cache = static_cast<uint4 *>(value_cache);
    p.dev_err = dev_err;
    p.num_slots = (int64_t)cache->num_blocks * cache->block_size;
    p.num_heads = num_heads;
    p.vecs_per_row = cache->head_dim * 2 / 16;
    p.block_size = cache->block_size;
    cudaError_t e = launch_pdl(write_kv_kernel, dim3(num_tokens), dim3(128), 0,
                               static_cast<cudaStream_t>(stream), p);
    if (e != cudaSuccess)
        return cuda_fail(e, "write_kv launch");
    return ok();
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size)
{
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        check_partition_request(partition_size) != PA_OK)
        return (size_t)-1;
    const int P = partition_size == 0 ? kMinAutoPartition : partition_size;
    if (max_context_len <= P)
        return 0;
    const int64_t parts = (max_context_len + P - 1) / P;
    return workspace_bytes_for((int64_t)num_seqs * num_heads, parts, head_dim);
}

int32_t pa_decode_partition_size(int32_t num_seqs, int32_t num_heads,
                                 const pa_cache_desc *cache, int32_t max_context_len,
                                 int32_t partition_size)
{
    if (check_cache(cache) != PA_OK || num_seqs < 0 || num_heads <= 0 ||
        num_heads % cache->num_kv_heads != 0 || max_context_len < 0 ||
        check_partition_request(partition_size) != PA_OK)
        return -1;
    return choose_partition(num_seqs, num_heads, cache, max_context_len, partition_size,
                            partition_size == 0 ? sm_count_of_current_device() : 148);
}

} // extern "C"

namespace {

// ---------------------------------------------------------------------------
// The built-in split workspace of pa_decode_noalloc: a fixed array of device
// memory compiled into the library, for callers that cannot allocate.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CtxGetCurrentFn ctx_get_current()
{
    static std::atomic<CtxGetCurrentFn> cached{nullptr};
    CtxGetCurrentFn f = cached.load(std::memory_order_acquire);
    if (f)
        return f;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return nullptr;
    }
    f = reinterpret_cast<CtxGetCurrentFn>(fn);
    cached.store(f, std::memory_order_release);
    return f;
}

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory: its device address is looked up with the device current, once per
// device and context (a device reset creates a new context whose copy of the
// array may sit elsewhere), and handed to the kernels.
pa_status noalloc_scratch(void **out)
{
    struct Entry {
        CUcontext ctx;
        void *addr;
    };
    static std::mutex mu;
    static Entry cache[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(PA_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    // The context current on this thread (none yet on a thread that has not
    // used the runtime: then the look-up below sets it up).
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (!get || get(&ctx) != CUDA_SUCCESS)
        ctx = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ctx || cache[dev].ctx != ctx || !cache[dev].addr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        if (!get || get(&ctx) != CUDA_SUCCESS)
            ctx = nullptr;
        cache[dev].ctx = ctx;
        cache[dev].addr = p;
    }
    *out = cache[dev].addr;
    return PA_OK;
}

// pa_decode, and pa_write_kv_decode when new_key/new_value are given. With
// builtin_scratch (pa_decode_noalloc) the split workspace is the library's
// own array instead of the caller's.
pa_status decode_common(void *out, pa_dtype out_dtype, const void *query, int32_t num_seqs,
                        int32_t num_heads, const void *key_cache, const void *value_cache,
                        const pa_cache_desc *cache, const int32_t *block_tables,
                        int32_t max_blocks_per_seq, const int32_t *context_lens,
                        int32_t max_context_len, float scale, int32_t partition_size,
                        void *workspace, size_t workspace_bytes, int32_t *dev_err,
                        void *stream, const void *new_key, const void *new_value,
                        bool builtin_scratch = false)
{
    pa_status s = check_cache(cache);
    if (s != PA_OK)
        return s;
    if (num_seqs < 0 || num_heads <= 0 || max_blocks_per_seq < 0 || max_context_len < 0)
        return fail(PA_ERR_INVALID_ARG, "negative size argument");
    if (num_heads % cache->num_kv_heads != 0)
        return fail(PA_ERR_UNSUPPORTED, "num_heads %d is not a multiple of num_kv_heads %d",
                    num_heads, cache->num_kv_heads);
    if (out_dtype != PA_F16 && out_dtype != PA_BF16 && out_dtype != PA_F32)
        return fail(PA_ERR_INVALID_ARG, "out_dtype %d", (int)out_dtype);
    if ((s = check_partition_request(partition_size)) != PA_OK)
        return s;
    if (num_seqs == 0)
        return ok();
    if (num_seqs > 65535)
        return fail(PA_ERR_UNSUPPORTED, "num_seqs %d > 65535", num_seqs);
    if (!out || !query || !key_cache || !value_cache || !context_lens ||
        (max_blocks_per_seq > 0 && !block_tables))
        return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID_ARG, "query and caches must be 16-byte aligned");
    if (new_key || new_value) {
        if (!new_key || !new_value)
            return fail(PA_ERR_INVALID_ARG, "NULL key or value");
        if (!aligned16(new_key) || !aligned16(new_value))
            return fail(PA_ERR_INVALID_ARG, "key and value must be 16-byte aligned");
    }
    if (!(scale == scale))
        return fail(PA_ERR_INVALID_ARG, "scale is NaN");
    if (cache->num_blocks == 0 && max_context_len > 0)
        return fail(PA_ERR_INVALID_ARG, "empty pool with max_context_len %d", max_context_len);

    const int P = choose_partition(num_seqs, num_heads, cache, max_context_len,
                                   partition_size, sm_count_of_current_device());
    const int64_t parts = max_context_len > P ? (max_context_len + P - 1) / P : 1;
    if (parts > 65535)
        return fail(PA_ERR_UNSUPPORTED, "too many partitions (%lld)", (long long)parts);
    DecodeParams p = {};
    p.out = out;
    p.query = query;
    p.key_cache = key_cache;
    p.value_cache = value_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.dev_err = dev_err;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.partition_size = P;
    p.num_parts = (int32_t)parts;
    p.rank_seqs = rank_sequences(num_seqs, num_heads, cache, P, parts) ? 1 : 0;
    p.out_dtype = (int32_t)out_dtype;
    p.qk_scale_log2 = scale * 1.4426950408889634f;
    p.new_key = new_key;
    p.new_value = new_value;
    if (parts > 1) {
        const int64_t units = (int64_t)num_seqs * num_heads;
        const size_t need = workspace_bytes_for(units, parts, cache->head_dim);
        if (builtin_scratch) {
            if (need > PA_NOALLOC_SCRATCH_BYTES)
                return fail(PA_ERR_WORKSPACE,
                            "split decode needs %zu bytes of scratch (partition %d); the "
                            "built-in scratch holds %u: use a larger partition_size or pa_decode",
                            need, P, (unsigned)PA_NOALLOC_SCRATCH_BYTES);
            if ((s = noalloc_scratch(&workspace)) != PA_OK)
                return s;
            workspace_bytes = PA_NOALLOC_SCRATCH_BYTES;
            // The array keeps whatever the last call left: clear the arrival
            // counters this call can use (the first S * H of them), in stream
            // order before the kernel.
            const size_t counters = (size_t)std::min<int64_t>(units, kSplitCounters) * 4;
            const cudaError_t e =
                cudaMemsetAsync(workspace, 0, counters, static_cast<cudaStream_t>(stream));
            if (e != cudaSuccess)
                return cuda_fail(e, "clearing the built-in scratch counters");
        }
        if (!workspace || workspace_bytes < need)
            return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes, need %zu", workspace_bytes,
                        need);
        if (!aligned16(workspace))
            return fail(PA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
        const size_t acc = (size_t)(units * parts * cache->head_dim) * sizeof(float);
        char *w = static_cast<char *>(workspace);
        // Counter slots: (sequence, query head) for decode_split_kernel,
        // (sequence, K/V head) for the grouped kernel; both < S * H. The
        // merging CTA keeps one weight per (head, partition) in its ring
        // memory (at least kMergeWeights floats in every instantiation).
        const int64_t heads_per_cta =
            use_group_kernel(cache, num_heads) ? num_heads / cache->num_kv_heads : 1;
        const bool in_kernel = units <= kSplitCounters && heads_per_cta * parts <= kMergeWeights;
        p.ws_count = in_kernel ? reinterpret_cast<int32_t *>(w) : nullptr;
        p.ws_acc = reinterpret_cast<float *>(w + kCounterBytes);
        p.ws_ml = reinterpret_cast<float *>(w + kCounterBytes + (acc + 255) / 256 * 256);
    }
    return dispatch_decode(p, cache, static_cast<cudaStream_t>(stream));
}

} // namespace

extern "C" {

pa_status pa_decode(void *out, pa_dtype out_dtype, const void *query, int32_t num_seqs,
                    int32_t num_heads, const void *key_cache, const void *value_cache,
                    const pa_cache_desc *cache, const int32_t *block_tables,
                    int32_t max_blocks_per_seq, const int32_t *context_lens,
                    int32_t max_context_len, float scale, int32_t partition_size,
                    void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream)
{
    return decode_common(out, out_dtype, query, num_seqs, num_heads, key_cache, value_cache,
                         cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                         scale, partition_size, workspace, workspace_bytes, dev_err, stream,
                         nullptr, nullptr);
}

pa_status pa_write_kv_decode(void *out, pa_dtype out_dtype, const void *query, const void *key,
                             const void *value, int32_t num_seqs, int32_t num_heads,
                             void *key_cache, void *value_cache, const pa_cache_desc *cache,
                             const int32_t *block_tables, int32_t max_blocks_per_seq,
                             const int32_t *context_lens, int32_t max_context_len, float scale,
                             int32_t partition_size, void *workspace, size_t workspace_bytes,
                             int32_t *dev_err, void *stream)
{
    if (num_seqs > 0 && (!key || !value))
        return fail(PA_ERR_INVALID_ARG, "NULL key or value");
    return decode_common(out, out_dtype, query, num_seqs, num_heads, key_cache, value_cache,
                         cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                         scale, partition_size, workspace, workspace_bytes, dev_err, stream,
                         num_seqs > 0 ? key : nullptr, num_seqs > 0 ? value : nullptr);
}

pa_status pa_copy_blocks(void *const *key_caches, void *const *value_caches, int32_t num_layers,
                         const int64_t *block_mapping, int32_t num_pairs,
                         const pa_cache_desc *cache, int32_t *dev_err, void *stream)
{
    pa_status s = check_cache(cache);
    if (s != PA_OK)
        return s;
    if (num_pairs < 0)
        return fail(PA_ERR_INVALID_ARG, "num_pairs %d < 0", num_pairs);
    if (num_layers < 1 || num_layers > PA_MAX_LAYERS)
        return fail(PA_ERR_INVALID_ARG, "num_layers %d outside [1, %d]", num_layers, PA_MAX_LAYERS);
    if (num_pairs == 0)
        return ok();
    if (!block_mapping || !key_caches || !value_caches)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    CopyParams p;
    for (int l = 0; l < num_layers; ++l) {
        if (!key_caches[l] || !value_caches[l])
            return fail(PA_ERR_INVALID_ARG, "NULL cache pointer for layer %d", l);
        if (!aligned16(key_caches[l]) || !aligned16(value_caches[l]))
            return fail(PA_ERR_INVALID_ARG, "cache of layer %d not 16-byte aligned", l);
        p.key_caches[l] = static_cast<uint4 *>(key_caches[l]);
        p.value_caches[l] = static_cast<uint4 *>(value_caches[l]);
    }
    for (int l = num_layers; l < PA_MAX_LAYERS; ++l)
        p.key_caches[l] = p.value_caches[l] = nullptr;
    p.block_mapping = block_mapping;
    p.dev_err = dev_err;
    p.block_vecs = (int64_t)(block_bytes(cache) / 16);
    p.num_blocks = cache->num_blocks;
    cudaError_t e = launch_pdl(copy_blocks_kernel, dim3(num_pairs, num_layers, 2), dim3(256), 0,
                               static_cast<cudaStream_t>(stream), p);
    if (e != cudaSuccess)
        return cuda_fail(e, "copy_blocks launch");
    return ok();
}

// Self-test of the bounded wait every kernel uses on its shared-memory
// copies: one warp waits on an mbarrier that nothing will complete.
__global__ void bounded_wait_selftest_kernel(int32_t *dev_err, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0)
        mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    __syncwarp();
    const bool ok = mbar_wait_bounded(smem_addr(&bar), 0, limit_ns);
    if (__any_sync(0xffffffffu, !ok) && threadIdx.x == 0)
        report(dev_err, PA_DEVERR_TIMEOUT);
}

pa_status pa_selftest_wait_timeout(int32_t *dev_err, uint32_t limit_us, void *stream)
{
    if (!dev_err)
        return fail(PA_ERR_INVALID_ARG, "dev_err is NULL");
    if (limit_us == 0 || limit_us > 1000000u)
        return fail(PA_ERR_INVALID_ARG, "limit_us %u outside [1, 1000000]", limit_us);
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        dev_err, (uint64_t)limit_us * 1000u);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, "self-test launch");
    return ok();
}

// The address a kernel uses for `p`: device memory as is, pinned host memory
// through its device mapping. Pageable host memory (which no kernel may
// touch) and unknown pointers are refused.
static pa_status device_view(const void *p, const char *what, const void **out)
{
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PA_ERR_INVALID_ARG, "%s: not a CUDA-visible pointer", what);
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
        *out = p;
        return PA_OK;
    }
    if (a.type == cudaMemoryTypeHost && a.devicePointer) {
        *out = a.devicePointer;
        return PA_OK;
    }
    return fail(PA_ERR_INVALID_ARG,
                "%s: pageable host memory (the GPU can only reach pinned host memory)", what);
}

pa_status pa_swap_blocks(void *const *src_key_caches, void *const *src_value_caches,
                         const pa_cache_desc *src, void *const *dst_key_caches,
                         void *const *dst_value_caches, const pa_cache_desc *dst,
                         int32_t num_layers, const int64_t *block_mapping, int32_t num_pairs,
                         int32_t *dev_err, void *stream)
{
    pa_status s = check_cache(src);
    if (s != PA_OK)
        return s;
    if ((s = check_cache(dst)) != PA_OK)
        return s;
    if (src->block_size != dst->block_size || src->num_kv_heads != dst->num_kv_heads ||
        src->head_dim != dst->head_dim || src->dtype != dst->dtype ||
        block_bytes(src) != block_bytes(dst))
        return fail(PA_ERR_INVALID_ARG, "source and destination pools differ in block shape");
    if (num_pairs < 0)
        return fail(PA_ERR_INVALID_ARG, "num_pairs %d < 0", num_pairs);
    if (num_layers < 1 || num_layers > PA_MAX_LAYERS)
        return fail(PA_ERR_INVALID_ARG, "num_layers %d outside [1, %d]", num_layers, PA_MAX_LAYERS);
    if (num_pairs == 0)
        return ok();
    if (!block_mapping || !src_key_caches || !src_value_caches || !dst_key_caches ||
        !dst_value_caches)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    SwapParams p;
    const void *v = nullptr;
    if ((s = device_view(block_mapping, "block_mapping", &v)) != PA_OK)
        return s;
    p.block_mapping = static_cast<const int64_t *>(v);
    void *const *arrays[4] = {src_key_caches, src_value_caches, dst_key_caches, dst_value_caches};
    const char *names[4] = {"source key cache", "source value cache", "destination key cache",
                            "destination value cache"};
    for (int l = 0; l < num_layers; ++l) {
        const void *views[4];
        for (int k = 0; k < 4; ++k) {
            const void *ptr = arrays[k][l];
            if (!ptr || !aligned16(ptr))
                return fail(PA_ERR_INVALID_ARG, "%s of layer %d is NULL or not 16-byte aligned",
                            names[k], l);
            if ((s = device_view(ptr, names[k], &views[k])) != PA_OK)
                return s;
        }
        p.src_k[l] = static_cast<const uint4 *>(views[0]);
        p.src_v[l] = static_cast<const uint4 *>(views[1]);
        p.dst_k[l] = static_cast<uint4 *>(const_cast<void *>(views[2]));
        p.dst_v[l] = static_cast<uint4 *>(const_cast<void *>(views[3]));
    }
    for (int l = num_layers; l < PA_MAX_LAYERS; ++l) {
        p.src_k[l] = p.src_v[l] = nullptr;
        p.dst_k[l] = p.dst_v[l] = nullptr;
    }
    p.dev_err = dev_err;
    p.block_vecs = (int64_t)(block_bytes(src) / 16);
    p.src_blocks = src->num_blocks;
    p.dst_blocks = dst->num_blocks;
    cudaError_t e = launch_pdl(swap_blocks_kernel, dim3(num_pairs, num_layers, 2), dim3(256), 0,
                               static_cast<cudaStream_t>(stream), p);
    if (e != cudaSuccess)
        return cuda_fail(e, "swap_blocks launch");
    return ok();
}

} // extern "C"

extern "C" pa_status pa_decode_noalloc(void *out, pa_dtype out_dtype, const void *query,
                                       int32_t num_seqs, int32_t num_heads,
                                       const void *key_cache, const void *value_cache,
                                       const pa_cache_desc *cache, const int32_t *block_tables,
                                       int32_t max_blocks_per_seq, const int32_t *context_lens,
                                       int32_t max_context_len, float scale,
                                       int32_t partition_size, int32_t *dev_err, void *stream)
{
    return decode_common(out, out_dtype, query, num_seqs, num_heads, key_cache, value_cache,
                         cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                         scale, partition_size, nullptr, 0, dev_err, stream, nullptr, nullptr,
                         true);
}
