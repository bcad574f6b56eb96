// decode.cuh - paged decode attention for sm_100a.
//
// out[s,h,:] = softmax(scale * q K^T) V over the context_len tokens that the
// block table of sequence s reaches. Paging changes where K/V bytes live, not
// the arithmetic ("VLLM源码解析", core technology: attention over key_cache /
// value_cache through physical block indices; "vLLM基础", §2.3 block table).
//
// A work unit is (sequence s, head h, partition p) = tokens
// [p*P, min((p+1)*P, ctx)) of one (sequence, head). A sequence that fits one
// partition is finished in place; a longer one leaves (running max, running
// sum, unnormalised output) per partition in the workspace and
// reduce_kernel merges them with the log-sum-exp rule.
//
// The K/V of a unit stream through shared memory in chunks of 4 KiB of K
// rows (16 tokens at head_dim 128, 32 at 64) plus the matching V rows. Each
// warp keeps its own NS-stage ring: lane 0 issues 1-D bulk copies
// (cp.async.bulk, the TMA unit's non-tensor path) of a chunk's K and V rows
// straight out of the scattered physical blocks, each stage completing on
// its own mbarrier, NS chunks ahead of the math.
//
// decode_split_kernel: a CTA takes one unit and its NW warps share it, every
// NW-th chunk each, merging their softmax states in shared memory at the
// end. (A mapping with one warp per head and NW heads of a sequence per CTA
// was measured slower on every workload here and is not built.)
//
// Math per chunk (fp32): each row (token) is covered by D/32 lanes holding
// 32 of its dims; q.k is 4 x 16-byte shared loads + 32 FMAs per lane and a
// shuffle reduction over the row's lanes. Online softmax in base 2 (q is
// pre-scaled by scale*log2(e)): running max m, running sum l, rescale of the
// accumulator when m grows. Rows past the context are excluded (score -inf,
// V row skipped), never multiplied by zero, so stale or NaN bytes in the
// tail of a block cannot leak in.
//
// Bank conflicts: a 16-byte shared load is served per quarter-warp (8 lanes,
// 128 bytes). The 16-byte sub-chunk a lane reads in register slot j is
// XOR-swizzled with its row so that the quarter-warp's 8 loads hit 8
// distinct 4-bank groups; the slots are put back in order before the
// cross-row reduction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "pagedkv.h"
#include "ptx.cuh"

namespace pagedkv {

constexpr uint64_t kWaitLimitNs = 1000000000ull; // 1 s: far above any copy latency
constexpr int kMaxPartition = 8192;              // tokens per work unit, upper bound

struct DecodeParams {
    void *out;
    const void *query;
    const void *key_cache;
    const void *value_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_acc; // [S][H][num_parts][D]
    float *ws_ml;  // [S][H][num_parts][2] = (max, sum), base-2 domain
    int32_t *dev_err;
    int32_t num_seqs, num_heads, num_blocks, max_blocks_per_seq, max_context_len;
    int32_t partition_size, num_parts;
    int32_t out_dtype; // 0 f16, 1 bf16, 2 f32
    float qk_scale_log2;
    // Fused append (pa_write_kv_decode): the new token of sequence s, at
    // position context_lens[s] - 1, has K/V rows new_key/new_value[s][h][:];
    // NULL for a plain decode.
    const void *new_key;
    const void *new_value;
};

template <typename T> struct Elem;
template <> struct Elem<__half> {
    static __device__ __forceinline__ float2 pair(uint32_t u)
    {
        __half2 h;
        memcpy(&h, &u, 4);
        return __half22float2(h);
    }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float2 pair(uint32_t u)
    {
        __nv_bfloat162 h;
        memcpy(&h, &u, 4);
        return __bfloat1622float2(h);
    }
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &raw, float (&f)[8])
{
    float2 a = Elem<T>::pair(raw.x), b = Elem<T>::pair(raw.y);
    float2 c = Elem<T>::pair(raw.z), d = Elem<T>::pair(raw.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

__device__ __forceinline__ void store_out(void *out, int dtype, size_t idx, float v)
{
    if (dtype == 2)
        static_cast<float *>(out)[idx] = v;
    else if (dtype == 0)
        static_cast<__half *>(out)[idx] = __float2half_rn(v);
    else
        static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
}

// Clamp a sequence's context length to what the grid and its table cover.
__device__ __forceinline__ int checked_context(const DecodeParams &p, int raw, int bs,
                                               bool report_it)
{
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * bs);
    if (raw < 0 || raw > cap) {
        if (report_it)
            report(p.dev_err, PA_DEVERR_CONTEXT_LEN);
        return raw < 0 ? 0 : cap;
    }
    return raw;
}

template <typename T, int D, int BS, int NS> struct ChunkCfg {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    static constexpr int kLPR = D / 32;                    // lanes per row
    static constexpr int kRPS = 32 / kLPR;                 // rows per warp step
    static constexpr int kQR = 8 / kLPR;                   // rows per quarter-warp
    static constexpr int kChunk = 4096 / (D * 2);          // tokens per stage (4 KiB of K)
    static constexpr int kSteps = kChunk / kRPS;
    static constexpr int kSeg = BS < kChunk ? BS : kChunk; // rows per bulk copy
    static constexpr int kTile = kChunk * D;               // elements of K (or V) per stage
    static constexpr int kRingBytes = NS * 2 * kTile * 2;  // one warp's stages
    static_assert(kSteps >= 1 && kChunk % kRPS == 0, "chunk geometry");
};

// One warp's online-softmax state over the chunks it streamed. After
// finish(), the lanes with r == 0 (lane < D/32) hold the warp's sums for
// dims (qd + LPR*j)*8 + e, j < 4, e < 8; every lane holds m and l.
template <typename T, int D, int BS, int NS> struct WarpStream {
    using C = ChunkCfg<T, D, BS, NS>;
    static constexpr int LPR = C::kLPR, RPS = C::kRPS, QR = C::kQR, CHUNK = C::kChunk;
    static constexpr int STEPS = C::kSteps, TILE = C::kTile;
    static constexpr unsigned FULL = 0xffffffffu;

    float qf[4][8];
    float acc[4][8];
    float m, l;
    int qd, r, rx, lane;
    int bad_id; // lane 0: a block id outside the pool was met
    // Fused append: local chunk patch_i holds the new token at row
    // patch_row. Lanes < 2*D/8 carry 16 bytes of its K (then V) row in
    // patch_val, which replace that row in shared memory once the chunk has
    // landed and go to the cache at patch_dst (NULL: the block id was bad).
    int patch_i, patch_row;
    uint4 patch_val;
    uint4 *patch_dst;

    __device__ __forceinline__ void init(const T *q, float qk_scale_log2, int lane_)
    {
        lane = lane_;
        qd = lane % LPR;
        r = lane / LPR;
        rx = r & (QR - 1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int u = qd + LPR * (j ^ rx);
            unpack8<T>(*reinterpret_cast<const uint4 *>(q + u * 8), qf[j]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qf[j][e] *= qk_scale_log2;
                acc[j][e] = 0.f;
            }
        }
        m = -INFINITY;
        l = 0.f;
        bad_id = 0;
        patch_i = -1;
        patch_row = 0;
        patch_dst = nullptr;
    }

    // Stream chunks c0, c0 + cstride, ... (count of them) of a unit with
    // n_tok tokens whose block ids are table[0..]. Lane 0 issues the copies;
    // an id outside [0, num_blocks) is replaced by block 0 and sets bad_id.
    // Returns false if a wait ran out of time (the copies in flight have been
    // waited for, boundedly, before returning).
    __device__ __forceinline__ bool run(const T *kc, const T *vc, size_t head_off,
                                        size_t block_elems, int num_blocks,
                                        const int32_t *table, int n_tok, int c0, int cstride,
                                        int count, T *ring, uint32_t bar0)
    {
        auto issue = [&](int i) {
            const int tok0 = (c0 + i * cstride) * CHUNK;
            const int rows = min(CHUNK, n_tok - tok0);
            const int st = i % NS;
            T *dk = ring + st * 2 * TILE;
            T *dv = dk + TILE;
            const uint32_t bar = bar0 + st * 8;
            mbar_arrive_expect_tx(bar, 2u * rows * D * sizeof(T));
            for (int r0 = 0; r0 < rows; r0 += C::kSeg) {
                const int tok = tok0 + r0;
                int b = table[tok / BS];
                if (b < 0 || b >= num_blocks) {
                    bad_id = 1;
                    b = 0;
                }
                const size_t src = (size_t)b * block_elems + head_off + (size_t)(tok % BS) * D;
                const uint32_t bytes = (uint32_t)(min(C::kSeg, rows - r0) * D * sizeof(T));
                bulk_g2s(smem_addr(dk + r0 * D), kc + src, bytes, bar);
                bulk_g2s(smem_addr(dv + r0 * D), vc + src, bytes, bar);
            }
        };

        if (lane == 0)
            for (int i = 0; i < min(NS, count); ++i)
                issue(i);
        int issued = min(NS, count);
        int i = 0;
        for (; i < count; ++i) {
            const int st = i % NS;
            const bool ok = mbar_wait_bounded(bar0 + st * 8, (i / NS) & 1, kWaitLimitNs);
            if (__any_sync(FULL, !ok))
                break;
            const int rows = min(CHUNK, n_tok - (c0 + i * cstride) * CHUNK);
            T *sk = ring + st * 2 * TILE;
            T *sv = sk + TILE;
            if (i == patch_i) { // warp-uniform
                constexpr int RV = D * 2 / 16;
                if (lane < 2 * RV) {
                    T *srow = (lane >= RV ? sv : sk) + patch_row * D;
                    reinterpret_cast<uint4 *>(srow)[lane % RV] = patch_val;
                    if (patch_dst)
                        *patch_dst = patch_val;
                    fence_proxy_async_smem(); // before the stage is refilled by a bulk copy
                }
                __syncwarp();
            }

            float sc[STEPS];
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int row = t * RPS + r;
                const T *kr = sk + row * D;
                float dot = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float kf[8];
                    unpack8<T>(*reinterpret_cast<const uint4 *>(kr + (qd + LPR * (j ^ rx)) * 8),
                               kf);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dot = fmaf(qf[j][e], kf[e], dot);
                }
#pragma unroll
                for (int o = 1; o < LPR; o <<= 1)
                    dot += __shfl_xor_sync(FULL, dot, o);
                sc[t] = row < rows ? dot : -INFINITY;
            }
            float cm = sc[0];
#pragma unroll
            for (int t = 1; t < STEPS; ++t)
                cm = fmaxf(cm, sc[t]);
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1)
                cm = fmaxf(cm, __shfl_xor_sync(FULL, cm, o));
            const float m_new = fmaxf(m, cm); // finite: row 0 of a chunk is always valid
            const float corr = exp2f(m - m_new);
            m = m_new;
            l *= corr;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[j][e] *= corr;
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int row = t * RPS + r;
                const float pt = exp2f(sc[t] - m_new);
                l += pt;
                if (row < rows) {
                    const T *vr = sv + row * D;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float vf[8];
                        unpack8<T>(
                            *reinterpret_cast<const uint4 *>(vr + (qd + LPR * (j ^ rx)) * 8), vf);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            acc[j][e] = fmaf(pt, vf[e], acc[j][e]);
                    }
                }
            }
            __syncwarp();
            if (i + NS < count) {
                if (lane == 0)
                    issue(i + NS);
                issued = i + NS + 1;
            }
        }
        if (i < count) {
            // Timed out: let the copies still in flight land before the
            // shared memory is reused or the CTA exits.
            for (int k = i; k < issued; ++k)
                mbar_wait_bounded(bar0 + (k % NS) * 8, (k / NS) & 1, kWaitLimitNs);
            return false;
        }
        return true;
    }

    // Put the swizzled slots back in order (slot j <- sub-chunk qd + LPR*j)
    // and sum acc and l over the rows the warp's lanes covered.
    __device__ __forceinline__ void finish()
    {
        if (rx & 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float t0 = acc[0][e]; acc[0][e] = acc[1][e]; acc[1][e] = t0;
                float t2 = acc[2][e]; acc[2][e] = acc[3][e]; acc[3][e] = t2;
            }
        }
        if (rx & 2) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float t0 = acc[0][e]; acc[0][e] = acc[2][e]; acc[2][e] = t0;
                float t1 = acc[1][e]; acc[1][e] = acc[3][e]; acc[3][e] = t1;
            }
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
            l += __shfl_xor_sync(FULL, l, o);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[j][e] += __shfl_xor_sync(FULL, acc[j][e], o);
        }
    }
};

// Shared prologue: read the context length and the partition's slice of the
// block table at the same time (one global latency). Returns false when the
// partition is past the sequence (the whole CTA returns).
struct UnitInfo {
    int ctx, num_parts, start, n_tok;
};

template <int BS>
__device__ __forceinline__ bool load_unit(const DecodeParams &p, int s, int part, int tid,
                                          int nthreads, bool report_ctx, int32_t *table,
                                          UnitInfo &u)
{
    const int P = p.partition_size;
    const int raw = p.context_lens[s];
    const int start_blk = part * (P / BS);
    const int n_load = min(P / BS, p.max_blocks_per_seq - start_blk);
    const int32_t *bt = p.block_tables + (size_t)s * p.max_blocks_per_seq + start_blk;
    for (int i = tid; i < n_load; i += nthreads)
        table[i] = bt[i];
    u.ctx = checked_context(p, raw, BS, report_ctx);
    u.num_parts = u.ctx > 0 ? (u.ctx + P - 1) / P : 1;
    u.start = part * P;
    u.n_tok = min(P, u.ctx - u.start); // 0 only when ctx == 0
    return part < u.num_parts;
}

// NW warps share one unit: CTA = (head blockIdx.x, sequence blockIdx.y,
// partition blockIdx.z).
template <typename T, int D, int BS, int NW, int NS> struct SplitCfg {
    using C = ChunkCfg<T, D, BS, NS>;
    static constexpr int kRingsBytes = NW * C::kRingBytes;
    static constexpr int kBarBytes = NW * NS * 8;
    static constexpr int kMergeBytes = NW * (D + 2) * 4;
    static constexpr int kFixedBytes = kRingsBytes + kBarBytes + kMergeBytes;
    static size_t smem_bytes(int partition)
    {
        return kFixedBytes + ((partition / BS) * 4 + 15) / 16 * 16;
    }
};

template <typename T, int D, int BS, int NW, int NS>
__global__ void __launch_bounds__(NW * 32)
    decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    using W = WarpStream<T, D, BS, NS>;
    using Cfg = SplitCfg<T, D, BS, NW, NS>;
    constexpr int LPR = W::LPR;
    extern __shared__ __align__(128) unsigned char smem[];
    T *rings = reinterpret_cast<T *>(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kRingsBytes);
    float *merge = reinterpret_cast<float *>(smem + Cfg::kRingsBytes + Cfg::kBarBytes);
    int32_t *table = reinterpret_cast<int32_t *>(smem + Cfg::kFixedBytes);
    __shared__ int cta_flags;

    // Dependent kernels (the reduce, the next layer's write) may launch now;
    // each of them waits for this grid before it touches data.
    pdl_launch_dependents();
    const int h = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads;

    if (tid == 0)
        cta_flags = 0;
    if (lane == 0)
        for (int k = 0; k < NS; ++k)
            mbar_init(smem_addr(&bars[warp * NS + k]), 1);
    fence_mbar_init();
    pdl_wait_prior_grid(); // every input may come from the previous kernel
    UnitInfo u;
    const bool live = load_unit<BS>(p, s, part, tid, NW * 32, tid == 0 && h == 0 && part == 0,
                                    table, u);
    if (!live)
        return; // uniform across the CTA
    __syncthreads();

    W ws;
    ws.init(static_cast<const T *>(p.query) + ((size_t)s * H + h) * D, p.qk_scale_log2, lane);
    const int n_chunks = (u.n_tok + W::CHUNK - 1) / W::CHUNK;
    const int my_chunks = n_chunks <= warp ? 0 : (n_chunks - warp + NW - 1) / NW;
    if (p.new_key != nullptr && part == u.num_parts - 1 && u.n_tok > 0) {
        // This CTA holds the sequence's last token: the warp owning its
        // chunk puts the new K/V row in place (shared memory and cache).
        const int c_last = (u.n_tok - 1) / W::CHUNK;
        if (c_last % NW == warp) {
            constexpr int RV = D * 2 / 16;
            ws.patch_i = c_last / NW;
            ws.patch_row = (u.n_tok - 1) - c_last * W::CHUNK;
            if (lane < 2 * RV) {
                const bool isv = lane >= RV;
                const int e = lane % RV;
                ws.patch_val = reinterpret_cast<const uint4 *>(isv ? p.new_value : p.new_key)
                    [((size_t)s * H + h) * RV + e];
                const int b = table[(u.n_tok - 1) / BS];
                if (b >= 0 && b < p.num_blocks) {
                    T *cache = const_cast<T *>(
                        static_cast<const T *>(isv ? p.value_cache : p.key_cache));
                    ws.patch_dst = reinterpret_cast<uint4 *>(
                                       cache + (size_t)b * H * BS * D + (size_t)h * BS * D +
                                       (size_t)((u.n_tok - 1) % BS) * D) +
                                   e;
                }
            }
        }
    }
    const bool ok = ws.run(static_cast<const T *>(p.key_cache),
                           static_cast<const T *>(p.value_cache), (size_t)h * BS * D,
                           (size_t)H * BS * D, p.num_blocks, table, u.n_tok, warp, NW,
                           my_chunks, rings + (size_t)warp * NS * 2 * W::TILE,
                           smem_addr(&bars[warp * NS]));
    if (lane == 0) {
        if (!ok) {
            report(p.dev_err, PA_DEVERR_TIMEOUT);
            atomicOr(&cta_flags, 2);
        }
        if (ws.bad_id)
            atomicOr(&cta_flags, 1);
    }
    ws.finish();
    float *mw = merge + warp * (D + 2);
    if (lane < LPR) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                mw[(ws.qd + LPR * j) * 8 + e] = ws.acc[j][e];
    }
    if (lane == 0) {
        mw[D] = ws.m;
        mw[D + 1] = ws.l;
    }
    __syncthreads();

    const bool failed = cta_flags != 0;
    if (tid == 0 && (cta_flags & 1))
        report(p.dev_err, PA_DEVERR_BLOCK_ID);
    for (int d = tid; d < D; d += NW * 32) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, merge[w * (D + 2) + D]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(merge[w * (D + 2) + D] - M);
                L = fmaf(merge[w * (D + 2) + D + 1], f, L);
                O = fmaf(merge[w * (D + 2) + d], f, O);
            }
        }
        if (failed)
            O = NAN;
        if (u.num_parts == 1) {
            store_out(p.out, p.out_dtype, ((size_t)s * H + h) * D + d, L > 0.f ? O / L : O);
        } else {
            const size_t unit = ((size_t)s * H + h) * p.num_parts + part;
            p.ws_acc[unit * D + d] = O;
            if (d == 0) {
                p.ws_ml[unit * 2] = failed ? 0.f : M;
                p.ws_ml[unit * 2 + 1] = failed ? 1.f : L;
            }
        }
    }
}

// Merge the partitions of every split sequence:
// M = max_p m_p, L = sum_p l_p 2^(m_p - M), out = sum_p o_p 2^(m_p - M) / L.
template <int D>
__global__ void __launch_bounds__(D) reduce_kernel(const __grid_constant__ DecodeParams p,
                                                   int block_size)
{
    pdl_wait_prior_grid();
    const int h = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
    const int ctx = checked_context(p, p.context_lens[s], block_size, false);
    const int P = p.partition_size;
    const int num_parts = ctx > 0 ? (ctx + P - 1) / P : 1;
    if (num_parts <= 1)
        return;
    const size_t unit0 = ((size_t)s * p.num_heads + h) * p.num_parts;
    float M = -INFINITY;
    for (int i = 0; i < num_parts; ++i)
        M = fmaxf(M, p.ws_ml[(unit0 + i) * 2]);
    float L = 0.f, O = 0.f;
    for (int i = 0; i < num_parts; ++i) {
        const float f = exp2f(p.ws_ml[(unit0 + i) * 2] - M);
        L = fmaf(p.ws_ml[(unit0 + i) * 2 + 1], f, L);
        O = fmaf(p.ws_acc[(unit0 + i) * D + d], f, O);
    }
    store_out(p.out, p.out_dtype, ((size_t)s * p.num_heads + h) * D + d, O / L);
}

} // namespace pagedkv
