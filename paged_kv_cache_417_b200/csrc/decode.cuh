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
// sum, unnormalised output) per partition in the workspace, and the last of
// its CTAs to finish merges them with the log-sum-exp rule (merge_if_last;
// reduce_kernel does it when the workspace has no arrival counters).
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
#include <cuda_fp8.h>

#include <cstdint>
#include <type_traits>

#include "pagedkv.h"
#include "ptx.cuh"

namespace pagedkv {

constexpr uint64_t kWaitLimitNs = 1000000000ull; // 1 s: far above any copy latency
constexpr int kMaxPartition = 8192;              // tokens per work unit, upper bound
constexpr int kSplitCounters = 65536;            // arrival counters in a split workspace

struct DecodeParams {
    void *out;
    const void *query;
    const void *key_cache;
    const void *value_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *ws_acc; // [S][H][num_parts][D]
    float *ws_ml;  // [S][H][num_parts][2] = (max, sum), base-2 domain
    // Arrival counters of split units, zero between calls: the last CTA of
    // a split (sequence, head slot) merges its partitions. NULL: a separate
    // reduce_kernel merges instead.
    int32_t *ws_count;
    int32_t *dev_err;
    int32_t num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq, max_context_len;
    int32_t partition_size, num_parts;
    int32_t rank_seqs; // 1: grid row y takes the sequence of rank y (ranked_sequence)
    int32_t out_dtype; // 0 f16, 1 bf16, 2 f32
    float qk_scale_log2;
    // Fused append (pa_write_kv_decode): the new token of sequence s, at
    // position context_lens[s] - 1, has K/V rows new_key/new_value[s][kv head][:];
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

template <typename T> __device__ __forceinline__ void unpack8_to(const uint4 &raw, float *f)
{
    float2 a = Elem<T>::pair(raw.x), b = Elem<T>::pair(raw.y);
    float2 c = Elem<T>::pair(raw.z), d = Elem<T>::pair(raw.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &raw, float (&f)[8])
{
    unpack8_to<T>(raw, f);
}

// Storage tag of an fp8 cache: OCP e4m3 codes, one fp32 scale per row.
struct E4M3 {};

// Four e4m3 codes (little-endian bytes of u) to two f16 pairs (codes 0, 1
// in lo; 2, 3 in hi; exact), with the hardware e4m3x2 -> f16x2 conversion
// applied to the register's two 16-bit halves directly.
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t u, uint32_t &lo, uint32_t &hi)
{
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(u));
}

// An f16 pair (low half first) to two floats.
__device__ __forceinline__ float2 h2_to_float2(uint32_t h)
{
    float2 f;
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\t"
        "cvt.f32.f16 %1, b;\n\t}"
        : "=f"(f.x), "=f"(f.y)
        : "r"(h));
    return f;
}

// Four e4m3 codes (little-endian bytes of u) to floats (exact).
__device__ __forceinline__ void e4m3x4_to_float(uint32_t u, float *f)
{
    uint32_t lo, hi;
    e4m3x4_to_h2x2(u, lo, hi);
    const float2 fa = h2_to_float2(lo), fb = h2_to_float2(hi);
    f[0] = fa.x; f[1] = fa.y; f[2] = fb.x; f[3] = fb.y;
}

// Mixed-precision FMAs of sm_100 (fp32 accumulator, f16 multiplicands):
// d = c + a.lo*b.lo + a.hi*b.hi for f16 pairs a, b (the products are exact in
// fp32), and (c0, c1) += p * (v.lo, v.hi).
__device__ __forceinline__ float fma2_f16(uint32_t a, uint32_t b, float c)
{
    float d;
    asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %3;\n\tfma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void axpy2_f16(uint16_t p, uint32_t v, float &c0, float &c1)
{
    asm("{\n\t.reg .f16 v0, v1;\n\tmov.b32 {v0, v1}, %2;\n\t"
        "fma.rn.f32.f16 %0, %3, v0, %0;\n\tfma.rn.f32.f16 %1, %3, v1, %1;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "r"(v), "h"(p));
}

// Packed fp32 FMA of sm_100: (d0, d1) = (a0*b0 + d0, a1*b1 + d1).
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rd, {%0, %1};\n\tfma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Bytes of K codes per stage for fp8 caches (16-bit caches: 4 KiB).
#ifndef PA_FP8_STAGE_BYTES
#define PA_FP8_STAGE_BYTES 2048
#endif

// Which arithmetic the stream uses. The macros exist for tuning sweeps.
#ifndef PA_QK_MIXED
#define PA_QK_MIXED 1 // q.k with fma.rn.f32.f16 for f16 queries on f16 or fp8 caches
#endif
#ifndef PA_FFMA2
#define PA_FFMA2 1 // packed fp32 FMAs on the fp32 (non-mixed) paths
#endif
#ifndef PA_PV_MIXED
#define PA_PV_MIXED 1 // p.v with fma.rn.f32.f16 (p rounded to f16) for f16 caches
#endif

// Cached element formats. kPer16: elements per 16-byte load.
template <typename T> struct Store {
    static constexpr int kBytes = 2, kPer16 = 8;
    static constexpr bool kScaled = false;
    static __device__ __forceinline__ void unpack(const uint4 &raw, float (&f)[8])
    {
        unpack8<T>(raw, f);
    }
    // The 16 bytes as f16 pairs (meaningful for __half storage).
    static __device__ __forceinline__ void to_h2(const uint4 &raw, uint32_t (&w)[4])
    {
        w[0] = raw.x; w[1] = raw.y; w[2] = raw.z; w[3] = raw.w;
    }
};
template <> struct Store<E4M3> {
    static constexpr int kBytes = 1, kPer16 = 16;
    static constexpr bool kScaled = true;
    static __device__ __forceinline__ void unpack(const uint4 &raw, float (&f)[16])
    {
        e4m3x4_to_float(raw.x, f);
        e4m3x4_to_float(raw.y, f + 4);
        e4m3x4_to_float(raw.z, f + 8);
        e4m3x4_to_float(raw.w, f + 12);
    }
    // 16 codes as 8 f16 pairs (e4m3 values are exact in f16).
    static __device__ __forceinline__ void to_h2(const uint4 &raw, uint32_t (&w)[8])
    {
        const uint32_t c[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            e4m3x4_to_h2x2(c[k], w[2 * k], w[2 * k + 1]);
    }
};

// Quantise 16 floats with a precomputed 448/amax to e4m3 codes (round to
// nearest even, saturating at 448), packed little-endian.
__device__ __forceinline__ uint4 quantize16_e4m3(const float (&x)[16], float inv)
{
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
            make_float2(x[4 * k] * inv, x[4 * k + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(x[4 * k + 2] * inv, x[4 * k + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        w[k] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
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

// Geometry of a warp's stream for cache format T (a 16-bit type or E4M3).
// Every lane holds 32 dims of a row, as J 16-byte pieces of E elements.
template <typename T, int D, int BS, int NS> struct ChunkCfg {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    using S = Store<T>;
    static constexpr int kE = S::kPer16;                   // elements per 16 bytes
    static constexpr int kJ = 32 / kE;                     // 16-byte pieces per lane and row
    static constexpr int kLPR = D / 32;                    // lanes per row
    static constexpr int kRPS = 32 / kLPR;                 // rows per warp step
    static constexpr int kQR = 8 / kLPR;                   // rows per quarter-warp
    static constexpr int kRow = D * S::kBytes;             // bytes of a cached row
    static constexpr int kRow16 = kRow / 16;
    static constexpr int kChunk = (S::kScaled ? PA_FP8_STAGE_BYTES : 4096) / kRow; // rows per stage
    static constexpr int kSteps = kChunk / kRPS;
    static constexpr int kSeg = BS < kChunk ? BS : kChunk; // rows per bulk copy
    static constexpr int kTileBytes = BS * kRow + (S::kScaled ? 4 * BS : 0); // (block, head)
    static constexpr int kData = kChunk * kRow;            // K (or V) codes of a stage
    static constexpr int kScales = S::kScaled ? 4 * kChunk : 0;
    static constexpr int kStage = 2 * (kData + kScales);
    static constexpr int kRingBytes = NS * kStage;         // one warp's stages
    static_assert(kSteps >= 1 && kChunk % kRPS == 0, "chunk geometry");
    static_assert((kRow16 % 8 == 0 && kQR <= kJ) || (kRow16 == 4 && kJ == 2 && kQR == 4),
                  "swizzle");
    static_assert(kChunk % 4 == 0, "scale copies start 16-byte aligned");
    static_assert(kTileBytes % 16 == 0 && kData % 16 == 0 && kScales % 16 == 0, "alignment");
};

// One warp's online-softmax state over the chunks it streamed. After
// finish(), lanes with r == 0 (lane < D/32) hold the warp's sums for dims
// (qd + LPR*j)*E + e, j < J, e < E; every lane holds m and l.
template <typename T, typename QT, int D, int BS, int NS> struct WarpStream {
    using C = ChunkCfg<T, D, BS, NS>;
    using S = typename C::S;
    static constexpr int LPR = C::kLPR, RPS = C::kRPS, QR = C::kQR, CHUNK = C::kChunk;
    static constexpr int STEPS = C::kSteps, E = C::kE, J = C::kJ, ROW = C::kRow;
    static constexpr int DATA = C::kData, SCL = C::kScales, STAGE = C::kStage;
    static constexpr unsigned FULL = 0xffffffffu;
    // q.k on raw f16 query pairs with mixed FMAs (f16 caches, and fp8 codes
    // widened to exact f16 pairs), the scale applied per row; else on fp32
    // copies of the query pre-scaled by scale*log2(e).
    static constexpr bool kQKMixed =
        PA_QK_MIXED && std::is_same<QT, __half>::value &&
        (std::is_same<T, __half>::value || std::is_same<T, E4M3>::value);
    static constexpr bool kPVMixed = PA_PV_MIXED && std::is_same<T, __half>::value;

    float qf[kQKMixed ? 1 : J][kQKMixed ? 1 : E];
    uint32_t qh[kQKMixed ? J : 1][kQKMixed ? E / 2 : 1];
    float qscale;
    float acc[J][E];
    float m, l;
    int qd, r, rx, lane;
    int bad_id; // lane 0: a block id outside the pool was met
    // Fused append: local chunk patch_i holds the new token at row
    // patch_row. Lanes < 2*ROW/16 carry 16 bytes of its K (then V) row in
    // patch_val (fp8: codes, plus the row scale in patch_scale on the first
    // lane of each half), which replace that row in shared memory once the
    // chunk has landed and go to the cache at patch_dst / patch_sdst (NULL:
    // the block id was bad).
    int patch_i, patch_row;
    uint4 patch_val;
    float patch_scale;
    uint4 *patch_dst;
    float *patch_sdst;

    // XOR key of the 16-byte piece a lane of row r reads in slot j, chosen
    // so the 8 lanes of a quarter-warp hit 8 distinct bank groups.
    static __device__ __forceinline__ int swizzle_key(int row)
    {
        if constexpr (C::kRow16 % 8 == 0)
            return row & (QR - 1);
        else
            return (row >> 1) & (J - 1);
    }

    __device__ __forceinline__ void init(const QT *q, float qk_scale_log2, int lane_)
    {
        lane = lane_;
        qd = lane % LPR;
        r = lane / LPR;
        rx = swizzle_key(r);
        qscale = qk_scale_log2;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int u = qd + LPR * (j ^ rx);
#pragma unroll
            for (int h8 = 0; h8 < E / 8; ++h8) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(q + u * E + h8 * 8);
                if constexpr (kQKMixed) {
                    qh[j][h8 * 4 + 0] = raw.x;
                    qh[j][h8 * 4 + 1] = raw.y;
                    qh[j][h8 * 4 + 2] = raw.z;
                    qh[j][h8 * 4 + 3] = raw.w;
                } else {
                    float t[8];
                    unpack8<QT>(raw, t);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        qf[j][h8 * 8 + e] = t[e] * qk_scale_log2;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[j][h8 * 8 + e] = 0.f;
            }
        }
        m = -INFINITY;
        l = 0.f;
        bad_id = 0;
        patch_i = -1;
        patch_row = 0;
        patch_scale = 0.f;
        patch_dst = nullptr;
        patch_sdst = nullptr;
    }

    // Stream chunks c0, c0 + cstride, ... (count of them) of a unit with
    // n_tok tokens whose block ids are table[0..]. kc/vc are the pools'
    // bytes; a block's tile for this head starts at b * block_bytes +
    // head_off. Lane 0 issues the copies; an id outside [0, num_blocks) is
    // replaced by block 0 and sets bad_id. Returns false if a wait ran out of
    // time (the copies in flight have been waited for, boundedly, before
    // returning).
    __device__ __forceinline__ bool run(const char *kc, const char *vc, size_t head_off,
                                        size_t block_bytes, int num_blocks,
                                        const int32_t *table, int n_tok, int c0, int cstride,
                                        int count, char *ring, uint32_t bar0)
    {
        auto issue = [&](int i) {
            const int tok0 = (c0 + i * cstride) * CHUNK;
            const int rows = min(CHUNK, n_tok - tok0);
            const int st = i % NS;
            char *dk = ring + st * STAGE;
            char *dks = dk + DATA;
            char *dv = dks + SCL;
            char *dvs = dv + DATA;
            const uint32_t bar = bar0 + st * 8;
            uint32_t tx = 2u * rows * ROW;
            if constexpr (S::kScaled) // one 4-byte scale per row, copied 16 bytes at a time
                tx += 2u * ((rows / C::kSeg) * C::kSeg + ((rows % C::kSeg + 3) & ~3)) * 4u;
            mbar_arrive_expect_tx(bar, tx);
            for (int r0 = 0; r0 < rows; r0 += C::kSeg) {
                const int tok = tok0 + r0;
                int b = table[tok / BS];
                if (b < 0 || b >= num_blocks) {
                    bad_id = 1;
                    b = 0;
                }
                const int rb = min(C::kSeg, rows - r0);
                const size_t tile = (size_t)b * block_bytes + head_off;
                const size_t src = tile + (size_t)(tok % BS) * ROW;
                bulk_g2s(smem_addr(dk + r0 * ROW), kc + src, (uint32_t)(rb * ROW), bar);
                bulk_g2s(smem_addr(dv + r0 * ROW), vc + src, (uint32_t)(rb * ROW), bar);
                if constexpr (S::kScaled) {
                    const size_t ssrc = tile + (size_t)BS * ROW + (size_t)(tok % BS) * 4;
                    const uint32_t sb = (uint32_t)((rb + 3) & ~3) * 4u;
                    bulk_g2s(smem_addr(dks + r0 * 4), kc + ssrc, sb, bar);
                    bulk_g2s(smem_addr(dvs + r0 * 4), vc + ssrc, sb, bar);
                }
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
            char *sk = ring + st * STAGE;
            const float *sks = reinterpret_cast<const float *>(sk + DATA);
            char *sv = sk + DATA + SCL;
            const float *svs = reinterpret_cast<const float *>(sv + DATA);
            if (i == patch_i) { // warp-uniform
                constexpr int RV = ROW / 16;
                if (lane < 2 * RV) {
                    char *base = lane >= RV ? sv : sk;
                    reinterpret_cast<uint4 *>(base + patch_row * ROW)[lane % RV] = patch_val;
                    if (patch_dst)
                        *patch_dst = patch_val;
                    if constexpr (S::kScaled) {
                        if (lane % RV == 0) {
                            reinterpret_cast<float *>(base + DATA)[patch_row] = patch_scale;
                            if (patch_sdst)
                                *patch_sdst = patch_scale;
                        }
                    }
                    fence_proxy_async_smem(); // before the stage is refilled by a bulk copy
                }
                __syncwarp();
            }

            float sc[STEPS];
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int row = t * RPS + r;
                const char *kr = sk + row * ROW;
                float dot = 0.f;
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const uint4 raw =
                        *reinterpret_cast<const uint4 *>(kr + (qd + LPR * (j ^ rx)) * 16);
                    if constexpr (kQKMixed) {
                        uint32_t kh[E / 2];
                        S::to_h2(raw, kh);
#pragma unroll
                        for (int w = 0; w < E / 2; ++w)
                            dot = fma2_f16(qh[j][w], kh[w], dot);
                    } else {
                        float kf[E];
                        S::unpack(raw, kf);
                        if constexpr (PA_FFMA2) {
                            float d1 = 0.f;
#pragma unroll
                            for (int e = 0; e < E; e += 2)
                                ffma2(dot, d1, qf[j][e], qf[j][e + 1], kf[e], kf[e + 1]);
                            dot += d1;
                        } else {
#pragma unroll
                            for (int e = 0; e < E; ++e)
                                dot = fmaf(qf[j][e], kf[e], dot);
                        }
                    }
                }
#pragma unroll
                for (int o = 1; o < LPR; o <<= 1)
                    dot += __shfl_xor_sync(FULL, dot, o);
                if constexpr (kQKMixed)
                    dot *= qscale;
                if constexpr (S::kScaled)
                    dot *= sks[row];
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
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    acc[j][e] *= corr;
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int row = t * RPS + r;
                const float pt = exp2f(sc[t] - m_new);
                l += pt;
                if (row < rows) {
                    const char *vr = sv + row * ROW;
                    float pv = pt;
                    if constexpr (S::kScaled)
                        pv *= svs[row];
                    if constexpr (kPVMixed) {
                        const uint16_t ph = __half_as_ushort(__float2half_rn(pv));
#pragma unroll
                        for (int j = 0; j < J; ++j) {
                            uint32_t vh[E / 2];
                            S::to_h2(*reinterpret_cast<const uint4 *>(
                                         vr + (qd + LPR * (j ^ rx)) * 16),
                                     vh);
#pragma unroll
                            for (int w = 0; w < E / 2; ++w)
                                axpy2_f16(ph, vh[w], acc[j][2 * w], acc[j][2 * w + 1]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < J; ++j) {
                            float vf[E];
                            S::unpack(*reinterpret_cast<const uint4 *>(
                                          vr + (qd + LPR * (j ^ rx)) * 16),
                                      vf);
                            if constexpr (PA_FFMA2) {
#pragma unroll
                                for (int e = 0; e < E; e += 2)
                                    ffma2(acc[j][e], acc[j][e + 1], pv, pv, vf[e], vf[e + 1]);
                            } else {
#pragma unroll
                                for (int e = 0; e < E; ++e)
                                    acc[j][e] = fmaf(pv, vf[e], acc[j][e]);
                            }
                        }
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

    // Put the swizzled slots back in order (slot j <- piece qd + LPR*j) and
    // sum acc and l over the rows the warp's lanes covered.
    __device__ __forceinline__ void finish()
    {
        if (rx & 1) {
#pragma unroll
            for (int j = 0; j < J; j += 2)
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    float t0 = acc[j][e]; acc[j][e] = acc[j + 1][e]; acc[j + 1][e] = t0;
                }
        }
        if constexpr (J >= 4) {
            if (rx & 2) {
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        float t0 = acc[j][e]; acc[j][e] = acc[j + 2][e]; acc[j + 2][e] = t0;
                    }
            }
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
            l += __shfl_xor_sync(FULL, l, o);
#pragma unroll
            for (int j = 0; j < J; ++j)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    acc[j][e] += __shfl_xor_sync(FULL, acc[j][e], o);
        }
    }
};

// Merge partitions of query head h of sequence s (unit0 = its first
// partial): M = max_p m_p, L = sum_p l_p 2^(m_p - M), out = sum_p o_p 2^(m_p
// - M) / L. Loads bypass L1 (the partials were written by other CTAs).
template <int D>
__device__ __forceinline__ void merge_partitions(const DecodeParams &p, int s, int h, int d,
                                                 int num_parts)
{
    const size_t unit0 = ((size_t)s * p.num_heads + h) * p.num_parts;
    float M = -INFINITY;
    for (int i = 0; i < num_parts; ++i)
        M = fmaxf(M, __ldcg(&p.ws_ml[(unit0 + i) * 2]));
    float L = 0.f, O = 0.f;
    for (int i = 0; i < num_parts; ++i) {
        const float f = exp2f(__ldcg(&p.ws_ml[(unit0 + i) * 2]) - M);
        L = fmaf(__ldcg(&p.ws_ml[(unit0 + i) * 2 + 1]), f, L);
        O = fmaf(__ldcg(&p.ws_acc[(unit0 + i) * D + d]), f, O);
    }
    store_out(p.out, p.out_dtype, ((size_t)s * p.num_heads + h) * D + d, O / L);
}

// Most output elements a thread merges in merge_if_last (16 heads x D 128
// over 128 threads).
constexpr int kMergeOutPerThread = 16;

// Arrival on a split counter: an atomic add with acquire-release semantics
// at GPU scope. Release publishes every write the CTA ordered before it
// (its barrier); acquire lets the last arriver see all earlier arrivers'
// writes.
__device__ __forceinline__ int arrive_acq_rel(int32_t *counter)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(counter)
                 : "memory");
    return old;
}

// Called by every thread of a CTA that has just written the partials of
// query heads h0 .. h0+nh-1 of sequence s: counts the CTA in on counter
// `slot`; the CTA that completes the count (the last of the num_parts
// partitions to finish) merges those heads into the output and resets the
// counter to zero for the next call (the classic last-block pattern). The
// merge turns each head's (m, l) pairs into normalised weights
// 2^(m_p - M) / L in shared memory `wbuf` (nh * num_parts floats; one warp
// per head, each lane holding up to kMergeLanePairs pairs, all heads' loads
// issued before any reduction), then every thread sums its output elements
// over the partitions with all loads of a partition issued together. The
// host guarantees nh * num_parts <= the buffer and nh * D <=
// kMergeOutPerThread * nthreads.
constexpr int kMergeLanePairs = 4; // partitions per lane held in registers
template <int D>
__device__ __forceinline__ void merge_if_last(const DecodeParams &p, int s, int h0, int nh,
                                              int slot, int num_parts, int tid, int nthreads,
                                              int *flag, float *wbuf)
{
    __syncthreads();
    if (tid == 0)
        *flag = arrive_acq_rel(&p.ws_count[slot]) == num_parts - 1;
    __syncthreads();
    if (!*flag)
        return;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads >> 5;
    const float2 *ml0 = reinterpret_cast<const float2 *>(p.ws_ml) +
                        ((size_t)s * p.num_heads + h0) * p.num_parts;
    for (int g0 = warp; g0 < nh; g0 += nwarps * kMergeLanePairs) {
        // Up to kMergeLanePairs heads per pass (g0, g0 + nwarps, ...), when
        // every lane holds its partitions of them in registers; else one.
        const bool fits = num_parts <= 32;
        float2 v[kMergeLanePairs];
#pragma unroll
        for (int j = 0; j < kMergeLanePairs; ++j) {
            const int g = g0 + j * nwarps;
            v[j] = make_float2(-INFINITY, 0.f);
            if (fits && g < nh && lane < num_parts)
                v[j] = __ldcg(ml0 + (size_t)g * p.num_parts + lane);
        }
#pragma unroll
        for (int j = 0; j < kMergeLanePairs; ++j) {
            const int g = g0 + j * nwarps;
            if (g >= nh || (!fits && j > 0))
                continue; // warp-uniform
            const float2 *ml = ml0 + (size_t)g * p.num_parts;
            float M = v[j].x;
            if (!fits)
                for (int i = lane; i < num_parts; i += 32)
                    M = fmaxf(M, __ldcg(ml + i).x);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            float L = lane < num_parts && fits ? v[j].y * exp2f(v[j].x - M) : 0.f;
            if (!fits)
                for (int i = lane; i < num_parts; i += 32) {
                    const float2 q = __ldcg(ml + i);
                    L = fmaf(q.y, exp2f(q.x - M), L);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                L += __shfl_xor_sync(0xffffffffu, L, o);
            if (fits) {
                if (lane < num_parts)
                    wbuf[g * num_parts + lane] = exp2f(v[j].x - M) / L;
            } else {
                for (int i = lane; i < num_parts; i += 32)
                    wbuf[g * num_parts + i] = exp2f(__ldcg(ml + i).x - M) / L;
            }
        }
        if (!fits)
            g0 -= nwarps * (kMergeLanePairs - 1); // advance by one head per warp
    }
    __syncthreads();
    float O[kMergeOutPerThread];
#pragma unroll
    for (int k = 0; k < kMergeOutPerThread; ++k)
        O[k] = 0.f;
    const float *acc0 = p.ws_acc + ((size_t)s * p.num_heads + h0) * p.num_parts * D;
    for (int i = 0; i < num_parts; ++i) {
#pragma unroll
        for (int k = 0; k < kMergeOutPerThread; ++k) {
            const int idx = tid + k * nthreads;
            if (idx < nh * D) {
                const int g = idx / D, d = idx - g * D;
                O[k] = fmaf(__ldcg(acc0 + ((size_t)g * p.num_parts + i) * D + d),
                            wbuf[g * num_parts + i], O[k]);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kMergeOutPerThread; ++k) {
        const int idx = tid + k * nthreads;
        if (idx < nh * D) {
            const int g = idx / D, d = idx - g * D;
            store_out(p.out, p.out_dtype, ((size_t)s * p.num_heads + h0 + g) * D + d, O[k]);
        }
    }
    if (tid == 0)
        p.ws_count[slot] = 0;
}

// Longest sequences first: when DecodeParams::rank_seqs is set (batches of
// up to kRankMaxSeqs sequences; the host decides per launch), a CTA on grid
// row y works on the sequence of rank y by (context length descending,
// index ascending), so the hardware hands out the longest units first and a
// launch ends on short ones (a per-CTA timeline of the grouped kernel on the
// Llama-7B layer showed a ~12 us drain of long last CTAs). Any order gives
// the same outputs. The ranking costs each CTA a dependent round trip for
// all context lengths and O(S^2 / threads) compares.
constexpr int kRankMaxSeqs = 128;

// Every thread of the CTA calls it (two barriers): the sequence of rank y.
// ctx_buf: kRankMaxSeqs ints of 16-byte aligned shared memory; out: one
// shared int. Sequence k gets the key (min(max(len, 0), 2^24 - 1) << 7) |
// (127 - k): keys are distinct, larger for longer sequences and, among equal
// (or clamped) lengths, for smaller indices; the rank of k is the number of
// larger keys, a permutation of 0 .. S-1 whatever the lengths. Keys are
// padded with -1 (below every key) to a multiple of 4 and compared four at
// a time.
__device__ __forceinline__ int ranked_sequence(const int32_t *context_lens, int S, int y,
                                               int tid, int nthreads, int32_t *ctx_buf, int *out)
{
    const int S4 = (S + 3) >> 2;
    for (int k = tid; k < 4 * S4; k += nthreads)
        ctx_buf[k] = k < S ? (min(max(context_lens[k], 0), (1 << 24) - 1) << 7) | (127 - k) : -1;
    __syncthreads();
    const int4 *c4 = reinterpret_cast<const int4 *>(ctx_buf);
    for (int k = tid; k < S; k += nthreads) {
        const int c = ctx_buf[k];
        int r = 0;
#pragma unroll 4
        for (int j = 0; j < S4; ++j) {
            const int4 v = c4[j];
            r += (v.x > c) + (v.y > c) + (v.z > c) + (v.w > c);
        }
        if (r == y)
            *out = k; // ranks are a permutation: exactly one writer
    }
    __syncthreads();
    return *out;
}

// Shared prologue: read the context length and the partition's slice of the
// block table at the same time (one global latency). Returns false when the
// partition is past the sequence (the whole CTA returns).
struct UnitInfo {
    int ctx, num_parts, start, n_tok;
};

template <int BS>
__device__ __forceinline__ bool load_unit(const DecodeParams &p, int s, int part, int P, int tid,
                                          int nthreads, bool report_ctx, int32_t *table,
                                          UnitInfo &u)
{
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
    static constexpr int kRankBytes = kRankMaxSeqs * 4;
    static constexpr int kFixedBytes = kRingsBytes + kBarBytes + kMergeBytes + kRankBytes;
    static_assert((kRingsBytes + kBarBytes + kMergeBytes) % 16 == 0, "ranking buffer alignment");
    static size_t smem_bytes(int partition)
    {
        return kFixedBytes + ((partition / BS) * 4 + 15) / 16 * 16;
    }
};

// T: cache format (__half, __nv_bfloat16 or E4M3); QT: query / new-row /
// output-element type (T itself for 16-bit caches).
template <typename T, typename QT, int D, int BS, int NW, int NS>
__global__ void __launch_bounds__(NW * 32)
    decode_split_kernel(const __grid_constant__ DecodeParams p)
{
    using W = WarpStream<T, QT, D, BS, NS>;
    using Cfg = SplitCfg<T, D, BS, NW, NS>;
    constexpr int LPR = W::LPR, E = W::E, J = W::J, ROW = W::ROW;
    constexpr int TILE = W::C::kTileBytes;
    extern __shared__ __align__(128) unsigned char smem[];
    char *rings = reinterpret_cast<char *>(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kRingsBytes);
    float *merge = reinterpret_cast<float *>(smem + Cfg::kRingsBytes + Cfg::kBarBytes);
    int32_t *rank_ctx = reinterpret_cast<int32_t *>(smem + Cfg::kRingsBytes + Cfg::kBarBytes +
                                                    Cfg::kMergeBytes);
    int32_t *table = reinterpret_cast<int32_t *>(smem + Cfg::kFixedBytes);
    __shared__ int cta_flags, ranked_seq;

    // Dependent kernels (the reduce, the next layer's write) may launch now;
    // each of them waits for this grid before it touches data.
    pdl_launch_dependents();
    const int h = blockIdx.x, part = blockIdx.z;
    int s = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads, HK = p.num_kv_heads;
    const int group = H / HK;  // query heads per K/V head
    const int kvh = h / group; // the K/V head this query head reads

    if (tid == 0)
        cta_flags = 0;
    if (lane == 0)
        for (int k = 0; k < NS; ++k)
            mbar_init(smem_addr(&bars[warp * NS + k]), 1);
    fence_mbar_init();
    pdl_wait_prior_grid(); // every input may come from the previous kernel
    if (p.rank_seqs)
        s = ranked_sequence(p.context_lens, p.num_seqs, blockIdx.y, tid, NW * 32, rank_ctx,
                            &ranked_seq);
    UnitInfo u;
    const bool live = load_unit<BS>(p, s, part, p.partition_size, tid, NW * 32,
                                    tid == 0 && h == 0 && part == 0, table, u);
    if (!live)
        return; // uniform across the CTA
    __syncthreads();

    W ws;
    ws.init(static_cast<const QT *>(p.query) + ((size_t)s * H + h) * D, p.qk_scale_log2, lane);
    const int n_chunks = (u.n_tok + W::CHUNK - 1) / W::CHUNK;
    const int my_chunks = n_chunks <= warp ? 0 : (n_chunks - warp + NW - 1) / NW;
    if (p.new_key != nullptr && part == u.num_parts - 1 && u.n_tok > 0) {
        // This CTA holds the sequence's last token: the warp owning its
        // chunk puts the new K/V row in place (shared memory and cache).
        const int c_last = (u.n_tok - 1) / W::CHUNK;
        if (c_last % NW == warp) { // warp-uniform
            constexpr int RV = ROW / 16; // lanes per cached row: K on lanes [0, RV), V after
            ws.patch_i = c_last / NW;
            ws.patch_row = (u.n_tok - 1) - c_last * W::CHUNK;
            const bool isv = lane >= RV;
            const int piece = lane % RV;
            const QT *src = static_cast<const QT *>(isv ? p.new_value : p.new_key) +
                            ((size_t)s * HK + kvh) * D + (size_t)piece * E;
            if constexpr (Store<T>::kScaled) {
                // Quantise the new row: amax over its D inputs, then
                // codes = e4m3(x * (448 / amax)) and scale = amax / 448.
                float x[16];
                float amax = 0.f;
                if (lane < 2 * RV) {
                    unpack8_to<QT>(*reinterpret_cast<const uint4 *>(src), x);
                    unpack8_to<QT>(*reinterpret_cast<const uint4 *>(src + 8), x + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        amax = fmaxf(amax, fabsf(x[e]));
                }
#pragma unroll
                for (int o = 1; o < RV; o <<= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(W::FULL, amax, o));
                if (lane < 2 * RV) {
                    const float inv = amax > 0.f ? 448.f / amax : 0.f;
                    ws.patch_val = quantize16_e4m3(x, inv);
                    ws.patch_scale = amax / 448.f;
                }
            } else {
                if (lane < 2 * RV)
                    ws.patch_val = *reinterpret_cast<const uint4 *>(src);
            }
            if (lane < 2 * RV && h % group == 0) { // one query head per group writes
                const int b = table[(u.n_tok - 1) / BS];
                if (b >= 0 && b < p.num_blocks) {
                    char *cache =
                        const_cast<char *>(static_cast<const char *>(isv ? p.value_cache
                                                                           : p.key_cache));
                    char *tile = cache + ((size_t)b * HK + kvh) * TILE;
                    const int off = (u.n_tok - 1) % BS;
                    ws.patch_dst = reinterpret_cast<uint4 *>(tile + (size_t)off * ROW) + piece;
                    if (Store<T>::kScaled && piece == 0)
                        ws.patch_sdst =
                            reinterpret_cast<float *>(tile + (size_t)BS * ROW) + off;
                }
            }
        }
    }
    const bool ok = ws.run(static_cast<const char *>(p.key_cache),
                           static_cast<const char *>(p.value_cache), (size_t)kvh * TILE,
                           (size_t)HK * TILE, p.num_blocks, table, u.n_tok, warp, NW, my_chunks,
                           rings + (size_t)warp * W::C::kRingBytes, smem_addr(&bars[warp * NS]));
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
        for (int j = 0; j < J; ++j)
#pragma unroll
            for (int e = 0; e < E; ++e)
                mw[(ws.qd + LPR * j) * E + e] = ws.acc[j][e];
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
    if (u.num_parts > 1 && p.ws_count)
        merge_if_last<D>(p, s, h, 1, s * H + h, u.num_parts, tid, NW * 32, &cta_flags,
                         reinterpret_cast<float *>(rings));
}

// Separate merge kernel, for grids with more (sequence, head) slots than a
// workspace holds counters: one CTA per (head, sequence).
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
    merge_partitions<D>(p, s, h, d, num_parts);
}

} // namespace pagedkv
