// decode_group.cuh - paged decode attention on warp-level tensor-core tiles
// for grouped query heads (num_heads = G * num_kv_heads, G <= 16) on
// sm_100a: 16-bit caches, and fp8 (e4m3) caches with f16 rows and head_dim
// 128 (2 <= G <= 16 for both; the kernel itself also handles G = 1).
//
// Query heads kvh*G .. kvh*G+G-1 all attend over K/V head kvh. A CTA takes
// the unit (K/V head kvh, sequence s, partition p) for the whole group, so
// each K/V byte crosses HBM once per group instead of once per query head,
// and the G query rows share every staged tile. The outputs, the split
// workspace and the merge of partitions are those of decode_split_kernel
// (per query head; the last CTA of a (K/V head, sequence) merges its G
// heads). The per-warp state and the math of one staged chunk are GroupWarp;
// the fused append's new rows, NewRow.
//
// Staging: each pool is viewed as a 3-D tensor for the TMA unit. 16-bit
// pools: (64 elements, D/64 128-byte units, rows), row = one token of one
// (block, head) tile, row index (block*Hkv + kvh)*bs + offset. fp8 pools:
// (D code bytes, bs rows, tiles), tile index block*Hkv + kvh, which steps
// over the tile's row scales. A warp's stage receives CH tokens of K and of
// V (16 at 16 bits, 32 at fp8: 8 KiB either way) through tiled copies
// (cp.async.bulk.tensor) of min(bs, 16) whole rows per box with the 128-byte
// swizzle: 16-byte piece c of 128-byte unit u of the stage lands at piece
// c ^ (u % 8). fp8 row scales follow by 1-D bulk copies into a small
// per-warp area. Every code area starts on a 1024-byte boundary; the 8 rows
// of an 8x8 ldmatrix tile hit 8 distinct bank groups when a row is one unit
// (fp8, 16-bit at D = 64) and 4 when it is two (2-way at D = 128).
//
// Math per 16-token step in one warp, on tensor-core tiles (mma.sync
// m16n8k16, f16/bf16 operands, fp32 accumulation), in one of two
// orientations. G <= 8 (GroupWarpT): S^T = K Q^T and O^T += V^T P^T, with
// tokens and d on the 16-row side of the tiles and the heads as their 8
// columns (described at GroupWarpT). G > 8 (GroupWarp), described here: the
// G query heads are the M rows, padded to 16 with zeros:
//   S = Q K^T      2 column tiles of 8 tokens x D/16 k-steps, K tiles by
//                  ldmatrix straight from the swizzled stage. fp8: a tile
//                  register holds 4 consecutive codes of one token; they are
//                  widened with the e4m3x2 -> f16x2 conversion into the two
//                  halves of the B fragment, and the query's k order is
//                  permuted the same way (any k order gives the same sum).
//                  The token's K scale multiplies its score.
//   online softmax in base 2 on the accumulator fragments: the 16 scores of
//                  a row live in one quad of lanes (2 shuffles per max);
//   O += P V       P goes from the S fragments into the A operand without
//                  leaving registers. 16-bit V tiles by ldmatrix.trans. fp8
//                  V: ldmatrix.trans on code pairs gives a lane tokens 2q,
//                  2q+1 at codes d = 2g, 2g+1 of a piece; one byte permute
//                  and the widening make the B fragments of two column
//                  tiles, d even and d odd (tile 2c + o: column n is d =
//                  16c + 2n + o). The token's V scale is
//                  folded into P relative to the largest V scale met so far
//                  (R): P' = p * s_v / R <= 1, so an f16 P' keeps its
//                  precision however small the scales; O is rescaled when R
//                  grows and multiplied by R at the end.
// P is rounded to the operand type for the product (the running sum keeps
// the fp32 weights). bf16 carries only 8 significant bits, so a bf16 P is
// split into a bf16 head and a bf16 remainder and multiplied twice, which
// keeps about 16 bits.
//
// Rows past the context (only in a partition's last step): their scores are
// set to -inf and their fp8 V scales to 0 by selection (never computed from
// the stale bytes), and the V rows of a partial last chunk are zeroed in
// shared memory before the product, so a weight of 0 meets a finite value
// (0 * NaN would otherwise reach the sum).
//
// These tiles are warp-sized on purpose: the group is at most 16 rows,
// below the 64-row minimum of a tcgen05 MMA, and the kernel is bound by HBM
// bandwidth, so the tensor cores only have to remove the per-element FMA,
// conversion and shuffle work of decode_split_kernel.
#pragma once

#include <cuda.h> // CUtensorMap (type only; maps are encoded on the host)

#include "decode.cuh"

namespace pagedkv {

constexpr int kGroupMaxHeads = 16;

struct GroupParams {
    CUtensorMap tk; // key pool (see the staging note above), 128B swizzle
    CUtensorMap tv; // value pool, same geometry
    DecodeParams p;
};

// Stage geometry of the grouped kernels (independent of the block size).
template <typename T, int D> struct GroupGeom {
    static_assert(D == 64 || D == 128, "head_dim");
    static constexpr bool kFp8 = std::is_same<T, E4M3>::value;
    static_assert(!kFp8 || D == 128, "fp8 rows of 128 bytes");
    static constexpr int kRow = D * (kFp8 ? 1 : 2);  // bytes per cached row
    static constexpr int kUnits = kRow / 128;        // 128-byte units per row
    static constexpr int kChunk = kFp8 ? 32 : 16;    // tokens per stage
    static constexpr int kHalf = kChunk * kRow;      // the K (or V) codes of a stage
    static constexpr int kStage = 2 * kHalf;
    static constexpr int kMergeStride = D + 4;       // a row's (O, m, l) in a merge area (16-byte rows)
    static_assert(kHalf % 1024 == 0, "swizzle atoms");

    // Piece p (16 bytes) of row t sits in unit t*kUnits + p/8 at position
    // (p % 8) ^ ((t*kUnits + p/8) % 8) of a swizzled stage.
    static __device__ __forceinline__ int piece_off(int t, int piece)
    {
        const int unit = t * kUnits + (piece >> 3);
        return unit * 128 + (((piece & 7) ^ (unit & 7)) << 4);
    }
};

template <typename T, int D, int BS, int NW, int NS> struct GroupCfg : GroupGeom<T, D> {
    using Geo = GroupGeom<T, D>;
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    static constexpr int kRing = NS * Geo::kStage;         // one warp's stages
    static constexpr int kSeg = BS < 16 ? BS : 16;         // rows per TMA box
    static constexpr int kRingsBytes = NW * kRing;
    static constexpr int kBarBytes = (NW * NS * 8 + 15) / 16 * 16; // mbarriers, 16-byte padded
    // fp8 row scales: per warp, [stage][K | V][kChunk] floats.
    static constexpr int kScaleBytes = Geo::kFp8 ? NW * NS * 2 * Geo::kChunk * 4 : 0;
    static constexpr int kRankBytes = kRankMaxSeqs * 4; // context lengths for ranking
    static constexpr int kFixedBytes = kRingsBytes + kBarBytes + kScaleBytes + kRankBytes;
    static_assert((kRingsBytes + kBarBytes + kScaleBytes) % 16 == 0, "ranking buffer alignment");
    // After its last chunk a warp of decode_group_kernel leaves (O, m, l) of
    // its rows in its ring; warp 0's ring then also holds, per row, the NW
    // weights of the warps and the row's (M, L) (kMergeWeights).
    static constexpr int kMergeWeights = kGroupMaxHeads * Geo::kMergeStride; // floats
    static_assert((kMergeWeights + kGroupMaxHeads * (NW + 2)) * 4 <= kRing,
                  "merge area fits a ring");
    static_assert((kSeg * Geo::kRow) % 1024 == 0, "swizzle atoms");
    static_assert(Geo::kChunk % kSeg == 0 && Geo::kChunk % 16 == 0, "chunk geometry");
    // 1 KiB of slack to align the rings to 1024 bytes.
    static size_t smem_bytes(int partition)
    {
        return 1024 + kFixedBytes + ((partition / BS) * 4 + 15) / 16 * 16;
    }
};

template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi)
{
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// The two floats a bf16 pair stands for.
__device__ __forceinline__ float2 unpack_bf2(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Transpose of an 8x8 tile of 16-bit elements held as one register per lane
// (lane l holds row l/4, columns 2(l%4), 2(l%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// One warp's share of a group: the G query rows of a (sequence, K/V head) as
// the A operand, the output accumulator fragments and the online-softmax
// state, and the math that consumes one staged chunk (the header comment
// above describes it), for 8 < G <= 16: both fragment row halves are live
// (G <= 8 takes GroupWarpT). T: __half, __nv_bfloat16 or E4M3.
template <typename T, int D> struct GroupWarp {
    using Geo = GroupGeom<T, D>;
    static constexpr bool kFp8 = Geo::kFp8;
    static constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    using QT = typename std::conditional<kFp8, __half, T>::type; // operand / row type
    static constexpr int CH = Geo::kChunk, ROW = Geo::kRow;
    static constexpr int KT = D / 16; // k-steps of q.k = pairs of 8-wide d tiles of O
    static constexpr int MS = Geo::kMergeStride;
    static constexpr unsigned FULL = 0xffffffffu;

    // Fragment coordinates: this lane holds rows g0 and g1 = g0 + 8 and, in
    // every 8-wide column tile, columns q2 and q2 + 1 (q = lane % 4).
    int lane, g0, g1, q, q2;
    // ldmatrix row addresses (rows within a 16-token step). 16-bit K
    // (non-transposed, B of S = Q K^T): lanes 0-7 / 8-15 / 16-23 / 24-31
    // give token rows 0-7 / 0-7 / 8-15 / 8-15 at pieces c / c+1 / c / c+1.
    // V (transposed, B of O = P V; fp8 on code pairs) and fp8 K
    // (non-transposed): rows 0-7 / 8-15 / 0-7 / 8-15 at pieces c / c / c+1 /
    // c+1, register = (token tile, piece).
    int kt, kc, vt, vc;
    uint32_t qa[KT][4]; // Q as the A operand, one 16x16 tile per k-step
    float o[2 * KT][4];
    float m0, m1, l0, l1;
    float vref; // fp8: largest V scale so far (R), floored at FLT_MIN
    float vinv; // fp8: 1 / vref

    static __device__ __forceinline__ int piece_off(int t, int piece)
    {
        return Geo::piece_off(t, piece);
    }

    // O tile j covers 8 d. 16-bit: d = 8j + q2 (+1 for the second
    // element). fp8, j = 2c + o: d = 16c + 2*q2 + o (+2 for the second), so
    // tiles 2c and 2c + 1 together hold d = 16c + 2*q2 .. 16c + 2*q2 + 3.
    // Elements 0, 1: row g0; 2, 3: row g1.
    __device__ __forceinline__ void store_row(float *row, int e, float scale) const
    {
#pragma unroll
        for (int j = 0; j < 2 * KT; j += 2) {
            if constexpr (kFp8) {
                const int d = 8 * j + 2 * q2; // 16c + 2*q2 with c = j / 2
                *reinterpret_cast<float2 *>(row + d) =
                    make_float2(o[j][e] * scale, o[j + 1][e] * scale);
                *reinterpret_cast<float2 *>(row + d + 2) =
                    make_float2(o[j][e + 1] * scale, o[j + 1][e + 1] * scale);
            } else {
                *reinterpret_cast<float2 *>(row + 8 * j + q2) =
                    make_float2(o[j][e] * scale, o[j][e + 1] * scale);
                *reinterpret_cast<float2 *>(row + 8 * j + 8 + q2) =
                    make_float2(o[j + 1][e] * scale, o[j + 1][e + 1] * scale);
            }
        }
    }

    __device__ __forceinline__ void init(int lane_)
    {
        lane = lane_;
        g0 = lane >> 2;
        g1 = g0 + 8;
        q = lane & 3;
        q2 = 2 * q;
        kt = kFp8 ? (lane & 7) + (((lane >> 3) & 1) << 3) : (lane & 7) + ((lane >> 4) << 3);
        kc = kFp8 ? lane >> 4 : (lane >> 3) & 1;
        vt = (lane & 7) + (((lane >> 3) & 1) << 3);
        vc = lane >> 4;
    }

    // The query rows of heads row0 .. row0 + G - 1 (row0 counts rows of D
    // elements); rows >= G are zero. k-slots (2q, 2q+1) / (2q+8, 2q+9) hold
    // d = 16kk + 2q (+1) / + 8 (+1); fp8: d = 16kk + 4q (+1) / + 2 (+1),
    // matching the widened K codes.
    __device__ __forceinline__ void load_q(const void *query, size_t row0, int G)
    {
        const uint32_t *qp = static_cast<const uint32_t *>(query); // element pairs
        const size_t r0 = (row0 + g0) * (D / 2);
        const size_t r1 = r0 + (size_t)8 * (D / 2);
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            const int c = kFp8 ? (16 * kk + 4 * q) / 2 : (16 * kk + q2) / 2;
            const int c2 = kFp8 ? c + 1 : c + 4;
            qa[kk][0] = g0 < G ? qp[r0 + c] : 0u;
            qa[kk][1] = g1 < G ? qp[r1 + c] : 0u;
            qa[kk][2] = g0 < G ? qp[r0 + c2] : 0u;
            qa[kk][3] = g1 < G ? qp[r1 + c2] : 0u;
        }
    }

    __device__ __forceinline__ void reset()
    {
#pragma unroll
        for (int j = 0; j < 2 * KT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[j][e] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
        vref = 1.17549435e-38f;
        vinv = 1.f / vref;
    }

    // One staged chunk: K codes at sk, V at sv (swizzled), fp8 row scales at
    // ksc / vsc, `rows` valid tokens (1 .. CH; only a unit's last chunk can
    // be partial), qs = scale * log2(e).
    __device__ __forceinline__ void chunk(char *sk, char *sv, const float *ksc, const float *vsc,
                                          int rows, float qs)
    {
        if (rows < CH) { // zero the V rows past the context
            for (int k = rows * (ROW / 16) + lane; k < CH * (ROW / 16); k += 32)
                reinterpret_cast<uint4 *>(sv)[k] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem(); // before the stage is refilled by a copy
            __syncwarp();
        }
        const uint32_t kb = smem_addr(sk), vb = smem_addr(sv);
#pragma unroll
        for (int sub = 0; sub < CH / 16; ++sub) {
            const int srows = rows - 16 * sub; // valid tokens of this step
            if (srows <= 0)
                break; // warp-uniform
            const int t0 = 16 * sub;

            // S = Q K^T for the step's 16 tokens, even and odd k-steps in
            // separate accumulators (two shorter dependency chains per tile).
            float sc[2][4], sd[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sc[j][e] = sd[j][e] = 0.f;
            if constexpr (kFp8) {
#pragma unroll
                for (int kp = 0; kp < KT / 2; ++kp) { // pieces 2kp, 2kp+1
                    uint32_t r[4];
                    ldsm_x4(kb + piece_off(t0 + kt, 2 * kp + kc), r);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kk = 2 * kp + h;
                        float(&acc0)[4] = h ? sd[0] : sc[0];
                        float(&acc1)[4] = h ? sd[1] : sc[1];
                        uint32_t b0l, b0h, b1l, b1h;
                        e4m3x4_to_h2x2(r[2 * h], b0l, b0h);
                        e4m3x4_to_h2x2(r[2 * h + 1], b1l, b1h);
                        mma_16816<false>(acc0, qa[kk], b0l, b0h);
                        mma_16816<false>(acc1, qa[kk], b1l, b1h);
                    }
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < KT; ++kk) {
                    uint32_t b[4];
                    ldsm_x4(kb + piece_off(t0 + kt, 2 * kk + kc), b);
                    mma_16816<kBf16>(kk & 1 ? sd[0] : sc[0], qa[kk], b[0], b[1]);
                    mma_16816<kBf16>(kk & 1 ? sd[1] : sc[1], qa[kk], b[2], b[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sc[j][e] += sd[j][e];

            // Online softmax (base 2). sc[j][e]: token t0 + 8j + q2 + (e & 1),
            // row g0 for e < 2, g1 otherwise.
            const bool partial = srows < 16; // warp-uniform
            float x[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float2 ks = make_float2(qs, qs);
                if constexpr (kFp8) {
                    const float2 k2 = *reinterpret_cast<const float2 *>(ksc + t0 + 8 * j + q2);
                    ks = make_float2(k2.x * qs, k2.y * qs);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x[j][e] = sc[j][e] * ((e & 1) ? ks.y : ks.x);
            }
            if (partial) {
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (8 * j + q2 + (e & 1) >= srows)
                            x[j][e] = -INFINITY;
            }
            float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 2));
            const float mn0 = fmaxf(m0, mx0); // finite: token 0 of a step is always valid
            const float c0 = exp2f(m0 - mn0);
            m0 = mn0;
            float pr[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                pr[j][0] = exp2f(x[j][0] - mn0);
                pr[j][1] = exp2f(x[j][1] - mn0);
            }
            l0 = fmaf(l0, c0, (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
            float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 2));
            const float mn1 = fmaxf(m1, mx1);
            const float c1 = exp2f(m1 - mn1);
            m1 = mn1;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                pr[j][2] = exp2f(x[j][2] - mn1);
                pr[j][3] = exp2f(x[j][3] - mn1);
            }
            l1 = fmaf(l1, c1, (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
            float cr = 1.f; // fp8: R_old / R_new
            if constexpr (kFp8) {
                // Fold the V scales into P relative to R (tokens past the
                // context get P' = 0 by selection).
                float vs[2][2];
                float vmax = 0.f;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float2 v2 = *reinterpret_cast<const float2 *>(vsc + t0 + 8 * j + q2);
                    vs[j][0] = v2.x;
                    vs[j][1] = v2.y;
                    if (partial) { // stale scales past the context must not reach P'
                        if (8 * j + q2 >= srows)
                            vs[j][0] = 0.f;
                        if (8 * j + q2 + 1 >= srows)
                            vs[j][1] = 0.f;
                    }
                    vmax = fmaxf(vmax, fmaxf(vs[j][0], vs[j][1]));
                }
                vmax = fmaxf(vmax, __shfl_xor_sync(FULL, vmax, 1));
                vmax = fmaxf(vmax, __shfl_xor_sync(FULL, vmax, 2));
                if (vmax > vref) { // warp-uniform; R (and 1/R) change only here
                    cr = vref / vmax;
                    vref = vmax;
                    vinv = 1.f / vmax;
                }
                // Tokens past the context have p = 0 and a zeroed scale.
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        pr[j][e] *= vs[j][e & 1] * vinv;
            }
            if (__any_sync(FULL, c0 != 1.f || c1 != 1.f || cr != 1.f)) { // a max moved
                const float f0 = c0 * cr, f1 = c1 * cr;
#pragma unroll
                for (int j = 0; j < 2 * KT; ++j) {
                    o[j][0] *= f0;
                    o[j][1] *= f0;
                    o[j][2] *= f1;
                    o[j][3] *= f1;
                }
            }

            // P as the A operand (16 rows x 16 tokens): the S fragment layout
            // of the two token tiles is exactly the A fragment layout.
            uint32_t pa[4];
            pa[0] = pack2<QT>(pr[0][0], pr[0][1]);
            pa[1] = pack2<QT>(pr[0][2], pr[0][3]);
            pa[2] = pack2<QT>(pr[1][0], pr[1][1]);
            pa[3] = pack2<QT>(pr[1][2], pr[1][3]);
            uint32_t pl[4]; // bf16: the remainder P - bf16(P)
            if constexpr (kBf16) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = k >> 1, e = (k & 1) * 2;
                    const float2 hh = unpack_bf2(pa[k]);
                    pl[k] = pack2<T>(pr[j][e] - hh.x, pr[j][e + 1] - hh.y);
                }
            }

            if constexpr (kFp8) {
                // O += P V per pair of pieces: r[2h] / r[2h + 1] hold tokens
                // 2q, 2q + 1 (of 0-7 / 8-15) at codes d = 2g, 2g + 1 of piece
                // c; reordered to (d 2g: both tokens | d 2g + 1: both) and
                // widened, they are b0 / b1 of the even and odd d tiles.
#pragma unroll
                for (int kp = 0; kp < KT / 2; ++kp) {
                    uint32_t r[4];
                    ldsm_x4_trans(vb + piece_off(t0 + vt, 2 * kp + vc), r);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = 2 * kp + h; // piece: d = 16c .. 16c + 15
                        uint32_t e0, o0, e1, o1;
                        e4m3x4_to_h2x2(__byte_perm(r[2 * h], 0u, 0x3120u), e0, o0);
                        e4m3x4_to_h2x2(__byte_perm(r[2 * h + 1], 0u, 0x3120u), e1, o1);
                        mma_16816<false>(o[2 * c], pa, e0, e1);
                        mma_16816<false>(o[2 * c + 1], pa, o0, o1);
                    }
                }
            } else {
                // O += P V, two 8-wide d tiles per transposed ldmatrix.
#pragma unroll
                for (int dp = 0; dp < KT; ++dp) {
                    uint32_t b[4];
                    ldsm_x4_trans(vb + piece_off(t0 + vt, 2 * dp + vc), b);
                    mma_16816<kBf16>(o[2 * dp], pa, b[0], b[1]);
                    mma_16816<kBf16>(o[2 * dp + 1], pa, b[2], b[3]);
                    if constexpr (kBf16) {
                        mma_16816<kBf16>(o[2 * dp], pl, b[0], b[1]);
                        mma_16816<kBf16>(o[2 * dp + 1], pl, b[2], b[3]);
                    }
                }
            }
        }
    }

    // Row sums over each quad, then this warp's (O, m, l) of rows < G into
    // mw (row stride MS; fp8: O back in the scale of the codes' values,
    // times R).
    __device__ __forceinline__ void store(float *mw, int G)
    {
        l0 += __shfl_xor_sync(FULL, l0, 1);
        l0 += __shfl_xor_sync(FULL, l0, 2);
        l1 += __shfl_xor_sync(FULL, l1, 1);
        l1 += __shfl_xor_sync(FULL, l1, 2);
        const float oscale = kFp8 ? vref : 1.f;
        __syncwarp();
        if (g0 < G) {
            store_row(mw + g0 * MS, 0, oscale);
            if ((lane & 3) == 0) {
                mw[g0 * MS + D] = m0;
                mw[g0 * MS + D + 1] = l0;
            }
        }
        if (g1 < G) {
            store_row(mw + g1 * MS, 2, oscale);
            if ((lane & 3) == 0) {
                mw[g1 * MS + D] = m1;
                mw[g1 * MS + D + 1] = l1;
            }
        }
    }
};

// One warp's share of a group of G <= 8 query heads in the transposed
// orientation: S^T = K Q^T and O^T += V^T P^T. The 16 tokens of a step (for
// S^T) and 16 values of d (for O^T) fill the 16 rows of each m16n8k16 tile
// and the heads its 8 columns, so every tile is fully used; GroupWarp's
// orientation (heads as rows) leaves rows 8-15 of every tile empty when
// G <= 8 and needs twice the tiles and accumulators. Same interface and
// merge-area output as GroupWarp. Heads >= G are zero query columns (their
// outputs are never stored).
//
// Fragment coordinates: g = lane / 4, q = lane % 4. S^T: rows = tokens g,
// g + 8, columns = heads 2q, 2q + 1. Q^T (B operand): k = d pair, n = head
// g. P^T (B operand): k = tokens 2q, 2q + 1 (and + 8), n = head g, made from
// the S^T fragments by one 8x8 register transpose (movmatrix) per 8 tokens.
// O^T tile j: rows = d (drow), columns = heads 2q, 2q + 1.
// K and V tiles both come from ldmatrix with rows (tokens) 0-7 / 8-15 /
// 0-7 / 8-15 at pieces c / c / c+1 / c+1: non-transposed K is exactly the A
// fragment of one k-step; transposed 16-bit V gives the A fragment of O^T
// tile j in register order 0, 2, 1, 3. fp8: each register holds 4 codes of
// one token; widened to f16 pairs (codes 0-1, 2-3) they are K's A fragment
// with the k order d = 4q, 4q+1 | 4q+2, 4q+3 (the query is loaded in the
// same order). fp8 V comes through transposed ldmatrix on code pairs (see
// chunk); the rows of O^T tile j are then d = 16j + 2g and 16j + 2g + 1.
template <typename T, int D> struct GroupWarpT {
    using Geo = GroupGeom<T, D>;
    static constexpr bool kFp8 = Geo::kFp8;
    static constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    using QT = typename std::conditional<kFp8, __half, T>::type; // operand / row type
    static constexpr int CH = Geo::kChunk, ROW = Geo::kRow;
    static constexpr int KT = D / 16; // 16-wide d pieces: k-steps of S^T, row tiles of O^T
    static constexpr int MS = Geo::kMergeStride;
    static constexpr unsigned FULL = 0xffffffffu;

    int lane, g, q;
    int rt, rc;          // ldmatrix row (token) and piece offset of this lane
    uint32_t qb[KT][2];  // Q^T as the B operand of each k-step
    float o[KT][4];      // O^T tiles
    float ma, mb;        // running maxima of heads 2q, 2q + 1
    float la, lb;        // this lane's tokens' share of their sums
    float vref;          // fp8: largest V scale so far (R), floored at FLT_MIN
    float vinv;          // fp8: 1 / vref

    static __device__ __forceinline__ int piece_off(int t, int piece)
    {
        return Geo::piece_off(t, piece);
    }

    // d of row g (hi = 0) or g + 8 (hi = 1) of O^T tile j.
    __device__ __forceinline__ int drow(int j, int hi) const
    {
        return kFp8 ? 16 * j + 2 * g + hi : 16 * j + g + 8 * hi;
    }

    __device__ __forceinline__ void init(int lane_)
    {
        lane = lane_;
        g = lane >> 2;
        q = lane & 3;
        rt = (lane & 7) + (((lane >> 3) & 1) << 3);
        rc = lane >> 4;
    }

    // Head g's query row (row0 + g) as B fragments: 16-bit k-slots (2q, 2q+1)
    // / (2q+8, 2q+9) hold d = 16kk + 2q (+1) / + 8 (+1); fp8: d = 16kk + 4q
    // (+1) / + 2 (+1), matching the widened K codes. Heads >= G: zero.
    __device__ __forceinline__ void load_q(const void *query, size_t row0, int G)
    {
        const uint32_t *qp = static_cast<const uint32_t *>(query); // element pairs
        const size_t r = (row0 + g) * (D / 2);
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            const int c0 = kFp8 ? 8 * kk + 2 * q : 8 * kk + q;
            const int c1 = kFp8 ? c0 + 1 : c0 + 4;
            qb[kk][0] = g < G ? qp[r + c0] : 0u;
            qb[kk][1] = g < G ? qp[r + c1] : 0u;
        }
    }

    __device__ __forceinline__ void reset()
    {
#pragma unroll
        for (int j = 0; j < KT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[j][e] = 0.f;
        ma = mb = -INFINITY;
        la = lb = 0.f;
        vref = 1.17549435e-38f;
        vinv = 1.f / vref;
    }

    // S^T of tokens t0 .. t0 + 15, even and odd k-steps in separate
    // accumulators (two shorter dependency chains).
    __device__ __forceinline__ void scores(uint32_t kb, int t0, float (&sa)[4]) const
    {
        float sb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            sa[e] = sb[e] = 0.f;
        if constexpr (kFp8) {
#pragma unroll
            for (int kp = 0; kp < KT / 2; ++kp) { // pieces 2kp, 2kp + 1
                uint32_t r[4];
                ldsm_x4(kb + piece_off(t0 + rt, 2 * kp + rc), r);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t a[4];
                    e4m3x4_to_h2x2(r[2 * h], a[0], a[2]);     // tokens 0-7
                    e4m3x4_to_h2x2(r[2 * h + 1], a[1], a[3]); // tokens 8-15
                    mma_16816<false>(h ? sb : sa, a, qb[2 * kp + h][0], qb[2 * kp + h][1]);
                }
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                uint32_t a[4];
                ldsm_x4(kb + piece_off(t0 + rt, 2 * kk + rc), a);
                mma_16816<kBf16>(kk & 1 ? sb : sa, a, qb[kk][0], qb[kk][1]);
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
            sa[e] += sb[e];
    }

    // One staged chunk (as GroupWarp::chunk): K codes at sk, V at sv, fp8 row
    // scales at ksc / vsc, `rows` valid tokens, qs = scale * log2(e).
    __device__ __forceinline__ void chunk(char *sk, char *sv, const float *ksc, const float *vsc,
                                          int rows, float qs)
    {
        if (rows < CH) { // zero the V rows past the context
            for (int k = rows * (ROW / 16) + lane; k < CH * (ROW / 16); k += 32)
                reinterpret_cast<uint4 *>(sv)[k] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem(); // before the stage is refilled by a copy
            __syncwarp();
        }
        const uint32_t kb = smem_addr(sk), vb = smem_addr(sv);
#pragma unroll
        for (int sub = 0; sub < CH / 16; ++sub) {
            const int srows = rows - 16 * sub; // valid tokens of this step
            if (srows <= 0)
                break; // warp-uniform
            const int t0 = 16 * sub;
            float sa[4];
            scores(kb, t0, sa);

            // Online softmax (base 2) per head over the step's tokens: sa[0]
            // / sa[1]: token t0 + g, heads 2q / 2q + 1; sa[2] / sa[3]: token
            // t0 + g + 8. The 16 tokens of a head live in the 8 lanes of one q.
            float k0 = qs, k1 = qs;
            if constexpr (kFp8) {
                k0 = ksc[t0 + g] * qs;
                k1 = ksc[t0 + g + 8] * qs;
            }
            float x0 = sa[0] * k0, x1 = sa[1] * k0, x2 = sa[2] * k1, x3 = sa[3] * k1;
            const bool partial = srows < 16; // warp-uniform
            if (partial) {
                if (g >= srows)
                    x0 = x1 = -INFINITY;
                if (g + 8 >= srows)
                    x2 = x3 = -INFINITY;
            }
            float mxa = fmaxf(x0, x2), mxb = fmaxf(x1, x3);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                mxa = fmaxf(mxa, __shfl_xor_sync(FULL, mxa, sh));
                mxb = fmaxf(mxb, __shfl_xor_sync(FULL, mxb, sh));
            }
            const float na = fmaxf(ma, mxa), nb = fmaxf(mb, mxb); // finite: token t0 is valid
            const float ca = exp2f(ma - na), cb = exp2f(mb - nb);
            ma = na;
            mb = nb;
            float p0 = exp2f(x0 - na), p1 = exp2f(x1 - nb);
            float p2 = exp2f(x2 - na), p3 = exp2f(x3 - nb);
            la = fmaf(la, ca, p0 + p2);
            lb = fmaf(lb, cb, p1 + p3);
            float cr = 1.f; // fp8: R_old / R_new
            if constexpr (kFp8) {
                // Fold the V scales into P relative to R (tokens past the
                // context get P' = 0 by selection).
                float v0 = vsc[t0 + g], v1 = vsc[t0 + g + 8];
                if (partial) { // stale scales past the context must not reach P'
                    if (g >= srows)
                        v0 = 0.f;
                    if (g + 8 >= srows)
                        v1 = 0.f;
                }
                float vmax = fmaxf(v0, v1);
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1)
                    vmax = fmaxf(vmax, __shfl_xor_sync(FULL, vmax, sh));
                if (vmax > vref) { // warp-uniform; R (and 1/R) change only here
                    cr = vref / vmax;
                    vref = vmax;
                    vinv = 1.f / vmax;
                }
                const float w0 = v0 * vinv, w1 = v1 * vinv;
                p0 *= w0;
                p1 *= w0;
                p2 *= w1;
                p3 *= w1;
            }
            if (__any_sync(FULL, ca != 1.f || cb != 1.f || cr != 1.f)) { // a max moved
                const float fa = ca * cr, fb = cb * cr;
#pragma unroll
                for (int j = 0; j < KT; ++j) {
                    o[j][0] *= fa;
                    o[j][2] *= fa;
                    o[j][1] *= fb;
                    o[j][3] *= fb;
                }
            }

            // P^T as the B operand: the S^T fragment pair of tokens g (and
            // g + 8), heads 2q, 2q + 1, transposed in registers, is head g at
            // tokens 2q, 2q + 1 (and + 8).
            const uint32_t pb0 = movmatrix_trans(pack2<QT>(p0, p1));
            const uint32_t pb1 = movmatrix_trans(pack2<QT>(p2, p3));
            uint32_t pl0 = 0u, pl1 = 0u; // bf16: the remainder P - bf16(P)
            if constexpr (kBf16) {
                const float2 h01 = unpack_bf2(pack2<T>(p0, p1));
                const float2 h23 = unpack_bf2(pack2<T>(p2, p3));
                pl0 = movmatrix_trans(pack2<T>(p0 - h01.x, p1 - h01.y));
                pl1 = movmatrix_trans(pack2<T>(p2 - h23.x, p3 - h23.y));
            }

            if constexpr (kFp8) {
                // O^T += V^T P^T per piece. Transposed ldmatrix on code
                // pairs: a lane gets tokens 2q, 2q + 1 at codes d = 2g, 2g + 1
                // of the piece; reordered to (d 2g: both tokens, d 2g + 1:
                // both tokens) and widened, these are the A fragment rows of
                // d = 2g (rows 0-7) and 2g + 1 (rows 8-15).
#pragma unroll
                for (int kp = 0; kp < KT / 2; ++kp) {
                    uint32_t r[4];
                    ldsm_x4_trans(vb + piece_off(t0 + rt, 2 * kp + rc), r);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t a[4];
                        e4m3x4_to_h2x2(__byte_perm(r[2 * h], 0u, 0x3120u), a[0], a[1]);
                        e4m3x4_to_h2x2(__byte_perm(r[2 * h + 1], 0u, 0x3120u), a[2], a[3]);
                        mma_16816<false>(o[2 * kp + h], a, pb0, pb1);
                    }
                }
            } else {
                // O^T += V^T P^T, one 16-row tile of d per transposed ldmatrix.
#pragma unroll
                for (int j = 0; j < KT; ++j) {
                    uint32_t r[4];
                    ldsm_x4_trans(vb + piece_off(t0 + rt, 2 * j + rc), r);
                    const uint32_t a[4] = {r[0], r[2], r[1], r[3]};
                    mma_16816<kBf16>(o[j], a, pb0, pb1);
                    if constexpr (kBf16)
                        mma_16816<kBf16>(o[j], a, pl0, pl1);
                }
            }
        }
    }

    // Sums over each head's 8 lanes, then this warp's (O, m, l) of heads < G
    // into mw (row stride MS; fp8: O back in the scale of the codes' values,
    // times R).
    __device__ __forceinline__ void store(float *mw, int G)
    {
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) {
            la += __shfl_xor_sync(FULL, la, sh);
            lb += __shfl_xor_sync(FULL, lb, sh);
        }
        const float oscale = kFp8 ? vref : 1.f;
        const int ha = 2 * q, hb = ha + 1;
        __syncwarp();
        if (ha < G) {
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                mw[ha * MS + drow(j, 0)] = o[j][0] * oscale;
                mw[ha * MS + drow(j, 1)] = o[j][2] * oscale;
            }
            if (g == 0) {
                mw[ha * MS + D] = ma;
                mw[ha * MS + D + 1] = la;
            }
        }
        if (hb < G) {
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                mw[hb * MS + drow(j, 0)] = o[j][1] * oscale;
                mw[hb * MS + drow(j, 1)] = o[j][3] * oscale;
            }
            if (g == 0) {
                mw[hb * MS + D] = mb;
                mw[hb * MS + D + 1] = lb;
            }
        }
    }
};

// The new token's K and V rows for the fused append (pa_write_kv_decode),
// one (sequence, K/V head) row per warp: lanes [0, RV) hold 16 bytes of the
// stored K row each, the next RV lanes the V row (fp8: 16 codes quantised
// from 16 inputs, with the row scale amax / 448 on every lane of the half).
template <typename T, int D, int BS> struct NewRow {
    using Geo = GroupGeom<T, D>;
    using QT = typename std::conditional<Geo::kFp8, __half, T>::type;
    static constexpr int RV = Geo::kRow / 16;
    static constexpr size_t kTile =
        Geo::kFp8 ? (size_t)BS * (D + 4) : (size_t)BS * D * 2; // one (block, head) tile
    uint4 val;
    float scale;

    // Every lane calls it; src_row = s * num_kv_heads + kvh.
    __device__ __forceinline__ void load(const DecodeParams &p, size_t src_row, int lane)
    {
        const bool isv = lane >= RV;
        const int piece = lane % RV;
        constexpr int EPL = Geo::kFp8 ? 16 : 8; // inputs per lane
        const QT *src = static_cast<const QT *>(isv ? p.new_value : p.new_key) + src_row * D +
                        (size_t)piece * EPL;
        val = make_uint4(0u, 0u, 0u, 0u);
        scale = 0.f;
        if constexpr (Geo::kFp8) {
            // codes = e4m3(x * (448 / amax)), scale = amax / 448.
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
            for (int o2 = 1; o2 < RV; o2 <<= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o2));
            if (lane < 2 * RV) {
                const float inv = amax > 0.f ? 448.f / amax : 0.f;
                val = quantize16_e4m3(x, inv);
                scale = amax / 448.f;
            }
        } else {
            if (lane < 2 * RV)
                val = *reinterpret_cast<const uint4 *>(src);
        }
    }

    // Where this lane's 16 bytes (and, on the first lane of each half, the
    // fp8 row scale) go in the cache: block b, K/V head kvh, slot offset off.
    // NULL for lanes without a part and for a block id outside the pool.
    __device__ __forceinline__ void locate(const DecodeParams &p, int b, int kvh, int off,
                                           int lane, uint4 *&d, float *&sd) const
    {
        d = nullptr;
        sd = nullptr;
        if (lane >= 2 * RV || b < 0 || b >= p.num_blocks)
            return;
        const bool isv = lane >= RV;
        const int piece = lane % RV;
        char *cache =
            const_cast<char *>(static_cast<const char *>(isv ? p.value_cache : p.key_cache));
        char *tile = cache + ((size_t)b * p.num_kv_heads + kvh) * kTile;
        d = reinterpret_cast<uint4 *>(tile + (size_t)off * Geo::kRow) + piece;
        if (Geo::kFp8 && piece == 0)
            sd = reinterpret_cast<float *>(tile + (size_t)BS * Geo::kRow) + off;
    }
};

// decode_group_kernel: one CTA per (K/V head, sequence, partition) of a
// fixed partition size; grid (num_kv_heads, num_seqs, num_parts). TWO: the
// launch has G > 8 (heads as tile rows, GroupWarp); else the transposed
// GroupWarpT.
template <typename T, int D, int BS, int NW, int NS, bool TWO>
__global__ void __launch_bounds__(NW * 32)
    decode_group_kernel(const __grid_constant__ GroupParams gp)
{
    using Cfg = GroupCfg<T, D, BS, NW, NS>;
    static_assert(kGroupMaxHeads * D <= kMergeOutPerThread * NW * 32, "merge_if_last capacity");
    // G > 8: heads as tile rows; G <= 8: the transposed orientation.
    using Wp = typename std::conditional<TWO, GroupWarp<T, D>, GroupWarpT<T, D>>::type;
    constexpr bool kFp8 = Cfg::kFp8;
    constexpr int CH = Cfg::kChunk, SEG = Cfg::kSeg, ROW = Cfg::kRow;
    constexpr int MS = Cfg::kMergeStride;
    constexpr unsigned FULL = 0xffffffffu;
    const DecodeParams &p = gp.p;

    extern __shared__ __align__(1024) unsigned char group_smem[];
    unsigned char *smem = group_smem + ((1024u - (smem_addr(group_smem) & 1023u)) & 1023u);
    char *rings = reinterpret_cast<char *>(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kRingsBytes);
    float *scales = reinterpret_cast<float *>(smem + Cfg::kRingsBytes + Cfg::kBarBytes);
    int32_t *rank_ctx =
        reinterpret_cast<int32_t *>(smem + Cfg::kRingsBytes + Cfg::kBarBytes + Cfg::kScaleBytes);
    int32_t *table = reinterpret_cast<int32_t *>(smem + Cfg::kFixedBytes);
    __shared__ int cta_flags, ranked_seq;

    pdl_launch_dependents();
    const int kvh = blockIdx.x, part = blockIdx.z, P = p.partition_size;
    int s = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads, HK = p.num_kv_heads, G = H / HK;

    if (tid == 0)
        cta_flags = 0;
    if (lane == 0)
        for (int k = 0; k < NS; ++k)
            mbar_init(smem_addr(&bars[warp * NS + k]), 1);
    fence_mbar_init();
    pdl_wait_prior_grid(); // every input may come from the previous kernel
    if (p.rank_seqs) // longest sequences first (ranked_sequence)
        s = ranked_sequence(p.context_lens, p.num_seqs, blockIdx.y, tid, NW * 32, rank_ctx,
                            &ranked_seq);

    Wp w;
    w.init(lane);
    // Loaded before the block table so that the two reads overlap.
    w.load_q(p.query, (size_t)s * H + (size_t)kvh * G, G);

    UnitInfo u;
    const bool live = load_unit<BS>(p, s, part, P, tid, NW * 32,
                                    tid == 0 && kvh == 0 && part == 0, table, u);
    if (!live)
        return; // uniform across the CTA
    __syncthreads();
    w.reset();

    const int n_chunks = (u.n_tok + CH - 1) / CH;
    const int my_chunks = n_chunks <= warp ? 0 : (n_chunks - warp + NW - 1) / NW;
    char *ring = rings + (size_t)warp * Cfg::kRing;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(&bars[warp * NS]);
    float *wscales = scales + (size_t)warp * NS * 2 * CH; // fp8: [stage][K | V][CH]

    // Fused append: the warp owning the chunk of the sequence's last token
    // puts the new K/V row into that chunk once it has landed, and into the
    // cache.
    constexpr int RV = ROW / 16;
    int patch_i = -1, patch_row = 0;
    NewRow<T, D, BS> nr;
    nr.val = make_uint4(0u, 0u, 0u, 0u);
    nr.scale = 0.f;
    uint4 *patch_dst = nullptr;
    float *patch_sdst = nullptr;
    if (p.new_key != nullptr && part == u.num_parts - 1 && u.n_tok > 0) {
        const int c_last = (u.n_tok - 1) / CH;
        if (c_last % NW == warp) { // warp-uniform
            patch_i = c_last / NW;
            patch_row = (u.n_tok - 1) - c_last * CH;
            nr.load(p, (size_t)s * HK + kvh, lane);
            nr.locate(p, table[(u.n_tok - 1) / BS], kvh, (u.n_tok - 1) % BS, lane, patch_dst,
                      patch_sdst);
        }
    }

    // Lane 0: the copies of local chunk i (global chunk warp + i*NW). Boxes
    // that start past the context are not fetched; a block id outside the
    // pool is replaced by block 0 and recorded.
    int bad_id = 0;
    const char *kpool = static_cast<const char *>(p.key_cache);
    const char *vpool = static_cast<const char *>(p.value_cache);
    auto issue = [&](int i) {
        const int tok0 = (warp + i * NW) * CH;
        const int rows = min(CH, u.n_tok - tok0);
        const int nseg = (rows + SEG - 1) / SEG;
        const int st = i % NS;
        const uint32_t dk = ring_s + st * Cfg::kStage, dv = dk + Cfg::kHalf;
        const uint32_t bar = bar0 + st * 8;
        mbar_arrive_expect_tx(bar, (uint32_t)(nseg * SEG * (ROW + (kFp8 ? 4 : 0)) * 2));
        for (int sg = 0; sg < nseg; ++sg) {
            const int tok = tok0 + sg * SEG;
            int b = table[tok / BS];
            if (b < 0 || b >= p.num_blocks) {
                bad_id = 1;
                b = 0;
            }
            const int tile = b * HK + kvh;
            if constexpr (kFp8) {
                const int off = tok % BS;
                tma_load_3d(dk + sg * SEG * ROW, &gp.tk, 0, off, tile, bar);
                tma_load_3d(dv + sg * SEG * ROW, &gp.tv, 0, off, tile, bar);
                const size_t sofs = (size_t)tile * (BS * (D + 4)) + BS * D + (size_t)off * 4;
                float *sk = wscales + (st * 2) * CH + sg * SEG;
                bulk_g2s(smem_addr(sk), kpool + sofs, SEG * 4, bar);
                bulk_g2s(smem_addr(sk + CH), vpool + sofs, SEG * 4, bar);
            } else {
                const int y = tile * BS + tok % BS;
                tma_load_3d(dk + sg * SEG * ROW, &gp.tk, 0, 0, y, bar);
                tma_load_3d(dv + sg * SEG * ROW, &gp.tv, 0, 0, y, bar);
            }
        }
    };

    if (lane == 0)
        for (int i = 0; i < min(NS, my_chunks); ++i)
            issue(i);
    int issued = min(NS, my_chunks);
    const float qs = p.qk_scale_log2;

    int i = 0;
    for (; i < my_chunks; ++i) {
        const int st = i % NS;
        const bool ok = mbar_wait_bounded(bar0 + st * 8, (i / NS) & 1, kWaitLimitNs);
        if (__any_sync(FULL, !ok))
            break;
        const int rows = min(CH, u.n_tok - (warp + i * NW) * CH);
        char *sk = ring + st * Cfg::kStage;
        char *sv = sk + Cfg::kHalf;
        float *ksc = wscales + (st * 2) * CH; // fp8 scales of the stage
        float *vsc = ksc + CH;
        if (i == patch_i) { // warp-uniform
            if (lane < 2 * RV) {
                const bool isv = lane >= RV;
                char *dst = (isv ? sv : sk) + Wp::piece_off(patch_row, lane % RV);
                *reinterpret_cast<uint4 *>(dst) = nr.val;
                if (patch_dst)
                    *patch_dst = nr.val;
                if constexpr (kFp8) {
                    if (lane % RV == 0) {
                        (isv ? vsc : ksc)[patch_row] = nr.scale;
                        if (patch_sdst)
                            *patch_sdst = nr.scale;
                    }
                }
                fence_proxy_async_smem(); // before the stage is refilled by a copy
            }
            __syncwarp();
        }
        w.chunk(sk, sv, ksc, vsc, rows, qs);
        __syncwarp();
        if (i + NS < my_chunks) {
            if (lane == 0)
                issue(i + NS);
            issued = i + NS + 1;
        }
    }
    const bool timed_out = i < my_chunks;
    if (timed_out) {
        // Let the copies still in flight land before the ring is reused.
        for (int k = i; k < issued; ++k)
            mbar_wait_bounded(bar0 + (k % NS) * 8, (k / NS) & 1, kWaitLimitNs);
    }
    if (lane == 0) {
        if (timed_out) {
            report(p.dev_err, PA_DEVERR_TIMEOUT);
            atomicOr(&cta_flags, 2);
        }
        if (bad_id)
            atomicOr(&cta_flags, 1);
    }

    // This warp's (O, m, l) into its ring, then the warps merged in two
    // passes: one thread per query row turns the NW (m, l) pairs into
    // weights 2^(m_w - M) (divided by L = sum_w l_w 2^(m_w - M) for a single
    // pass), then every thread sums four columns of a row at a time.
    __syncwarp();
    w.store(reinterpret_cast<float *>(ring), G);
    __syncthreads();

    const bool failed = cta_flags != 0;
    if (tid == 0 && (cta_flags & 1))
        report(p.dev_err, PA_DEVERR_BLOCK_ID);
    constexpr int WS = NW + 2; // per row: NW weights, M, L
    float *wts = reinterpret_cast<float *>(rings) + Cfg::kMergeWeights;
    if (tid < G) {
        const int g = tid;
        float mw[NW], M = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) {
            mw[w2] = reinterpret_cast<const float *>(rings + w2 * Cfg::kRing)[g * MS + D];
            M = fmaxf(M, mw[w2]);
        }
        float L = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) {
            // A warp without tokens has m = -inf and weight 0; so has every
            // warp of an empty unit (M = -inf, output 0).
            mw[w2] = M == -INFINITY ? 0.f : exp2f(mw[w2] - M);
            L = fmaf(reinterpret_cast<const float *>(rings + w2 * Cfg::kRing)[g * MS + D + 1],
                     mw[w2], L);
        }
        const bool normalise = u.num_parts == 1 && L > 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2)
            wts[g * WS + w2] = normalise ? mw[w2] / L : mw[w2];
        if (u.num_parts > 1) {
            const size_t unit = ((size_t)s * H + kvh * G + g) * p.num_parts + part;
            p.ws_ml[unit * 2] = failed ? 0.f : M;
            p.ws_ml[unit * 2 + 1] = failed ? 1.f : L;
        }
    }
    __syncthreads();
    constexpr int D4 = D / 4;
    constexpr int kPasses = (kGroupMaxHeads * D4 + NW * 32 - 1) / (NW * 32);
#pragma unroll
    for (int k = 0; k < kPasses; ++k) {
        const int idx = tid + k * NW * 32;
        if (idx < G * D4) {
            const int g = idx / D4, d = (idx - g * D4) * 4;
            float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) {
                const float f = wts[g * WS + w2];
                const float4 v = *reinterpret_cast<const float4 *>(
                    reinterpret_cast<const float *>(rings + w2 * Cfg::kRing) + g * MS + d);
                o4.x = fmaf(v.x, f, o4.x);
                o4.y = fmaf(v.y, f, o4.y);
                o4.z = fmaf(v.z, f, o4.z);
                o4.w = fmaf(v.w, f, o4.w);
            }
            if (failed)
                o4 = make_float4(NAN, NAN, NAN, NAN);
            const int h = kvh * G + g;
            if (u.num_parts == 1) {
                const size_t o = ((size_t)s * H + h) * D + d;
                store_out(p.out, p.out_dtype, o, o4.x);
                store_out(p.out, p.out_dtype, o + 1, o4.y);
                store_out(p.out, p.out_dtype, o + 2, o4.z);
                store_out(p.out, p.out_dtype, o + 3, o4.w);
            } else {
                const size_t unit = ((size_t)s * H + h) * p.num_parts + part;
                *reinterpret_cast<float4 *>(p.ws_acc + unit * D + d) = o4;
            }
        }
    }
    if (u.num_parts > 1 && p.ws_count)
        merge_if_last<D>(p, s, kvh * G, G, s * HK + kvh, u.num_parts, tid, NW * 32, &cta_flags,
                         reinterpret_cast<float *>(rings));
}

} // namespace pagedkv
