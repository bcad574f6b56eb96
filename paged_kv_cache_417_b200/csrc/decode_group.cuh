// decode_group.cuh - paged decode attention for grouped query heads
// (num_heads = G * num_kv_heads, 2 <= G <= 16, 16-bit caches) on sm_100a.
//
// Query heads kvh*G .. kvh*G+G-1 all attend over K/V head kvh. A CTA takes
// the unit (K/V head kvh, sequence s, partition p) for the whole group, so
// each K/V byte crosses HBM once per group instead of once per query head,
// and the G query rows share every staged tile. The outputs, the split
// workspace and the merge of partitions are those of decode_split_kernel
// (per query head; the last CTA of a (K/V head, sequence) merges its G
// heads).
//
// Staging: each pool is viewed as a tensor of rows (row = one token of one
// (block, head) tile, D 16-bit elements; row index (block*Hkv + kvh)*bs +
// offset), each row split into D/64 128-byte units: dims (64 elements,
// D/64 units, rows). A warp's stage receives 16 tokens of K and of V
// through tiled TMA copies (cp.async.bulk.tensor) of min(bs, 16) whole rows
// per box, contiguous in global memory, with the 128-byte swizzle: 16-byte
// piece c of 128-byte unit u of the stage lands at piece c ^ (u % 8) of that
// unit. A stage is [K | V] x [16 rows x D*2 bytes], each half starting on a
// 1024-byte boundary; row t's unit h is unit t*D/64 + h, so the 8 rows of an
// 8x8 ldmatrix tile hit 8 distinct bank groups at D = 64 and 4 (2-way) at
// D = 128.
//
// Math per 16-token chunk in one warp, on tensor-core tiles (mma.sync
// m16n8k16, fp32 accumulation); the G query heads are the M rows, padded to
// 16 with zeros (G <= 8 uses rows 0-7 only):
//   S = Q K^T      2 column tiles of 8 tokens x D/16 k-steps, K tiles by
//                  ldmatrix straight from the swizzled stage;
//   online softmax in base 2 on the accumulator fragments: the 16 scores of
//                  a row live in one quad of lanes (2 shuffles per max);
//   O += P V       P goes from the S fragments into the A operand without
//                  leaving registers; V tiles by ldmatrix.trans.
// P is rounded to the cache's type for the product (the running sum keeps
// the fp32 weights). bf16 carries only 8 significant bits, so a bf16 P is
// split into a bf16 head and a bf16 remainder and multiplied twice, which
// keeps about 16 bits.
//
// Rows past the context: their scores are set to -inf (never computed from
// the stale bytes), and the V rows of a partial last chunk are zeroed in
// shared memory before the product, so a weight of 0 meets a finite value
// (0 * NaN would otherwise reach the sum).
//
// These tiles are warp-sized on purpose: the group is at most 16 rows,
// below the 64-row minimum of a tcgen05 MMA, and the kernel is bound by HBM
// bandwidth, so the tensor cores only have to remove the per-element FMA
// and shuffle work of decode_split_kernel.
#pragma once

#include <cuda.h> // CUtensorMap (type only; maps are encoded on the host)

#include "decode.cuh"

namespace pagedkv {

constexpr int kGroupMaxHeads = 16;

struct GroupParams {
    CUtensorMap tk; // key pool: dims (64, D/64, NB*Hkv*bs), box (64, D/64, min(bs, 16)), 128B swizzle
    CUtensorMap tv; // value pool, same geometry
    DecodeParams p;
};

template <int D, int BS, int NW, int NS> struct GroupCfg {
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block_size");
    static constexpr int kChunk = 16;                      // tokens per warp step
    static constexpr int kUnits = D / 64;                  // 128-byte units per row
    static constexpr int kRow = D * 2;                     // bytes per row
    static constexpr int kHalf = kChunk * kRow;            // the K (or V) rows of a stage
    static constexpr int kStage = 2 * kHalf;
    static constexpr int kRing = NS * kStage;              // one warp's stages
    static constexpr int kSeg = BS < kChunk ? BS : kChunk; // rows per TMA box
    static constexpr int kRingsBytes = NW * kRing;
    static constexpr int kBarBytes = NW * NS * 8;
    static constexpr int kFixedBytes = kRingsBytes + kBarBytes;
    // After its last chunk a warp leaves (O, m, l) of its rows in its ring.
    static constexpr int kMergeStride = D + 2;
    static_assert(kGroupMaxHeads * kMergeStride * 4 <= kRing, "merge area fits a ring");
    static_assert(kHalf % 1024 == 0 && (kSeg * kRow) % 1024 == 0, "swizzle atoms");
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

// T: __half or __nv_bfloat16 (cache, query and new-row type). TWO: G > 8
// (fragment rows 8-15 are live).
template <typename T, int D, int BS, int NW, int NS, bool TWO>
__global__ void __launch_bounds__(NW * 32)
    decode_group_kernel(const __grid_constant__ GroupParams gp)
{
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    using Cfg = GroupCfg<D, BS, NW, NS>;
    constexpr int CH = Cfg::kChunk, SEG = Cfg::kSeg, ROW = Cfg::kRow, U = Cfg::kUnits;
    constexpr int KT = D / 16; // k-steps of q.k = pairs of 8-wide d tiles of O
    constexpr int MS = Cfg::kMergeStride;
    constexpr unsigned FULL = 0xffffffffu;
    const DecodeParams &p = gp.p;

    extern __shared__ __align__(1024) unsigned char group_smem[];
    unsigned char *smem = group_smem + ((1024u - (smem_addr(group_smem) & 1023u)) & 1023u);
    char *rings = reinterpret_cast<char *>(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kRingsBytes);
    int32_t *table = reinterpret_cast<int32_t *>(smem + Cfg::kFixedBytes);
    __shared__ int cta_flags;

    pdl_launch_dependents();
    const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads, HK = p.num_kv_heads, G = H / HK;

    if (tid == 0)
        cta_flags = 0;
    if (lane == 0)
        for (int k = 0; k < NS; ++k)
            mbar_init(smem_addr(&bars[warp * NS + k]), 1);
    fence_mbar_init();
    pdl_wait_prior_grid(); // every input may come from the previous kernel

    // Fragment coordinates: this lane holds rows g0 and g1 = g0 + 8 and, in
    // every 8-wide column tile, columns q2 and q2 + 1.
    const int g0 = lane >> 2, g1 = g0 + 8, q2 = 2 * (lane & 3);

    // Q as the A operand, one 16x16 tile per k-step; rows >= G are zero.
    // Loaded before the block table so that the two reads overlap.
    uint32_t qa[KT][4];
    {
        const uint32_t *q = static_cast<const uint32_t *>(p.query); // element pairs
        const size_t r0 = ((size_t)s * H + (size_t)kvh * G + g0) * (D / 2);
        const size_t r1 = r0 + (size_t)8 * (D / 2);
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            const int c = (16 * kk + q2) / 2;
            qa[kk][0] = g0 < G ? q[r0 + c] : 0u;
            qa[kk][1] = TWO && g1 < G ? q[r1 + c] : 0u;
            qa[kk][2] = g0 < G ? q[r0 + c + 4] : 0u;
            qa[kk][3] = TWO && g1 < G ? q[r1 + c + 4] : 0u;
        }
    }

    UnitInfo u;
    const bool live = load_unit<BS>(p, s, part, tid, NW * 32, tid == 0 && kvh == 0 && part == 0,
                                    table, u);
    if (!live)
        return; // uniform across the CTA
    __syncthreads();

    float o[2 * KT][4]; // 8-wide d tile j: d = 8j + q2 (+1); rows g0 (0, 1), g1 (2, 3)
#pragma unroll
    for (int j = 0; j < 2 * KT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[j][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const int n_chunks = (u.n_tok + CH - 1) / CH;
    const int my_chunks = n_chunks <= warp ? 0 : (n_chunks - warp + NW - 1) / NW;
    char *ring = rings + (size_t)warp * Cfg::kRing;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar0 = smem_addr(&bars[warp * NS]);

    // Fused append: the warp owning the chunk of the sequence's last token
    // puts the new K/V row into that chunk once it has landed, and into the
    // cache. Lanes [0, D/8) carry 16 bytes of the K row each, the next D/8
    // lanes the V row.
    constexpr int RV = D / 8;
    int patch_i = -1, patch_row = 0;
    uint4 patch_val = make_uint4(0u, 0u, 0u, 0u);
    uint4 *patch_dst = nullptr;
    if (p.new_key != nullptr && part == u.num_parts - 1 && u.n_tok > 0) {
        const int c_last = (u.n_tok - 1) / CH;
        if (c_last % NW == warp) { // warp-uniform
            patch_i = c_last / NW;
            patch_row = (u.n_tok - 1) - c_last * CH;
            if (lane < 2 * RV) {
                const bool isv = lane >= RV;
                const int piece = lane % RV;
                const T *src = static_cast<const T *>(isv ? p.new_value : p.new_key) +
                               ((size_t)s * HK + kvh) * D + (size_t)piece * 8;
                patch_val = *reinterpret_cast<const uint4 *>(src);
                const int b = table[(u.n_tok - 1) / BS];
                if (b >= 0 && b < p.num_blocks) {
                    char *cache = const_cast<char *>(
                        static_cast<const char *>(isv ? p.value_cache : p.key_cache));
                    const size_t row = ((size_t)b * HK + kvh) * BS + (u.n_tok - 1) % BS;
                    patch_dst = reinterpret_cast<uint4 *>(cache + row * (D * 2)) + piece;
                }
            }
        }
    }

    // Lane 0: the TMA boxes of local chunk i (global chunk warp + i*NW).
    // Boxes that start past the context are not fetched; a block id outside
    // the pool is replaced by block 0 and recorded.
    int bad_id = 0;
    auto issue = [&](int i) {
        const int tok0 = (warp + i * NW) * CH;
        const int rows = min(CH, u.n_tok - tok0);
        const int nseg = (rows + SEG - 1) / SEG;
        const int st = i % NS;
        const uint32_t dk = ring_s + st * Cfg::kStage, dv = dk + Cfg::kHalf;
        const uint32_t bar = bar0 + st * 8;
        mbar_arrive_expect_tx(bar, (uint32_t)(nseg * SEG * ROW * 2));
        for (int sg = 0; sg < nseg; ++sg) {
            const int tok = tok0 + sg * SEG;
            int b = table[tok / BS];
            if (b < 0 || b >= p.num_blocks) {
                bad_id = 1;
                b = 0;
            }
            const int y = (b * HK + kvh) * BS + tok % BS;
            tma_load_3d(dk + sg * SEG * ROW, &gp.tk, 0, 0, y, bar);
            tma_load_3d(dv + sg * SEG * ROW, &gp.tv, 0, 0, y, bar);
        }
    };

    if (lane == 0)
        for (int i = 0; i < min(NS, my_chunks); ++i)
            issue(i);
    int issued = min(NS, my_chunks);

    // ldmatrix row addresses. K (non-transposed, B of S = Q K^T): lanes
    // 0-7 / 8-15 / 16-23 / 24-31 give token rows 0-7 / 0-7 / 8-15 / 8-15 at
    // pieces c / c+1 / c / c+1, i.e. both k-halves of both token tiles.
    // V (transposed, B of O = P V): token rows 0-7 / 8-15 / 0-7 / 8-15 at
    // pieces c / c / c+1 / c+1, i.e. both token halves of two d tiles.
    // Piece p (16 bytes, d = 8p..8p+7) of row t sits in unit t*U + p/8 at
    // position (p % 8) ^ ((t*U + p/8) % 8).
    const int kt = (lane & 7) + ((lane >> 4) << 3), kc = (lane >> 3) & 1;
    const int vt = (lane & 7) + (((lane >> 3) & 1) << 3), vc = lane >> 4;
    auto piece_off = [](int t, int piece) {
        const int unit = t * U + (piece >> 3);
        return unit * 128 + (((piece & 7) ^ (unit & 7)) << 4);
    };
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
        if (i == patch_i) { // warp-uniform
            if (lane < 2 * RV) {
                char *dst = (lane >= RV ? sv : sk) + piece_off(patch_row, lane % RV);
                *reinterpret_cast<uint4 *>(dst) = patch_val;
                if (patch_dst)
                    *patch_dst = patch_val;
                fence_proxy_async_smem();
            }
            __syncwarp();
        }
        if (rows < CH) { // the partition's last chunk: zero the V rows past it
            for (int k = rows * (ROW / 16) + lane; k < CH * (ROW / 16); k += 32)
                reinterpret_cast<uint4 *>(sv)[k] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();
            __syncwarp();
        }

        // S = Q K^T for the chunk's 16 tokens, even and odd k-steps in
        // separate accumulators (two shorter dependency chains per tile).
        const uint32_t kb = smem_addr(sk), vb = smem_addr(sv);
        float sc[2][4], sd[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sc[j][e] = sd[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            uint32_t b[4];
            ldsm_x4(kb + piece_off(kt, 2 * kk + kc), b);
            mma_16816<kBf16>(kk & 1 ? sd[0] : sc[0], qa[kk], b[0], b[1]);
            mma_16816<kBf16>(kk & 1 ? sd[1] : sc[1], qa[kk], b[2], b[3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sc[j][e] += sd[j][e];

        // Online softmax (base 2). sc[j][e]: token 8j + q2 + (e & 1), row g0
        // for e < 2, g1 otherwise.
        float x[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                x[j][e] = 8 * j + q2 + (e & 1) < rows ? sc[j][e] * qs : -INFINITY;
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 2));
        const float mn0 = fmaxf(m0, mx0); // finite: token 0 of a chunk is always valid
        const float c0 = exp2f(m0 - mn0);
        m0 = mn0;
        float pr[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            pr[j][0] = exp2f(x[j][0] - mn0);
            pr[j][1] = exp2f(x[j][1] - mn0);
        }
        l0 = fmaf(l0, c0, (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
        float c1 = 1.f;
        if constexpr (TWO) {
            float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 2));
            const float mn1 = fmaxf(m1, mx1);
            c1 = exp2f(m1 - mn1);
            m1 = mn1;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                pr[j][2] = exp2f(x[j][2] - mn1);
                pr[j][3] = exp2f(x[j][3] - mn1);
            }
            l1 = fmaf(l1, c1, (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
        } else {
#pragma unroll
            for (int j = 0; j < 2; ++j)
                pr[j][2] = pr[j][3] = 0.f;
        }
        if (__any_sync(FULL, c0 != 1.f || c1 != 1.f)) { // a running max moved
#pragma unroll
            for (int j = 0; j < 2 * KT; ++j) {
                o[j][0] *= c0;
                o[j][1] *= c0;
                if constexpr (TWO) {
                    o[j][2] *= c1;
                    o[j][3] *= c1;
                }
            }
        }

        // P as the A operand (16 rows x 16 tokens): the S fragment layout of
        // the two token tiles is exactly the A fragment layout.
        uint32_t pa[4];
        pa[0] = pack2<T>(pr[0][0], pr[0][1]);
        pa[1] = pack2<T>(pr[0][2], pr[0][3]);
        pa[2] = pack2<T>(pr[1][0], pr[1][1]);
        pa[3] = pack2<T>(pr[1][2], pr[1][3]);
        uint32_t pl[4]; // bf16: the remainder P - bf16(P)
        if constexpr (kBf16) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = k >> 1, e = (k & 1) * 2;
                const float2 h = unpack_bf2(pa[k]);
                pl[k] = pack2<T>(pr[j][e] - h.x, pr[j][e + 1] - h.y);
            }
        }

        // O += P V, two 8-wide d tiles per transposed ldmatrix.
#pragma unroll
        for (int dp = 0; dp < KT; ++dp) {
            uint32_t b[4];
            ldsm_x4_trans(vb + piece_off(vt, 2 * dp + vc), b);
            mma_16816<kBf16>(o[2 * dp], pa, b[0], b[1]);
            mma_16816<kBf16>(o[2 * dp + 1], pa, b[2], b[3]);
            if constexpr (kBf16) {
                mma_16816<kBf16>(o[2 * dp], pl, b[0], b[1]);
                mma_16816<kBf16>(o[2 * dp + 1], pl, b[2], b[3]);
            }
        }
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

    // Row sums over the quad; then this warp's (O, m, l) into its ring.
    l0 += __shfl_xor_sync(FULL, l0, 1);
    l0 += __shfl_xor_sync(FULL, l0, 2);
    l1 += __shfl_xor_sync(FULL, l1, 1);
    l1 += __shfl_xor_sync(FULL, l1, 2);
    __syncwarp();
    float *mw = reinterpret_cast<float *>(ring);
    if (g0 < G) {
#pragma unroll
        for (int j = 0; j < 2 * KT; ++j)
            *reinterpret_cast<float2 *>(mw + g0 * MS + 8 * j + q2) = make_float2(o[j][0], o[j][1]);
        if ((lane & 3) == 0) {
            mw[g0 * MS + D] = m0;
            mw[g0 * MS + D + 1] = l0;
        }
    }
    if constexpr (TWO) {
        if (g1 < G) {
#pragma unroll
            for (int j = 0; j < 2 * KT; ++j)
                *reinterpret_cast<float2 *>(mw + g1 * MS + 8 * j + q2) =
                    make_float2(o[j][2], o[j][3]);
            if ((lane & 3) == 0) {
                mw[g1 * MS + D] = m1;
                mw[g1 * MS + D + 1] = l1;
            }
        }
    }
    __syncthreads();

    const bool failed = cta_flags != 0;
    if (tid == 0 && (cta_flags & 1))
        report(p.dev_err, PA_DEVERR_BLOCK_ID);
    for (int idx = tid; idx < G * D; idx += NW * 32) {
        const int g = idx / D, d = idx - g * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            M = fmaxf(M, reinterpret_cast<const float *>(rings + w * Cfg::kRing)[g * MS + D]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float *mv = reinterpret_cast<const float *>(rings + w * Cfg::kRing) + g * MS;
                const float f = exp2f(mv[D] - M);
                L = fmaf(mv[D + 1], f, L);
                O = fmaf(mv[d], f, O);
            }
        }
        if (failed)
            O = NAN;
        const int h = kvh * G + g;
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
        merge_if_last<D>(p, s, kvh * G, G, s * HK + kvh, u.num_parts, tid, NW * 32, &cta_flags,
                         reinterpret_cast<float *>(rings));
}

} // namespace pagedkv
