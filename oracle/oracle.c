/*
 * oracle.c - plain, slow, fp64 CPU oracle for one decode step of paged
 * attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do. It shares no code, header or table with the CUDA library.
 *
 * What it follows:
 *   - The KV cache is a pool of fixed-size physical blocks; a sequence's
 *     logical block i lives in the physical block its block table names
 *     ("vLLM基础: 架构、推理流程与关键组件", §2.3, block-table sketch;
 *     "啃透vLLM源码", §2.2). Token t of a sequence sits in logical block
 *     t / block_size at offset t % block_size (the in-order fill of
 *     LogicalTokenBlock.append_tokens, "啃透vLLM源码", §2.2).
 *   - Attention reads the caches through the physical block indices
 *     ("VLLM源码解析", core technology: attention_forward calling
 *     paged_attention_forward with key_cache, value_cache and the physical
 *     block indices). Paging moves bytes, not arithmetic, so the result is
 *     exact attention: gather the sequence's tokens into contiguous K and V,
 *     then softmax(scale * q K^T) V, evaluated here in fp64 with the
 *     textbook two-pass softmax (subtract the maximum, exponentiate,
 *     normalise).
 *   - Copy-on-write duplicates a shared block before a sequence writes into
 *     it ("vLLM基础", §2.3).
 *
 * Layout (a reading; the pages never print one): each pool is
 * [num_blocks][num_heads][block_size][head_dim], elements as raw 16-bit
 * patterns (fp16 or bf16). query/key/value/out are [rows][num_heads][head_dim].
 * Grouped heads (a reading; not on the pages): with num_heads query heads
 * over num_kv_heads K/V heads, query head h reads K/V head
 * h / (num_heads / num_kv_heads).
 * An fp8 pool (KV-cache quantisation, named by "vLLM基础", §2.5 as further
 * tuning on top of paging; the format below is a reading) holds per
 * (block, head) block_size rows of head_dim OCP e4m3 codes followed by
 * block_size fp32 row scales; a row's values are its codes times its scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };

/* IEEE 754 binary16: sign, 5-bit exponent (bias 15), 10-bit fraction. */
static double widen_f16(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* zero / subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 0x400), e - 25);  /* 1.f * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: the upper half of an IEEE binary32. */
static double widen_bf16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double widen(uint16_t x, int dtype)
{
    return dtype == ORACLE_BF16 ? widen_bf16(x) : widen_f16(x);
}

double oracle_widen(uint16_t x, int dtype) { return widen(x, dtype); }

/* Bytes of K and V cache for `tokens` tokens of every one of `layers` layers:
 * 2 (K and V) x layers x tokens x heads x head_dim x element bytes
 * ("vLLM基础", §2.3, the per-sequence preallocation estimate). */
int64_t oracle_kv_cache_bytes(int64_t layers, int64_t tokens, int64_t heads,
                              int64_t head_dim, int64_t elem_bytes)
{
    return 2 * layers * tokens * heads * head_dim * elem_bytes;
}

/* Write each new token's K and V into its slot. slot < 0 = padding, skipped.
 * Returns 0, or -1 if a slot lies outside the pool (nothing written then). */
int oracle_write_kv(const uint16_t *key, const uint16_t *value, int64_t num_tokens,
                    int32_t num_heads, int32_t head_dim, const int64_t *slot_mapping,
                    uint16_t *key_cache, uint16_t *value_cache, int64_t num_blocks,
                    int32_t block_size)
{
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * block_size)
            return -1;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        int64_t block = slot / block_size, offset = slot % block_size;
        for (int32_t h = 0; h < num_heads; ++h) {
            size_t dst = (size_t)(((block * num_heads + h) * block_size + offset) * head_dim);
            size_t src = (size_t)((t * num_heads + h) * head_dim);
            memcpy(key_cache + dst, key + src, (size_t)head_dim * sizeof(uint16_t));
            memcpy(value_cache + dst, value + src, (size_t)head_dim * sizeof(uint16_t));
        }
    }
    return 0;
}

/* Copy whole blocks src -> dst in every layer's K and V pool.
 * mapping is [num_pairs][2] = (src, dst). Returns -1 on an id outside the
 * pool (nothing copied then). */
int oracle_copy_blocks(uint16_t **key_caches, uint16_t **value_caches, int32_t num_layers,
                       const int64_t *mapping, int64_t num_pairs, int64_t num_blocks,
                       int64_t block_elems)
{
    for (int64_t i = 0; i < 2 * num_pairs; ++i)
        if (mapping[i] < 0 || mapping[i] >= num_blocks)
            return -1;
    for (int32_t l = 0; l < num_layers; ++l)
        for (int64_t i = 0; i < num_pairs; ++i) {
            int64_t src = mapping[2 * i], dst = mapping[2 * i + 1];
            memcpy(key_caches[l] + dst * block_elems, key_caches[l] + src * block_elems,
                   (size_t)block_elems * sizeof(uint16_t));
            memcpy(value_caches[l] + dst * block_elems, value_caches[l] + src * block_elems,
                   (size_t)block_elems * sizeof(uint16_t));
        }
    return 0;
}

/* Swap: copy whole blocks from one pool set to another of the same block
 * shape (a GPU pool and a pool in host memory, "啃透vLLM源码", §3: blocks go
 * to CPU memory when GPU memory runs short and come back when needed).
 * mapping is [num_pairs][2] = (block in the source pools, block in the
 * destination pools). Returns -1 on an id outside its pool (nothing copied). */
int oracle_swap_blocks(uint16_t **src_k, uint16_t **src_v, int64_t src_blocks, uint16_t **dst_k,
                       uint16_t **dst_v, int64_t dst_blocks, int32_t num_layers,
                       const int64_t *mapping, int64_t num_pairs, int64_t block_elems)
{
    for (int64_t i = 0; i < num_pairs; ++i)
        if (mapping[2 * i] < 0 || mapping[2 * i] >= src_blocks || mapping[2 * i + 1] < 0 ||
            mapping[2 * i + 1] >= dst_blocks)
            return -1;
    for (int32_t l = 0; l < num_layers; ++l)
        for (int64_t i = 0; i < num_pairs; ++i) {
            int64_t a = mapping[2 * i], b = mapping[2 * i + 1];
            memcpy(dst_k[l] + b * block_elems, src_k[l] + a * block_elems,
                   (size_t)block_elems * sizeof(uint16_t));
            memcpy(dst_v[l] + b * block_elems, src_v[l] + a * block_elems,
                   (size_t)block_elems * sizeof(uint16_t));
        }
    return 0;
}

/* Textbook attention over contiguous fp64 K and V (ctx >= 1 rows):
 * s_j = scale * q . k_j; subtract the maximum, exponentiate, normalise;
 * out = sum_j p_j v_j. */
static void attend(double *out, const double *q, const double *K, const double *V, int32_t ctx,
                   int32_t head_dim, double scale, double *w)
{
    /* 2. Scores s_j = scale * q . k_j. */
    for (int32_t j = 0; j < ctx; ++j) {
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d)
            dot += q[d] * K[(size_t)j * head_dim + d];
        w[j] = scale * dot;
    }

    /* 3. Softmax: subtract the maximum, exponentiate, normalise. */
    double m = w[0];
    for (int32_t j = 1; j < ctx; ++j)
        if (w[j] > m)
            m = w[j];
    double z = 0.0;
    for (int32_t j = 0; j < ctx; ++j) {
        w[j] = exp(w[j] - m);
        z += w[j];
    }

    /* 4. Output o = sum_j p_j v_j. */
    for (int32_t d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int32_t j = 0; j < ctx; ++j)
            acc += w[j] * V[(size_t)j * head_dim + d];
        out[d] = acc / z;
    }
}

/* OCP FP8 E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; the largest finite magnitude is
 * 1.75 * 2^8 = 448; exponent field 0 holds subnormals m/8 * 2^-6. */
static double e4m3_decode(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 0xf, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

double oracle_e4m3_decode(uint8_t c) { return e4m3_decode(c); }

/* Nearest e4m3 value to x, ties to an even mantissa, magnitudes at or above
 * 448 clamped to 448 (saturating to the largest finite value). x finite. */
static uint8_t e4m3_encode(float x)
{
    uint8_t sign = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0)
        return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {           /* subnormal range: multiples of 2^-9 */
        double m = rint(a * 512.0);     /* round to nearest, ties to even */
        return sign | (uint8_t)m;       /* m == 8 is the smallest normal, 0x08 */
    }
    int e = ilogb(a);                   /* a in [2^e, 2^(e+1)) */
    double m = rint((a / ldexp(1.0, e) - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        e += 1;
    }
    return sign | (uint8_t)(((e + 7) << 3) | (int)m);
}

uint8_t oracle_e4m3_encode(float x) { return e4m3_encode(x); }

/* Quantise one row of n inputs to e4m3 codes with one fp32 scale: amax is
 * the largest magnitude, scale = amax / 448 and code = e4m3(x * (448 /
 * amax)), each step rounded to fp32 (zero row: scale 0, codes 0). */
static void quantize_row(const uint16_t *x, int dtype, int32_t n, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int32_t i = 0; i < n; ++i) {
        float a = (float)fabs(widen(x[i], dtype));
        if (a > amax)
            amax = a;
    }
    float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
    *scale = amax / 448.0f;
    for (int32_t i = 0; i < n; ++i) {
        float v = (float)widen(x[i], dtype) * inv;
        codes[i] = e4m3_encode(v);
    }
}

/* fp8 pools: each (block, head) tile is block_size rows of head_dim e4m3
 * codes followed by block_size fp32 row scales. */
static size_t fp8_tile_bytes(int32_t block_size, int32_t head_dim)
{
    return (size_t)block_size * (size_t)head_dim + 4 * (size_t)block_size;
}

/* Write new tokens into fp8 pools: quantise each (token, head) row. */
int oracle_write_kv_fp8(const uint16_t *key, const uint16_t *value, int io_dtype,
                        int64_t num_tokens, int32_t num_heads, int32_t head_dim,
                        const int64_t *slot_mapping, uint8_t *key_cache, uint8_t *value_cache,
                        int64_t num_blocks, int32_t block_size)
{
    for (int64_t t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= num_blocks * block_size)
            return -1;
    size_t tile = fp8_tile_bytes(block_size, head_dim);
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        int64_t block = slot / block_size, offset = slot % block_size;
        for (int32_t h = 0; h < num_heads; ++h) {
            size_t base = (size_t)(block * num_heads + h) * tile;
            size_t src = (size_t)((t * num_heads + h) * head_dim);
            float sk, sv;
            quantize_row(key + src, io_dtype, head_dim, key_cache + base + offset * head_dim, &sk);
            quantize_row(value + src, io_dtype, head_dim, value_cache + base + offset * head_dim,
                         &sv);
            memcpy(key_cache + base + (size_t)block_size * head_dim + 4 * offset, &sk, 4);
            memcpy(value_cache + base + (size_t)block_size * head_dim + 4 * offset, &sv, 4);
        }
    }
    return 0;
}

/* One (sequence, head) of a 16-bit cache: gather the context through the
 * block table, then textbook attention. */
static int decode_one(double *out, const uint16_t *q16, const uint16_t *key_cache,
                      const uint16_t *value_cache, int64_t num_blocks, int32_t num_kv_heads,
                      int32_t block_size, int32_t head_dim, int dtype, const int32_t *table,
                      int32_t table_len, int32_t ctx, int32_t kvh, double scale)
{
    if (ctx <= 0) {
        for (int32_t d = 0; d < head_dim; ++d)
            out[d] = 0.0;
        return 0;
    }
    if ((int64_t)(ctx - 1) / block_size >= table_len)
        return -1;
    double *q = malloc(sizeof(double) * (size_t)head_dim);
    double *K = malloc(sizeof(double) * (size_t)ctx * (size_t)head_dim);
    double *V = malloc(sizeof(double) * (size_t)ctx * (size_t)head_dim);
    double *w = malloc(sizeof(double) * (size_t)ctx);
    int rc = 0;
    if (!q || !K || !V || !w) {
        rc = -2;
        goto done;
    }
    for (int32_t d = 0; d < head_dim; ++d)
        q[d] = widen(q16[d], dtype);

    /* 1. Gather: token j of the sequence -> physical block table[j / bs],
     *    offset j % bs. */
    for (int32_t j = 0; j < ctx; ++j) {
        int64_t block = table[j / block_size];
        if (block < 0 || block >= num_blocks) {
            rc = -1;
            goto done;
        }
        size_t base =
            (size_t)(((block * num_kv_heads + kvh) * block_size + j % block_size) * head_dim);
        for (int32_t d = 0; d < head_dim; ++d) {
            K[(size_t)j * head_dim + d] = widen(key_cache[base + d], dtype);
            V[(size_t)j * head_dim + d] = widen(value_cache[base + d], dtype);
        }
    }
    attend(out, q, K, V, ctx, head_dim, scale, w);
done:
    free(q);
    free(K);
    free(V);
    free(w);
    return rc;
}

/* One (sequence, head) of an fp8 cache: the gathered K/V values are the
 * codes times their row scales. */
static int decode_one_fp8(double *out, const uint16_t *q16, int io_dtype,
                          const uint8_t *key_cache, const uint8_t *value_cache,
                          int64_t num_blocks, int32_t num_kv_heads, int32_t block_size,
                          int32_t head_dim, const int32_t *table, int32_t table_len, int32_t ctx,
                          int32_t kvh, double scale)
{
    if (ctx <= 0) {
        for (int32_t d = 0; d < head_dim; ++d)
            out[d] = 0.0;
        return 0;
    }
    if ((int64_t)(ctx - 1) / block_size >= table_len)
        return -1;
    double *q = malloc(sizeof(double) * (size_t)head_dim);
    double *K = malloc(sizeof(double) * (size_t)ctx * (size_t)head_dim);
    double *V = malloc(sizeof(double) * (size_t)ctx * (size_t)head_dim);
    double *w = malloc(sizeof(double) * (size_t)ctx);
    int rc = 0;
    size_t tile = fp8_tile_bytes(block_size, head_dim);
    if (!q || !K || !V || !w) {
        rc = -2;
        goto done;
    }
    for (int32_t d = 0; d < head_dim; ++d)
        q[d] = widen(q16[d], io_dtype);
    for (int32_t j = 0; j < ctx; ++j) {
        int64_t block = table[j / block_size];
        if (block < 0 || block >= num_blocks) {
            rc = -1;
            goto done;
        }
        size_t base = (size_t)(block * num_kv_heads + kvh) * tile;
        int32_t off = j % block_size;
        float sk, sv;
        memcpy(&sk, key_cache + base + (size_t)block_size * head_dim + 4 * off, 4);
        memcpy(&sv, value_cache + base + (size_t)block_size * head_dim + 4 * off, 4);
        for (int32_t d = 0; d < head_dim; ++d) {
            K[(size_t)j * head_dim + d] = e4m3_decode(key_cache[base + off * head_dim + d]) * sk;
            V[(size_t)j * head_dim + d] = e4m3_decode(value_cache[base + off * head_dim + d]) * sv;
        }
    }
    attend(out, q, K, V, ctx, head_dim, scale, w);
done:
    free(q);
    free(K);
    free(V);
    free(w);
    return rc;
}

/* Decode attention for one query token per sequence and head.
 * out is fp64 [num_seqs][num_heads][head_dim]. `scale` is used as given
 * (callers pass the fp32 scale widened to double). num_threads <= 0 uses the
 * OpenMP default. Returns 0, or -1 if some block id or context length does
 * not fit the pool or the table (that (seq, head) is then left unwritten). */
int oracle_decode(double *out, const uint16_t *query, int32_t num_seqs, int32_t num_heads,
                  int32_t num_kv_heads, int32_t head_dim, const uint16_t *key_cache,
                  const uint16_t *value_cache, int64_t num_blocks, int32_t block_size, int dtype,
                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                  const int32_t *context_lens, double scale, int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads)
        return -1;
    int32_t group = num_heads / num_kv_heads;
    int rc = 0;
    int64_t units = (int64_t)num_seqs * num_heads;
#ifdef _OPENMP
    if (num_threads <= 0)
        num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(min : rc)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int32_t s = (int32_t)(u / num_heads), h = (int32_t)(u % num_heads);
        int r = decode_one(out + u * head_dim, query + u * head_dim, key_cache, value_cache,
                           num_blocks, num_kv_heads, block_size, head_dim, dtype,
                           block_tables + (int64_t)s * max_blocks_per_seq,
                           max_blocks_per_seq, context_lens[s], h / group, scale);
        if (r < rc)
            rc = r;
    }
    (void)num_threads;
    return rc;
}

/* oracle_decode for fp8 pools (uint8, tiles of codes then row scales);
 * query in io_dtype. */
int oracle_decode_fp8(double *out, const uint16_t *query, int io_dtype, int32_t num_seqs,
                      int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                      const uint8_t *key_cache, const uint8_t *value_cache, int64_t num_blocks,
                      int32_t block_size, const int32_t *block_tables,
                      int32_t max_blocks_per_seq, const int32_t *context_lens, double scale,
                      int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads)
        return -1;
    int32_t group = num_heads / num_kv_heads;
    int rc = 0;
    int64_t units = (int64_t)num_seqs * num_heads;
#ifdef _OPENMP
    if (num_threads <= 0)
        num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(min : rc)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int32_t s = (int32_t)(u / num_heads), h = (int32_t)(u % num_heads);
        int r = decode_one_fp8(out + u * head_dim, query + u * head_dim, io_dtype, key_cache,
                               value_cache, num_blocks, num_kv_heads, block_size, head_dim,
                               block_tables + (int64_t)s * max_blocks_per_seq,
                               max_blocks_per_seq, context_lens[s], h / group, scale);
        if (r < rc)
            rc = r;
    }
    (void)num_threads;
    return rc;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
