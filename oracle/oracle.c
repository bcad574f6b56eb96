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

/* One (sequence, head): gather, then textbook softmax attention in fp64. */
static int decode_one(double *out, const uint16_t *q16, const uint16_t *key_cache,
                      const uint16_t *value_cache, int64_t num_blocks, int32_t num_heads,
                      int32_t block_size, int32_t head_dim, int dtype, const int32_t *table,
                      int32_t table_len, int32_t ctx, int32_t h, double scale)
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
        size_t base = (size_t)(((block * num_heads + h) * block_size + j % block_size) * head_dim);
        for (int32_t d = 0; d < head_dim; ++d) {
            K[(size_t)j * head_dim + d] = widen(key_cache[base + d], dtype);
            V[(size_t)j * head_dim + d] = widen(value_cache[base + d], dtype);
        }
    }

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
                  int32_t head_dim, const uint16_t *key_cache, const uint16_t *value_cache,
                  int64_t num_blocks, int32_t block_size, int dtype,
                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                  const int32_t *context_lens, double scale, int num_threads)
{
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
                           num_blocks, num_heads, block_size, head_dim, dtype,
                           block_tables + (int64_t)s * max_blocks_per_seq,
                           max_blocks_per_seq, context_lens[s], h, scale);
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
