/*
 * pagedkv.h - C ABI of a B200 (sm_100a) paged-KV-cache decode library.
 *
 * The method: PagedAttention keeps the KV cache in fixed-size physical blocks
 * (16 tokens by default) that may lie anywhere in a pool; each sequence
 * reaches its blocks through a block table that maps logical block i to a
 * physical block id ("vLLM基础：架构、推理流程与关键组件", §2.3;
 * "啃透vLLM源码", §2.2). Decode-step attention reads the caches through
 * those physical block indices ("VLLM源码解析", core technology,
 * paged_attention_forward). Shared blocks are copied before a sequence
 * writes into them (copy-on-write, "vLLM基础", §2.3).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Cache layout: key_cache and value_cache are two separate device arrays
 *   [num_blocks][num_kv_heads][block_size][head_dim] of 16-bit elements
 *   (fp16 or bf16), row-major. Token t of a sequence lives in physical block
 *   block_table[t / block_size] at offset t % block_size; its "slot" is
 *   block * block_size + offset.
 * - fp8 caches (PA_FP8_E4M3; KV-cache quantisation, which "vLLM基础", §2.5
 *   names as further tuning on top of paging): each (block, head) tile is
 *   block_size rows of head_dim OCP e4m3 codes followed by block_size fp32
 *   row scales, [num_blocks][num_kv_heads][block_size*head_dim + 4*block_size]
 *   bytes; a row's values are its codes times its scale. Writes quantise a
 *   row x as scale = amax/448, codes = e4m3(x * (448/amax)) (fp32 steps,
 *   round to nearest even, saturating). Query, key, value and outputs are
 *   then of the descriptor's io_dtype (PA_F16 or PA_BF16).
 * - Supported shapes: head_dim 64 or 128; block_size 8, 16 or 32; num_heads
 *   a multiple of num_kv_heads. With G = num_heads / num_kv_heads > 1
 *   (grouped heads, not on the pages), query head h reads K/V head h / G.
 * - Ownership: the caller owns every buffer, including the decode
 *   workspace. The library allocates no memory, keeps no per-call state and
 *   never synchronises; every call only enqueues kernels on `stream` (a
 *   cudaStream_t passed as void*, NULL = the legacy default stream) on the
 *   current CUDA device. Calls are safe from several host threads.
 * - Errors: arguments are checked on the host before anything is launched;
 *   a failed check returns a status and launches nothing
 *   (pa_last_error() then describes it). PA_ERR_CUDA means a launch failed.
 *   Device-side checks (block ids, slots, context lengths, bounded waits)
 *   cannot return a status; each call takes an optional device int32
 *   `dev_err` (may be NULL) into which the kernels OR the PA_DEVERR_* bits
 *   below. The caller zeroes it and reads it after synchronising.
 * - Alignment: cache, key, value and query pointers must be 16-byte aligned,
 *   and so must the workspace.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad alignment ... */
    PA_ERR_UNSUPPORTED = 2, /* valid but not built: head_dim, block_size, GQA ... */
    PA_ERR_WORKSPACE = 3,   /* decode workspace missing or too small */
    PA_ERR_CUDA = 4         /* a CUDA launch or attribute call failed */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_F32 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

/* Shape of one layer's K (and, identically, V) cache. dtype is the storage:
 * PA_F16, PA_BF16 or PA_FP8_E4M3. io_dtype is read for fp8 caches only: the
 * type of query, key and value rows (PA_F16 or PA_BF16); 16-bit caches take
 * rows of their own dtype. */
typedef struct {
    int32_t num_blocks;
    int32_t block_size;
    int32_t num_kv_heads;
    int32_t head_dim;
    pa_dtype dtype;
    pa_dtype io_dtype;
} pa_cache_desc;

/* Bits the kernels OR into *dev_err. */
#define PA_DEVERR_BLOCK_ID 1    /* a block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 2 /* context_len < 0, > max_context_len, or past the table */
#define PA_DEVERR_SLOT 4        /* a slot >= num_blocks * block_size */
#define PA_DEVERR_TIMEOUT 8     /* a bounded wait on a shared-memory copy ran out */
#define PA_DEVERR_COPY_PAIR 16  /* a copy pair id outside [0, num_blocks) */

/* pa_write_kv - store the K and V of new tokens in their cache slots.
 *
 * Follows the request lifecycle's allocation and append steps ("vLLM基础",
 * §2.2 steps 4-6) and the in-order slot fill of a logical block
 * ("啃透vLLM源码", §2.2, append_tokens): token t's K/V go to
 * (slot / block_size, head, slot % block_size, :) for every head.
 *
 * key, value    device [num_tokens][num_heads][head_dim], cache dtype.
 * slot_mapping  device int64 [num_tokens]; a negative slot is padding and is
 *               skipped; a slot >= num_blocks*block_size sets
 *               PA_DEVERR_SLOT and is skipped.
 * key_cache, value_cache  device, layout above; written in place.
 * num_tokens == 0 is a no-op. Two tokens mapped to one slot race.
 */
pa_status pa_write_kv(const void *key, const void *value, int32_t num_tokens,
                      int32_t num_heads, const int64_t *slot_mapping, void *key_cache,
                      void *value_cache, const pa_cache_desc *cache, int32_t *dev_err,
                      void *stream);

/* Bytes of workspace pa_decode needs. partition_size as for pa_decode; with
 * 0 (automatic) the bound covers every partition size the automatic choice
 * can take. Returns 0 when no workspace is needed and (size_t)-1 on
 * invalid arguments. */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size);

/* The partition size pa_decode uses for these arguments (tokens per CTA
 * work unit); >= max_context_len means a single pass without partitions to
 * merge. The cache descriptor decides the kernel and so the work units: one
 * CTA row per (sequence, query head), or per (sequence, K/V head) when
 * grouped query heads take the grouped kernel (2 <= G <= 16 with a 16-bit
 * cache, or with an fp8 cache of f16 rows and head_dim 128). Returns -1 on
 * invalid arguments. */
int32_t pa_decode_partition_size(int32_t num_seqs, int32_t num_heads,
                                 const pa_cache_desc *cache, int32_t max_context_len,
                                 int32_t partition_size);

/* pa_decode - one decode step of paged attention: for every sequence s and
 * head h, out[s,h,:] = softmax(scale * q K^T) V over the context_lens[s]
 * tokens that the block table of s reaches ("VLLM源码解析", core technology:
 * attention over key_cache/value_cache through physical block indices;
 * "vLLM基础", §2.3 block table).
 *
 * out           device [num_seqs][num_heads][head_dim] of out_dtype
 *               (PA_F16, PA_BF16 or PA_F32).
 * query         device [num_seqs][num_heads][head_dim], cache dtype (fp8
 *               caches: the descriptor's io_dtype). num_heads must be a
 *               multiple of cache->num_kv_heads.
 * block_tables  device int32 [num_seqs][max_blocks_per_seq]; only the first
 *               ceil(context_len / block_size) entries of a row are read.
 * context_lens  device int32 [num_seqs]; 0 gives a zero output row.
 * max_context_len  host; >= every context_lens[s] (a larger value is
 *               allowed; a smaller one sets PA_DEVERR_CONTEXT_LEN).
 * scale         multiplies q.k before the softmax (1/sqrt(head_dim) usually).
 * partition_size  0 = automatic; else tokens per work unit, a positive
 *               multiple of 32 up to 8192. A sequence longer than it is split
 *               into partitions whose partial results (running max, sum and
 *               unnormalised output, fp32) go to the workspace; the last CTA
 *               of a sequence to finish merges them with the log-sum-exp
 *               rule (when num_seqs * num_heads > 65536, a second kernel).
 * workspace     device, >= pa_decode_workspace_size(...) bytes when that is
 *               non-zero (may be NULL otherwise). Its first 256 KiB hold
 *               arrival counters that must be zero before the first call
 *               that uses the workspace; every call leaves them zero
 *               (zero-fill a new workspace once and keep it for this
 *               library). The rest is scratch. Two calls sharing one
 *               workspace on different streams race.
 * Precision: q.k products and sums, the softmax (running max, exponentials,
 * running sum) and the P.V sums are fp32. The softmax weight p of the P.V
 * products is rounded to the operand type first in three cases: to f16 with
 * f16 rows (a product of two f16 values is exact in fp32); to a bf16 head
 * plus a bf16 remainder (about 16 significant bits) with bf16 rows on the
 * grouped-heads kernel; and, with fp8 caches on the grouped-heads kernel,
 * p times the row's V scale over the largest V scale seen so far, to f16.
 * Otherwise (bf16 rows, and fp8 caches, with one CTA per query head) p
 * stays fp32. The output is rounded once, to out_dtype. A block id outside
 * the pool sets PA_DEVERR_BLOCK_ID and makes that sequence's output NaN.
 */
pa_status pa_decode(void *out, pa_dtype out_dtype, const void *query, int32_t num_seqs,
                    int32_t num_heads, const void *key_cache, const void *value_cache,
                    const pa_cache_desc *cache, const int32_t *block_tables,
                    int32_t max_blocks_per_seq, const int32_t *context_lens,
                    int32_t max_context_len, float scale, int32_t partition_size,
                    void *workspace, size_t workspace_bytes, int32_t *dev_err,
                    void *stream);

/* pa_write_kv_decode - pa_write_kv followed by pa_decode for a batch in
 * which every sequence appends exactly one token, in one launch.
 *
 * The request lifecycle appends each sequence's new token and runs attention
 * over all its tokens ("vLLM基础", §2.2 steps 4-6); here the new token of
 * sequence s is its last context token, position context_lens[s] - 1, and
 * its slot is the one the block table gives that position (the in-order
 * fill of "啃透vLLM源码", §2.2 append_tokens). key/value (device
 * [num_seqs][num_kv_heads][head_dim], cache io dtype, 16-byte aligned)
 * hold the new rows, one per K/V head.
 * The result equals pa_write_kv with that slot mapping followed by
 * pa_decode; the kernel that reads the sequence's last chunk puts the new
 * row into its staged copy and into the cache, so no other launch is needed.
 * Preconditions: the block that receives the new token is read by no other
 * sequence of the call (copy-on-write has already run); context_lens[s] = 0
 * appends nothing. All other arguments and errors are as for pa_decode.
 */
pa_status pa_write_kv_decode(void *out, pa_dtype out_dtype, const void *query, const void *key,
                             const void *value, int32_t num_seqs, int32_t num_heads,
                             void *key_cache, void *value_cache, const pa_cache_desc *cache,
                             const int32_t *block_tables, int32_t max_blocks_per_seq,
                             const int32_t *context_lens, int32_t max_context_len, float scale,
                             int32_t partition_size, void *workspace, size_t workspace_bytes,
                             int32_t *dev_err, void *stream);

/* pa_decode_noalloc - pa_decode without a caller-provided workspace, for
 * callers that cannot allocate device memory when they decode.
 *
 * The pages have no counterpart to this call; it exists for library users.
 * Some programs cannot call cudaMalloc on the path that runs decode: a
 * serving engine that reserved almost all device memory for its KV block
 * pool at start-up (a later allocation fails, or could only succeed by
 * giving up cache blocks), or a runtime that forbids allocation after
 * initialisation because cudaMalloc/cudaFree can synchronise the device and
 * stall every stream. This call takes the same arguments as pa_decode except
 * the workspace, and allocates nothing: split partitions are merged through
 * a fixed PA_NOALLOC_SCRATCH_BYTES array of device memory compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *
 * - Limit: if the partial results need more than PA_NOALLOC_SCRATCH_BYTES
 *   (see pa_decode_workspace_size with the partition size actually used,
 *   pa_decode_partition_size), the call returns PA_ERR_WORKSPACE and
 *   launches nothing; a larger partition_size needs less scratch. Argument
 *   checks run in the same order as pa_decode's, so both calls return the
 *   same status for the same arguments wherever the workspace is not the
 *   cause.
 * - Set-up: the call looks up the array's device address with the device
 *   current, once per device and CUDA context (again after a device reset,
 *   which gives the device a new context); make the first call on each
 *   device before any stream capture.
 * - Sharing: every call in the process on a device uses the same array and
 *   leaves its contents behind. The array's first 256 KiB are the split
 *   arrival counters, which must be zero when a split call's kernel starts:
 *   each split call clears the ones it uses with a cudaMemsetAsync on
 *   `stream` before its kernel (one extra operation in the stream; nothing
 *   is allocated). The rest is scratch that every call writes before it
 *   reads. Calls whose kernels overlap on the GPU (different streams or host
 *   threads) race on the array and give wrong output for the overlapping
 *   calls, with no error reported: serialise them. Since every call clears
 *   its counters first, a race does not reach later, serialised calls.
 * Everything else (arguments, errors, dev_err) is as for pa_decode.
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u << 20)
pa_status pa_decode_noalloc(void *out, pa_dtype out_dtype, const void *query, int32_t num_seqs,
                            int32_t num_heads, const void *key_cache, const void *value_cache,
                            const pa_cache_desc *cache, const int32_t *block_tables,
                            int32_t max_blocks_per_seq, const int32_t *context_lens,
                            int32_t max_context_len, float scale, int32_t partition_size,
                            int32_t *dev_err, void *stream);

/* pa_copy_blocks - copy-on-write duplication of shared blocks ("vLLM基础",
 * §2.3): for each pair i and each layer l, the whole block
 * block_mapping[i][0] of key_caches[l] and value_caches[l] (all heads, all
 * slots) is copied to block block_mapping[i][1].
 *
 * key_caches, value_caches  HOST arrays of num_layers device pointers
 *               (1 <= num_layers <= PA_MAX_LAYERS), every layer shaped by
 *               `cache`.
 * block_mapping device int64 [num_pairs][2] = (src, dst). Destinations must
 *               be distinct and no destination may also be a source (else
 *               the copies race). Ids outside the pool set
 *               PA_DEVERR_COPY_PAIR and that pair is skipped.
 * num_pairs == 0 is a no-op.
 */
#define PA_MAX_LAYERS 256
pa_status pa_copy_blocks(void *const *key_caches, void *const *value_caches,
                         int32_t num_layers, const int64_t *block_mapping,
                         int32_t num_pairs, const pa_cache_desc *cache, int32_t *dev_err,
                         void *stream);

/* pa_swap_blocks - move whole blocks between two pools of the same block
 * shape, typically the GPU pool and a pool in pinned host memory: swap out
 * when GPU memory runs short, swap in before the sequence runs again
 * ("啃透vLLM源码", §3, blocks_to_swap_out / blocks_to_swap_in). For each pair i
 * and layer l, block block_mapping[i][0] of the source K and V caches of
 * layer l is copied to block block_mapping[i][1] of the destination caches.
 *
 * src_key_caches ... dst_value_caches  HOST arrays of num_layers pointers,
 *               each to device memory or to pinned host memory that CUDA has
 *               mapped for the device (cudaHostAlloc / cudaHostRegister);
 *               pageable host memory is refused (PA_ERR_INVALID_ARG) before
 *               any launch. 16-byte aligned.
 * src, dst      pool shapes; block_size, heads, head_dim and dtype must match,
 *               num_blocks may differ.
 * block_mapping int64 [num_pairs][2], device or pinned host memory. Ids
 *               outside their pool set PA_DEVERR_COPY_PAIR and are skipped.
 *               Destinations must be distinct. num_pairs == 0 is a no-op.
 * One launch moves every pair of every layer; the GPU reads or writes the
 * host pool directly over the host link.
 */
pa_status pa_swap_blocks(void *const *src_key_caches, void *const *src_value_caches,
                         const pa_cache_desc *src, void *const *dst_key_caches,
                         void *const *dst_value_caches, const pa_cache_desc *dst,
                         int32_t num_layers, const int64_t *block_mapping, int32_t num_pairs,
                         int32_t *dev_err, void *stream);

/* Self-test of failure detection: one warp waits on a shared-memory barrier
 * that nothing will complete, through the same bounded wait every kernel
 * uses on its bulk copies, giving up after limit_us microseconds (1 ..
 * 1000000). It must then OR PA_DEVERR_TIMEOUT into *dev_err (device memory)
 * and return, leaving the context usable: the way a kernel stuck on a copy
 * reports instead of hanging. No counterpart on the pages. */
pa_status pa_selftest_wait_timeout(int32_t *dev_err, uint32_t limit_us, void *stream);

/* Static text for a status. */
const char *pa_status_string(pa_status status);

/* Details of the last failed call on this host thread ("" if none). */
const char *pa_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
