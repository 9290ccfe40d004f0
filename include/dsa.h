/*
 * dsa.h -- libdsa: the DeepSeek Sparse Attention (DSA) hot path on NVIDIA B200
 * (sm_100a).  Plain C ABI: device pointers, sizes and a CUDA stream; no C++ or
 * framework types cross it.
 *
 * The method (sources named by page title and section):
 *   "SGLang Day-0 support for DeepSeek-V3.2" (winzheng.jp review), section
 *   "DeepSeek Sparse Attention": a Lightning Indexer -- a light FP8 scorer --
 *   rates, for every query, the tokens before it; top-k token selection keeps
 *   the most relevant key/value entries; core attention then runs on those
 *   entries only, so its cost falls from O(L^2) to O(Lk).  The same section
 *   fixes the caches: the indexer key & key_scale cache uses page size 64, the
 *   token-level sparse operator page size 1.
 *   "DeepSeek-V3.2-Exp DSA deployment guide" (m.nxbn.cn), section 3.1: topk
 *   2048, FP8 indexer, fp8_e4m3 KV cache; section 5.1: a sequence shorter than
 *   topk falls back to dense attention (all positions are kept).
 *   "DeepSeek V3.2 usage guide" (SGLang docs), attention-kernel section: the
 *   sparse MLA kernels take bf16 q with a bf16 or FP8 KV cache.
 *
 * The operations (the pages print no formulas; these are the problem's
 * definitions):
 *   indexer   I[t,s] = k_scale[s] * q_scale[t] * sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:]),
 *             for s <= pos(t)
 *   top-k     the min(k, pos+1) positions with the largest I[t,.]; equal scores
 *             go to the lower position; -1 pads the rest
 *   MLA       per head h: z_s = softmax_scale * q[t,h,:] . kv_s  over the
 *             selected s (kv_s = stored row * kv_scale[s]),
 *             o[t,h,:] = softmax(z) . kv[:, 0:d_v],  lse[t,h] = log sum_s exp(z_s)
 *
 * Conventions shared by every call:
 *   - Batch: sequence b owns query rows cu_q[b] .. cu_q[b+1]-1, which are its
 *     LAST nq_b tokens, so query i of sequence b sits at position
 *     pos = seq_lens[b] - nq_b + i and attends to positions 0..pos.
 *   - All array pointers are DEVICE pointers owned by the caller and borrowed
 *     until the work queued on `stream` has finished.  The library allocates no
 *     memory, creates no streams and never synchronises (except
 *     dsa_device_check).  Work is queued on `stream` in call order.
 *   - Every argument is validated on the host before anything is queued; on
 *     failure the call returns an error status, queues nothing and sets a
 *     thread-local message (dsa_last_error_message).  A valid batch with
 *     total_q == 0 is a no-op that returns DSA_OK without looking further.
 *   - Data pointers must be 16-byte aligned; row strides are given in elements.
 *   - Index and table entries read on the device are range-checked; a bad entry
 *     is skipped (contributes nothing) and recorded in a per-device check word
 *     that dsa_device_check reads.  Kernels never trap.
 */
#ifndef LIBDSA_DSA_H_
#define LIBDSA_DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

/* A cudaStream_t.  NULL means the legacy default stream. */
typedef void* dsa_stream_t;

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARGUMENT = 1,    /* null pointer, bad size, misalignment */
    DSA_ERR_UNSUPPORTED = 2,         /* valid, but a shape/dtype this build has no kernel for */
    DSA_ERR_WORKSPACE_TOO_SMALL = 3,
    DSA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
    DSA_ERR_DEVICE_CHECK = 5         /* a kernel recorded a bad index/table entry or a timeout */
} dsa_status_t;

typedef enum dsa_dtype {
    DSA_F32 = 0,
    DSA_BF16 = 1,
    DSA_FP8_E4M3 = 2                 /* OCP e4m3 ("fn": no infinities, max 448) */
} dsa_dtype_t;

/* Device check codes (dsa_device_check). */
#define DSA_CHECK_NONE 0
#define DSA_CHECK_BAD_PAGE 1         /* block-table entry outside [0, num_pages), or a
                                        cache_store slot outside [0, num_rows) */
#define DSA_CHECK_BAD_INDEX 2        /* top-k index outside [-1, pos] */
#define DSA_CHECK_BAD_BATCH 3        /* nq_b > seq_lens[b], seq_lens[b] > max_seq_len, ... */
#define DSA_CHECK_TIMEOUT 4          /* a bounded on-chip wait gave up */
#define DSA_CHECK_FP16_RANGE 5       /* the tensor-core attention met a bf16 query or
                                        latent-KV value of magnitude > 65504 (or a
                                        non-finite one): its fp16 operands saturate
                                        there, so that output is not exact */

/* A ragged batch of sequences.  Host fields are upper bounds used to size
 * grids and check strides; device arrays are read by the kernels. */
typedef struct dsa_batch {
    int32_t num_seqs;               /* B >= 1 */
    int32_t total_q;                /* T = cu_q[B] (host copy) */
    int32_t max_seq_len;            /* >= every seq_lens[b] (host) */
    int32_t reserved;
    const int32_t* cu_q;            /* device [B+1], non-decreasing, cu_q[0] = 0 */
    const int32_t* seq_lens;        /* device [B], L_b >= nq_b */
} dsa_batch_t;

/* A paged per-token cache: logical token s of sequence b lives in physical page
 * block_table[b * bt_stride + s / page_size], row s % page_size.
 *   indexer key cache: page_size 64, dim d_I, dtype FP8 (or F32), scale = k_scale
 *   latent KV cache:   page_size 1 (block_table is then a slot table), dim d_qk,
 *                      dtype BF16 / FP8 (or F32), scale = per-token kv scale */
typedef struct dsa_paged_cache {
    const void* data;               /* device [num_pages][page_size][dim] of dtype */
    const float* scale;             /* device [num_pages][page_size] fp32, or NULL (= 1) */
    const int32_t* block_table;     /* device [num_seqs][bt_stride] int32 */
    int64_t num_pages;
    int32_t page_size;
    int32_t dim;
    int32_t bt_stride;              /* >= ceil(max_seq_len / page_size) */
    dsa_dtype_t dtype;
} dsa_paged_cache_t;

/*
 * dsa_indexer_logits -- Lightning Indexer scores.
 *   q       [T][heads][dim] of q_dtype; q_scale [T] fp32 or NULL (= 1)
 *   w       [T][heads] fp32 per-head weights
 *   k_cache page_size 64, dim == dim, dtype == q_dtype
 *   logits  [T][ld_logits] fp32 output, ld_logits >= batch->max_seq_len.
 *           Row t holds I[t, s] for s in [0, pos(t)]; entries after pos(t) are
 *           unspecified (some are written with -inf).
 * Kernels: FP8 e4m3 q/k with heads = 64, dim = 128 (tcgen05 tensor cores);
 *          F32 q/k with heads <= 64, dim <= 128, dim % 4 == 0 (CUDA cores).
 */
DSA_API dsa_status_t dsa_indexer_logits(const void* q, dsa_dtype_t q_dtype, const float* q_scale,
                                        const float* w, int32_t heads, int32_t dim,
                                        const dsa_paged_cache_t* k_cache, const dsa_batch_t* batch,
                                        float* logits, int64_t ld_logits, dsa_stream_t stream);

/*
 * dsa_topk -- per-row top-k selection over logits[t][0..pos(t)].
 *   idx [T][k] int32 output: the selected positions in ascending order, then
 *   -1 padding.  1 <= k <= 65536.  The result is deterministic.
 *   Ties at the k-th score keep the lowest positions; -0.0 equals +0.0.
 *   Logits must not be NaN.
 */
DSA_API dsa_status_t dsa_topk(const float* logits, int64_t ld_logits, const dsa_batch_t* batch,
                              int32_t k, int32_t* idx, dsa_stream_t stream);

/*
 * dsa_sparse_mla_prefill -- attention of each query row over its selected
 * latent-KV rows (one pass per query; no workspace).
 *   q        [T][heads][d_qk] of q_dtype
 *   kv       page_size 1, dim == d_qk; V is the first d_v columns of each row
 *   idx      [T][k] logical positions from dsa_topk (-1 entries are skipped)
 *   out      [T][heads][d_v] of out_dtype;  lse [T][heads] fp32 or NULL
 *            (natural log; -inf and o = 0 for a row with no valid index)
 * Kernels: BF16 q with BF16 or FP8 (per-token scale) KV, heads = 128,
 *          d_qk = 576, d_v = 512, out BF16 (tcgen05 tensor cores on pairs of
 *          SMs; S = q.kv^T and P.V on fp16 operands: fp8 codes convert exactly,
 *          bf16 q and rows within +-65504; a value fp16 cannot hold saturates and
 *          is reported as DSA_CHECK_FP16_RANGE);
 *          F32 q/KV with heads <= 16, d_qk <= 576, d_v <= 512, d_v % 4 == 0
 *          (CUDA cores).
 */
DSA_API dsa_status_t dsa_sparse_mla_prefill(const void* q, dsa_dtype_t q_dtype, int32_t heads,
                                            int32_t d_qk, int32_t d_v, float softmax_scale,
                                            const dsa_paged_cache_t* kv, const dsa_batch_t* batch,
                                            const int32_t* idx, int32_t k, void* out,
                                            dsa_dtype_t out_dtype, float* lse, dsa_stream_t stream);

/*
 * dsa_sparse_mla_decode -- as dsa_sparse_mla_prefill, for few query rows: the
 * selected list of each row is split across CTAs and the partial results are
 * merged by log-sum-exp.  Needs a caller-owned workspace of at least
 * dsa_sparse_mla_decode_workspace_size(...) bytes (16-byte aligned).
 */
DSA_API size_t dsa_sparse_mla_decode_workspace_size(int32_t total_q, int32_t heads, int32_t d_v,
                                                    int32_t k);
DSA_API dsa_status_t dsa_sparse_mla_decode(const void* q, dsa_dtype_t q_dtype, int32_t heads,
                                           int32_t d_qk, int32_t d_v, float softmax_scale,
                                           const dsa_paged_cache_t* kv, const dsa_batch_t* batch,
                                           const int32_t* idx, int32_t k, void* out,
                                           dsa_dtype_t out_dtype, float* lse, void* workspace,
                                           size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_sparse_mla_decode_noalloc -- dsa_sparse_mla_decode for callers that cannot
 * hand over a workspace: the split partials go to a fixed array that the library
 * holds in device memory (a file-scope __device__ array of
 * DSA_NOALLOC_SCRATCH_BYTES per device) instead.  This call is an addition of
 * this library; the DeepSeek-V3.2 pages describe no such variant.
 *
 * Who needs it: a caller with no device allocator of its own (a plain C host
 * program, a plug-in that must not touch the host framework's memory pool), or
 * one that has committed every free byte of HBM to its KV caches at start-up
 * and so has no room left to carve a workspace from.  Nothing in the call
 * allocates or frees device memory; the array is set aside by the CUDA runtime
 * when the library's module holding it is loaded on the device.
 *
 * Limits and rules:
 *   - dsa_sparse_mla_decode_workspace_size(total_q, heads, d_v, k) must not
 *     exceed DSA_NOALLOC_SCRATCH_BYTES (20 MiB); a larger need returns
 *     DSA_ERR_WORKSPACE_TOO_SMALL with a message and queues nothing.  The split
 *     rule of this version keeps rows x splits <= 74, so its largest need is
 *     74 x 128 heads x 512 x 4 B plus the lse (19.4 MB) and every call the
 *     kernels accept fits (32 decode rows at k = 2048 need 16.03 MiB).
 *   - The first call on each device looks the array's address up (with that
 *     device current) and caches it; make that first call before beginning any
 *     stream capture.
 *   - There is one array per device: two calls on one device whose executions
 *     may overlap (different streams not ordered by events, or different host
 *     threads) race on it and give wrong results.  Calls on one stream are safe.
 *   - The array keeps whatever the last call left in it.  Every call writes each
 *     partial it reads before reading it, so nothing needs to start at zero.
 * Other arguments, the kernels used and the results are those of
 * dsa_sparse_mla_decode.
 */
#define DSA_NOALLOC_SCRATCH_BYTES ((size_t)20 << 20)
DSA_API dsa_status_t dsa_sparse_mla_decode_noalloc(const void* q, dsa_dtype_t q_dtype,
                                                   int32_t heads, int32_t d_qk, int32_t d_v,
                                                   float softmax_scale, const dsa_paged_cache_t* kv,
                                                   const dsa_batch_t* batch, const int32_t* idx,
                                                   int32_t k, void* out, dsa_dtype_t out_dtype,
                                                   float* lse, dsa_stream_t stream);

/*
 * dsa_decode -- the whole decode step in one call: indexer logits -> top-k ->
 * sparse MLA (split + merge), queued back to back on `stream`.  The logits and
 * the index lists live in the workspace; idx_out (nullable, [T][k]) receives a
 * copy of the selection.  Arguments mean what they mean in the calls above.
 */
DSA_API size_t dsa_decode_workspace_size(const dsa_batch_t* batch, int32_t k, int32_t heads,
                                         int32_t d_v);
DSA_API dsa_status_t dsa_decode(const void* q_idx, dsa_dtype_t q_idx_dtype,
                                const float* q_idx_scale, const float* w, int32_t idx_heads,
                                int32_t idx_dim, const dsa_paged_cache_t* k_cache, int32_t k,
                                const void* q, dsa_dtype_t q_dtype, int32_t heads, int32_t d_qk,
                                int32_t d_v, float softmax_scale, const dsa_paged_cache_t* kv,
                                const dsa_batch_t* batch, int32_t* idx_out, void* out,
                                dsa_dtype_t out_dtype, float* lse, void* workspace,
                                size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_indexer_topk -- the indexer and the top-k without the full logits matrix
 * ("SGLang Day-0 support for DeepSeek-V3.2", its launch lines' FUSE_TOPK switch: the
 * selection fused with the scoring).  The query rows are processed in blocks whose
 * logits take at most 80 MB of the L2 (592 rows at 32K context, 148 at 128K); each
 * block's logits go to the workspace and are selected from at once, so they do not
 * round-trip through HBM and the memory needed is one block, not [T][L].
 * Arguments and results are those of dsa_indexer_logits followed by dsa_topk
 * (idx [T][k]: identical lists); workspace: at least dsa_indexer_topk_workspace_size
 * bytes, 16-byte aligned, contents undefined afterwards.  A larger workspace takes
 * larger blocks (the whole batch if its logits fit, else 148 x 2^m rows): fewer,
 * longer launches whose logits no longer stay in L2 -- with the whole batch in one
 * block this is dsa_indexer_logits followed by dsa_topk.  Meant for prefill-sized batches;
 * for decode, dsa_decode keeps the whole step in one call.
 */
DSA_API size_t dsa_indexer_topk_workspace_size(const dsa_batch_t* batch);
DSA_API dsa_status_t dsa_indexer_topk(const void* q, dsa_dtype_t q_dtype, const float* q_scale,
                                      const float* w, int32_t heads, int32_t dim,
                                      const dsa_paged_cache_t* k_cache, const dsa_batch_t* batch,
                                      int32_t k, int32_t* idx, void* workspace,
                                      size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_cache_store -- writes n new tokens into a cache, the step before the
 * indexer and the attention read them: the indexer key cache (page size 64,
 * FP8 with a per-token key scale) and the latent-KV cache (page size 1, BF16
 * or FP8 with a per-token scale).  Sources: "SGLang Day-0 support for
 * DeepSeek-V3.2", section "DeepSeek Sparse Attention" (the key & key_scale
 * cache, the token-level cache) and section "Future work" (FP8 KV cache);
 * "DeepSeek-V3.2-Exp DSA deployment guide", section 3.1 (fp8_e4m3 KV cache).
 *   x             [n][dim] of x_dtype (DSA_F32 or DSA_BF16), row-major
 *   slot_mapping  [n] int64: the cache row of token i, i.e. physical page *
 *                 page_size + position within the page (for a dsa_paged_cache_t:
 *                 block_table[b][s / page_size] * page_size + s % page_size);
 *                 a negative entry skips token i
 *   cache_data    [num_rows][dim] of cache_dtype -- the page array of a cache
 *                 seen as num_pages * page_size rows
 *   cache_scale   [num_rows] fp32, written for an FP8 cache; ignored (may be
 *                 NULL) for BF16 / F32 caches
 * FP8 cache: scale = amax / 448 in fp32 with amax = max |x_e| of the row (1 for
 * an all-zero row, or when amax / 448 underflows to 0), code_e = e4m3(x_e /
 * scale): the quotient is an IEEE fp32 division (correctly rounded), rounded to
 * e4m3 to nearest even and saturated at +-448, so that code * scale
 * dequantises.  BF16
 * cache: x rounded to nearest even.  F32 cache: x widened exactly.
 * dim must be a multiple of 16 in [16, 1024]; pointers 16-byte aligned
 * (slot_mapping 8, cache_scale 4).  A slot >= num_rows is skipped and recorded
 * as DSA_CHECK_BAD_PAGE.  Two tokens with the same slot race (either may win).
 */
DSA_API dsa_status_t dsa_cache_store(const void* x, dsa_dtype_t x_dtype, int32_t n, int32_t dim,
                                     const int64_t* slot_mapping, void* cache_data,
                                     dsa_dtype_t cache_dtype, float* cache_scale, int64_t num_rows,
                                     dsa_stream_t stream);

/* Synchronises `stream`, then reads the current device's check word into *code
 * (a DSA_CHECK_* value, 0 if nothing was recorded) and clears it if `reset`.
 * Returns DSA_ERR_DEVICE_CHECK when a code was recorded.  The word is shared by
 * all streams of the device. */
DSA_API dsa_status_t dsa_device_check(dsa_stream_t stream, int32_t* code, int32_t reset);

/* The message of the last failed call on this thread ("" if none). */
DSA_API const char* dsa_last_error_message(void);
DSA_API const char* dsa_status_string(dsa_status_t status);
DSA_API int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LIBDSA_DSA_H_ */
