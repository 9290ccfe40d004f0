// api.cu -- the libdsa C ABI (include/dsa.h): host-side validation, workspace
// carving and kernel launches.  Nothing here allocates, synchronises (except
// dsa_device_check) or creates streams.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "dsa.h"
#include "kernels.h"

namespace {

using namespace dsa;

thread_local std::string g_msg;

// An NVTX range around each entry point (visible in Nsight timelines; a no-op when no
// tool is attached).
struct Range {
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
};

dsa_status_t fail(dsa_status_t st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_msg = buf;
    return st;
}

dsa_status_t ok() {
    g_msg.clear();
    return DSA_OK;
}

dsa_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// The per-device check word: kernels record the first bad table entry / index /
// timeout here (atomicCAS from 0), dsa_device_check reads and clears it.
__device__ int g_check_word;

constexpr int kMaxDevices = 64;
std::mutex g_check_mu;
int* g_check_ptr[kMaxDevices];

cudaError_t check_word(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_check_mu);
    if (!g_check_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_check_word);
        if (e != cudaSuccess) return e;
        g_check_ptr[dev] = static_cast<int*>(p);
    }
    *out = g_check_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool valid_dtype(int d) { return d == DSA_F32 || d == DSA_BF16 || d == DSA_FP8_E4M3; }

constexpr int kMaxSeqLen = 1 << 22;

dsa_status_t check_batch(const dsa_batch_t* b, BatchView* v) {
    if (!b) return fail(DSA_ERR_INVALID_ARGUMENT, "batch is NULL");
    if (b->num_seqs < 1) return fail(DSA_ERR_INVALID_ARGUMENT, "batch.num_seqs must be >= 1");
    if (b->total_q < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "batch.total_q must be >= 0");
    if (b->max_seq_len < 1 || b->max_seq_len > kMaxSeqLen)
        return fail(DSA_ERR_INVALID_ARGUMENT, "batch.max_seq_len must be in [1, %d]", kMaxSeqLen);
    if (!b->cu_q || !b->seq_lens || !aligned4(b->cu_q) || !aligned4(b->seq_lens))
        return fail(DSA_ERR_INVALID_ARGUMENT, "batch.cu_q / batch.seq_lens must be non-NULL, 4-byte aligned");
    *v = BatchView{b->num_seqs, b->total_q, b->max_seq_len, b->cu_q, b->seq_lens};
    return DSA_OK;
}

dsa_status_t check_cache(const dsa_paged_cache_t* c, const char* name, int page_size, int dim,
                         const BatchView& bv, CacheView* v) {
    if (!c) return fail(DSA_ERR_INVALID_ARGUMENT, "%s is NULL", name);
    if (!c->data || !aligned16(c->data))
        return fail(DSA_ERR_INVALID_ARGUMENT, "%s.data must be non-NULL and 16-byte aligned", name);
    if (c->scale && !aligned16(c->scale))
        return fail(DSA_ERR_INVALID_ARGUMENT, "%s.scale must be 16-byte aligned", name);
    if (!c->block_table || !aligned4(c->block_table))
        return fail(DSA_ERR_INVALID_ARGUMENT, "%s.block_table must be non-NULL, 4-byte aligned", name);
    if (!valid_dtype(c->dtype)) return fail(DSA_ERR_INVALID_ARGUMENT, "%s.dtype is not a dsa_dtype_t", name);
    if (c->num_pages < 1) return fail(DSA_ERR_INVALID_ARGUMENT, "%s.num_pages must be >= 1", name);
    if (c->page_size != page_size)
        return fail(DSA_ERR_UNSUPPORTED, "%s.page_size must be %d (got %d)", name, page_size, c->page_size);
    if (c->dim != dim)
        return fail(DSA_ERR_INVALID_ARGUMENT, "%s.dim (%d) must equal the query dim (%d)", name, c->dim, dim);
    const long long need = ((long long)bv.max_seq_len + page_size - 1) / page_size;
    if (c->bt_stride < need)
        return fail(DSA_ERR_INVALID_ARGUMENT, "%s.bt_stride (%d) < ceil(max_seq_len / page_size) = %lld",
                    name, c->bt_stride, need);
    *v = CacheView{c->data, c->scale, c->block_table, (long long)c->num_pages, c->page_size, c->dim,
                   c->bt_stride, (int)c->dtype};
    return DSA_OK;
}

// ---------------------------------------------------------------- indexer
dsa_status_t indexer_validate(const void* q, dsa_dtype_t q_dtype, const float* q_scale,
                              const float* w, int heads, int dim,
                              const dsa_paged_cache_t* k_cache, const BatchView& bv,
                              const float* logits, long long ld, CacheView* kc) {
    dsa_status_t s = check_cache(k_cache, "k_cache", kIndexerPage, dim, bv, kc);
    if (s != DSA_OK) return s;
    if (!q || !aligned16(q)) return fail(DSA_ERR_INVALID_ARGUMENT, "q must be non-NULL, 16-byte aligned");
    if (!w || !aligned16(w)) return fail(DSA_ERR_INVALID_ARGUMENT, "w must be non-NULL, 16-byte aligned");
    if (q_scale && !aligned4(q_scale)) return fail(DSA_ERR_INVALID_ARGUMENT, "q_scale must be 4-byte aligned");
    if (!logits || !aligned16(logits)) return fail(DSA_ERR_INVALID_ARGUMENT, "logits must be non-NULL, 16-byte aligned");
    if (ld < bv.max_seq_len || ld % 4 != 0)
        return fail(DSA_ERR_INVALID_ARGUMENT, "ld_logits (%lld) must be >= max_seq_len and a multiple of 4", ld);
    if (!valid_dtype(q_dtype)) return fail(DSA_ERR_INVALID_ARGUMENT, "q_dtype is not a dsa_dtype_t");
    if ((int)q_dtype != kc->dtype)
        return fail(DSA_ERR_UNSUPPORTED, "indexer q and key cache dtypes must match");
    if (heads < 1 || dim < 1) return fail(DSA_ERR_INVALID_ARGUMENT, "heads and dim must be >= 1");
    if (q_dtype == DSA_FP8_E4M3) {
        if (heads != 64 || dim != 128)
            return fail(DSA_ERR_UNSUPPORTED, "fp8 indexer supports heads = 64, dim = 128");
    } else if (q_dtype == DSA_F32) {
        if (heads > 64 || dim > 128 || dim % 4 != 0)
            return fail(DSA_ERR_UNSUPPORTED, "fp32 indexer supports heads <= 64, dim <= 128, dim %% 4 == 0");
    } else {
        return fail(DSA_ERR_UNSUPPORTED, "indexer supports fp8 e4m3 or fp32 inputs");
    }
    return DSA_OK;
}

cudaError_t indexer_launch(const void* q, const float* q_scale, const float* w, int heads, int dim,
                           const CacheView& kc, const BatchView& bv, float* logits, long long ld,
                           int* check, cudaStream_t st, bool pdl = false, int row0 = 0) {
    if (kc.dtype == kE4M3)  // validated: 64 heads x 128 dims
        return launch_indexer_fp8_tc(q, q_scale, w, kc, bv, logits, ld, check, st, pdl, row0);
    return launch_indexer_generic(q, q_scale, w, heads, dim, kc, bv, logits, ld, check, st, row0);
}

// ---------------------------------------------------------------- top-k
dsa_status_t topk_validate(const float* logits, long long ld, const BatchView& bv, int k,
                           const int* idx) {
    if (!logits || !aligned16(logits)) return fail(DSA_ERR_INVALID_ARGUMENT, "logits must be non-NULL, 16-byte aligned");
    if (!idx || !aligned16(idx)) return fail(DSA_ERR_INVALID_ARGUMENT, "idx must be non-NULL, 16-byte aligned");
    if (ld < bv.max_seq_len || ld % 4 != 0)
        return fail(DSA_ERR_INVALID_ARGUMENT, "ld_logits (%lld) must be >= max_seq_len and a multiple of 4", ld);
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARGUMENT, "k must be in [1, 65536]");
    return DSA_OK;
}

// ---------------------------------------------------------------- sparse MLA
enum class MlaKind { kGenericF32, kTensorCore };

struct MlaPlan {
    MlaKind kind;
    CacheView kv;
};

dsa_status_t mla_check(const void* q, dsa_dtype_t q_dtype, int heads, int d_qk, int d_v,
                       float scale, const dsa_paged_cache_t* kv, const BatchView& bv,
                       const int* idx, int k, const void* out, dsa_dtype_t out_dtype,
                       const float* lse, MlaPlan* plan) {
    dsa_status_t s = check_cache(kv, "kv", 1, d_qk, bv, &plan->kv);
    if (s != DSA_OK) return s;
    if (!q || !aligned16(q)) return fail(DSA_ERR_INVALID_ARGUMENT, "q must be non-NULL, 16-byte aligned");
    if (!idx || !aligned16(idx)) return fail(DSA_ERR_INVALID_ARGUMENT, "idx must be non-NULL, 16-byte aligned");
    if (!out || !aligned16(out)) return fail(DSA_ERR_INVALID_ARGUMENT, "out must be non-NULL, 16-byte aligned");
    if (lse && !aligned16(lse)) return fail(DSA_ERR_INVALID_ARGUMENT, "lse must be 16-byte aligned");
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARGUMENT, "k must be in [1, 65536]");
    if (!(scale > 0.f) || scale != scale) return fail(DSA_ERR_INVALID_ARGUMENT, "softmax_scale must be > 0");
    if (heads < 1 || d_qk < 1 || d_v < 1 || d_v > d_qk)
        return fail(DSA_ERR_INVALID_ARGUMENT, "need heads >= 1 and 1 <= d_v <= d_qk");
    if (!valid_dtype(q_dtype) || !valid_dtype(out_dtype))
        return fail(DSA_ERR_INVALID_ARGUMENT, "q_dtype / out_dtype is not a dsa_dtype_t");
    if (q_dtype == DSA_F32 && plan->kv.dtype == kF32) {
        if (d_qk > 576 || d_v > 512 || heads > 16 || d_v % 4 != 0)
            return fail(DSA_ERR_UNSUPPORTED, "fp32 sparse MLA supports heads <= 16, d_qk <= 576, "
                        "d_v <= 512 with d_v %% 4 == 0");
        if (out_dtype != DSA_F32 && out_dtype != DSA_BF16)
            return fail(DSA_ERR_UNSUPPORTED, "fp32 sparse MLA writes fp32 or bf16 output");
        plan->kind = MlaKind::kGenericF32;
        return DSA_OK;
    }
    if (q_dtype == DSA_BF16 && (plan->kv.dtype == kBF16 || plan->kv.dtype == kE4M3)) {
        if (heads != 128 || d_qk != 576 || d_v != 512)
            return fail(DSA_ERR_UNSUPPORTED, "bf16 sparse MLA supports heads = 128, d_qk = 576, d_v = 512");
        if (out_dtype != DSA_BF16) return fail(DSA_ERR_UNSUPPORTED, "bf16 sparse MLA writes bf16 output");
        if (plan->kv.num_pages >= 0x7FFFFFFFLL)
            return fail(DSA_ERR_UNSUPPORTED, "latent KV caches are limited to 2^31 - 1 rows");
        plan->kind = MlaKind::kTensorCore;
        return DSA_OK;
    }
    return fail(DSA_ERR_UNSUPPORTED, "sparse MLA supports fp32 q + fp32 KV, or bf16 q + bf16/fp8 KV");
}

cudaError_t mla_launch(const MlaPlan& plan, const void* q, int heads, int d_qk, int d_v,
                       float scale, const BatchView& bv, const int* idx, int k, int nsplit,
                       void* out, int out_dtype, float* lse, void* o_part, float* lse_part,
                       int* check, cudaStream_t st, bool pdl = false) {
    // (pdl: the tensor-core kernel waits for its predecessor before reading idx; the
    // CUDA-core kernel does not, so it is always launched plainly)
    if (plan.kind == MlaKind::kTensorCore)
        return launch_mla_tc(q, scale, plan.kv, bv, idx, k, nsplit, out, lse, o_part, lse_part,
                             check, st, pdl);
    return launch_mla_generic(q, heads, d_qk, d_v, scale, plan.kv, bv, idx, k, nsplit, out,
                              out_dtype, lse, static_cast<float*>(o_part), lse_part, check, st);
}

// Split of each row's selection list for decode: enough CTAs to cover the GPU,
// at least 256 selected rows per split, at most 16 splits.
int decode_splits(int total_q, int k) {
    if (total_q <= 0) return 1;
    int by_gpu = (kNumSMs / 2) / total_q;
    int by_k = (k + 255) / 256;
    int n = by_gpu < by_k ? by_gpu : by_k;
    if (n > 16) n = 16;
    return n < 1 ? 1 : n;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t mla_decode_ws(int total_q, int heads, int d_v, int k) {
    const int ns = decode_splits(total_q, k);
    if (ns == 1) return 0;
    const size_t o = (size_t)total_q * ns * heads * d_v * sizeof(float);
    const size_t l = (size_t)total_q * ns * heads * sizeof(float);
    return align_up(o, 256) + align_up(l, 256);
}

dsa_status_t mla_decode_validate(const BatchView& bv, int heads, int d_v, int k, const void* ws,
                                 size_t ws_bytes) {
    const size_t need = mla_decode_ws(bv.total_q, heads, d_v, k);
    if (need && (!ws || !aligned16(ws)))
        return fail(DSA_ERR_INVALID_ARGUMENT, "workspace must be non-NULL and 16-byte aligned");
    if (ws_bytes < need)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need, ws_bytes);
    return DSA_OK;
}

cudaError_t mla_decode_launch(const MlaPlan& plan, const void* q, int heads, int d_qk, int d_v,
                              float scale, const BatchView& bv, const int* idx, int k, void* out,
                              dsa_dtype_t out_dtype, float* lse, void* ws, int* check,
                              cudaStream_t st, bool pdl = false) {
    const int ns = decode_splits(bv.total_q, k);
    if (ns == 1)
        return mla_launch(plan, q, heads, d_qk, d_v, scale, bv, idx, k, 1, out, out_dtype, lse,
                          nullptr, nullptr, check, st, pdl);
    // partials o/l: fp16 from the tensor-core kernel (|o| <= max |v|, 11 significant
    // bits), fp32 from the CUDA-core one; the workspace is sized for fp32 either way
    void* o_part = ws;
    float* l_part = reinterpret_cast<float*>(
        static_cast<char*>(ws) + align_up((size_t)bv.total_q * ns * heads * d_v * 4, 256));
    cudaError_t e = mla_launch(plan, q, heads, d_qk, d_v, scale, bv, idx, k, ns, nullptr,
                               out_dtype, nullptr, o_part, l_part, check, st, pdl);
    if (e != cudaSuccess) return e;
    return launch_mla_combine(o_part, plan.kind == MlaKind::kTensorCore, l_part, bv.total_q, ns,
                              heads, d_v, out, out_dtype, lse, st, pdl);
}

long long decode_ld(int max_seq_len) { return ((long long)max_seq_len + 63) / 64 * 64; }

}  // namespace

extern "C" {

DSA_API dsa_status_t dsa_indexer_logits(const void* q, dsa_dtype_t q_dtype, const float* q_scale,
                                        const float* w, int32_t heads, int32_t dim,
                                        const dsa_paged_cache_t* k_cache, const dsa_batch_t* batch,
                                        float* logits, int64_t ld_logits, dsa_stream_t stream) {
    Range nvtx_range("dsa_indexer_logits");
    BatchView bv;
    CacheView kc;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    s = indexer_validate(q, q_dtype, q_scale, w, heads, dim, k_cache, bv, logits, ld_logits, &kc);
    if (s != DSA_OK) return s;
    if (bv.total_q == 0) return ok();
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    if (e == cudaSuccess)
        e = indexer_launch(q, q_scale, w, heads, dim, kc, bv, logits, ld_logits, check,
                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "indexer launch");
}

DSA_API dsa_status_t dsa_topk(const float* logits, int64_t ld_logits, const dsa_batch_t* batch,
                              int32_t k, int32_t* idx, dsa_stream_t stream) {
    Range nvtx_range("dsa_topk");
    BatchView bv;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    s = topk_validate(logits, ld_logits, bv, k, idx);
    if (s != DSA_OK) return s;
    if (bv.total_q == 0) return ok();
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    if (e == cudaSuccess)
        e = launch_topk(logits, ld_logits, bv, k, idx, check, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "top-k launch");
}

DSA_API dsa_status_t dsa_sparse_mla_prefill(const void* q, dsa_dtype_t q_dtype, int32_t heads,
                                            int32_t d_qk, int32_t d_v, float softmax_scale,
                                            const dsa_paged_cache_t* kv, const dsa_batch_t* batch,
                                            const int32_t* idx, int32_t k, void* out,
                                            dsa_dtype_t out_dtype, float* lse, dsa_stream_t stream) {
    Range nvtx_range("dsa_sparse_mla_prefill");
    BatchView bv;
    MlaPlan plan;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    s = mla_check(q, q_dtype, heads, d_qk, d_v, softmax_scale, kv, bv, idx, k, out, out_dtype,
                      lse, &plan);
    if (s != DSA_OK) return s;
    if (bv.total_q == 0) return ok();
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    if (e == cudaSuccess)
        e = mla_launch(plan, q, heads, d_qk, d_v, softmax_scale, bv, idx, k, 1, out, out_dtype,
                       lse, nullptr, nullptr, check, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sparse MLA launch");
}

DSA_API size_t dsa_sparse_mla_decode_workspace_size(int32_t total_q, int32_t heads, int32_t d_v,
                                                    int32_t k) {
    if (total_q < 0 || heads < 1 || d_v < 1 || k < 1) return 0;
    return mla_decode_ws(total_q, heads, d_v, k);
}

DSA_API dsa_status_t dsa_sparse_mla_decode(const void* q, dsa_dtype_t q_dtype, int32_t heads,
                                           int32_t d_qk, int32_t d_v, float softmax_scale,
                                           const dsa_paged_cache_t* kv, const dsa_batch_t* batch,
                                           const int32_t* idx, int32_t k, void* out,
                                           dsa_dtype_t out_dtype, float* lse, void* workspace,
                                           size_t workspace_bytes, dsa_stream_t stream) {
    Range nvtx_range("dsa_sparse_mla_decode");
    BatchView bv;
    MlaPlan plan;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    s = mla_check(q, q_dtype, heads, d_qk, d_v, softmax_scale, kv, bv, idx, k, out, out_dtype,
                      lse, &plan);
    if (s == DSA_OK) s = mla_decode_validate(bv, heads, d_v, k, workspace, workspace_bytes);
    if (s != DSA_OK) return s;
    if (bv.total_q == 0) return ok();
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    if (e == cudaSuccess)
        e = mla_decode_launch(plan, q, heads, d_qk, d_v, softmax_scale, bv, idx, k, out, out_dtype,
                              lse, workspace, check, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sparse MLA decode launch");
}

DSA_API dsa_status_t dsa_sparse_mla_decode_noalloc(const void* q, dsa_dtype_t q_dtype,
                                                   int32_t heads, int32_t d_qk, int32_t d_v,
                                                   float softmax_scale, const dsa_paged_cache_t* kv,
                                                   const dsa_batch_t* batch, const int32_t* idx,
                                                   int32_t k, void* out, dsa_dtype_t out_dtype,
                                                   float* lse, dsa_stream_t stream) {
    Range nvtx_range("dsa_sparse_mla_decode_noalloc");
    static_assert(kStaticScratchBytes == DSA_NOALLOC_SCRATCH_BYTES, "scratch size mismatch");
    BatchView bv;
    MlaPlan plan;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    s = mla_check(q, q_dtype, heads, d_qk, d_v, softmax_scale, kv, bv, idx, k, out, out_dtype,
                  lse, &plan);
    if (s != DSA_OK) return s;
    const size_t need = mla_decode_ws(bv.total_q, heads, d_v, k);
    if (need > kStaticScratchBytes)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL,
                    "dsa_sparse_mla_decode_noalloc: this batch needs %zu bytes of split scratch "
                    "but the built-in array holds %zu; use dsa_sparse_mla_decode with a workspace",
                    need, kStaticScratchBytes);
    int* check = nullptr;
    void* scratch = nullptr;
    cudaError_t e = check_word(&check);
    if (e != cudaSuccess) return cuda_fail(e, "check word address");
    if (need) {
        e = static_scratch(&scratch);
        if (e != cudaSuccess) return cuda_fail(e, "static scratch address");
    }
    e = mla_decode_launch(plan, q, heads, d_qk, d_v, softmax_scale, bv, idx, k, out, out_dtype, lse,
                          scratch, check, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sparse MLA decode (static scratch) launch");
}

DSA_API size_t dsa_decode_workspace_size(const dsa_batch_t* batch, int32_t k, int32_t heads,
                                         int32_t d_v) {
    if (!batch || batch->total_q < 0 || batch->max_seq_len < 1 || k < 1 || heads < 1 || d_v < 1)
        return 0;
    const size_t T = (size_t)batch->total_q;
    return align_up(T * decode_ld(batch->max_seq_len) * sizeof(float), 256) +
           align_up(T * (size_t)k * sizeof(int32_t), 256) +
           mla_decode_ws(batch->total_q, heads, d_v, k);
}

DSA_API dsa_status_t dsa_decode(const void* q_idx, dsa_dtype_t q_idx_dtype,
                                const float* q_idx_scale, const float* w, int32_t idx_heads,
                                int32_t idx_dim, const dsa_paged_cache_t* k_cache, int32_t k,
                                const void* q, dsa_dtype_t q_dtype, int32_t heads, int32_t d_qk,
                                int32_t d_v, float softmax_scale, const dsa_paged_cache_t* kv,
                                const dsa_batch_t* batch, int32_t* idx_out, void* out,
                                dsa_dtype_t out_dtype, float* lse, void* workspace,
                                size_t workspace_bytes, dsa_stream_t stream) {
    Range nvtx_range("dsa_decode");
    BatchView bv;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARGUMENT, "k must be in [1, 65536]");
    if (idx_out && !aligned16(idx_out))
        return fail(DSA_ERR_INVALID_ARGUMENT, "idx_out must be 16-byte aligned");
    if (!workspace || !aligned16(workspace))
        return fail(DSA_ERR_INVALID_ARGUMENT, "workspace must be non-NULL and 16-byte aligned");
    const size_t need = dsa_decode_workspace_size(batch, k, heads, d_v);
    if (workspace_bytes < need)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need,
                    workspace_bytes);
    // Carve the workspace: logits [T][ld], the selection [T][k], the MLA partials.
    const long long ld = decode_ld(bv.max_seq_len);
    char* p = static_cast<char*>(workspace);
    float* logits = reinterpret_cast<float*>(p);
    p += align_up((size_t)bv.total_q * ld * sizeof(float), 256);
    int* sel = idx_out ? idx_out : reinterpret_cast<int*>(p);
    p += align_up((size_t)bv.total_q * (size_t)k * sizeof(int32_t), 256);
    void* mla_ws = p;

    // Validate every stage before the first launch.
    CacheView kc;
    MlaPlan plan;
    s = indexer_validate(q_idx, q_idx_dtype, q_idx_scale, w, idx_heads, idx_dim, k_cache, bv,
                         logits, ld, &kc);
    if (s == DSA_OK) s = topk_validate(logits, ld, bv, k, sel);
    if (s == DSA_OK)
        s = mla_check(q, q_dtype, heads, d_qk, d_v, softmax_scale, kv, bv, sel, k, out, out_dtype,
                      lse, &plan);
    if (s != DSA_OK) return s;
    if (bv.total_q == 0) return ok();
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (e == cudaSuccess)
        e = indexer_launch(q_idx, q_idx_scale, w, idx_heads, idx_dim, kc, bv, logits, ld, check, st,
                           true);
    // every kernel of the chain starts as a programmatic dependent of the kernel before
    // it and waits for that kernel before touching memory it may write: the tensor-core
    // indexer before reading anything (its predecessor is the caller's earlier work),
    // top-k before the logits, attention before the selection, the merge before the
    // partials; each kernel finishes only after its own wait, so the chain is ordered
    // after everything earlier on the stream (the CUDA-core indexer ignores pdl)
    if (e == cudaSuccess) e = launch_topk(logits, ld, bv, k, sel, check, st, true);
    if (e == cudaSuccess)
        e = mla_decode_launch(plan, q, heads, d_qk, d_v, softmax_scale, bv, sel, k, out, out_dtype,
                              lse, mla_ws, check, st, true);
    return e == cudaSuccess ? ok() : cuda_fail(e, "decode launch");
}

// Rows per block of dsa_indexer_topk for a workspace of `bytes` (by default the minimum:
// the logits of one block take at most 80 MB of the 126 MB L2, so the top-k reads them
// while they are still on chip).  The whole batch if it fits; else, where the workspace
// allows 148 rows or more, 148 x 2^m rows: the top-k runs one CTA per row and the indexer
// 4 rows per CTA over 592 / (rows / 4) key chunks, so both fill whole waves of the 148
// SMs.
constexpr size_t kL2BlockBytes = (size_t)80 << 20;

int indexer_topk_block_rows(int total_q, long long ld, size_t bytes = kL2BlockBytes) {
    const long long budget = (long long)(bytes / ((size_t)ld * sizeof(float)));
    long long rows;
    if (budget >= total_q) {
        rows = total_q;                    // the whole batch in one block
    } else if (budget >= kNumSMs) {
        rows = kNumSMs;
        while (rows * 2 <= budget) rows *= 2;
    } else {
        rows = budget & ~3LL;
    }
    if (rows < 4) rows = 4;
    if (rows > total_q) rows = total_q;
    return (int)rows;
}

DSA_API size_t dsa_indexer_topk_workspace_size(const dsa_batch_t* batch) {
    if (!batch || batch->total_q < 0 || batch->max_seq_len < 1) return 0;
    const long long ld = decode_ld(batch->max_seq_len);
    const int rows = indexer_topk_block_rows(batch->total_q, ld);
    return align_up((size_t)(rows > 0 ? rows : 0) * (size_t)ld * sizeof(float), 256);
}

DSA_API dsa_status_t dsa_indexer_topk(const void* q, dsa_dtype_t q_dtype, const float* q_scale,
                                      const float* w, int32_t heads, int32_t dim,
                                      const dsa_paged_cache_t* k_cache, const dsa_batch_t* batch,
                                      int32_t k, int32_t* idx, void* workspace,
                                      size_t workspace_bytes, dsa_stream_t stream) {
    Range nvtx_range("dsa_indexer_topk");
    BatchView bv;
    dsa_status_t s = check_batch(batch, &bv);
    if (s != DSA_OK || bv.total_q == 0) return s == DSA_OK ? ok() : s;
    if (!workspace || !aligned16(workspace))
        return fail(DSA_ERR_INVALID_ARGUMENT, "workspace must be non-NULL and 16-byte aligned");
    const size_t need = dsa_indexer_topk_workspace_size(batch);
    if (workspace_bytes < need)
        return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need,
                    workspace_bytes);
    const long long ld = decode_ld(bv.max_seq_len);
    float* logits = static_cast<float*>(workspace);
    CacheView kc;
    s = indexer_validate(q, q_dtype, q_scale, w, heads, dim, k_cache, bv, logits, ld, &kc);
    if (s == DSA_OK) s = topk_validate(logits, ld, bv, k, idx);
    if (s != DSA_OK) return s;
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Blocks of rows: the indexer writes a block's logits, the top-k selects from them
    // (programmatic dependents; each kernel waits for its predecessor before touching
    // the shared buffer, so block i+1's logits never overwrite what block i still reads).
    // a workspace larger than the minimum takes larger blocks (fewer, longer launches)
    const int rows = indexer_topk_block_rows(bv.total_q, ld, workspace_bytes > kL2BlockBytes
                                                                 ? workspace_bytes : kL2BlockBytes);
    for (int r0 = 0; e == cudaSuccess && r0 < bv.total_q; r0 += rows) {
        BatchView blk = bv;
        blk.total_q = r0 + rows < bv.total_q ? r0 + rows : bv.total_q;
        e = indexer_launch(q, q_scale, w, heads, dim, kc, blk, logits, ld, check, st, true, r0);
        if (e == cudaSuccess) e = launch_topk(logits, ld, blk, k, idx, check, st, true, r0);
    }
    return e == cudaSuccess ? ok() : cuda_fail(e, "indexer + top-k launch");
}

DSA_API dsa_status_t dsa_cache_store(const void* x, dsa_dtype_t x_dtype, int32_t n, int32_t dim,
                                     const int64_t* slot_mapping, void* cache_data,
                                     dsa_dtype_t cache_dtype, float* cache_scale, int64_t num_rows,
                                     dsa_stream_t stream) {
    Range nvtx_range("dsa_cache_store");
    if (n < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "n must be >= 0");
    if (n == 0) return ok();
    if (x_dtype != DSA_F32 && x_dtype != DSA_BF16)
        return fail(valid_dtype(x_dtype) ? DSA_ERR_UNSUPPORTED : DSA_ERR_INVALID_ARGUMENT,
                    "x_dtype must be DSA_F32 or DSA_BF16");
    if (!valid_dtype(cache_dtype))
        return fail(DSA_ERR_INVALID_ARGUMENT, "cache_dtype is not a dsa_dtype_t");
    if (dim < 16 || dim > 1024 || dim % 16 != 0)
        return fail(DSA_ERR_UNSUPPORTED, "dim (%d) must be a multiple of 16 in [16, 1024]", dim);
    if (num_rows < 1) return fail(DSA_ERR_INVALID_ARGUMENT, "num_rows must be >= 1");
    if (!x || !aligned16(x)) return fail(DSA_ERR_INVALID_ARGUMENT, "x must be non-NULL, 16-byte aligned");
    if (!slot_mapping || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return fail(DSA_ERR_INVALID_ARGUMENT, "slot_mapping must be non-NULL, 8-byte aligned");
    if (!cache_data || !aligned16(cache_data))
        return fail(DSA_ERR_INVALID_ARGUMENT, "cache_data must be non-NULL, 16-byte aligned");
    if (cache_dtype == DSA_FP8_E4M3 && (!cache_scale || !aligned4(cache_scale)))
        return fail(DSA_ERR_INVALID_ARGUMENT, "an FP8 cache needs a 4-byte aligned cache_scale");
    int* check = nullptr;
    cudaError_t e = check_word(&check);
    if (e == cudaSuccess)
        e = launch_cache_store(x, x_dtype, n, dim, reinterpret_cast<const long long*>(slot_mapping),
                               cache_data, cache_dtype, cache_scale, num_rows, check,
                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "cache store launch");
}

DSA_API dsa_status_t dsa_device_check(dsa_stream_t stream, int32_t* code, int32_t reset) {
    Range nvtx_range("dsa_device_check");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_check_word, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read check word");
    if (reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_check_word, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clear check word");
    }
    if (code) *code = v;
    if (v != 0) return fail(DSA_ERR_DEVICE_CHECK, "device check recorded code %d", v);
    return ok();
}

DSA_API const char* dsa_last_error_message(void) { return g_msg.c_str(); }

DSA_API const char* dsa_status_string(dsa_status_t status) {
    switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARGUMENT: return "DSA_ERR_INVALID_ARGUMENT";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "DSA_ERR_WORKSPACE_TOO_SMALL";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_DEVICE_CHECK: return "DSA_ERR_DEVICE_CHECK";
    }
    return "unknown dsa_status_t";
}

DSA_API int32_t dsa_version(void) { return 100; }

}  // extern "C"
