// kernels.h -- internal launchers of libdsa (host side, C++).  The public C ABI
// in include/dsa.h validates arguments and then calls these.
#pragma once

#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace dsa {

// Launch; with pdl, as a programmatic dependent of the previous kernel in the stream
// (the kernel must then pdl_wait() before reading that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int kIndexerPage = 64;
constexpr int kNumSMs = 148;

// 2-D tensor map [rows][inner] (row stride in bytes) with a box_inner x box_rows box.
cudaError_t make_tensor_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype,
                               int elem_bytes, unsigned long long inner, unsigned long long rows,
                               unsigned long long row_stride_bytes, unsigned box_inner,
                               unsigned box_rows, CUtensorMapSwizzle swizzle);

// Lightning Indexer on CUDA cores (fp32 q/k; any heads <= 64, dim <= 128, dim % 4 == 0).
cudaError_t launch_indexer_generic(const void* q, const float* q_scale, const float* w, int heads,
                                   int dim, const CacheView& k, const BatchView& bv, float* logits,
                                   long long ld, int* check, cudaStream_t st, int row0 = 0);

// Lightning Indexer on tcgen05 tensor cores (fp8 e4m3 q/k, 64 heads x 128 dims).
cudaError_t launch_indexer_fp8_tc(const void* q, const float* q_scale, const float* w,
                                  const CacheView& k, const BatchView& bv, float* logits,
                                  long long ld, int* check, cudaStream_t st, bool pdl = false, int row0 = 0);

// Writes n token rows of x (fp32 or bf16, [n][dim], dim % 16 == 0, dim <= 1024) into
// cache rows slots[i] (negative: skipped) as fp8 e4m3 + amax/448 scale, bf16 or fp32.
cudaError_t launch_cache_store(const void* x, int x_dtype, int n, int dim, const long long* slots,
                               void* data, int cache_dtype, float* scale, long long num_rows,
                               int* check, cudaStream_t st);

// Per-row top-k by radix select.  Launches with row0 > 0 cover rows [row0, bv.total_q)
// (the indexer writes, and the top-k reads, logits row t at (t - row0) * ld).
cudaError_t launch_topk(const float* logits, long long ld, const BatchView& bv, int k, int* idx,
                        int* check, cudaStream_t st, bool pdl = false, int row0 = 0);

// Sparse MLA on CUDA cores (fp32 q/KV).  nsplit > 1 writes partials (o/l, lse) to
// o_part [T][nsplit][heads][d_v] / lse_part [T][nsplit][heads] instead of out/lse.
cudaError_t launch_mla_generic(const void* q, int heads, int d_qk, int d_v, float scale,
                               const CacheView& kv, const BatchView& bv, const int* idx, int k,
                               int nsplit, void* out, int out_dtype, float* lse, float* o_part,
                               float* lse_part, int* check, cudaStream_t st);

// Sparse MLA on tcgen05 tensor cores: bf16 q, bf16 or fp8 KV, 128 heads, 576 / 512.
// nsplit > 1 writes partials o/l in fp16 to o_part [T][nsplit][128][512] (each is
// bounded by the largest V value) and lse to lse_part [T][nsplit][128] fp32.
cudaError_t launch_mla_tc(const void* q, float scale, const CacheView& kv, const BatchView& bv,
                          const int* idx, int k, int nsplit, void* out, float* lse, void* o_part,
                          float* lse_part, int* check, cudaStream_t st, bool pdl = false);

// Size of the fixed device array behind dsa_sparse_mla_decode_noalloc
// (equals DSA_NOALLOC_SCRATCH_BYTES in include/dsa.h).
constexpr size_t kStaticScratchBytes = size_t(20) << 20;

// Address of that array on the current device (looked up once per device).
cudaError_t static_scratch(void** ptr);

// Log-sum-exp merge of split partials (fp16 when half_part, else fp32) into out
// (out_dtype) and lse.
cudaError_t launch_mla_combine(const void* o_part, bool half_part, const float* lse_part,
                               int total_q, int nsplit, int heads, int d_v, void* out,
                               int out_dtype, float* lse, cudaStream_t st, bool pdl = false);

}  // namespace dsa
