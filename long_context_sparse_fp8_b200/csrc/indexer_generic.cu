// indexer_generic.cu -- Lightning Indexer scores on CUDA cores (fp32 or fp8 inputs).
//
// I[t,s] = k_scale[s] * q_scale[t] * sum_j w[t,j] * ReLU(q[t,j,:] . k[s,:]),  s <= pos(t)
// (the indexer of "SGLang Day-0 support for DeepSeek-V3.2", section "DeepSeek
// Sparse Attention"; score definition as this library's header states it).
//
// One CTA scores one query row against one 64-token page of the key cache: the
// query (heads x dim) and the page are staged in shared memory as fp32, four
// threads share a key and split its heads, and a two-step shuffle adds their parts.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;

template <int DT>
__global__ void __launch_bounds__(kThreads)
indexer_generic_kernel(const void* __restrict__ q, const float* __restrict__ q_scale,
                       const float* __restrict__ w, int heads, int dim, CacheView kc, BatchView bv,
                       float* __restrict__ logits, long long ld, int row0, int* check) {
    extern __shared__ float sm[];
    const int t = row0 + blockIdx.x, tile = blockIdx.y, tid = threadIdx.x;
    float* lrow = logits + (long long)blockIdx.x * ld;   // row t is logits row t - row0
    const RowInfo ri = row_info(bv, t, check);
    if (!ri.ok) return;
    const int s0 = tile * kIndexerPage;
    if (s0 > ri.pos) return;

    const int qstride = dim + 1;  // padded rows: no bank conflicts between heads / keys
    float* qs = sm;                                  // [heads][dim+1]
    float* ks = qs + heads * qstride;                // [64][dim+1]
    float* ws = ks + kIndexerPage * qstride;         // [heads]
    float* kscale = ws + heads;                      // [64]
    __shared__ long long page_row0;

    if (tid == 0) {
        long long r = cache_row(kc, ri.b, s0, check);
        page_row0 = r;
    }
    for (int i = tid; i < heads * dim; i += kThreads)
        qs[(i / dim) * qstride + i % dim] = load_as_f32<DT>(q, (long long)t * heads * dim + i);
    for (int i = tid; i < heads; i += kThreads) ws[i] = __ldg(w + (long long)t * heads + i);
    __syncthreads();
    const long long r0 = page_row0;
    if (r0 < 0) {  // bad page: recorded; the tile's scores are -inf
        for (int i = tid; i < kIndexerPage; i += kThreads)
            if (s0 + i <= ri.pos) lrow[s0 + i] = -INFINITY;
        return;
    }
    for (int i = tid; i < kIndexerPage * dim; i += kThreads)
        ks[(i / dim) * qstride + i % dim] = load_as_f32<DT>(kc.data, r0 * dim + i);
    for (int i = tid; i < kIndexerPage; i += kThreads)
        kscale[i] = kc.scale ? __ldg(kc.scale + r0 + i) : 1.0f;
    __syncthreads();

    const int key = tid >> 2, part = tid & 3;
    float acc = 0.f;
    for (int j = part; j < heads; j += 4) {
        float dot = 0.f;
        const float* qr = qs + j * qstride;
        const float* kr = ks + key * qstride;
        for (int d = 0; d < dim; ++d) dot = fmaf(qr[d], kr[d], dot);
        acc = fmaf(ws[j], fmaxf(dot, 0.f), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) {
        const int s = s0 + key;
        const float qsc = q_scale ? __ldg(q_scale + t) : 1.0f;
        if (s <= ri.pos) lrow[s] = kscale[key] * qsc * acc;
        else if (s < ld) lrow[s] = -INFINITY;
    }
}

}  // namespace

cudaError_t launch_indexer_generic(const void* q, const float* q_scale, const float* w, int heads,
                                   int dim, const CacheView& k, const BatchView& bv, float* logits,
                                   long long ld, int* check, cudaStream_t st, int row0) {
    const int tiles = (bv.max_seq_len + kIndexerPage - 1) / kIndexerPage;
    const size_t smem = sizeof(float) * ((size_t)(heads + kIndexerPage) * (dim + 1) + heads + 64);
    auto kern = k.dtype == kE4M3 ? indexer_generic_kernel<kE4M3> : indexer_generic_kernel<kF32>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(bv.total_q - row0, tiles);
    kern<<<grid, kThreads, smem, st>>>(q, q_scale, w, heads, dim, k, bv, logits, ld, row0, check);
    return cudaGetLastError();
}

}  // namespace dsa
