// topk.cu -- per-query top-k token selection (k = 2048 in DeepSeek-V3.2 serving:
// "DeepSeek-V3.2-Exp DSA deployment guide", section 3.1; selection of the most
// relevant key/value entries: "SGLang Day-0 support for DeepSeek-V3.2", section
// "DeepSeek Sparse Attention").  A row with pos+1 <= k keeps every position
// (dense fallback, same guide, section 5.1).
//
// Method: exact radix select on order-preserving 32-bit keys.  One 1024-thread CTA
// owns one row.  Three histogram passes (11 + 11 + 10 bits, shared-memory
// atomics) pin down the exact k-th largest key T and how many keys equal to T
// are still needed; a final two-pass emission writes every key > T and the
// lowest-position keys == T in ascending position order (deterministic output).  Rows of up to kSmemKeys candidates are staged once in shared
// memory; longer rows are re-read from global memory (L2) on each pass.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemKeys = 48 * 1024;  // 192 KB of staged keys

// Monotone map float -> uint32 (larger float, larger key); -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one int per thread; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sums[lane];
        int s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_sums[lane] = s - w;        // exclusive per warp
        if (lane == 31) warp_sums[32] = s;
    }
    __syncthreads();
    const int r = warp_sums[warp] + x - v;
    *total = warp_sums[32];
    __syncthreads();  // warp_sums may be reused right after
    return r;
}

struct Row {
    const float* g;       // global row
    const uint32_t* s;    // staged keys or nullptr
    __device__ __forceinline__ uint32_t operator()(int i) const {
        return s ? s[i] : order_key(__ldg(g + i));
    }
};

__global__ void __launch_bounds__(kThreads)
topk_kernel(const float* __restrict__ logits, long long ld, BatchView bv, int k,
            int* __restrict__ idx, int* check, int smem_keys) {
    extern __shared__ uint32_t skeys[];
    __shared__ int hist[2048];
    __shared__ int warp_sums[kWarps + 1];
    __shared__ int s_bin, s_above;

    const int t = blockIdx.x, tid = threadIdx.x;
    int* out = idx + (long long)t * k;
    const RowInfo ri = row_info(bv, t, check);
    if (!ri.ok) {
        for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    const int n = ri.pos + 1;
    if (n <= k) {  // every causal position is selected
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* grow = logits + (long long)t * ld;
    Row row{grow, nullptr};
    if (n <= smem_keys) {
        for (int i = tid; i < n; i += kThreads) skeys[i] = order_key(__ldg(grow + i));
        row.s = skeys;
        __syncthreads();
    }

    // ---- radix select: find the exact k-th largest key -------------------------
    uint32_t prefix = 0u, pmask = 0u;
    int remaining = k;   // how many of the keys matching `prefix` still have to be taken
    const int shifts[3] = {21, 10, 0};
    const int nbits[3] = {11, 11, 10};
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int nb = 1 << nbits[p], shift = shifts[p];
        for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const uint32_t key = row(i);
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
        }
        __syncthreads();
        // Suffix counts from the top bin down: thread tid owns reversed bins
        // [tid*per, tid*per + per).
        const int per = nb / kThreads;
        int local[2] = {0, 0};
        int tsum = 0;
        for (int j = 0; j < per; ++j) {
            local[j] = hist[nb - 1 - (tid * per + j)];
            tsum += local[j];
        }
        int total;
        int run = block_excl_scan(tsum, warp_sums, &total);
        for (int j = 0; j < per; ++j) {
            const int bin = nb - 1 - (tid * per + j);
            const int above = run;
            run += local[j];
            if (run >= remaining && above < remaining) {
                s_bin = bin;
                s_above = above;
            }
        }
        __syncthreads();
        const int bin = s_bin;
        remaining -= s_above;
        prefix |= (uint32_t)bin << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;          // the k-th largest key
    const int need_eq = remaining;      // keys == T to take (>= 1)

    // ---- emit, deterministic and in position order --------------------------
    // Warp w owns the contiguous segment [w*seg, (w+1)*seg).  Pass A counts its
    // keys > T and == T; a block scan turns the counts into offsets; pass B
    // writes every key > T and the first need_eq keys == T (lowest positions).
    const int lane = tid & 31, warp = tid >> 5;
    const int seg = ((n + kWarps - 1) / kWarps + 31) & ~31;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    int c_gt = 0, c_eq = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < w1 ? row(i) : 0u;
        c_gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > T));
        c_eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == T));
    }
    __shared__ int s_gt[kWarps], s_eq[kWarps];
    if (lane == 0) {
        s_gt[warp] = c_gt;
        s_eq[warp] = c_eq;
    }
    __syncthreads();
    int gt_before = 0, eq_before = 0;
    for (int v = 0; v < warp; ++v) {
        gt_before += s_gt[v];
        eq_before += s_eq[v];
    }
    int taken = gt_before + min(eq_before, need_eq);   // output slot of the next taken key
    int eq_seen = eq_before;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < w1 ? row(i) : 0u;
        const bool gt = i < w1 && key > T;
        const bool eq = i < w1 && key == T;
        const unsigned meq = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(meq & ((1u << lane) - 1u));
        const bool take = gt || (eq && eq_rank < need_eq);
        const unsigned mt = __ballot_sync(0xffffffffu, take);
        if (take) out[taken + __popc(mt & ((1u << lane) - 1u))] = i;
        taken += __popc(mt);
        eq_seen += __popc(meq);
    }
}

}  // namespace

cudaError_t launch_topk(const float* logits, long long ld, const BatchView& bv, int k, int* idx,
                        int* check, cudaStream_t st) {
    const int staged = bv.max_seq_len < kSmemKeys ? bv.max_seq_len : kSmemKeys;
    const size_t smem = (size_t)staged * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    topk_kernel<<<bv.total_q, kThreads, smem, st>>>(logits, ld, bv, k, idx, check, staged);
    return cudaGetLastError();
}

}  // namespace dsa
