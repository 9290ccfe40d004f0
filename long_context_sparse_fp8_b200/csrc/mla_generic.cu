// mla_generic.cu -- sparse MLA on CUDA cores for fp32 inputs, and the log-sum-exp
// merge of split partial results (shared with the tensor-core kernel).
//
// For query row t and head h, over the selected positions s (idx[t][.], -1 skipped):
//   z_s = softmax_scale * q[t,h,:] . (kv_s * kv_scale[s]),  p = softmax(z),
//   o[t,h,:] = sum_s p_s * kv_s[0:d_v] * kv_scale[s],  lse = log sum_s exp(z_s)
// (core attention over the top-k entries only: "SGLang Day-0 support for
// DeepSeek-V3.2", section "DeepSeek Sparse Attention"; V is the first d_v columns
// of the latent row).
//
// One warp owns one (query, head): it keeps q and its slice of o in registers,
// walks the selected rows with an online softmax, and reduces each dot product
// with shuffles.  With nsplit > 1 the selection list is cut into nsplit equal
// chunks and each chunk writes a normalised partial (o/l, lse) for the merge.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kWarpsPerBlock = 4;
constexpr int kMaxQK = 576;  // 18 per lane
constexpr int kMaxV = 512;   // 16 per lane

template <int QDT, int KVDT>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
mla_generic_kernel(const void* __restrict__ q, int heads, int d_qk, int d_v, float scale,
                   CacheView kv, BatchView bv, const int* __restrict__ idx, int k, int nsplit,
                   void* __restrict__ out, int out_dtype, float* __restrict__ lse,
                   float* __restrict__ o_part, float* __restrict__ lse_part, int* check) {
    const int t = blockIdx.x, split = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * kWarpsPerBlock + warp;
    if (h >= heads) return;
    const RowInfo ri = row_info(bv, t, check);

    float qv[kMaxQK / 32];
#pragma unroll
    for (int j = 0; j < kMaxQK / 32; ++j) {
        const int d = lane + 32 * j;
        qv[j] = d < d_qk ? load_as_f32<QDT>(q, ((long long)t * heads + h) * d_qk + d) : 0.f;
    }
    float o[kMaxV / 32];
#pragma unroll
    for (int j = 0; j < kMaxV / 32; ++j) o[j] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int chunk = (k + nsplit - 1) / nsplit;
    const int i0 = split * chunk, i1 = min(k, i0 + chunk);
    for (int i = i0; ri.ok && i < i1; ++i) {
        const int s = __ldg(idx + (long long)t * k + i);
        if (s < 0) continue;
        if (s > ri.pos) {
            if (lane == 0) report(check, kCheckBadIndex);
            continue;
        }
        const long long r = cache_row(kv, ri.b, s, check);
        if (r < 0) continue;
        const float sc = kv.scale ? __ldg(kv.scale + r) : 1.0f;
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxQK / 32; ++j) {
            const int d = lane + 32 * j;
            if (d < d_qk) dot = fmaf(qv[j], load_as_f32<KVDT>(kv.data, r * d_qk + d), dot);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float z = dot * sc * scale;
        const float m_new = fmaxf(m, z);
        const float alpha = __expf(m - m_new);
        const float p = __expf(z - m_new);
        l = l * alpha + p;
        const float ps = p * sc;
#pragma unroll
        for (int j = 0; j < kMaxV / 32; ++j) {
            const int d = lane + 32 * j;
            const float v = d < d_v ? load_as_f32<KVDT>(kv.data, r * d_qk + d) : 0.f;
            o[j] = fmaf(o[j], alpha, ps * v);
        }
        m = m_new;
    }
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const float lse_v = l > 0.f ? m + logf(l) : -INFINITY;
    if (nsplit == 1) {
        const long long base = ((long long)t * heads + h) * d_v;
#pragma unroll
        for (int j = 0; j < kMaxV / 32; ++j) {
            const int d = lane + 32 * j;
            if (d >= d_v) continue;
            const float v = o[j] * inv;
            if (out_dtype == kBF16) reinterpret_cast<__nv_bfloat16*>(out)[base + d] = __float2bfloat16_rn(v);
            else reinterpret_cast<float*>(out)[base + d] = v;
        }
        if (lse && lane == 0) lse[(long long)t * heads + h] = lse_v;
    } else {
        const long long pbase = (((long long)t * nsplit + split) * heads + h);
#pragma unroll
        for (int j = 0; j < kMaxV / 32; ++j) {
            const int d = lane + 32 * j;
            if (d < d_v) o_part[pbase * d_v + d] = o[j] * inv;
        }
        if (lane == 0) lse_part[pbase] = lse_v;
    }
}

// Merge of split partials: o = sum_i exp(lse_i - lse) o_i with lse = log sum_i exp(lse_i).
// One thread per 4 output values of one (query, head); a block covers 2 heads x 512.
// With NS > 0 (= nsplit, known at compile time) every partial a thread needs is
// loaded before any is used, so the loads overlap instead of forming a dependent
// chain; NS = 0 handles any nsplit <= 16 the same way in a fixed-size frame.
template <typename PT>
__device__ __forceinline__ float4 load_part4(const PT* p) {
    if constexpr (sizeof(PT) == 4) {
        return __ldg(reinterpret_cast<const float4*>(p));
    } else {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
}

template <int NS, typename PT>
__global__ void __launch_bounds__(256)
mla_combine_kernel(const PT* __restrict__ o_part, const float* __restrict__ lse_part,
                   int nsplit_rt, int heads, int d_v, void* __restrict__ out, int out_dtype,
                   float* __restrict__ lse) {
    constexpr int kMaxSplit = NS > 0 ? NS : 16;
    const int nsplit = NS > 0 ? NS : nsplit_rt;
    const int t = blockIdx.x;
    const int per_head = d_v / 4;                       // threads per head
    const int h = blockIdx.y * (blockDim.x / per_head) + threadIdx.x / per_head;
    const int d4 = threadIdx.x % per_head;
    pdl_wait();                                         // partials of the previous kernel
    if (h >= heads) return;
    float li[kMaxSplit];
    float4 ov[kMaxSplit];
#pragma unroll
    for (int i = 0; i < kMaxSplit; ++i) {
        if (i < nsplit) {
            const long long pb = ((long long)t * nsplit + i) * heads + h;
            li[i] = __ldg(lse_part + pb);
            ov[i] = load_part4(o_part + pb * d_v + 4 * d4);
        }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxSplit; ++i)
        if (i < nsplit) mx = fmaxf(mx, li[i]);
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kMaxSplit; ++i) {
        if (i < nsplit && li[i] != -INFINITY) {
            const float wgt = __expf(li[i] - mx);
            wsum += wgt;
            acc.x = fmaf(wgt, ov[i].x, acc.x);
            acc.y = fmaf(wgt, ov[i].y, acc.y);
            acc.z = fmaf(wgt, ov[i].z, acc.z);
            acc.w = fmaf(wgt, ov[i].w, acc.w);
        }
    }
    const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
    const long long ob = ((long long)t * heads + h) * d_v + 4 * d4;
    if (out_dtype == kBF16) {
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out) + ob);
        o2[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        o2[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + ob) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (lse && d4 == 0)
        lse[(long long)t * heads + h] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_mla_generic(const void* q, int heads, int d_qk, int d_v, float scale,
                               const CacheView& kv, const BatchView& bv, const int* idx, int k,
                               int nsplit, void* out, int out_dtype, float* lse, float* o_part,
                               float* lse_part, int* check, cudaStream_t st) {
    dim3 grid(bv.total_q, (heads + kWarpsPerBlock - 1) / kWarpsPerBlock, nsplit);
    dim3 block(32 * kWarpsPerBlock);
    // fp32 q with fp32 KV (bf16 / fp8 KV runs on the tensor-core kernel)
    mla_generic_kernel<kF32, kF32><<<grid, block, 0, st>>>(q, heads, d_qk, d_v, scale, kv, bv,
        idx, k, nsplit, out, out_dtype, lse, o_part, lse_part, check);
    return cudaGetLastError();
}

namespace {

template <typename PT>
cudaError_t combine_for(const PT* o_part, const float* lse_part, int total_q, int nsplit,
                        int heads, int d_v, void* out, int out_dtype, float* lse, cudaStream_t st,
                        bool pdl) {
    // d_v % 4 == 0 and d_v <= 512 (validated by the callers)
    const int per_head = d_v / 4;
    const int heads_per_block = per_head >= 256 ? 1 : 256 / per_head;
    dim3 grid(total_q, (heads + heads_per_block - 1) / heads_per_block);
    const int threads = per_head * heads_per_block;
    auto kern = nsplit == 2 ? mla_combine_kernel<2, PT> : nsplit == 3 ? mla_combine_kernel<3, PT>
              : nsplit == 4 ? mla_combine_kernel<4, PT> : nsplit == 8 ? mla_combine_kernel<8, PT>
                                                                      : mla_combine_kernel<0, PT>;
    cudaError_t e = launch_kernel(kern, grid, dim3(threads), 0, st, pdl, o_part, lse_part, nsplit,
                                  heads, d_v, out, out_dtype, lse);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

// Partials: fp16 from the tensor-core kernel, fp32 from the CUDA-core one.
cudaError_t launch_mla_combine(const void* o_part, bool half_part, const float* lse_part,
                               int total_q, int nsplit, int heads, int d_v, void* out,
                               int out_dtype, float* lse, cudaStream_t st, bool pdl) {
    return half_part
               ? combine_for(static_cast<const __half*>(o_part), lse_part, total_q, nsplit, heads,
                             d_v, out, out_dtype, lse, st, pdl)
               : combine_for(static_cast<const float*>(o_part), lse_part, total_q, nsplit, heads,
                             d_v, out, out_dtype, lse, st, pdl);
}

}  // namespace dsa
