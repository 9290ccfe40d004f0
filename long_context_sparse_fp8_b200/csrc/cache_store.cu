// cache_store.cu -- writes new tokens into the paged caches the indexer and the
// sparse attention read.
//
// "SGLang Day-0 support for DeepSeek-V3.2" (winzheng.jp review), section "DeepSeek
// Sparse Attention": the indexer keeps a key & key_scale cache (page size 64) and
// the sparse operator a token-level cache (page size 1); its "Future work" section
// and the KV_CACHE_STORE_FP8 switch of its launch lines: the KV cache may be stored
// in FP8, halving what attention reads.  "DeepSeek-V3.2-Exp DSA deployment guide"
// (m.nxbn.cn), section 3.1: fp8_e4m3 KV cache.  The FP8 scaling is one fp32 scale
// per token, amax / 448.
//
// Rows are spread over lane groups: 16 lanes per row when the row has at most 16
// chunks of 8 elements (the 128-wide indexer key), else 32.  Each lane group takes four
// rows per pass, so every warp keeps 4-8 rows of loads in flight (up to four 16-B or
// 32-B loads per lane per row, all issued before use, kept packed until converted);
// |x| is max-reduced within the group, the scale amax/448 is formed once per row, and
// each lane converts and stores its chunks (8 B of e4m3 codes, 16 B of bf16 or 32 B of
// fp32).  HBM-bound: dim x (input + output bytes) + 4 B scale + 8 B slot per token.
//
// The FP8 codes are e4m3(x / scale) with the quotient correctly rounded to fp32.  A
// division per element would make the kernel compute-bound, so each quotient is first
// taken as x * (1/scale), which lies within 3 fp32 ulps of the correctly rounded
// quotient.  In the normal e4m3 range (|q| >= 2^-6) the codes change only at the
// midpoints between neighbouring e4m3 values, fp32 numbers whose low 20 mantissa bits
// are 0x80000; a product more than 3 ulps from such a midpoint has the code of the
// exact quotient (rounding is monotone).  An 8-element chunk with any element within 3
// ulps of a midpoint, or nonzero below 2^-6 (e4m3 subnormals), takes its codes from the
// divisions instead (out of line: about one chunk in 10^4 on Gaussian rows).  Scales
// below the smallest normal fp32, whose reciprocal may overflow, divide always.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kThreads = 128;
constexpr int kRowsPerGroup = 4;       // rows each lane group loads before converting

// A chunk = 8 consecutive elements, kept as loaded (bf16: one 16-B word; fp32: two).
template <int XT>
struct Chunk {
    uint4 w[XT == kBF16 ? 1 : 2];
};

template <int XT>
__device__ __forceinline__ void load_chunk(const void* x, long long e, Chunk<XT>& c) {
    if constexpr (XT == kBF16) {
        c.w[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + e));
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + e);
        c.w[0] = __ldg(p);
        c.w[1] = __ldg(p + 1);
    }
}

template <int XT>
__device__ __forceinline__ float elem(const Chunk<XT>& c, int e) {
    if constexpr (XT == kBF16) {
        const uint32_t u = (e >> 1) == 0 ? c.w[0].x : (e >> 1) == 1 ? c.w[0].y : (e >> 1) == 2 ? c.w[0].z : c.w[0].w;
        return __uint_as_float((e & 1) ? (u & 0xFFFF0000u) : (u << 16));
    } else {
        const uint4 q = c.w[e >> 2];
        const uint32_t u = (e & 3) == 0 ? q.x : (e & 3) == 1 ? q.y : (e & 3) == 2 ? q.z : q.w;
        return __uint_as_float(u);
    }
}

// Two fp32 values to e4m3 codes (round to nearest even, saturating at +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// e4m3 codes of the 8 quotients f[e] / sc, each correctly rounded to fp32 first: the
// divisions themselves (the rare path; kept out of line).
__device__ __noinline__ uint2 e4m3x8_divide(float f0, float f1, float f2, float f3, float f4,
                                            float f5, float f6, float f7, float sc) {
    return make_uint2(e4m3x2(__fdiv_rn(f0, sc), __fdiv_rn(f1, sc)) |
                          (e4m3x2(__fdiv_rn(f2, sc), __fdiv_rn(f3, sc)) << 16),
                      e4m3x2(__fdiv_rn(f4, sc), __fdiv_rn(f5, sc)) |
                          (e4m3x2(__fdiv_rn(f6, sc), __fdiv_rn(f7, sc)) << 16));
}

// Whether the product q = x * (1/sc) may round to another e4m3 code than the correctly
// rounded quotient (see the head of the file).
__device__ __forceinline__ bool e4m3_risky(float q) {
    const uint32_t m = __float_as_uint(q) & 0x7FFFFFFFu;
    return (m != 0u && m < 0x3C800000u) || ((m & 0xFFFFFu) - 0x7FFFDu) <= 6u;
}

// e4m3 codes of an 8-element chunk divided by sc (rcp = 1/sc correctly rounded).
template <int XT>
__device__ __forceinline__ uint2 e4m3x8_quotients(const Chunk<XT>& c, float sc, float rcp,
                                                  bool divide_all) {
    float q[8];
    bool risky = divide_all;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        q[e] = __fmul_rn(elem<XT>(c, e), rcp);
        risky |= e4m3_risky(q[e]);
    }
    if (risky)
        return e4m3x8_divide(elem<XT>(c, 0), elem<XT>(c, 1), elem<XT>(c, 2), elem<XT>(c, 3),
                             elem<XT>(c, 4), elem<XT>(c, 5), elem<XT>(c, 6), elem<XT>(c, 7), sc);
    return make_uint2(e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16),
                      e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16));
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int XT, int CT, int LPR, int CPL>
__global__ void __launch_bounds__(kThreads) cache_store_kernel(
    const void* __restrict__ x, int n, int dim, const long long* __restrict__ slots,
    void* __restrict__ data, float* __restrict__ scale, long long num_rows, int* check) {
    constexpr int kGroups = 32 / LPR;            // row groups per warp
    constexpr int kPerPass = kRowsPerGroup * kGroups;
    const int lane = threadIdx.x & 31, g = lane / LPR, gl = lane % LPR;
    const int nch = dim >> 3;
    const long long warps = (long long)gridDim.x * (kThreads / 32);
    const long long w = (long long)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (long long base = w * kPerPass; base < n; base += warps * kPerPass) {
        long long slot[kRowsPerGroup];
        Chunk<XT> v[kRowsPerGroup][CPL];
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            const long long row = base + u * kGroups + g;
            slot[u] = row < n ? __ldg(slots + row) : -1;
            // the row is loaded whatever its slot, so that its loads do not wait for the
            // slot's (a skipped token costs one wasted read)
#pragma unroll
            for (int r = 0; r < CPL; ++r) {
                const int c = gl + LPR * r;
                if (row < n && c < nch) {
                    load_chunk<XT>(x, row * dim + 8 * c, v[u][r]);
                } else {
#pragma unroll
                    for (int k = 0; k < (XT == kBF16 ? 1 : 2); ++k) v[u][r].w[k] = make_uint4(0, 0, 0, 0);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            if (slot[u] >= num_rows) {
                if (gl == 0) report(check, kCheckBadPage);
                slot[u] = -1;
            }
            if constexpr (CT == kE4M3) {
                float amax = 0.f;
#pragma unroll
                for (int r = 0; r < CPL; ++r)
#pragma unroll
                    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(elem<XT>(v[u][r], e)));
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (slot[u] < 0) continue;
                // scale = amax / 448 (1 for a zero row or an underflowed quotient);
                // codes = e4m3(x / scale)
                float sc = __fdiv_rn(amax, 448.0f);
                if (!(sc > 0.f)) sc = 1.0f;
                const float rcp = __frcp_rn(sc);
                const bool divide_all = sc < 1.17549435e-38f;     // subnormal scale
                uint8_t* dst = static_cast<uint8_t*>(data) + slot[u] * dim;
#pragma unroll
                for (int r = 0; r < CPL; ++r) {
                    const int c = gl + LPR * r;
                    if (c >= nch) continue;
                    *reinterpret_cast<uint2*>(dst + 8 * c) = e4m3x8_quotients<XT>(v[u][r], sc, rcp, divide_all);
                }
                if (gl == 0) scale[slot[u]] = sc;
            } else if constexpr (CT == kBF16) {
                if (slot[u] < 0) continue;
                uint16_t* dst = static_cast<uint16_t*>(data) + slot[u] * dim;
#pragma unroll
                for (int r = 0; r < CPL; ++r) {
                    const int c = gl + LPR * r;
                    if (c >= nch) continue;
                    uint4 o;
                    if constexpr (XT == kBF16) {
                        o = v[u][r].w[0];
                    } else {
                        const Chunk<XT>& a = v[u][r];
                        o = make_uint4(bf16x2(elem<XT>(a, 0), elem<XT>(a, 1)), bf16x2(elem<XT>(a, 2), elem<XT>(a, 3)),
                                       bf16x2(elem<XT>(a, 4), elem<XT>(a, 5)), bf16x2(elem<XT>(a, 6), elem<XT>(a, 7)));
                    }
                    *reinterpret_cast<uint4*>(dst + 8 * c) = o;
                }
            } else {
                if (slot[u] < 0) continue;
                float* dst = static_cast<float*>(data) + slot[u] * dim;
#pragma unroll
                for (int r = 0; r < CPL; ++r) {
                    const int c = gl + LPR * r;
                    if (c >= nch) continue;
                    const Chunk<XT>& a = v[u][r];
                    float4* p = reinterpret_cast<float4*>(dst + 8 * c);
                    p[0] = make_float4(elem<XT>(a, 0), elem<XT>(a, 1), elem<XT>(a, 2), elem<XT>(a, 3));
                    p[1] = make_float4(elem<XT>(a, 4), elem<XT>(a, 5), elem<XT>(a, 6), elem<XT>(a, 7));
                }
            }
        }
    }
}

template <int XT, int CT, int LPR, int CPL>
cudaError_t launch_shape(const void* x, int n, int dim, const long long* slots, void* data,
                         float* scale, long long num_rows, int* check, cudaStream_t st) {
    constexpr int kRowsPerBlock = (kThreads / 32) * kRowsPerGroup * (32 / LPR);
    // one wave: as many blocks as fit on the SMs at once (queried once per shape)
    static std::atomic<int> cached{0};
    int per_sm = cached.load(std::memory_order_relaxed);
    if (per_sm == 0) {
        int b = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &b, cache_store_kernel<XT, CT, LPR, CPL>, kThreads, 0);
        if (e != cudaSuccess) return e;
        per_sm = b > 0 ? b : 1;
        cached.store(per_sm, std::memory_order_relaxed);
    }
    const long long blocks = ((long long)n + kRowsPerBlock - 1) / kRowsPerBlock;
    const long long wave = (long long)per_sm * kNumSMs;
    const int grid = (int)(blocks < wave ? blocks : wave);
    cache_store_kernel<XT, CT, LPR, CPL><<<grid, kThreads, 0, st>>>(x, n, dim, slots, data, scale,
                                                                   num_rows, check);
    return cudaGetLastError();
}

template <int XT, int CT>
cudaError_t launch_for(const void* x, int n, int dim, const long long* slots, void* data,
                       float* scale, long long num_rows, int* check, cudaStream_t st) {
    const int nch = dim / 8;
    if (nch <= 16) return launch_shape<XT, CT, 16, 1>(x, n, dim, slots, data, scale, num_rows, check, st);
    if (nch <= 32) return launch_shape<XT, CT, 32, 1>(x, n, dim, slots, data, scale, num_rows, check, st);
    if (nch <= 64) return launch_shape<XT, CT, 32, 2>(x, n, dim, slots, data, scale, num_rows, check, st);
    if (nch <= 96) return launch_shape<XT, CT, 32, 3>(x, n, dim, slots, data, scale, num_rows, check, st);
    return launch_shape<XT, CT, 32, 4>(x, n, dim, slots, data, scale, num_rows, check, st);
}

template <int XT>
cudaError_t launch_x(const void* x, int n, int dim, const long long* slots, void* data, int ct,
                     float* scale, long long num_rows, int* check, cudaStream_t st) {
    if (ct == kE4M3) return launch_for<XT, kE4M3>(x, n, dim, slots, data, scale, num_rows, check, st);
    if (ct == kBF16) return launch_for<XT, kBF16>(x, n, dim, slots, data, scale, num_rows, check, st);
    return launch_for<XT, kF32>(x, n, dim, slots, data, scale, num_rows, check, st);
}

}  // namespace

cudaError_t launch_cache_store(const void* x, int x_dtype, int n, int dim, const long long* slots,
                               void* data, int cache_dtype, float* scale, long long num_rows,
                               int* check, cudaStream_t st) {
    return x_dtype == kBF16
               ? launch_x<kBF16>(x, n, dim, slots, data, cache_dtype, scale, num_rows, check, st)
               : launch_x<kF32>(x, n, dim, slots, data, cache_dtype, scale, num_rows, check, st);
}

}  // namespace dsa
