// topk.cu -- per-query top-k token selection (k = 2048 in DeepSeek-V3.2 serving:
// "DeepSeek-V3.2-Exp DSA deployment guide", section 3.1; selection of the most
// relevant key/value entries: "SGLang Day-0 support for DeepSeek-V3.2", section
// "DeepSeek Sparse Attention").  A row with pos+1 <= k keeps every position
// (dense fallback, same guide, section 5.1).
//
// Method: exact radix select on order-preserving 32-bit keys, one 1024-thread CTA
// per row, output in ascending position order (deterministic; equal keys at the
// threshold go to the lowest positions).
//
//   1. One vectorised read of the row stages the keys in shared memory (up to the
//      staging capacity; the rest is re-read from L2) and builds a histogram of the
//      top 11 key bits.  Logits crowd into a few exponent bins, so each lane adds to
//      one of four interleaved histogram copies to cut same-address conflicts.  The
//      histogram fixes the bin b1 of the k-th key: every key in a higher bin is in.
//   2. One sweep over 32-key groups writes a selection bitmap straight from warp
//      ballots (bit set = bin above b1) and appends the keys of bin b1 with their
//      positions to the sweeping warp's own segment of a candidate list C.
//   3. Two radix passes (11 + 10 bits) over C fix the exact k-th key T and how many
//      keys equal to T are needed; keys above T get their bit, and the equal keys
//      go to a second bitmap from which the lowest positions are taken.
//   4. A block scan over the bitmap's popcounts turns it into the ascending list.
// If C would overflow (thousands of keys in one bin, e.g. equal scores, or more than
// a segment's worth in one warp's share), steps 2-3 fall back to radix passes over
// the whole row and one marking sweep.
// Rows of at least 24k keys first try a sampled threshold (step 0): the m-th largest of
// 2048 evenly spaced keys (low 10 bits cleared), m chosen so that about 2k keys of the row are expected at or
// above it; one coalesced read of the row then gathers those keys (and positions) as
// the candidates, and the exact selection runs on them as in step 3 with full 32-bit
// keys.  The candidates hold the whole top k whenever at least k keys reach the
// threshold, which is checked; otherwise (or on overflow) steps 1-4 run as above, so
// the result is the same either way -- only the reads differ (one pass over the row,
// no per-key shared-memory atomics).  Rows longer
// than the bitmap capacity use a second kernel that refines over the whole row and
// emits in two ordered sweeps.  Batches of a few dozen long rows (>= 32768 keys)
// split every row over a thread-block cluster (topk_cluster_kernel, below).
#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kTopBits = 11;
constexpr uint32_t kLowMask = (1u << (32 - kTopBits)) - 1u;   // 21 low key bits
constexpr int kCopies = 4;                 // interleaved copies of the first histogram
constexpr int kCandCap = 8192;             // candidates: low 21 key bits + position
constexpr int kSeg = kCandCap / 32;        // per-warp candidate segment
constexpr int kMaxWords = 8192;            // bitmap words: rows up to 262144 keys
constexpr int kSmemLimit = 232448;
constexpr int kSample = 2048;              // keys sampled for the step-0 threshold
constexpr int kPrefilterRatio = 24;       // step 0 for rows of at least 24k keys
constexpr int kStaticReserve = 1024;

// Monotone map float -> uint32 (larger float, larger key); -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
    int warp_sums[kWarps + 1];
    int bin, above, count;
    int seg_n[32];            // candidates found by each warp
};

// Block-wide exclusive prefix sum of one int per thread; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, Shared& sh, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh.warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = sh.warp_sums[lane];
        int s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        sh.warp_sums[lane] = s - w;        // exclusive per warp
        if (lane == 31) sh.warp_sums[32] = s;
    }
    __syncthreads();
    const int r = sh.warp_sums[warp] + x - v;
    *total = sh.warp_sums[32];
    __syncthreads();  // warp_sums may be reused right after
    return r;
}

// The bin (of nb = 1024 or 2048, counted from the top) holding the remaining-th
// largest key, summing `copies` histograms spaced 2048 apart; *above = keys in
// higher bins, *count = keys in the bin.  Ends synchronised.
__device__ __forceinline__ int scan_bins(Shared& sh, const int* local, int nb, int remaining,
                                         int* above, int* count);

__device__ __forceinline__ int find_bin(Shared& sh, const int* hist, int copies, int nb,
                                        int remaining, int* above, int* count) {
    const int tid = threadIdx.x;
    const int per = nb / kThreads;
    int local[2] = {0, 0};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (j < per) {
            const int bin = nb - 1 - (tid * per + j);
            for (int c = 0; c < copies; ++c) local[j] += hist[c * 2048 + bin];
        }
    }
    return scan_bins(sh, local, nb, remaining, above, count);
}

// The scan behind find_bin: thread tid holds the counts of bins nb-1-(tid*per+j).
__device__ __forceinline__ int scan_bins(Shared& sh, const int* local, int nb, int remaining,
                                         int* above, int* count) {
    const int tid = threadIdx.x;
    const int per = nb / kThreads;
    int total;
    int run = block_excl_scan(local[0] + local[1], sh, &total);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (j < per) {
            const int ab = run;
            run += local[j];
            if (run >= remaining && ab < remaining) {
                sh.bin = nb - 1 - (tid * per + j);
                sh.above = ab;
                sh.count = local[j];
            }
        }
    }
    __syncthreads();
    *above = sh.above;
    *count = sh.count;
    const int b = sh.bin;
    __syncthreads();
    return b;
}

// Keys of the row: staged prefix in shared memory, the rest re-read from global.
struct Row {
    const float* g;
    const uint32_t* s;
    int cap;
    __device__ __forceinline__ uint32_t operator()(int i) const {
        return i < cap ? s[i] : order_key(__ldg(g + i));
    }
};

// One radix refinement pass over n keys: histogram (copy 0) of bits
// [shift, shift+nbits) of the keys matching prefix/pmask, then the bin of the
// remaining-th largest; *count = keys in that bin.
// for_each(f) calls f(key) for this thread's share of the keys.
template <class ForEach>
__device__ __forceinline__ void refine(Shared& sh, int* hist, ForEach for_each, int shift,
                                       int nbits, uint32_t& prefix, uint32_t& pmask,
                                       int& remaining, int* count) {
    const int nb = 1 << nbits, tid = threadIdx.x;
    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t pf = prefix, pm = pmask;
    for_each([&](uint32_t key) {
        if ((key & pm) == pf) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
    });
    __syncthreads();
    int above;
    const int bin = find_bin(sh, hist, 1, nb, remaining, &above, count);
    remaining -= above;
    prefix |= (uint32_t)bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
}

// Stage the row's keys (first `cap`) and build the interleaved top-bit histogram.
__device__ __forceinline__ void stage_and_histogram(const float* grow, int n, uint32_t* skeys,
                                                    int cap, int* hist) {
    const int tid = threadIdx.x;
    int* my_hist = hist + (tid & (kCopies - 1)) * 2048;
    for (int base = 0; base < n; base += 8 * kThreads) {
        float v[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i0 = base + h * 4 * kThreads + 4 * tid;
            if (i0 + 3 < n) {
                const float4 f = __ldg(reinterpret_cast<const float4*>(grow + i0));
                v[4 * h] = f.x; v[4 * h + 1] = f.y; v[4 * h + 2] = f.z; v[4 * h + 3] = f.w;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[4 * h + j] = i0 + j < n ? __ldg(grow + i0 + j) : 0.f;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = base + h * 4 * kThreads + 4 * tid + j;
                if (i < n) {
                    const uint32_t key = order_key(v[4 * h + j]);
                    if (i < cap) skeys[i] = key;
                    atomicAdd(&my_hist[key >> (32 - kTopBits)], 1);
                }
            }
        }
    }
}

// The `need` lowest positions among the keys equal to the threshold (eqmap, n_eq of
// them) join the selection bitmap.  Ends synchronised.
__device__ __forceinline__ void take_lowest_equal(Shared& sh, uint32_t* bitmap, const uint32_t* eqmap,
                                                  int words, int need, int n_eq) {
    const int tid = threadIdx.x;
    if (n_eq == need) {
        for (int w = tid; w < words; w += kThreads) bitmap[w] |= eqmap[w];
    } else {
        const int wpt = (words + kThreads - 1) / kThreads;
        const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
        int c = 0;
        for (int w = w0; w < w1; ++w) c += __popc(eqmap[w]);
        int total;
        int before = block_excl_scan(c, sh, &total);
        for (int w = w0; w < w1 && before < need; ++w) {
            uint32_t e = eqmap[w];
            const int pc = __popc(e);
            if (before + pc > need) {               // keep only the lowest bits
                for (int drop = before + pc - need; drop > 0; --drop)
                    e &= ~(0x80000000u >> __clz(e));
            }
            bitmap[w] |= e;
            before += pc;
        }
    }
    __syncthreads();
}

// Bitmap of the selected positions (ascending) -> out[0, count).
__device__ __forceinline__ void bitmap_to_list(Shared& sh, const uint32_t* bits, int words,
                                               int* out, int base = 0) {
    const int tid = threadIdx.x;
    const int wpt = (words + kThreads - 1) / kThreads;
    const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
    int total;
    int at = block_excl_scan(c, sh, &total);
    for (int w = w0; w < w1; ++w) {
        uint32_t b = bits[w];
        while (b) {
            const int bit = __ffs(b) - 1;
            out[at++] = base + 32 * w + bit;
            b &= b - 1u;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(const float* __restrict__ logits, long long ld, BatchView bv, int k,
            int* __restrict__ idx, int* check, int words_cap, int stage_cap, int row0) {
    extern __shared__ __align__(16) uint8_t dyn[];
    int* hist = reinterpret_cast<int*>(dyn);                                   // [4][2048]
    uint32_t* ckey = reinterpret_cast<uint32_t*>(dyn + kCopies * 2048 * 4);      // [kCandCap]
    int* cpos = reinterpret_cast<int*>(ckey + kCandCap);                         // [kCandCap]
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(cpos + kCandCap);             // [words_cap]
    uint32_t* eqmap = bitmap + words_cap;                                        // [words_cap]
    uint32_t* skeys = eqmap + words_cap;                                         // [stage_cap]
    __shared__ Shared sh;

    const int t = row0 + blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();
    int* out = idx + (long long)t * k;
    const RowInfo ri = row_info(bv, t, check);
    // the logits may come from the previous kernel, and an earlier kernel of the stream
    // may still read the selection buffer: wait before the first load or store
    pdl_wait();
    if (!ri.ok) {
        for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    const int n = ri.pos + 1;
    if (n <= k) {  // every causal position is selected
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* grow = logits + (long long)(t - row0) * ld;
    const Row row{grow, skeys, stage_cap};
    const int words = (n + 31) >> 5;

    // ---- 0. sampled threshold; candidates at or above it --------------------------
    if (n >= kPrefilterRatio * k && 3 * k <= kCandCap) {
        uint32_t* samp = reinterpret_cast<uint32_t*>(cpos);      // [kSample], before C is built
        for (int s = tid; s < kSample; s += kThreads)
            samp[s] = order_key(__ldg(grow + (int)(((long long)s * n) / kSample)));
        for (int w = tid; w < words; w += kThreads) {
            bitmap[w] = 0u;
            eqmap[w] = 0u;
        }
        __syncthreads();
        // T0 = the m-th largest sample key with its low 10 bits cleared, m = ceil(2 k
        // kSample / n): about 2k keys of the row are expected at or above it (the count
        // is checked below)
        const int m = (int)min((long long)kSample, (2LL * k * kSample + n - 1) / n);
        auto samp_each = [&](auto f) {
            for (int s2 = tid; s2 < kSample; s2 += kThreads) f(samp[s2]);
        };
        uint32_t prefix = 0u, pmask = 0u;
        int rem = m, cnt;
        refine(sh, hist, samp_each, 21, 11, prefix, pmask, rem, &cnt);
        refine(sh, hist, samp_each, 10, 11, prefix, pmask, rem, &cnt);
        const uint32_t T0 = prefix;
        // one coalesced read of the row (a warp takes 128 consecutive keys at a time,
        // interleaved over the warps): keys >= T0 with their positions into the
        // sweeping warp's segment of C
        int c_at = 0;
        constexpr int kU = 4;                              // 128-key blocks in flight per warp
        for (int b0 = 128 * warp; b0 < n; b0 += kU * 128 * kWarps) {        // warp-uniform
            float4 f[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i4 = b0 + u * 128 * kWarps + 4 * lane;
                if (i4 + 3 < n) {
                    f[u] = __ldg(reinterpret_cast<const float4*>(grow + i4));
                } else {
                    f[u].x = i4 < n ? __ldg(grow + i4) : 0.f;
                    f[u].y = i4 + 1 < n ? __ldg(grow + i4 + 1) : 0.f;
                    f[u].z = i4 + 2 < n ? __ldg(grow + i4 + 2) : 0.f;
                    f[u].w = i4 + 3 < n ? __ldg(grow + i4 + 3) : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i4 = b0 + u * 128 * kWarps + 4 * lane;
                const uint32_t kk[4] = {order_key(f[u].x), order_key(f[u].y), order_key(f[u].z),
                                        order_key(f[u].w)};
                bool c4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) c4[j] = i4 + j < n && kk[j] >= T0;
                if (!__any_sync(0xffffffffu, c4[0] || c4[1] || c4[2] || c4[3])) continue;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const unsigned mc = __ballot_sync(0xffffffffu, c4[j]);
                    if (mc) {
                        const int c = c_at + __popc(mc & ((1u << lane) - 1u));
                        if (c4[j] && c < kSeg) {
                            ckey[warp * kSeg + c] = kk[j];
                            cpos[warp * kSeg + c] = i4 + j;
                        }
                        c_at += __popc(mc);
                    }
                }
            }
        }
        if (lane == 0) sh.seg_n[warp] = c_at;
        int total;
        block_excl_scan(min(c_at, kSeg + 1) * (lane == 0 ? 1 : 0), sh, &total);
        const bool ok = !__syncthreads_or(c_at > kSeg) && total >= k;
        if (ok) {
            // ---- exact threshold among the candidates (full keys); mark them --------
            const int seg_cnt = sh.seg_n[warp];
            auto cand_each = [&](auto f) {
                for (int c = lane; c < seg_cnt; c += 32) f(ckey[warp * kSeg + c]);
            };
            uint32_t pf = 0u, pm = 0u;
            int remaining = k, n_eq;
            refine(sh, hist, cand_each, 21, 11, pf, pm, remaining, &n_eq);
            refine(sh, hist, cand_each, 10, 11, pf, pm, remaining, &n_eq);
            refine(sh, hist, cand_each, 0, 10, pf, pm, remaining, &n_eq);
            const uint32_t T = pf;
            for (int c = lane; c < seg_cnt; c += 32) {
                const uint32_t key = ckey[warp * kSeg + c];
                const int p = cpos[warp * kSeg + c];
                if (key > T) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
                else if (key == T) atomicOr(&eqmap[p >> 5], 1u << (p & 31));
            }
            __syncthreads();
            take_lowest_equal(sh, bitmap, eqmap, words, remaining, n_eq);
            bitmap_to_list(sh, bitmap, words, out);
            return;
        }
        // too few keys reached T0, or a segment overflowed: the full method below
    }

    // ---- 1. stage + top-bit histogram ------------------------------------------
    for (int i = tid; i < kCopies * 2048; i += kThreads) hist[i] = 0;
    __syncthreads();
    stage_and_histogram(grow, n, skeys, stage_cap, hist);
    __syncthreads();
    int n_def, n_cand;
    const uint32_t b1 = (uint32_t)find_bin(sh, hist, kCopies, 2048, k, &n_def, &n_cand);
    int remaining = k - n_def;          // keys of bin b1 still to take (>= 1)
    uint32_t T;                         // the k-th largest key
    int n_eq;                           // keys equal to T

    // whole-row iteration for the radix passes of the fallback
    auto row_each = [&](auto f) {
        for (int i = tid; i < n; i += kThreads) f(row(i));
    };
    bool fast = n_cand <= kCandCap;
    if (fast) {
        // ---- 2. bitmap of the higher bins; candidates of bin b1 -> per-warp segments
        // of C (no shared counter: one would serialise every warp on one address)
        int c_at = 0;
        for (int g0 = warp; g0 < words; g0 += 4 * kWarps) {
            uint32_t kk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = 32 * (g0 + u * kWarps) + lane;
                kk[u] = i < n ? row(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int g = g0 + u * kWarps;
                if (g >= words) break;
                const int i = 32 * g + lane;
                const uint32_t bin = kk[u] >> (32 - kTopBits);
                const unsigned md = __ballot_sync(0xffffffffu, i < n && bin > b1);
                const bool cand = i < n && bin == b1;
                const unsigned mc = __ballot_sync(0xffffffffu, cand);
                if (lane == 0) {
                    bitmap[g] = md;
                    eqmap[g] = 0u;
                }
                if (mc) {
                    const int c = c_at + __popc(mc & ((1u << lane) - 1u));
                    if (cand && c < kSeg) {
                        ckey[warp * kSeg + c] = kk[u] & kLowMask;
                        cpos[warp * kSeg + c] = i;
                    }
                    c_at += __popc(mc);
                }
            }
        }
        if (lane == 0) sh.seg_n[warp] = c_at;
        fast = !__syncthreads_or(c_at > kSeg);   // a full segment: take the fallback
    }
    if (fast) {
        // ---- 3. exact threshold among the candidates; mark them ------------------
        const int seg_cnt = sh.seg_n[warp];        // <= kSeg here
        auto cand_each = [&](auto f) {
            for (int c = lane; c < seg_cnt; c += 32) f(ckey[warp * kSeg + c]);
        };
        uint32_t prefix = 0u, pmask = 0u;
        refine(sh, hist, cand_each, 10, 11, prefix, pmask, remaining, &n_eq);
        refine(sh, hist, cand_each, 0, 10, prefix, pmask, remaining, &n_eq);
        T = prefix;
        for (int c = lane; c < seg_cnt; c += 32) {
            const uint32_t key = ckey[warp * kSeg + c];
            const int p = cpos[warp * kSeg + c];
            if (key > T) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
            else if (key == T) atomicOr(&eqmap[p >> 5], 1u << (p & 31));
        }
    } else {
        // ---- fallback: refine over the whole row, then one marking sweep ---------
        uint32_t prefix = b1 << (32 - kTopBits);
        uint32_t pmask = ~kLowMask;
        refine(sh, hist, row_each, 10, 11, prefix, pmask, remaining, &n_eq);
        refine(sh, hist, row_each, 0, 10, prefix, pmask, remaining, &n_eq);
        T = prefix;
        for (int g0 = warp; g0 < words; g0 += 4 * kWarps) {
            uint32_t kk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = 32 * (g0 + u * kWarps) + lane;
                kk[u] = i < n ? row(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int g = g0 + u * kWarps;
                if (g >= words) break;
                const int i = 32 * g + lane;
                const unsigned mg = __ballot_sync(0xffffffffu, i < n && kk[u] > T);
                const unsigned me = __ballot_sync(0xffffffffu, i < n && kk[u] == T);
                if (lane == 0) {
                    bitmap[g] = mg;
                    eqmap[g] = me;
                }
            }
        }
    }
    __syncthreads();

    take_lowest_equal(sh, bitmap, eqmap, words, remaining, n_eq);

    // ---- 4. ascending output -------------------------------------------------------
    bitmap_to_list(sh, bitmap, words, out);
}

// Rows longer than the bitmap capacity: three radix passes over the whole row, then
// an ordered two-sweep emission (warp w owns a contiguous segment; one sweep counts,
// the second writes).
__global__ void __launch_bounds__(kThreads, 1)
topk_long_kernel(const float* __restrict__ logits, long long ld, BatchView bv, int k,
                 int* __restrict__ idx, int* check, int stage_cap, int row0) {
    extern __shared__ __align__(16) uint8_t dyn[];
    int* hist = reinterpret_cast<int*>(dyn);                                // [4][2048]
    uint32_t* skeys = reinterpret_cast<uint32_t*>(dyn + kCopies * 2048 * 4);
    __shared__ Shared sh;
    __shared__ int s_gt[kWarps], s_eq[kWarps];

    const int t = row0 + blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int* out = idx + (long long)t * k;
    const RowInfo ri = row_info(bv, t, check);
    pdl_wait();                                  // before the first load or store (see topk_kernel)
    if (!ri.ok) {
        for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    const int n = ri.pos + 1;
    if (n <= k) {
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float* grow = logits + (long long)(t - row0) * ld;
    const Row row{grow, skeys, stage_cap};
    for (int i = tid; i < kCopies * 2048; i += kThreads) hist[i] = 0;
    __syncthreads();
    stage_and_histogram(grow, n, skeys, stage_cap, hist);
    __syncthreads();
    int n_def, cnt;
    const uint32_t b1 = (uint32_t)find_bin(sh, hist, kCopies, 2048, k, &n_def, &cnt);
    int remaining = k - n_def;
    uint32_t prefix = b1 << (32 - kTopBits), pmask = ~kLowMask;
    auto row_each = [&](auto f) {
        for (int i = tid; i < n; i += kThreads) f(row(i));
    };
    refine(sh, hist, row_each, 10, 11, prefix, pmask, remaining, &cnt);
    refine(sh, hist, row_each, 0, 10, prefix, pmask, remaining, &cnt);
    const uint32_t T = prefix;
    const int need_eq = remaining;

    const int seg = ((n + kWarps - 1) / kWarps + 31) & ~31;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    int c_gt = 0, c_eq = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < w1 ? row(i) : 0u;
        c_gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > T));
        c_eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == T));
    }
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
    int taken = gt_before + min(eq_before, need_eq);
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

// ---------------------------------------------------------------------------------
// Short batches (a few dozen rows): each row is split over the C CTAs of a thread-block
// cluster (C = 2, 4 or 8), CTA r owning the contiguous segment r of the row.  The
// method is the one above; the three histograms that fix the threshold are summed
// across the cluster through distributed shared memory (every thread reads its bins
// from every CTA), the equal keys at the threshold go to the lowest positions across
// segments in rank order, and each CTA writes its selected positions at the offset
// given by the counts of the lower ranks.  All decisions derive from cluster-summed
// values, so every CTA takes the same branches and the same cluster barriers.
constexpr int kCCand = 4096;               // candidates per CTA
constexpr int kCSeg = kCCand / kWarps;     // per-warp candidate segment

struct ClusterEx {
    int slot[2][8];                        // all-gather buffers, used alternately
};

__device__ __forceinline__ int ld_cluster_s32(uint32_t caddr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
    return v;
}

__device__ __forceinline__ void st_cluster_s32(uint32_t caddr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(caddr), "r"(v) : "memory");
}

// Every CTA contributes v; returns the cluster total and *before = the sum over lower
// ranks.  Uses buffer (*use)++ & 1 (each buffer is rewritten only after a later cluster
// barrier that every reader of its previous values has passed).
__device__ __forceinline__ int cluster_allgather_sum(ClusterEx& ex, int v, int nrank, int rank,
                                                     int* use, int* before) {
    const int b = (*use)++ & 1;
    if (threadIdx.x < nrank) st_cluster_s32(sm100::mapa(sm100::smem_u32(&ex.slot[b][rank]), threadIdx.x), v);
    sm100::cluster_sync();
    int tot = 0, bef = 0;
    for (int q = 0; q < nrank; ++q) {
        const int x = ex.slot[b][q];
        tot += x;
        if (q < rank) bef += x;
    }
    *before = bef;
    return tot;
}

// The bin of the remaining-th largest key over the cluster-summed histogram `hist`
// (nb bins; complete in this CTA).  Ends after every CTA has read every histogram.
__device__ __forceinline__ int cluster_find_bin(Shared& sh, const int* hist, int nb, int nrank,
                                                int remaining, int* above, int* count) {
    sm100::cluster_sync();                          // every CTA's histogram is complete
    const int per = nb / kThreads;
    int local[2] = {0, 0};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        if (j < per) {
            const uint32_t a = sm100::smem_u32(hist + (nb - 1 - (threadIdx.x * per + j)));
            int v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = q < nrank ? ld_cluster_s32(sm100::mapa(a, q)) : 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) local[j] += v[q];
        }
    }
    const int b = scan_bins(sh, local, nb, remaining, above, count);
    sm100::cluster_sync();                          // all reads done: hist may be reused
    return b;
}

template <class ForEach>
__device__ __forceinline__ void cluster_refine(Shared& sh, int* hist, ForEach for_each, int shift,
                                               int nbits, uint32_t& prefix, uint32_t& pmask,
                                               int& remaining, int* count, int nrank) {
    const int nb = 1 << nbits, tid = threadIdx.x;
    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t pf = prefix, pm = pmask;
    for_each([&](uint32_t key) {
        if ((key & pm) == pf) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1);
    });
    __syncthreads();
    int above;
    const int bin = cluster_find_bin(sh, hist, nb, nrank, remaining, &above, count);
    remaining -= above;
    prefix |= (uint32_t)bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
}

__global__ void __launch_bounds__(kThreads, 1)
topk_cluster_kernel(const float* __restrict__ logits, long long ld, BatchView bv, int k,
                    int* __restrict__ idx, int* check, int words_cap, int stage_cap, int row0) {
    extern __shared__ __align__(16) uint8_t dyn[];
    int* hist = reinterpret_cast<int*>(dyn);                                   // [4][2048]
    uint32_t* ckey = reinterpret_cast<uint32_t*>(dyn + kCopies * 2048 * 4);      // [kCCand]
    int* cpos = reinterpret_cast<int*>(ckey + kCCand);                           // [kCCand]
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(cpos + kCCand);               // [words_cap]
    uint32_t* eqmap = bitmap + words_cap;                                        // [words_cap]
    uint32_t* skeys = eqmap + words_cap;                                         // [stage_cap]
    __shared__ Shared sh;
    __shared__ ClusterEx ex;

    uint32_t nrank_u;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(nrank_u));
    const int nrank = (int)nrank_u, rank = (int)sm100::cluster_ctarank();
    const int t = row0 + blockIdx.x / nrank, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();
    int* out = idx + (long long)t * k;
    const RowInfo ri = row_info(bv, t, check);
    pdl_wait();                                  // before the first load or store (see topk_kernel)
    if (!ri.ok) {
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    const int n = ri.pos + 1;
    if (n <= k) {
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    // this CTA's segment of the row: [seg0, seg0 + sn), 32-aligned
    const int seg = (((n + nrank - 1) / nrank) + 31) & ~31;
    const int seg0 = min(n, rank * seg), sn = min(n, seg0 + seg) - seg0;
    const float* grow = logits + (long long)(t - row0) * ld + seg0;
    const Row row{grow, skeys, stage_cap};
    const int words = (sn + 31) >> 5;
    int use = 0;

    // ---- 1. stage + top-bit histogram, summed over the cluster ---------------------
    for (int i = tid; i < kCopies * 2048; i += kThreads) hist[i] = 0;
    __syncthreads();
    stage_and_histogram(grow, sn, skeys, stage_cap, hist);
    __syncthreads();
    for (int b = tid; b < 2048; b += kThreads)
        hist[b] = hist[b] + hist[2048 + b] + hist[4096 + b] + hist[6144 + b];
    __syncthreads();
    int n_def, n_cand;
    const uint32_t b1 = (uint32_t)cluster_find_bin(sh, hist, 2048, nrank, k, &n_def, &n_cand);
    int remaining = k - n_def;
    uint32_t T;
    int n_eq;
    auto row_each = [&](auto f) {
        for (int i = tid; i < sn; i += kThreads) f(row(i));
    };

    // ---- 2. bitmap of the higher bins; candidates of bin b1 into per-warp segments
    int c_at = 0;
    for (int g0 = warp; g0 < words; g0 += 4 * kWarps) {
        uint32_t kk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = 32 * (g0 + u * kWarps) + lane;
            kk[u] = i < sn ? row(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int g = g0 + u * kWarps;
            if (g >= words) break;
            const int i = 32 * g + lane;
            const uint32_t bin = kk[u] >> (32 - kTopBits);
            const unsigned md = __ballot_sync(0xffffffffu, i < sn && bin > b1);
            const bool cand = i < sn && bin == b1;
            const unsigned mc = __ballot_sync(0xffffffffu, cand);
            if (lane == 0) {
                bitmap[g] = md;
                eqmap[g] = 0u;
            }
            if (mc) {
                const int c = c_at + __popc(mc & ((1u << lane) - 1u));
                if (cand && c < kCSeg) {
                    ckey[warp * kCSeg + c] = kk[u] & kLowMask;
                    cpos[warp * kCSeg + c] = i;
                }
                c_at += __popc(mc);
            }
        }
    }
    if (lane == 0) sh.seg_n[warp] = c_at;
    const int over_local = __syncthreads_or(c_at > kCSeg) ? 1 : 0;
    int dummy;
    const bool fast = cluster_allgather_sum(ex, over_local, nrank, rank, &use, &dummy) == 0;

    if (fast) {
        // ---- 3. exact threshold among the cluster's candidates; mark them ----------
        const int seg_cnt = sh.seg_n[warp];
        auto cand_each = [&](auto f) {
            for (int c = lane; c < seg_cnt; c += 32) f(ckey[warp * kCSeg + c]);
        };
        uint32_t prefix = 0u, pmask = 0u;
        cluster_refine(sh, hist, cand_each, 10, 11, prefix, pmask, remaining, &n_eq, nrank);
        cluster_refine(sh, hist, cand_each, 0, 10, prefix, pmask, remaining, &n_eq, nrank);
        T = prefix;
        for (int c = lane; c < seg_cnt; c += 32) {
            const uint32_t key = ckey[warp * kCSeg + c];
            const int p = cpos[warp * kCSeg + c];
            if (key > T) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
            else if (key == T) atomicOr(&eqmap[p >> 5], 1u << (p & 31));
        }
    } else {
        // ---- fallback: refine over the segments, then one marking sweep --------------
        uint32_t prefix = b1 << (32 - kTopBits);
        uint32_t pmask = ~kLowMask;
        cluster_refine(sh, hist, row_each, 10, 11, prefix, pmask, remaining, &n_eq, nrank);
        cluster_refine(sh, hist, row_each, 0, 10, prefix, pmask, remaining, &n_eq, nrank);
        T = prefix;
        for (int g0 = warp; g0 < words; g0 += kWarps) {
            const int i = 32 * g0 + lane;
            const uint32_t key = i < sn ? row(i) : 0u;
            const unsigned mg = __ballot_sync(0xffffffffu, i < sn && key > T);
            const unsigned me = __ballot_sync(0xffffffffu, i < sn && key == T);
            if (lane == 0) {
                bitmap[g0] = mg;
                eqmap[g0] = me;
            }
        }
    }
    __syncthreads();

    // ---- equal keys: the `remaining` lowest positions of the whole row -------------
    {
        const int wpt = (words + kThreads - 1) / kThreads;
        const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
        int c = 0;
        for (int w = w0; w < w1; ++w) c += __popc(eqmap[w]);
        int local_eq;
        int before = block_excl_scan(c, sh, &local_eq);
        int eq_lower;
        cluster_allgather_sum(ex, local_eq, nrank, rank, &use, &eq_lower);
        const int take = max(0, min(local_eq, remaining - eq_lower));
        for (int w = w0; w < w1 && before < take; ++w) {
            uint32_t e = eqmap[w];
            const int pc = __popc(e);
            if (before + pc > take) {
                for (int drop = before + pc - take; drop > 0; --drop)
                    e &= ~(0x80000000u >> __clz(e));
            }
            bitmap[w] |= e;
            before += pc;
        }
    }
    __syncthreads();

    // ---- 4. ascending output: this segment's positions after the lower ranks' -------
    {
        const int wpt = (words + kThreads - 1) / kThreads;
        const int w0 = min(words, tid * wpt), w1 = min(words, w0 + wpt);
        int c = 0;
        for (int w = w0; w < w1; ++w) c += __popc(bitmap[w]);
        int local_sel;
        block_excl_scan(c, sh, &local_sel);
        int sel_lower;
        cluster_allgather_sum(ex, local_sel, nrank, rank, &use, &sel_lower);
        bitmap_to_list(sh, bitmap, words, out + sel_lower, seg0);
    }
}


// Per-device launch state: every top-k kernel's dynamic shared-memory limit is raised
// once to the largest size any launch asks for (so no launch ever lowers it under a
// launch on another host thread), and whether a cluster of 2, 4 or 8 CTAs at that
// size fits on the device is asked once.
constexpr int kMaxDynSmem = kSmemLimit - kStaticReserve;
constexpr int kMaxDevices = 64;

struct TopkDeviceState {
    std::once_flag once;
    cudaError_t err = cudaSuccess;
    bool cluster_fits[4] = {false, false, false, false};   // index: C = 1, 2, 4, 8
};
TopkDeviceState g_topk_dev[kMaxDevices];

cudaError_t topk_device_state(const TopkDeviceState** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    TopkDeviceState& s = g_topk_dev[dev];
    std::call_once(s.once, [&s] {
        for (auto kern : {topk_kernel, topk_cluster_kernel}) {
            s.err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
            if (s.err != cudaSuccess) return;
        }
        s.err = cudaFuncSetAttribute(topk_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kMaxDynSmem);
        if (s.err != cudaSuccess) return;
        for (int slot = 1; slot < 4; ++slot) {
            cudaLaunchConfig_t probe = {};
            const unsigned C = 1u << slot;
            probe.gridDim = dim3(C);
            probe.blockDim = dim3(kThreads);
            probe.dynamicSmemBytes = kMaxDynSmem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = C;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            probe.attrs = attr;
            probe.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &probe) != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
            s.cluster_fits[slot] = n > 0;
        }
    });
    if (s.err != cudaSuccess) return s.err;
    *out = &s;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_topk(const float* logits, long long ld, const BatchView& bv, int k, int* idx,
                        int* check, cudaStream_t st, bool pdl, int row0) {
    const TopkDeviceState* ds = nullptr;
    cudaError_t de = topk_device_state(&ds);
    if (de != cudaSuccess) return de;
    const int hist_bytes = kCopies * 2048 * 4;
    const int words = ((bv.max_seq_len + 31) / 32 + 3) & ~3;
    // A few dozen long rows would leave most SMs idle with one CTA per row, and a row
    // beyond the staging capacity is re-read from L2: split each row over a cluster of
    // C CTAs instead.  (Rows of ~8K keys measured slower this way: the cluster barriers
    // and exchanges cost more than the split saves.)
    const int T = bv.total_q - row0;
    const int C = T <= kNumSMs / 8 ? 8 : T <= kNumSMs / 4 ? 4 : T <= kNumSMs / 2 ? 2 : 1;
    const int cseg = (((bv.max_seq_len + C - 1) / C) + 31) & ~31;
    const int slot = C == 2 ? 1 : C == 4 ? 2 : 3;
    if (C > 1 && bv.max_seq_len >= 32768 && bv.max_seq_len > 2 * k && cseg <= 32 * kMaxWords &&
        ds->cluster_fits[slot]) {
        const int seg = cseg;
        const int cwords = ((seg / 32) + 3) & ~3;
        const int fixed = hist_bytes + kCCand * 8 + 2 * cwords * 4;
        int stage = (kMaxDynSmem - fixed) / 4 & ~3;
        if (stage > seg) stage = seg;
        const size_t smem = (size_t)fixed + (size_t)stage * 4;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(T * C);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 2 : 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, logits, ld, bv, k, idx, check,
                                           cwords, stage, row0);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (words <= kMaxWords) {
        const int fixed = hist_bytes + kCandCap * 8 + 2 * words * 4;
        int stage = (kMaxDynSmem - fixed) / 4 & ~3;
        if (stage > bv.max_seq_len) stage = bv.max_seq_len;
        const size_t smem = (size_t)fixed + (size_t)stage * 4;
        cudaError_t e = launch_kernel(topk_kernel, dim3(T), dim3(kThreads), smem, st, pdl, logits, ld,
                          bv, k, idx, check, words, stage, row0);
        if (e != cudaSuccess) return e;
    } else {
        const int stage = (kMaxDynSmem - hist_bytes) / 4 & ~3;
        const size_t smem = (size_t)hist_bytes + (size_t)stage * 4;
        cudaError_t e = launch_kernel(topk_long_kernel, dim3(T), dim3(kThreads), smem, st, pdl, logits,
                          ld, bv, k, idx, check, stage, row0);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace dsa
