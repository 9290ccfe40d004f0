// mla_tc.cu -- sparse MLA over the selected latent-KV rows on sm_100a tensor cores.
//
// Per query row t and head h, over the selected positions s:
//   z_s = softmax_scale * q[t,h,:] . kv_s,  o[t,h,:] = softmax(z) . kv[:, 0:512],
//   lse[t,h] = log sum_s exp(z_s)
// (core attention over only the top-k entries: "SGLang Day-0 support for
// DeepSeek-V3.2", section "DeepSeek Sparse Attention"; bf16 q with a bf16 or FP8
// KV cache: "DeepSeek V3.2 usage guide", attention-kernel section; 128 heads,
// 576 = 512 latent + 64 rope, V = the 512 latent columns).
//
// Why two CTAs per query.  The fp32 output tile O (128 heads x 512) would fill all
// 512 TMEM columns of an SM, leaving no room for the scores.  So CTA v (v = 0, 1)
// of a (query, split) owns V columns [256v, 256v+256): it computes the full score
// tile S = Q . KV^T (K = 576) itself, runs the softmax, and accumulates its half of
// O.  The two CTAs repeat the QK product (1.5x the unique tensor work) but never
// talk to each other: exchanging partial score tiles through distributed shared
// memory moves only ~8 bytes per cycle between a CTA pair, slower than recomputing.
//
// Roles (352 threads): warps 0-3 = softmax (thread = head = TMEM lane), warps 4-9 =
// gather (3 threads per selected row), warp 10 = TMEM owner and MMA issuer.  The
// gather is software-pipelined over tiles, per thread: the index of tile j+4, the
// slot of tile j+3, an L2 bulk prefetch of the rows of tile j+2 and the register
// loads of tile j+1 are all in flight while tile j is written to shared memory.  The MMAs run on fp16 operands: e4m3 and bf16 values
// convert to fp16 exactly (bf16 magnitudes above 65504 saturate), and P keeps 11
// significant bits.
//
// Tensor memory: O_v (256 columns), S (64), P (32 = 64 fp16) and query dims 0..319
// (160 columns); dims 320..575 of the query sit in shared memory next to a 2-stage
// ring of gathered 64-row tiles (72 KB each, 128-byte swizzled K-major regions of
// 64 dims).  Per tile: 36 MMAs (M=128, N=64, K=16) for S -- A from TMEM or shared
// memory -- and 4 MMAs (M=128, N=256, K=16) for P.V_v with A = P in TMEM.  Online
// softmax in base 2 with lazy rescaling (O and l are rescaled only when the running
// max grows by more than 2^8).
#include <climits>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kHeads = 128;
constexpr int kTile = 64;
constexpr int kThreads = 352;
constexpr int kGatherWarp0 = 4;
constexpr int kGatherThreads = 192;    // 3 per row of a 64-row tile
constexpr int kMmaWarp = 10;

constexpr int kStages = 2;
constexpr int kRegions = 9;                              // 64-dim regions of a 576-dim row
constexpr uint32_t kQsRegions = 4;                       // query dims 320..575 in smem
constexpr uint32_t kQsBytes = kQsRegions * 16384;        // 128 rows x 128 B per region
constexpr uint32_t kStageBytes = kRegions * 8192;        // 64 rows x 128 B per region
constexpr uint32_t kOffQs = 0;
constexpr uint32_t kOffKV = kOffQs + kQsBytes;
constexpr uint32_t kOffFlag = kOffKV + kStages * kStageBytes;   // [stage][64] validity bytes
constexpr uint32_t kOffScale = kOffFlag + kStages * 64;         // [stage][64] fp32 kv scale
constexpr uint32_t kOffBar = kOffScale + kStages * 256;
constexpr uint32_t kNumBars = 12;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // 256 output columns
constexpr uint32_t kColS = 256;    // 64 score columns
constexpr uint32_t kColP = 320;    // 32 columns = 64 fp16 probabilities
constexpr uint32_t kColQ = 352;    // 160 columns = query dims 0..319 as fp16 pairs
constexpr int kQtSteps = 20;       // K-steps of 16 dims with A in TMEM

struct Params {
    const uint4* q;            // bf16 [T][128][576] as 16-byte chunks (72 per head)
    const uint8_t* kv;         // [slots][576] bf16 (1152 B) or fp8 (576 B)
    const float* kv_scale;     // [slots] or nullptr
    const int* slot_table;
    int st_stride;
    long long num_slots;
    BatchView bv;
    const int* idx;
    int k;
    int nsplit;
    int chunk;                 // selected entries per split (multiple of 64)
    float sc_log2;             // softmax_scale * log2(e)
    __nv_bfloat16* out;
    float* lse;
    float* o_part;
    float* lse_part;
    int* check;
};

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint4 ldg16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void sts16(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                 ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Two e4m3 codes (low byte first) -> two fp16 (exact: every e4m3 value is an fp16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Two floats -> fp16x2 (lo in the low half), round to nearest, saturating at 65504.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two bf16 (one 32-bit word) -> two fp16; exact for magnitudes in [2^-14, 65504].
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    return pack_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 a) {
    return make_uint4(bf16x2_to_f16x2(a.x), bf16x2_to_f16x2(a.y), bf16x2_to_f16x2(a.z),
                      bf16x2_to_f16x2(a.w));
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
mla_tc_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(base);
    uint8_t* vflag = base + kOffFlag;
    float* colscale = reinterpret_cast<float*>(base + kOffScale);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBar);
    uint64_t* kvfull = bars + 0;    // [2] gather -> MMA / softmax     (192 arrivals)
    uint64_t* kvempty = bars + 2;   // [2] PV done -> gather           (commit)
    uint64_t* sfull = bars + 4;     // scores ready                    (commit)
    uint64_t* sempty = bars + 5;    // scores read                     (128)
    uint64_t* pfull = bars + 6;     // P (and any O rescale) ready     (128)
    uint64_t* pvdone = bars + 7;    // PV finished                     (commit)
    uint64_t* qfull = bars + 8;     // query in TMEM + shared memory   (128)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int vh = blockIdx.x & 1;                   // which half of the V columns
    const int cid = blockIdx.x >> 1;
    const int t = cid / p.nsplit, split = cid % p.nsplit;
    const RowInfo ri = row_info(p.bv, t, threadIdx.x == 0 ? p.check : nullptr);
    const int i0 = split * p.chunk, i1 = min(p.k, i0 + p.chunk);
    __shared__ int s_skip;

    if (threadIdx.x == 0) {
        s_skip = timed_out_before(p.check) ? 1 : 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&kvfull[i], kGatherThreads);
            mbar_init(&kvempty[i], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(sempty, 128);
        mbar_init(pfull, 128);
        mbar_init(pvdone, 1);
        mbar_init(qfull, 128);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = (ri.ok && i1 > i0 && !s_skip) ? (i1 - i0 + kTile - 1) / kTile : 0;

    if (warp >= kGatherWarp0 && warp < kMmaWarp) {
        // ============================================================ gather
        const int gt = threadIdx.x - kGatherWarp0 * 32;     // 0..191
        const int c = gt / 3, part = gt % 3;                // row of the tile, third of the row
        constexpr int kN = kFp8 ? 12 : 24;                  // 16-byte loads per thread per tile
        constexpr int kRowBytes = kFp8 ? 576 : 1152;
        const long long seq_base = (long long)ri.b * p.st_stride;
        // Per-thread pipeline state for its row c of upcoming tiles: no load result is
        // consumed in the iteration that issues the load.
        int idx5 = -1;                                  // index of tile j+5
        int raw_s4 = -1;                                // slot-table entry of tile j+4 (unchecked)
        long long slot1 = -1, slot2 = -1, slot3 = -1;   // checked slots of tiles j+1..j+3
        auto fetch_idx = [&](int j) -> int {
            const int i = i0 + j * kTile + c;
            return (j < n_tiles && i < i1) ? __ldg(p.idx + (long long)t * p.k + i) : -1;
        };
        // Slot-table entry for index s, or a sentinel for a skipped entry / an index
        // past the query position (table entries are checked separately).
        constexpr int kSkip = INT_MIN, kPastPos = INT_MIN + 1;
        auto fetch_slot = [&](int s) -> int {
            if (s < 0) return kSkip;
            if (s > ri.pos) return kPastPos;
            return __ldg(p.slot_table + seq_base + s);
        };
        auto check_slot = [&](int raw) -> long long {   // -1 for skipped / bad entries
            if (raw == kSkip) return -1;
            if (raw == kPastPos || raw < 0 || (long long)raw >= p.num_slots) {
                if (part == 0) report(p.check, raw == kPastPos ? kCheckBadIndex : kCheckBadPage);
                return -1;
            }
            return raw;
        };
        auto prefetch_row = [&](long long sl) {
            if (sl >= 0)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                             ::"l"(p.kv + sl * kRowBytes + part * kN * 16), "r"(kN * 16) : "memory");
        };
        uint4 v[kN];
        float scale = 1.0f;
        auto load_regs = [&](long long sl) {
            const uint4* row = reinterpret_cast<const uint4*>(p.kv + (sl < 0 ? 0 : sl) * kRowBytes) + part * kN;
#pragma unroll
            for (int u = 0; u < kN; ++u) v[u] = sl >= 0 ? ldg16(row + u) : make_uint4(0, 0, 0, 0);
            scale = (sl >= 0 && kFp8 && p.kv_scale) ? __ldg(p.kv_scale + sl) : 1.0f;
        };
        // prologue: tiles 0..4 in flight
        long long slot0 = -1;
        if (n_tiles > 0) {
            const int x0 = fetch_idx(0), x1 = fetch_idx(1), x2 = fetch_idx(2), x3 = fetch_idx(3),
                      x4 = fetch_idx(4);
            idx5 = fetch_idx(5);
            const int r0 = fetch_slot(x0), r1 = fetch_slot(x1), r2 = fetch_slot(x2),
                      r3 = fetch_slot(x3);
            raw_s4 = fetch_slot(x4);
            slot0 = check_slot(r0);
            slot1 = check_slot(r1);
            slot2 = check_slot(r2);
            slot3 = check_slot(r3);
            prefetch_row(slot1);
            load_regs(slot0);
        }
        long long cur = slot0;                          // slot of the tile held in v
        for (int j = 0; j < n_tiles; ++j) {
            const int stage = j % kStages;
            if (!mbar_wait_warp(&kvempty[stage], ((j / kStages) & 1) ^ 1, p.check)) break;
            const uint32_t st = sb + kOffKV + stage * kStageBytes;
            if constexpr (kFp8) {
#pragma unroll
                for (int u = 0; u < kN; ++u) {
                    const int g = 2 * (part * kN + u);      // first of the two fp16 chunks
                    const uint4 a = v[u];
                    const uint4 lo = make_uint4(e4m3x2_to_f16x2(a.x & 0xFFFF), e4m3x2_to_f16x2(a.x >> 16),
                                                e4m3x2_to_f16x2(a.y & 0xFFFF), e4m3x2_to_f16x2(a.y >> 16));
                    const uint4 hi = make_uint4(e4m3x2_to_f16x2(a.z & 0xFFFF), e4m3x2_to_f16x2(a.z >> 16),
                                                e4m3x2_to_f16x2(a.w & 0xFFFF), e4m3x2_to_f16x2(a.w >> 16));
                    sts16(st + (g >> 3) * 8192 + sw128(c, g & 7), lo);
                    sts16(st + ((g + 1) >> 3) * 8192 + sw128(c, (g + 1) & 7), hi);
                }
            } else {
#pragma unroll
                for (int u = 0; u < kN; ++u) {
                    const int g = part * kN + u;
                    sts16(st + (g >> 3) * 8192 + sw128(c, g & 7), bf16x8_to_f16x8(v[u]));
                }
            }
            if (part == 0) {
                vflag[stage * 64 + c] = cur >= 0 ? 1 : 0;
                colscale[stage * 64 + c] = scale;
            }
            fence_proxy_async_smem();
            mbar_arrive(&kvfull[stage]);
            // advance the pipeline by one tile
            if (j + 1 < n_tiles) load_regs(slot1);
            prefetch_row(slot2);
            const long long s4 = check_slot(raw_s4);   // loaded one iteration ago
            raw_s4 = fetch_slot(idx5);                  // index loaded one iteration ago
            idx5 = fetch_idx(j + 6);
            cur = slot1;
            slot1 = slot2;
            slot2 = slot3;
            slot3 = s4;
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (elect_one() && n_tiles > 0) {
            bool alive = mbar_wait(qfull, 0, p.check);
            tc_fence_after();
            const uint32_t idesc_qk = instr_desc(0, 0, 0, 0, kTile, kHeads);   // fp16 x fp16
            const uint32_t idesc_pv = instr_desc(0, 0, 0, 1, 256, kHeads);
            const uint32_t qs = sb + kOffQs;
            for (int j = 0; alive && j <= n_tiles; ++j) {
                if (j < n_tiles) {
                    const int stage = j % kStages;
                    if (!mbar_wait(&kvfull[stage], (j / kStages) & 1, p.check)) break;
                    if (j >= 1 && !mbar_wait(sempty, (j - 1) & 1, p.check)) break;
                    tc_fence_after();
                    const uint32_t kva = sb + kOffKV + stage * kStageBytes;
#pragma unroll
                    for (int s = 0; s < 36; ++s) {
                        const uint64_t bdesc =
                            smem_desc(kva + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024, kLayoutSw128);
                        if (s < kQtSteps)
                            mma_f16_ts(tmem + kColS, tmem + kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
                        else
                            mma_f16(tmem + kColS,
                                    smem_desc(qs + ((s - kQtSteps) >> 2) * 16384 + (s & 3) * 32, 16, 1024,
                                              kLayoutSw128),
                                    bdesc, idesc_qk, 1u);
                    }
                    mma_commit(sfull);
                }
                if (j >= 1) {
                    const int jj = j - 1, stage = jj % kStages;
                    if (!mbar_wait(pfull, jj & 1, p.check)) break;
                    tc_fence_after();
                    const uint32_t va = sb + kOffKV + stage * kStageBytes + vh * 4 * 8192;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem + kColO, tmem + kColP + 8 * kk,
                                   smem_desc(va + kk * 2048, 8192, 1024, kLayoutSw128), idesc_pv,
                                   (jj > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&kvempty[stage]);
                    mma_commit(pvdone);
                }
            }
        }
    } else {
        // ============================================================ softmax
        const int h = threadIdx.x;                       // head == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        {   // query row h: dims 0..319 into TMEM as fp16 pairs, 320..575 into smem
            const uint4* qrow = p.q + ((long long)t * kHeads + h) * 72;
            if (ri.ok) asm volatile("cp.async.bulk.prefetch.L2.global [%0], 1152;" ::"l"(qrow) : "memory");
#pragma unroll
            for (int g0 = 0; g0 < 72; g0 += 24) {
                uint4 qv[24];
#pragma unroll
                for (int g = 0; g < 24; ++g) qv[g] = ri.ok ? ldg16(qrow + g0 + g) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int g = 0; g < 24; g += 2) {
                    const int gg = g0 + g;
                    const uint4 a = bf16x8_to_f16x8(qv[g]), b = bf16x8_to_f16x8(qv[g + 1]);
                    if (gg < 40) {
                        tmem_st8(lane_base + kColQ + 4 * gg, a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w);
                    } else {
                        const int c0 = gg - 40;              // chunk index within dims 320..575
                        sts16(sb + kOffQs + (c0 >> 3) * 16384 + sw128(h, c0 & 7), a);
                        sts16(sb + kOffQs + ((c0 + 1) >> 3) * 16384 + sw128(h, (c0 + 1) & 7), b);
                    }
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(qfull);
        }
        float m_run = -INFINITY, l_run = 0.f;
        bool alive = true;
        for (int j = 0; alive && j < n_tiles; ++j) {
            const int stage = j % kStages;
            float x[64];
            {   // ---- scores of tile j
                if (!mbar_wait_warp(sfull, j & 1, p.check)) { alive = false; break; }
                tc_fence_after();
                uint32_t a[32], c[32];
                tmem_ld32(lane_base + kColS, a);
                tmem_ld32(lane_base + kColS + 32, c);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(sempty);                       // the next QK may overwrite S
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = __uint_as_float(a[i]);
                    x[32 + i] = __uint_as_float(c[i]);
                }
            }
            // ---- online softmax (base 2)
            if (!mbar_wait_warp(&kvfull[stage], (j / kStages) & 1, p.check)) { alive = false; break; }
            const float* cs = colscale + stage * 64;
            {   // invalid entries (skipped or bad indices) score -inf
                const uint4* f4 = reinterpret_cast<const uint4*>(vflag + stage * 64);
                uint4 w[4];
                bool all = true;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    w[q] = f4[q];
                    all = all && w[q].x == 0x01010101u && w[q].y == 0x01010101u &&
                          w[q].z == 0x01010101u && w[q].w == 0x01010101u;
                }
                if (!all) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t ws[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
                        for (int b = 0; b < 16; ++b)
                            if (!((ws[b >> 2] >> (8 * (b & 3))) & 1u)) x[16 * q + b] = -INFINITY;
                    }
                }
            }
            // scores in base 2: x * sc (fp8: times each row's kv scale)
            float sc = p.sc_log2;
            if constexpr (kFp8) {
#pragma unroll
                for (int i = 0; i < 64; ++i) x[i] *= p.sc_log2 * cs[i];
                sc = 1.0f;
            }
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx[i] = fmaxf(fmaxf(fmaxf(x[8 * i], x[8 * i + 1]), fmaxf(x[8 * i + 2], x[8 * i + 3])),
                              fmaxf(fmaxf(x[8 * i + 4], x[8 * i + 5]), fmaxf(x[8 * i + 6], x[8 * i + 7])));
            const float m_tile = sc * fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                            fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + 8.0f;           // rescale only past 2^8 growth
            const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
            if (need) m_run = m_new;
            const bool warp_rescale = __any_sync(0xffffffffu, need) && j > 0;
            const float msub = m_run == -INFINITY ? 0.f : m_run;   // exp2(-inf) = +0
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
                const float e0 = fast_exp2(fmaf(x[i], sc, -msub));
                const float e1 = fast_exp2(fmaf(x[i + 1], sc, -msub));
                ls[(i >> 1) & 3] += e0 + e1;
                pk[i / 2] = kFp8 ? pack_f16(e0 * cs[i], e1 * cs[i + 1]) : pack_f16(e0, e1);
            }
            l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            // ---- P (and O) are free once the previous PV has finished
            if (j >= 1 && !mbar_wait_warp(pvdone, (j - 1) & 1, p.check)) { alive = false; break; }
            tc_fence_after();
            if (warp_rescale) {
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(lane_base + kColO + cc * 32, o);
                }
            }
            tmem_st32(lane_base + kColP, pk);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(pfull);
        }
        // ---- epilogue: O_v / l and lse
        const bool have = alive && n_tiles > 0 && mbar_wait_warp(pvdone, (n_tiles - 1) & 1, p.check);
        tc_fence_after();
        const float inv = (have && l_run > 0.f) ? 1.0f / l_run : 0.f;
        const float lse_v = (have && l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994531f
                                                  : -INFINITY;
        if (p.nsplit == 1) {
            uint4* orow = reinterpret_cast<uint4*>(p.out + ((long long)t * kHeads + h) * 512 + vh * 256);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t o[32];
                if (have) {
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 w;
                    w.x = have ? pack_bf16(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv) : 0u;
                    w.y = have ? pack_bf16(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv) : 0u;
                    w.z = have ? pack_bf16(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv) : 0u;
                    w.w = have ? pack_bf16(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv) : 0u;
                    orow[cc * 4 + q4] = w;
                }
            }
            if (vh == 0 && p.lse) p.lse[(long long)t * kHeads + h] = lse_v;
        } else {
            const long long pb = ((long long)t * p.nsplit + split) * kHeads + h;
            float4* orow = reinterpret_cast<float4*>(p.o_part + pb * 512 + vh * 256);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t o[32];
                if (have) {
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    orow[cc * 8 + q4] = have ? make_float4(__uint_as_float(o[4 * q4]) * inv,
                                                           __uint_as_float(o[4 * q4 + 1]) * inv,
                                                           __uint_as_float(o[4 * q4 + 2]) * inv,
                                                           __uint_as_float(o[4 * q4 + 3]) * inv)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (vh == 0) p.lse_part[pb] = lse_v;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_mla_tc(const void* q, float scale, const CacheView& kv, const BatchView& bv,
                          const int* idx, int k, int nsplit, void* out, float* lse, float* o_part,
                          float* lse_part, int* check, cudaStream_t st) {
    Params p;
    p.q = reinterpret_cast<const uint4*>(q);
    p.kv = reinterpret_cast<const uint8_t*>(kv.data);
    p.kv_scale = kv.scale;
    p.slot_table = kv.table;
    p.st_stride = kv.bt_stride;
    p.num_slots = kv.num_pages;
    p.bv = bv;
    p.idx = idx;
    p.k = k;
    p.nsplit = nsplit;
    p.chunk = ((k + nsplit - 1) / nsplit + kTile - 1) / kTile * kTile;
    p.sc_log2 = scale * 1.4426950408889634f;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.check = check;
    const bool fp8 = kv.dtype == kE4M3;
    auto kern = fp8 ? mla_tc_kernel<true> : mla_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * bv.total_q * nsplit);
    kern<<<grid, kThreads, kSmemBytes, st>>>(p);
    return cudaGetLastError();
}

}  // namespace dsa
