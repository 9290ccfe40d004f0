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
// gather runs a per-thread pipeline over tiles: the index of tile j+5, the slot of
// tile j+4 and an L2 prefetch of the rows of tile j+2 are in flight while tile j is
// copied.  bf16 rows go to shared memory by asynchronous 16-byte copies (no register
// staging); e4m3 rows are loaded one tile ahead into registers and converted to bf16
// (exact).  S = Q.K^T runs on bf16 operands.  P is kept in fp16 (11 significant
// bits; bf16 P loses up to 2^-9 relative per term, too much for rows dominated by a
// few large values), so once S_j has read a tile, the gather group converts this
// CTA's V columns of it in place from bf16 to fp16 (exact for magnitudes in
// [2^-14, 65504]; larger ones saturate) while the softmax runs, and P.V runs on fp16.
//
// Tensor memory: O_v (256 columns), two 64-column score buffers (S_j in fp32, then
// P_j in fp16 written over it, so S_{j+1} never waits for the softmax of tile j) and query dims 0..255 (128 columns); dims 256..575 of the query sit in shared memory
// next to a 2-stage ring of gathered 64-row tiles (72 KB each, 128-byte swizzled
// K-major regions of 64 dims).  Per tile: 36 MMAs (M=128, N=64, K=16) for S -- A
// from TMEM or shared memory -- and 4 MMAs (M=128, N=256, K=16) for P.V_v with A =
// P in TMEM.  Online softmax in base 2 with lazy rescaling (O and l are
// rescaled only when the running max grows by more than 2^8).
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
constexpr int kGatherThreads = 192;    // two groups of 96, one per KV stage
constexpr int kGroupThreads = 96;
constexpr int kMmaWarp = 10;

constexpr int kStages = 2;
constexpr int kRegions = 9;                              // 64-dim regions of a 576-dim row
constexpr uint32_t kQsRegions = 5;                       // query dims 256..575 in smem
constexpr uint32_t kQsBytes = kQsRegions * 16384;        // 128 rows x 128 B per region
constexpr uint32_t kStageBytes = kRegions * 8192;        // 64 rows x 128 B per region
constexpr uint32_t kOffQs = 0;
constexpr uint32_t kOffKV = kOffQs + kQsBytes;
constexpr uint32_t kOffFlag = kOffKV + kStages * kStageBytes;   // [stage][64] validity bytes
constexpr uint32_t kOffScale = kOffFlag + kStages * 64;         // [stage][64] fp32 kv scale
constexpr uint32_t kOffSlot = kOffScale + kStages * 256;       // [stage][64] int slot
constexpr uint32_t kOffBar = kOffSlot + kStages * 256;
constexpr uint32_t kNumBars = 16;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // 256 output columns
constexpr uint32_t kColS = 256;    // two 64-column buffers: S_j (fp32), then P_j (fp16,
                                   // 32 columns) over it
constexpr uint32_t kColQ = 384;    // 128 columns = query dims 0..255 as bf16 pairs
constexpr int kQtSteps = 16;       // K-steps of 16 dims with A in TMEM
constexpr int kQtChunks = 32;      // 16-byte query chunks held in TMEM

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
    __half* o_part;            // split partials o / l in fp16 (|o| <= max |v|)
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

__device__ __forceinline__ void group_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint4 lds16(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr) : "memory");
    return v;
}

__device__ __forceinline__ void sts16(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                 ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Two e4m3 codes (low byte first) -> two bf16 (exact: every e4m3 value is a bf16;
// the hardware conversion goes through fp16, which also holds every e4m3 value).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(saddr), "l"(gptr), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Two floats -> fp16x2 (lo in the low half), round to nearest, saturating at 65504.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight bf16 -> eight fp16: exact for magnitudes in [2^-14, 65504] (larger ones
// saturate; smaller ones keep an absolute precision of 2^-24).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 a) {
    auto cv = [](uint32_t v) {
        return pack_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
    };
    return make_uint4(cv(a.x), cv(a.y), cv(a.z), cv(a.w));
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
mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(base);
    uint8_t* vflag = base + kOffFlag;
    float* colscale = reinterpret_cast<float*>(base + kOffScale);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBar);
    uint64_t* kvfull = bars + 0;    // [2] gather -> MMA / softmax     (192 arrivals)
    uint64_t* kvempty = bars + 2;   // [2] PV done -> gather           (commit)
    uint64_t* sfull = bars + 4;     // [2] S_j ready in buffer j%2     (commit)
    uint64_t* pfull = bars + 6;     // [2] P_j (and any O rescale) ready (128)
    uint64_t* pvdone = bars + 8;    // [2] P_j.V finished; buffer j%2 free (commit)
    uint64_t* qfull = bars + 10;    // query in TMEM + shared memory   (128)
    uint64_t* qload = bars + 11;    // query tiles landed (TMA bytes)
    uint64_t* vconv = bars + 12;    // [2] V_v of stage s converted to fp16 (96)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    pdl_trigger();
    const int vh = blockIdx.x & 1;                   // which half of the V columns
    const int cid = blockIdx.x >> 1;
    const int t = cid / p.nsplit, split = cid % p.nsplit;
    const RowInfo ri = row_info(p.bv, t, threadIdx.x == 0 ? p.check : nullptr);
    const int i0 = split * p.chunk, i1 = min(p.k, i0 + p.chunk);
    __shared__ int s_skip;

    if (threadIdx.x == 0) {
        s_skip = timed_out_before(p.check) ? 1 : 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&kvfull[i], kGroupThreads);
            mbar_init(&kvempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            mbar_init(&pfull[i], 128);
            mbar_init(&pvdone[i], 1);
        }
        mbar_init(qfull, 128);
        mbar_init(qload, 1);
        mbar_init(&vconv[0], kGroupThreads);
        mbar_init(&vconv[1], kGroupThreads);
        fence_barrier_init();
        // the query row block [128 heads][576] as nine 64-dim swizzled tiles: dims
        // 256..575 straight into their shared-memory home, dims 0..255 into KV stage 0
        // for the softmax threads to move into TMEM
        if (ri.ok) {
            prefetch_tmap(&tm_q);
            mbar_arrive_expect_tx(qload, 9 * 16384);
            for (int r = 0; r < 9; ++r)
                tma_load_2d(base + (r < 4 ? kOffKV + r * 16384 : kOffQs + (r - 4) * 16384), &tm_q,
                            64 * r, t * kHeads, qload);
        }
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
        // Group g (warps 4-6 or 7-9) fills KV stage g with tiles g, g+2, g+4, ...:
        // the two groups' copies of consecutive tiles overlap.  Thread r < 64 of a
        // group owns row r: it runs the index -> slot pipeline for the group's
        // upcoming tiles and publishes the tile's slots in shared memory; then every
        // warp copies whole 128-byte lines (8 lanes per line, 4 rows per instruction).
        const int gt = threadIdx.x - kGatherWarp0 * 32;     // 0..191
        const int grp = gt / kGroupThreads, gl = gt % kGroupThreads;
        const int gw = gl >> 5, lane = gl & 31;
        constexpr int kRowBytes = kFp8 ? 576 : 1152;
        int* srow = reinterpret_cast<int*>(base + kOffSlot) + grp * 64;
        const long long seq_base = (long long)ri.b * p.st_stride;
        auto fetch_idx = [&](int j) -> int {
            const int i = i0 + j * kTile + gl;
            return (gl < kTile && j < n_tiles && i < i1) ? __ldg(p.idx + (long long)t * p.k + i) : -1;
        };
        // Slot-table entry for index s, or a sentinel for a skipped entry / an index
        // past the query position (table entries are checked separately).
        constexpr int kSkip = INT_MIN, kPastPos = INT_MIN + 1;
        auto fetch_slot = [&](int s) -> int {
            if (s < 0) return kSkip;
            if (s > ri.pos) return kPastPos;
            return __ldg(p.slot_table + seq_base + s);
        };
        auto check_slot = [&](int raw) -> int {   // -1 for skipped / bad entries
            if (raw == kSkip) return -1;
            if (raw == kPastPos || raw < 0 || (long long)raw >= p.num_slots) {
                report(p.check, raw == kPastPos ? kCheckBadIndex : kCheckBadPage);
                return -1;
            }
            return raw;
        };
        // pipeline over the group's own tiles: slots of tiles j and j+2, the table
        // entry of tile j+4 and the index of tile j+6 are in flight at tile j
        int sl_cur = -1, sl_next = -1, raw_n2 = kSkip, idx_n3 = -1;
        pdl_wait();                                  // the selection may come from the previous kernel
        if (grp < n_tiles) {
            const int x0 = fetch_idx(grp), x1 = fetch_idx(grp + 2), x2 = fetch_idx(grp + 4);
            idx_n3 = fetch_idx(grp + 6);
            const int r0 = fetch_slot(x0), r1 = fetch_slot(x1);
            raw_n2 = fetch_slot(x2);
            sl_cur = check_slot(r0);
            sl_next = check_slot(r1);
        }
        const int stage = grp;
        const uint32_t st = sb + kOffKV + stage * kStageBytes;
        if (grp == 0 && n_tiles > 0) mbar_wait_warp(qfull, 0, p.check);   // stage 0 held query tiles
        for (int j = grp; j < n_tiles; j += kStages) {
            if (sl_next >= 0)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                             ::"l"(p.kv + (long long)sl_next * kRowBytes), "r"(kRowBytes) : "memory");
            if (!mbar_wait_warp(&kvempty[stage], ((j / kStages) & 1) ^ 1, p.check)) break;
            if (gl < kTile) {
                srow[gl] = sl_cur;
                vflag[stage * 64 + gl] = sl_cur >= 0 ? 1 : 0;
                colscale[stage * 64 + gl] =
                    (kFp8 && sl_cur >= 0 && p.kv_scale) ? __ldg(p.kv_scale + sl_cur) : 1.0f;
            }
            group_sync(1 + grp, kGroupThreads);
            if constexpr (!kFp8) {
                // 64 rows x 9 regions of 128 bytes = 144 units of 4 rows; warp gw takes
                // units gw, gw+3, ...; a skipped or bad row becomes zeros (score masked)
                const int chunk = lane & 7;
#pragma unroll 8
                for (int u = gw; u < 144; u += 3) {
                    const int rg = u / 9, region = u - rg * 9;
                    const int row = 4 * rg + (lane >> 3);
                    const int sl = srow[row];
                    const uint8_t* src = p.kv + (long long)(sl < 0 ? 0 : sl) * 1152 + region * 128 + chunk * 16;
                    cp_async16(st + region * 8192 + sw128(row, chunk), src, sl >= 0 ? 16u : 0u);
                }
            } else {
                // 64 rows x 36 pieces of 16 e4m3 codes; thread gl takes pieces gl + 96 i
                uint4 v[24];
#pragma unroll
                for (int i = 0; i < 24; ++i) {
                    const int q = gl + kGroupThreads * i, row = q / 36, pc = q - row * 36;
                    const int sl = srow[row];
                    v[i] = sl >= 0 ? ldg16(p.kv + (long long)sl * 576 + pc * 16) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int i = 0; i < 24; ++i) {
                    const int q = gl + kGroupThreads * i, row = q / 36, pc = q - row * 36;
                    const int g = 2 * pc;                       // first of the two bf16 chunks
                    const uint4 a = v[i];
                    const uint4 lo = make_uint4(e4m3x2_to_bf16x2(a.x & 0xFFFF), e4m3x2_to_bf16x2(a.x >> 16),
                                                e4m3x2_to_bf16x2(a.y & 0xFFFF), e4m3x2_to_bf16x2(a.y >> 16));
                    const uint4 hi = make_uint4(e4m3x2_to_bf16x2(a.z & 0xFFFF), e4m3x2_to_bf16x2(a.z >> 16),
                                                e4m3x2_to_bf16x2(a.w & 0xFFFF), e4m3x2_to_bf16x2(a.w >> 16));
                    sts16(st + (g >> 3) * 8192 + sw128(row, g & 7), lo);
                    sts16(st + ((g + 1) >> 3) * 8192 + sw128(row, (g + 1) & 7), hi);
                }
            }
            // advance the pipeline (independent loads, issued before waiting on the copies)
            const int nxt = check_slot(raw_n2);     // loaded one round ago
            raw_n2 = fetch_slot(idx_n3);             // index loaded one round ago
            idx_n3 = fetch_idx(j + 8);
            if constexpr (!kFp8) cp_async_commit_wait_all();
            fence_proxy_async_smem();
            mbar_arrive(&kvfull[stage]);
            // once S_j has read the bf16 rows, convert this CTA's V columns in place to
            // fp16 for P.V (P is fp16: bf16 P keeps too few bits, see above)
            if (!mbar_wait_warp(&sfull[stage], (j >> 1) & 1, p.check)) break;
            tc_fence_after();
            const uint32_t vb = st + vh * 4 * 8192;
#pragma unroll 4
            for (int q = gl; q < 4 * 512; q += kGroupThreads) {
                const uint32_t a = vb + q * 16;
                sts16(a, bf16x8_to_f16x8(lds16(a)));
            }
            fence_proxy_async_smem();
            mbar_arrive(&vconv[stage]);
            sl_cur = sl_next;
            sl_next = nxt;
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (elect_one() && n_tiles > 0) {
            bool alive = mbar_wait(qfull, 0, p.check);
            tc_fence_after();
            const uint32_t idesc_qk = instr_desc(1, 1, 0, 0, kTile, kHeads);   // bf16 x bf16
            const uint32_t idesc_pv = instr_desc(0, 0, 0, 1, 256, kHeads);   // fp16 P x fp16 V
            const uint32_t qs = sb + kOffQs;
            // S_j = Q . KV_j^T (36 K-steps of 16: dims 0..255 with A in TMEM, the rest
            // with A in shared memory)
            auto issue_qk = [&](int jt) {
                const uint32_t kva = sb + kOffKV + (jt % kStages) * kStageBytes;
                const uint32_t sbuf = tmem + kColS + 64 * (jt & 1);
#pragma unroll
                for (int s = 0; s < 36; ++s) {
                    const uint64_t bdesc =
                        smem_desc(kva + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024, kLayoutSw128);
                    if (s < kQtSteps)
                        mma_f16_ts(sbuf, tmem + kColQ + 8 * s, bdesc, idesc_qk, s > 0 ? 1u : 0u);
                    else
                        mma_f16(sbuf,
                                smem_desc(qs + ((s - kQtSteps) >> 2) * 16384 + (s & 3) * 32, 16, 1024,
                                          kLayoutSw128),
                                bdesc, idesc_qk, 1u);
                }
                mma_commit(&sfull[jt & 1]);
            };
            // O_v += P . V_v (fp16 operands; K = 64 tokens in four steps of 16)
            auto issue_pv = [&](int jt) {
                const int stage = jt % kStages;
                const uint32_t va = sb + kOffKV + stage * kStageBytes + vh * 4 * 8192;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16_ts(tmem + kColO, tmem + kColS + 64 * (jt & 1) + 8 * kk,
                               smem_desc(va + kk * 2048, 8192, 1024, kLayoutSw128), idesc_pv,
                               (jt > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&kvempty[stage]);
                mma_commit(&pvdone[jt & 1]);
            };
            // Round j issues S_j and P_{j-1}.V in whichever order their inputs arrive
            // (P.V first when both are ready: it frees a KV stage for the gather).
            // S_j reuses buffer j%2 once P_{j-2}.V has read the P stored there.
            for (int j = 0; alive && j <= n_tiles; ++j) {
                bool qk = j < n_tiles, pv = j >= 1;
                const uint32_t kv_par = (j / kStages) & 1;
                const long long t0 = clock64();
                while (qk || pv) {
                    if (pv && mbar_test(&pfull[(j - 1) & 1], ((j - 1) >> 1) & 1) &&
                        mbar_test(&vconv[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
                        tc_fence_after();
                        issue_pv(j - 1);
                        pv = false;
                    } else if (qk && mbar_test(&kvfull[j % kStages], kv_par) &&
                               (j < 2 || mbar_test(&pvdone[j & 1], ((j - 2) >> 1) & 1))) {
                        tc_fence_after();
                        issue_qk(j);
                        qk = false;
                    } else if (clock64() - t0 > kWaitLimitCycles) {
                        report(p.check, kCheckTimeout);
                        alive = false;
                        break;
                    }
                }
            }
        }
    } else {
        // ============================================================ softmax
        const int h = threadIdx.x;                       // head == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        {   // query row h, dims 0..255: from the staging tiles in KV stage 0 into TMEM
            // (waited for whenever issued: no copy may still be in flight at exit)
            if (ri.ok) mbar_wait_warp(qload, 0, p.check);
#pragma unroll
            for (int g = 0; g < kQtChunks; g += 2) {
                uint4 a = make_uint4(0, 0, 0, 0), b = a;
                if (ri.ok) {
                    const uint32_t src = sb + kOffKV + (g >> 3) * 16384;
                    a = lds16(src + sw128(h, g & 7));
                    b = lds16(src + sw128(h, (g + 1) & 7));
                }
                tmem_st8(lane_base + kColQ + 4 * g, a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(qfull);                         // also: KV stage 0 may be refilled
        }
        float m_run = -INFINITY, l_run = 0.f;
        bool alive = true;
        for (int j = 0; alive && j < n_tiles; ++j) {
            const int stage = j % kStages;
            float x[64];
            const uint32_t sb_col = kColS + 64 * (j & 1);  // S_j, then P_j
            {   // ---- scores of tile j
                if (!mbar_wait_warp(&sfull[j & 1], (j >> 1) & 1, p.check)) { alive = false; break; }
                tc_fence_after();
                uint32_t a[32], c[32];
                tmem_ld32(lane_base + sb_col, a);
                tmem_ld32(lane_base + sb_col + 32, c);
                tmem_ld_wait();
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
            // ---- O may be rescaled only once the previous PV has finished
            if (warp_rescale) {
                if (!mbar_wait_warp(&pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, p.check)) { alive = false; break; }
                tc_fence_after();
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
            tmem_st32(lane_base + sb_col, pk);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&pfull[j & 1]);
        }
        // ---- epilogue: O_v / l and lse (after the predecessor kernel: an earlier kernel
        // of the stream may still read the output or partial buffers)
        pdl_wait();
        const bool have = alive && n_tiles > 0 &&
                          mbar_wait_warp(&pvdone[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.check);
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
            uint4* orow = reinterpret_cast<uint4*>(p.o_part + pb * 512 + vh * 256);
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t o[32];
                if (have) {
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint4 w = make_uint4(0u, 0u, 0u, 0u);
                    if (have) {
                        w.x = pack_f16(__uint_as_float(o[8 * q8 + 0]) * inv, __uint_as_float(o[8 * q8 + 1]) * inv);
                        w.y = pack_f16(__uint_as_float(o[8 * q8 + 2]) * inv, __uint_as_float(o[8 * q8 + 3]) * inv);
                        w.z = pack_f16(__uint_as_float(o[8 * q8 + 4]) * inv, __uint_as_float(o[8 * q8 + 5]) * inv);
                        w.w = pack_f16(__uint_as_float(o[8 * q8 + 6]) * inv, __uint_as_float(o[8 * q8 + 7]) * inv);
                    }
                    orow[cc * 4 + q8] = w;
                }
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
                          const int* idx, int k, int nsplit, void* out, float* lse, void* o_part,
                          float* lse_part, int* check, cudaStream_t st, bool pdl) {
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
    p.o_part = static_cast<__half*>(o_part);
    p.lse_part = lse_part;
    p.check = check;
    CUtensorMap tm_q;
    cudaError_t me = make_tensor_map_2d(&tm_q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 576,
                                        (unsigned long long)bv.total_q * kHeads, 1152, 64, kHeads,
                                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (me != cudaSuccess) return me;
    const bool fp8 = kv.dtype == kE4M3;
    auto kern = fp8 ? mla_tc_kernel<true> : mla_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * bv.total_q * nsplit);
    e = launch_kernel(kern, grid, dim3(kThreads), kSmemBytes, st, pdl, tm_q, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dsa
