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
// Why a CTA pair.  The fp32 output tile O (128 heads x 512) fills all 512 TMEM
// columns of an SM, leaving no room for the score tile.  So a 2-CTA cluster works
// on one (query, split): rank r owns V columns [256r, 256r+256) and the 288 dims
// D_r = [256r, 256r+256) u [512+32r, 512+32r+32) of the QK contraction.  Each rank
// gathers only D_r of every selected row (no byte is fetched twice), computes the
// partial scores S_r = Q[:, D_r] . KV[:, D_r]^T on tcgen05, and the two partial
// tiles are swapped through distributed shared memory.  Both ranks add them
// (S_0 + S_1 == S_1 + S_0 bit for bit), so both run an identical online softmax,
// write the same P tile, and accumulate O[:, 256r:256r+256] += P . V_r.
//
// Roles (288 threads per CTA): warps 0-3 = softmax (thread = head = TMEM lane),
// warps 4-7 = gather (2 threads per selected row, loads issued one tile ahead),
// warp 8 = TMEM owner and MMA issuer.  The MMAs run on fp16 operands: e4m3 and
// bf16 values convert to fp16 exactly (bf16 magnitudes above 65504 saturate), and
// the probabilities P get 11 significant bits instead of bf16's 8.
// Per 64-row tile: 18 MMAs (M=128, N=64, K=16) for S_r, 4 MMAs (M=128, N=256,
// K=16) for P.V_r.  Online softmax in base 2 with lazy rescaling: O and l are only
// rescaled when the running max grows by more than 2^8.
//
// Shared memory (one CTA per SM): Q_r 72 KB, 2 KV stages x 36 KB, one exchange
// buffer of 32 KB, 2 P buffers x 16 KB.  Tiles of 64 dims are 128-byte swizzled K-major; the
// 32 rope dims of a rank use the no-swizzle core-matrix layout.
#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kHeads = 128;
constexpr int kTile = 64;
constexpr int kThreads = 288;
constexpr int kGatherWarp0 = 4;
constexpr int kMmaWarp = 8;

constexpr uint32_t kQBytes = 4 * 16384 + 8192;
constexpr uint32_t kStageBytes = 4 * 8192 + 4096;
constexpr uint32_t kXBytes = kHeads * kTile * 4;
constexpr uint32_t kPBytes = kHeads * kTile * 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kOffQ + kQBytes;
constexpr uint32_t kOffX = kOffKV + 2 * kStageBytes;
constexpr uint32_t kOffP = kOffX + kXBytes;             // [2] P tiles
constexpr uint32_t kOffFlag = kOffP + 2 * kPBytes;      // [2][64] validity bytes
constexpr uint32_t kOffScale = kOffFlag + 128;          // [2][64] fp32 per-row kv scale
constexpr uint32_t kOffBar = kOffScale + 512;
constexpr uint32_t kSmemBytes = kOffBar + 16 * 8 + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // two 64-column score buffers
constexpr uint32_t kColO = 256;    // 256 output columns

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
// Byte offset of 16-byte chunk c (0..3) of row r in a no-swizzle tile of 64-byte
// rows: 8x16-byte core matrices, K-adjacent ones 128 B apart, 8-row groups 512 B.
__device__ __forceinline__ uint32_t il64(int r, int c) {
    return (uint32_t)((r >> 3) * 512 + c * 128 + ((r & 7) << 4));
}
// Rank-local bf16 chunk g (0..35) of a row: chunk index in the 72-chunk global row.
__device__ __forceinline__ int global_chunk(int rank, int g) {
    return g < 32 ? 32 * rank + g : 64 + 4 * rank + (g - 32);
}
// Shared-memory offset of local chunk g of `row` (region stride rs, rope region r4).
__device__ __forceinline__ uint32_t local_off(int row, int g, uint32_t rs, uint32_t r4) {
    return g < 32 ? (uint32_t)(g >> 3) * rs + sw128(row, g & 7) : r4 + il64(row, g - 32);
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

__device__ __forceinline__ float4 lds16f(uint32_t saddr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(saddr));
    return v;
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_tc_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(base);
    uint8_t* vflag = base + kOffFlag;
    float* colscale = reinterpret_cast<float*>(base + kOffScale);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBar);
    uint64_t* kvfull = bars + 0;    // [2] gather -> MMA / softmax     (128 arrivals)
    uint64_t* kvempty = bars + 2;   // [2] PV done -> gather           (commit)
    uint64_t* sfull = bars + 4;     // [2] S_r ready -> softmax        (commit)
    uint64_t* sempty = bars + 6;    // [2] S_r read -> MMA             (128)
    uint64_t* xfull = bars + 8;     // peer's partial landed           (4 remote, one per warp)
    uint64_t* xempty = bars + 9;    // peer consumed our partial       (4 remote)
    uint64_t* pfull = bars + 10;    // [2] P (and any O rescale) ready (128)
    uint64_t* pvdone = bars + 12;   // [2] PV of that P buffer done    (commit)
    uint64_t* qfull = bars + 14;    // Q_r in place                    (128)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);

    const int warp = threadIdx.x >> 5;
    const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
    const int cid = blockIdx.x >> 1;
    const int t = cid / p.nsplit, split = cid % p.nsplit;
    const RowInfo ri = row_info(p.bv, t, threadIdx.x == 0 ? p.check : nullptr);
    const int i0 = split * p.chunk, i1 = min(p.k, i0 + p.chunk);
    __shared__ int s_skip;
    if (threadIdx.x == 0) s_skip = timed_out_before(p.check) ? 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kvfull[i], 128);
            mbar_init(&kvempty[i], 1);
            mbar_init(&sfull[i], 1);
            mbar_init(&sempty[i], 128);
            mbar_init(&pfull[i], 128);
            mbar_init(&pvdone[i], 1);
        }
        mbar_init(xfull, 4);
        mbar_init(xempty, 4);
        mbar_init(qfull, 128);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // the peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = (ri.ok && i1 > i0 && !s_skip) ? (i1 - i0 + kTile - 1) / kTile : 0;

    if (warp >= kGatherWarp0 && warp < kMmaWarp) {
        // ============================================================ gather
        const int gt = threadIdx.x - kGatherWarp0 * 32;     // 0..127
        {   // Q_r: head gt, its 36 rank-local chunks, as fp16
            const uint4* qrow = p.q + ((long long)t * kHeads + gt) * 72;
#pragma unroll
            for (int g0 = 0; g0 < 36; g0 += 18) {
                uint4 qv[18];
#pragma unroll
                for (int g = 0; g < 18; ++g)
                    qv[g] = ri.ok ? ldg16(qrow + global_chunk(rank, g0 + g)) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int g = 0; g < 18; ++g)
                    sts16(sb + kOffQ + local_off(gt, g0 + g, 16384, 65536), bf16x8_to_f16x8(qv[g]));
            }
            fence_proxy_async_smem();
            mbar_arrive(qfull);
        }
        const int c = gt >> 1, half = gt & 1;      // selected row of the tile, which half
        constexpr int kN = kFp8 ? 9 : 18;          // 16-byte global loads per thread per tile
        uint4 v[kN];
        bool valid = false;
        float scale = 0.f;
        auto load = [&](int j) {
            const int i = i0 + j * kTile + c;
            const int s = i < i1 ? __ldg(p.idx + (long long)t * p.k + i) : -1;
            valid = s >= 0 && s <= ri.pos;
            if (s > ri.pos && half == 0) report(p.check, kCheckBadIndex);
            long long slot = 0;
            if (valid) {
                slot = __ldg(p.slot_table + (long long)ri.b * p.st_stride + s);
                if (slot < 0 || slot >= p.num_slots) {
                    if (half == 0) report(p.check, kCheckBadPage);
                    valid = false;
                }
            }
            scale = (valid && kFp8 && p.kv_scale) ? __ldg(p.kv_scale + slot) : 1.0f;
            if constexpr (kFp8) {
                const uint8_t* row = p.kv + slot * 576;
#pragma unroll
                for (int u = 0; u < kN; ++u) {
                    const int gg = half * 9 + u;
                    const int off = gg < 16 ? 256 * (int)rank + 16 * gg : 512 + 32 * (int)rank + 16 * (gg - 16);
                    v[u] = valid ? ldg16(row + off) : make_uint4(0, 0, 0, 0);
                }
            } else {
                const uint4* row = reinterpret_cast<const uint4*>(p.kv + slot * 1152);
#pragma unroll
                for (int u = 0; u < kN; ++u)
                    v[u] = valid ? ldg16(row + global_chunk(rank, half * 18 + u)) : make_uint4(0, 0, 0, 0);
            }
        };
        if (n_tiles > 0) load(0);
        for (int j = 0; j < n_tiles; ++j) {
            const int stage = j & 1;
            if (!mbar_wait(&kvempty[stage], ((j >> 1) & 1) ^ 1, p.check)) break;
            const uint32_t st = sb + kOffKV + stage * kStageBytes;
            if constexpr (kFp8) {
#pragma unroll
                for (int u = 0; u < kN; ++u) {
                    const int gg = half * 9 + u;
                    const uint4 a = v[u];
                    const uint4 lo = make_uint4(e4m3x2_to_f16x2(a.x & 0xFFFF), e4m3x2_to_f16x2(a.x >> 16),
                                                e4m3x2_to_f16x2(a.y & 0xFFFF), e4m3x2_to_f16x2(a.y >> 16));
                    const uint4 hi = make_uint4(e4m3x2_to_f16x2(a.z & 0xFFFF), e4m3x2_to_f16x2(a.z >> 16),
                                                e4m3x2_to_f16x2(a.w & 0xFFFF), e4m3x2_to_f16x2(a.w >> 16));
                    sts16(st + local_off(c, 2 * gg, 8192, 32768), lo);
                    sts16(st + local_off(c, 2 * gg + 1, 8192, 32768), hi);
                }
            } else {
#pragma unroll
                for (int u = 0; u < kN; ++u)
                    sts16(st + local_off(c, half * 18 + u, 8192, 32768), bf16x8_to_f16x8(v[u]));
            }
            if (half == 0) {
                vflag[stage * 64 + c] = valid ? 1 : 0;
                colscale[stage * 64 + c] = scale;
            }
            fence_proxy_async_smem();
            mbar_arrive(&kvfull[stage]);
            if (j + 1 < n_tiles) load(j + 1);
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (elect_one() && n_tiles > 0) {
            bool alive = mbar_wait(qfull, 0, p.check);
            tc_fence_after();
            const uint32_t idesc_qk = instr_desc(0, 0, 0, 0, kTile, kHeads);   // fp16 x fp16
            const uint32_t idesc_pv = instr_desc(0, 0, 0, 1, 256, kHeads);
            const uint32_t qa = sb + kOffQ;
            const uint32_t pa = sb + kOffP;
            for (int j = 0; alive && j <= n_tiles; ++j) {
                if (j < n_tiles) {
                    const int stage = j & 1, buf = j & 1;
                    if (!mbar_wait(&kvfull[stage], (j >> 1) & 1, p.check)) break;
                    if (!mbar_wait(&sempty[buf], ((j >> 1) & 1) ^ 1, p.check)) break;
                    tc_fence_after();
                    const uint32_t kva = sb + kOffKV + stage * kStageBytes;
                    const uint32_t d = tmem + kColS + buf * kTile;
                    uint32_t acc = 0;
#pragma unroll
                    for (int reg = 0; reg < 4; ++reg) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            mma_f16(d, smem_desc(qa + reg * 16384 + kk * 32, 16, 1024, kLayoutSw128),
                                    smem_desc(kva + reg * 8192 + kk * 32, 16, 1024, kLayoutSw128),
                                    idesc_qk, acc);
                            acc = 1;
                        }
                    }
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        mma_f16(d, smem_desc(qa + 65536 + kk * 256, 128, 512, kLayoutNone),
                                smem_desc(kva + 32768 + kk * 256, 128, 512, kLayoutNone), idesc_qk, 1);
                    mma_commit(&sfull[buf]);
                }
                if (j >= 1) {
                    const int jj = j - 1, stage = jj & 1;
                    if (!mbar_wait(&pfull[jj & 1], (jj >> 1) & 1, p.check)) break;
                    tc_fence_after();
                    const uint32_t kva = sb + kOffKV + stage * kStageBytes;
                    const uint32_t pb = pa + (jj & 1) * kPBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + kColO, smem_desc(pb + kk * 32, 16, 1024, kLayoutSw128),
                                smem_desc(kva + kk * 2048, 8192, 1024, kLayoutSw128), idesc_pv,
                                (jj > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&kvempty[stage]);
                    mma_commit(&pvdone[jj & 1]);
                }
            }
        }
    } else {
        // ============================================================ softmax
        const int h = threadIdx.x;                       // head == TMEM lane
        const int lane = threadIdx.x & 31;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t xa = sb + kOffX;
        const uint32_t peer_x = mapa(xa, peer);
        const uint32_t peer_xfull = mapa(smem_u32(xfull), peer);   // the peer's own barriers
        const uint32_t peer_xempty = mapa(smem_u32(xempty), peer);
        float m_run = -INFINITY, l_run = 0.f;
        bool alive = true;
        for (int j = 0; alive && j < n_tiles; ++j) {
            const int buf = j & 1, u = j >> 1;
            // ---- this rank's partial scores
            if (!mbar_wait(&sfull[buf], u & 1, p.check)) { alive = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            {
                uint32_t a[32], b[32];
                tmem_ld32(lane_base + kColS + buf * kTile, a);
                tmem_ld32(lane_base + kColS + buf * kTile + 32, b);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    sr[i] = a[i];
                    sr[32 + i] = b[i];
                }
            }
            tc_fence_before();
            mbar_arrive(&sempty[buf]);
            // ---- swap partial tiles with the peer rank (one exchange buffer each)
            if (j >= 1 && !mbar_wait_cluster(xempty, (j - 1) & 1, p.check)) { alive = false; break; }
            const uint32_t xrow = (uint32_t)h * 256;
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4)
                st_cluster_v4(peer_x + xrow + ((c4 ^ (h & 7)) << 4), __uint_as_float(sr[4 * c4]),
                              __uint_as_float(sr[4 * c4 + 1]), __uint_as_float(sr[4 * c4 + 2]),
                              __uint_as_float(sr[4 * c4 + 3]));
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_xfull);
            if (!mbar_wait_cluster(xfull, j & 1, p.check)) { alive = false; break; }
            float x[64];
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                const float4 o = lds16f(xa + xrow + ((c4 ^ (h & 7)) << 4));
                x[4 * c4 + 0] = __uint_as_float(sr[4 * c4 + 0]) + o.x;
                x[4 * c4 + 1] = __uint_as_float(sr[4 * c4 + 1]) + o.y;
                x[4 * c4 + 2] = __uint_as_float(sr[4 * c4 + 2]) + o.z;
                x[4 * c4 + 3] = __uint_as_float(sr[4 * c4 + 3]) + o.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_xempty);
            // ---- online softmax (base 2)
            if (!mbar_wait(&kvfull[buf], u & 1, p.check)) { alive = false; break; }
            const uint8_t* fl = vflag + buf * 64;
            const float* cs = colscale + buf * 64;
            float m_tile = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float sc = kFp8 ? p.sc_log2 * cs[i] : p.sc_log2;
                x[i] = fl[i] ? x[i] * sc : -INFINITY;
                m_tile = fmaxf(m_tile, x[i]);
            }
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + 8.0f;           // rescale only past 2^8 growth
            const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
            if (need) m_run = m_new;
            const bool warp_rescale = __any_sync(0xffffffffu, need) && j > 0;
            float lsum = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
                const float e0 = (x[i] == -INFINITY) ? 0.f : fast_exp2(x[i] - m_run);
                const float e1 = (x[i + 1] == -INFINITY) ? 0.f : fast_exp2(x[i + 1] - m_run);
                lsum += e0 + e1;
                pk[i / 2] = kFp8 ? pack_f16(e0 * cs[i], e1 * cs[i + 1]) : pack_f16(e0, e1);
            }
            l_run = l_run * alpha + lsum;
            // ---- O may be rescaled once PV(j-1) is done; P[j&1] is free once PV(j-2) is
            if (warp_rescale && !mbar_wait(&pvdone[(j - 1) & 1], ((j - 1) >> 1) & 1, p.check)) {
                alive = false;
                break;
            }
            if (j >= 2 && !mbar_wait(&pvdone[j & 1], ((j - 2) >> 1) & 1, p.check)) { alive = false; break; }
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
                tmem_st_wait();
            }
            const uint32_t prow = sb + kOffP + (j & 1) * kPBytes;
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                sts16(prow + sw128(h, c8), make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]));
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&pfull[j & 1]);
        }
        // ---- epilogue: O_r / l and lse
        const bool have = alive && n_tiles > 0 &&
                          mbar_wait(&pvdone[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.check);
        tc_fence_after();
        const float inv = (have && l_run > 0.f) ? 1.0f / l_run : 0.f;
        const float lse_v = (have && l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994531f
                                                  : -INFINITY;
        if (p.nsplit == 1) {
            uint4* orow = reinterpret_cast<uint4*>(p.out + ((long long)t * kHeads + h) * 512 + rank * 256);
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
            if (rank == 0 && p.lse) p.lse[(long long)t * kHeads + h] = lse_v;
        } else {
            const long long pb = ((long long)t * p.nsplit + split) * kHeads + h;
            float4* orow = reinterpret_cast<float4*>(p.o_part + pb * 512 + rank * 256);
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
            if (rank == 0) p.lse_part[pb] = lse_v;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no remote shared-memory traffic after this point
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
