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
// One (query, split) runs on a pair of SMs: a cluster of two CTAs whose tensor cores
// act as one (tcgen05 cta_group::2, issued by the even CTA).  The fp32 output tile O
// (128 heads x 512) needs all 512 TMEM columns of one SM, so it is split by heads:
// CTA r holds heads [64r, 64r+64).  A tile of 64 selected keys is split by keys: CTA r
// gathers keys [32r, 32r+32) of the tile, whole rows, into its shared memory, and the
// paired MMA  S = Q . K^T  (M = 128 heads over the pair, N = 64 keys, K = 576) reads each
// CTA's query rows and both CTAs' key halves, so every selected row enters one SM for
// the scores.  For O += P . V (M = 128, N = 2 x 256 V dims, K = 64 keys) each CTA
// supplies half of the N columns -- V dims {128r..128r+127, 256+128r..+127} -- for all
// 64 keys, so it also gathers those 512 bytes of the peer's 32 rows (1.44x the
// algorithmic bytes into the SMs, against 2x when each SM of a pair gathers every row).
//
// Operands are fp16: the query and the rows are converted on the way into shared memory
// (bf16 -> fp16 is exact for magnitudes in [2^-14, 65504]; smaller ones keep an
// absolute precision of 2^-24, larger or non-finite ones saturate and are reported as
// DSA_CHECK_FP16_RANGE; e4m3 -> fp16 is always exact), so S and P.V take the same
// operands and P keeps 11 significant bits (bf16 P loses too many for rows dominated by
// a few large values).  FP8 rows keep their codes; the per-row scale multiplies S and P
// in fp32.
//
// Tensor memory, per CTA (both CTAs allocate the same 512 columns; the paired MMA
// writes each CTA's rows into its own TMEM): O at columns 0..255 (lanes 0-63 hold dims
// {0..127, 256..383} of heads 0..63 of this CTA, lanes 64-127 dims {128..255,
// 384..511}); two score buffers of 32 columns (lanes 0-63: keys 0..31 of the tile,
// lanes 64-127: keys 32..63); query dims 0..383 at columns 320..511, each head's row
// held twice (lanes h and h+64), the A layout of a paired MMA with A in TMEM.  Query
// dims 384..575 stay in shared memory.
//
// Roles (416 threads per CTA): warps 0-3 = softmax (thread = TMEM lane: head h = lane %
// 64, key half lane / 64; the two threads of a head exchange row maxima through shared
// memory); warps 4-11 = gather, two groups of four warps, group g filling stage g with
// tiles g, g+2, ... (a stage = this CTA's 32 key rows, 36 KB, + the V block of all 64
// keys, 32 KB); warp 12 = TMEM owner and, in the even CTA, the MMA issuer.  Online
// softmax in base 2 with lazy rescaling (O and l are rescaled only when the running
// max grows by more than 2^8).
#include <climits>
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kHeads = 128;
constexpr int kTile = 64;                 // keys per tile (32 per CTA)
constexpr int kThreads = 416;
constexpr int kGatherWarp0 = 4;
constexpr int kMmaWarp = 12;
constexpr int kStages = 2;

constexpr uint32_t kQsBytes = 3 * 8192;                  // query dims 384..575, 64 rows
constexpr uint32_t kPBytes = 8192;                       // P: 64 heads x 64 keys fp16
constexpr uint32_t kSbufBytes = 9 * 4096;                // 32 rows x 9 regions of 64 dims
constexpr uint32_t kVblkBytes = 4 * 8192;                // 64 keys x 4 blocks of 64 V dims
constexpr uint32_t kStageBytes = kSbufBytes + kVblkBytes;
constexpr uint32_t kOffQs = 0;
constexpr uint32_t kOffP = kOffQs + kQsBytes;
constexpr uint32_t kOffStage = kOffP + 2 * kPBytes;
constexpr uint32_t kOffSlot = kOffStage + kStages * kStageBytes;   // [stage][64] int
constexpr uint32_t kOffScale = kOffSlot + kStages * 256;           // [stage][64] fp32
constexpr uint32_t kOffRed = kOffScale + kStages * 256;            // [3][128] fp32
constexpr uint32_t kOffRing = kOffRed + 3 * 128 * 4;              // [4][64] int slots
constexpr uint32_t kOffRingSc = kOffRing + 4 * 256;                // [4][64] fp32 scales
constexpr uint32_t kOffBar = kOffRingSc + 4 * 256;
constexpr uint32_t kNumBars = 23;
constexpr uint32_t kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kStageBytes % 1024 == 0 && kOffStage % 1024 == 0, "swizzled tiles need 1 KB alignment");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;             // 256 columns
constexpr uint32_t kColS = 256;           // 2 x 32 columns
constexpr uint32_t kColQ = 320;           // 192 columns: query dims 0..383 (fp16 pairs)
constexpr int kQtSteps = 24;              // K-steps of 16 dims with A in TMEM

struct Params {
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

// ---------------------------------------------------------------- pair plumbing
// Arrives on the barrier at the same offset in the even CTA of the cluster.  The
// arrive keeps the default release semantics at CTA scope: a cluster-scope release
// holds the issuing thread ~1000 cycles (measured), and what the even CTA consumes
// after the barrier is read through the async proxy (each writer has already fenced
// its shared-memory stores to that proxy) or is TMEM ordered by tcgen05 fences.
__device__ __forceinline__ void arrive_leader(uint64_t* bar) {
    const uint32_t a = mapa(smem_u32(bar), 0);
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}

// Phase test / bounded wait with cluster-scope acquire (barriers the peer arrives on).
__device__ __forceinline__ bool mbar_test_cl(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, int* check) {
    const long long t0 = clock64();
    while (!mbar_test_cl(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            report(check, kCheckTimeout);
            return false;
        }
    }
    return true;
}

// Paired MMAs (issued by one thread of the even CTA): D (+)= A . B with fp16 operands,
// A from shared memory or from TMEM.
__device__ __forceinline__ void mma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma2_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// Arrives on `bar` in both CTAs of the pair once the paired MMAs issued so far are done.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}"
        ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- conversions
// Two floats -> fp16x2 (lo in the low half), round to nearest, saturating at 65504.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight bf16 -> eight fp16 (see the head of the file).  `flag` collects bit 15 of each
// half of (|x| bits + 0x3880): set exactly when |x| >= 65536 (the bf16 neighbour above
// 65280), i.e. when the value lies beyond the fp16 range, or is inf / NaN.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, uint32_t& flag) {
    flag |= ((v & 0x7FFF7FFFu) + 0x38803880u) & 0x80008000u;
    return pack_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 a, uint32_t& flag) {
    return make_uint4(bf16x2_to_f16x2(a.x, flag), bf16x2_to_f16x2(a.y, flag),
                      bf16x2_to_f16x2(a.z, flag), bf16x2_to_f16x2(a.w, flag));
}

// Two e4m3 codes (low byte first) -> two fp16 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}
// 16 codes -> two 16-byte chunks of fp16.
__device__ __forceinline__ void e4m3x16_to_f16(uint4 a, uint4& lo, uint4& hi) {
    lo = make_uint4(e4m3x2_to_f16x2(a.x & 0xFFFF), e4m3x2_to_f16x2(a.x >> 16),
                    e4m3x2_to_f16x2(a.y & 0xFFFF), e4m3x2_to_f16x2(a.y >> 16));
    hi = make_uint4(e4m3x2_to_f16x2(a.z & 0xFFFF), e4m3x2_to_f16x2(a.z >> 16),
                    e4m3x2_to_f16x2(a.w & 0xFFFF), e4m3x2_to_f16x2(a.w >> 16));
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

// The 64-dim region that V block b (0..3) of CTA `rank` covers: dims
// {128r..128r+127, 256+128r..256+128r+127} = regions 2r, 2r+1, 4+2r, 5+2r.
__device__ __forceinline__ int vblock_region(int b, int rank) {
    return (b & 1) + 2 * rank + 4 * (b >> 1);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
mla_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(base);
    int* srow = reinterpret_cast<int*>(base + kOffSlot);
    float* kscale = reinterpret_cast<float*>(base + kOffScale);
    float* red = reinterpret_cast<float*>(base + kOffRed);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBar);
    uint64_t* full = bars + 0;      // [2] even CTA: stage gathered in both CTAs   (8 warps)
    uint64_t* meta = bars + 2;      // [2] this CTA's slots / scales of the stage  (4 warps)
    uint64_t* sfull = bars + 4;     // [2] S_j in TMEM buffer j%2                  (commit)
    uint64_t* pfull = bars + 6;     // [2] even CTA: P_j written, O rescaled       (8 warps)
    uint64_t* pvdone = bars + 8;    // [2] P_j.V done: P buffer j%2 free           (commit)
    uint64_t* sempty = bars + 10;   // [2] stage free                              (commit)
    uint64_t* qready = bars + 12;   // even CTA: queries in place in both CTAs     (8 warps)
    uint64_t* qfree = bars + 13;    // query staging (in stage 0) consumed         (4 warps)
    uint64_t* qload = bars + 14;    // query tiles landed (TMA bytes)
    uint64_t* mmadone = bars + 15;  // every paired MMA finished                   (commit)
    uint64_t* slots = bars + 16;    // [4] tile j's slots published in ring j%4    (2 warps)
    uint64_t* redfull = bars + 20;  // [2] row-max halves of tile j%2 written       (4 warps)
    uint64_t* lfull = bars + 22;    // the heads' partial sums written             (4 warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    int* s_skip = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    pdl_trigger();
    const int pair = blockIdx.x >> 1;
    const int t = pair / p.nsplit, split = pair % p.nsplit;
    const RowInfo ri = row_info(p.bv, t, (threadIdx.x == 0 && rank == 0) ? p.check : nullptr);
    const int i0 = split * p.chunk, i1 = min(p.k, i0 + p.chunk);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], 16);
            mbar_init(&meta[i], 2);
            mbar_init(&sfull[i], 1);
            mbar_init(&pfull[i], 8);
            mbar_init(&pvdone[i], 1);
            mbar_init(&sempty[i], 1);
        }
        mbar_init(qready, 8);
        mbar_init(qfree, 4);
        mbar_init(qload, 1);
        mbar_init(mmadone, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&slots[i], 2);
        for (int i = 0; i < 2; ++i) mbar_init(&redfull[i], 4);
        mbar_init(lfull, 4);
        fence_barrier_init();
        if (rank == 0) {   // one decision for both CTAs: skip the work after a timeout
            const int skip = timed_out_before(p.check) ? 1 : 0;
            *s_skip = skip;
            asm volatile("st.shared::cluster.u32 [%0], %1;"
                         ::"r"(mapa(smem_u32(s_skip), 1)), "r"(skip) : "memory");
        }
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();      // barriers of both CTAs initialised, skip flag delivered, TMEM held
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = (ri.ok && i1 > i0 && !*s_skip) ? (i1 - i0 + kTile - 1) / kTile : 0;

    if (threadIdx.x == 0 && n_tiles > 0) {
        // this CTA's 64 query rows as nine 64-dim swizzled tiles: dims 384..575 straight
        // into their shared-memory home, dims 0..383 into stage 0 for the softmax threads
        // to move into TMEM
        prefetch_tmap(&tm_q);
        mbar_arrive_expect_tx(qload, 9 * 8192);
        for (int r = 0; r < 9; ++r)
            tma_load_2d(base + (r < 6 ? kOffStage + r * 8192 : kOffQs + (r - 6) * 8192), &tm_q,
                        64 * r, t * kHeads + 64 * rank, qload);
    }

    if (warp >= kGatherWarp0 && warp < kMmaWarp) {
        // ============================================================ gather
        // All eight warps gather every tile.  Thread gt < 64 owns key gt of each tile
        // (index -> slot pipeline, three tiles ahead) and publishes the tile's slots in a
        // four-entry ring; every thread then issues its share of the tile's loads (whole
        // 16-byte chunks, a warp covering 512 contiguous bytes of a row) into registers
        // BEFORE waiting for the tile's stage to be released, so the loads' latency
        // overlaps the compute of the two tiles in the stages; then it converts to fp16
        // and stores into the swizzled stage: this CTA's 32 rows into the key buffer
        // (and their V dims of this CTA's half into the V block), the peer's 32 rows'
        // V dims of this half into the V block.  (A thread is at most two tiles ahead of
        // the slowest gather thread -- a stage is released only after every thread has
        // gathered into it -- so a ring entry is rewritten only after every thread has
        // read it.)
        const int gt = threadIdx.x - kGatherWarp0 * 32;       // 0..255
        constexpr int kRowBytes = kFp8 ? 576 : 1152;
        constexpr int kOwnChunks = kFp8 ? 32 * 36 : 32 * 72;   // 16-byte loads per tile
        constexpr int kPeerChunks = kFp8 ? 32 * 16 : 32 * 32;
        constexpr int kLoads = (kOwnChunks + kPeerChunks + 255) / 256;
        int* ring = reinterpret_cast<int*>(base + kOffRing);
        float* ring_sc = reinterpret_cast<float*>(base + kOffRingSc);
        const long long seq_base = (long long)ri.b * p.st_stride;
        auto fetch_idx = [&](int j) -> int {
            const int i = i0 + j * kTile + gt;
            return (gt < kTile && j < n_tiles && i < i1) ? __ldg(p.idx + (long long)t * p.k + i) : -1;
        };
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
        auto fetch_scale = [&](int sl) -> float {
            return (kFp8 && sl >= 0 && p.kv_scale) ? __ldg(p.kv_scale + sl) : 1.0f;
        };
        // index pipeline (threads gt < 64): the checked slot and scale of the next tile to
        // publish, the slot of the one after, the raw table entry and the index beyond
        int sl_cur = -1, sl_next = -1, raw_n2 = kSkip, idx_n3 = -1;
        float sc_cur = 1.0f;
        pdl_wait();                                  // the selection may come from the previous kernel
        if (n_tiles > 0 && gt < kTile) {
            const int x0 = fetch_idx(0), x1 = fetch_idx(1), x2 = fetch_idx(2);
            idx_n3 = fetch_idx(3);
            const int r0 = fetch_slot(x0), r1 = fetch_slot(x1);
            raw_n2 = fetch_slot(x2);
            sl_cur = check_slot(r0);
            sl_next = check_slot(r1);
            sc_cur = fetch_scale(sl_cur);
        }
        uint32_t range = 0;
        // Publishes tile j's slots in ring entry j % 4 (the next tile in order) and waits
        // until the whole gather may read them.
        auto publish = [&](int j) -> bool {
            const int e = j & 3;
            if (gt < kTile) {
                ring[e * 64 + gt] = sl_cur;
                ring_sc[e * 64 + gt] = sc_cur;
                __syncwarp();
                if (lane == 0) mbar_arrive(&slots[e]);
                const int nxt = check_slot(raw_n2);
                raw_n2 = fetch_slot(idx_n3);
                idx_n3 = fetch_idx(j + 4);
                sl_cur = sl_next;
                sl_next = nxt;
                sc_cur = fetch_scale(sl_cur);
            }
            return mbar_wait_warp(&slots[e], (j >> 2) & 1, p.check);
        };
        // Issues this thread's loads I0 .. I0+N-1 of tile j into v (the slot of every load
        // first, all shared-memory reads in flight at once, then the global loads).
        auto issue = [&](int j, auto& v, auto i0_tag) {
            constexpr int I0 = decltype(i0_tag)::value;
            constexpr int N = sizeof(v) / sizeof(v[0]);
            const uint32_t rs_s = sb + kOffRing + (j & 3) * 256;
            int slv[N];
            int offv[N];
#pragma unroll
            for (int ii = 0; ii < N; ++ii) {
                const int q = gt + 256 * (I0 + ii);
                int key = 0;
                offv[ii] = -1;
                if (q < kOwnChunks) {
                    const int row = kFp8 ? q / 36 : q / 72, c = kFp8 ? q - row * 36 : q - row * 72;
                    key = 32 * rank + row;
                    offv[ii] = c * 16;
                } else if (q < kOwnChunks + kPeerChunks) {
                    const int qp = q - kOwnChunks;
                    const int row = kFp8 ? qp >> 4 : qp >> 5, jq = kFp8 ? qp & 15 : qp & 31;
                    const int reg = vblock_region(kFp8 ? jq >> 2 : jq >> 3, rank);
                    key = 32 * (1 - rank) + row;
                    offv[ii] = kFp8 ? reg * 64 + (jq & 3) * 16 : reg * 128 + (jq & 7) * 16;
                }
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(slv[ii]) : "r"(rs_s + 4 * key) : "memory");
            }
#pragma unroll
            for (int ii = 0; ii < N; ++ii) {
                v[ii] = make_uint4(0u, 0u, 0u, 0u);
                if (offv[ii] >= 0 && slv[ii] >= 0)
                    v[ii] = ldg16(p.kv + (long long)slv[ii] * kRowBytes + offv[ii]);
            }
        };
        // Waits for tile j's stage (free once P_{j-2}.V has finished; stage 0 first holds
        // the query tiles until the softmax warps have moved them) and hands the tile's
        // slots and scales to the softmax.
        auto claim = [&](int j) -> bool {
            const int stage = j & 1;
            if (j == 0 && !mbar_wait_warp(qfree, 0, p.check)) return false;
            if (!mbar_wait_warp(&sempty[stage], ((j >> 1) & 1) ^ 1, p.check)) return false;
            if (gt < kTile) {
                srow[stage * 64 + gt] = ring[(j & 3) * 64 + gt];
                kscale[stage * 64 + gt] = ring_sc[(j & 3) * 64 + gt];
            }
            return true;
        };
        // Converts loads I0 .. I0+N-1 of tile j (in v) to fp16 and stores them into its
        // stage: this CTA's rows into the key buffer (and their V dims of this CTA's half
        // into the V block), the peer's rows' V dims into the V block.
        auto put = [&](int j, const auto& v, auto i0_tag) {
            constexpr int I0 = decltype(i0_tag)::value;
            constexpr int N = sizeof(v) / sizeof(v[0]);
            const uint32_t sbuf = sb + kOffStage + (j & 1) * kStageBytes;
            const uint32_t vblk = sbuf + kSbufBytes;
#pragma unroll
            for (int ii = 0; ii < N; ++ii) {
                const int q = gt + 256 * (I0 + ii);
                if (q < kOwnChunks) {
                    if constexpr (!kFp8) {
                        const int row = q / 72, c = q - row * 72, reg = c >> 3, ch = c & 7;
                        const uint4 f = bf16x8_to_f16x8(v[ii], range);
                        sts16(sbuf + reg * 4096 + sw128(row, ch), f);
                        if (reg < 8 && ((reg >> 1) & 1) == rank)
                            sts16(vblk + (((reg >> 2) << 1) | (reg & 1)) * 8192 + sw128(32 * rank + row, ch), f);
                    } else {
                        const int row = q / 36, c = q - row * 36, reg = c >> 2, ch = 2 * (c & 3);
                        uint4 lo, hi;
                        e4m3x16_to_f16(v[ii], lo, hi);
                        sts16(sbuf + reg * 4096 + sw128(row, ch), lo);
                        sts16(sbuf + reg * 4096 + sw128(row, ch + 1), hi);
                        if (reg < 8 && ((reg >> 1) & 1) == rank) {
                            const uint32_t vb = vblk + (((reg >> 2) << 1) | (reg & 1)) * 8192;
                            sts16(vb + sw128(32 * rank + row, ch), lo);
                            sts16(vb + sw128(32 * rank + row, ch + 1), hi);
                        }
                    }
                } else if (q < kOwnChunks + kPeerChunks) {
                    const int qp = q - kOwnChunks;
                    if constexpr (!kFp8) {
                        const int row = qp >> 5, jq = qp & 31;
                        sts16(vblk + (jq >> 3) * 8192 + sw128(32 * (1 - rank) + row, jq & 7),
                              bf16x8_to_f16x8(v[ii], range));
                    } else {
                        const int row = qp >> 4, jq = qp & 15, ch = 2 * (jq & 3);
                        const uint32_t vb = vblk + (jq >> 2) * 8192;
                        uint4 lo, hi;
                        e4m3x16_to_f16(v[ii], lo, hi);
                        sts16(vb + sw128(32 * (1 - rank) + row, ch), lo);
                        sts16(vb + sw128(32 * (1 - rank) + row, ch + 1), hi);
                    }
                }
            }
        };
        // Tile j is in its stage: tell the MMA issuer (both CTAs) and the softmax.
        auto done = [&](int j) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                arrive_leader(&full[j & 1]);
                if (gt < kTile) mbar_arrive(&meta[j & 1]);
            }
        };
        using I0_0 = std::integral_constant<int, 0>;
        bool alive = n_tiles > 0;
        if constexpr (kFp8) {
            // two tiles of loads in flight: tile j+1's are issued before tile j is stored
            uint4 va[kLoads], vb[kLoads];
            if (alive && (alive = publish(0))) issue(0, va, I0_0{});
            for (int j = 0; alive && j < n_tiles; j += 2) {
                if (j + 1 < n_tiles) {
                    if (!(alive = publish(j + 1))) break;
                    issue(j + 1, vb, I0_0{});
                }
                if (!(alive = claim(j))) break;
                put(j, va, I0_0{});
                done(j);
                if (j + 1 >= n_tiles) break;
                if (j + 2 < n_tiles) {
                    if (!(alive = publish(j + 2))) break;
                    issue(j + 2, va, I0_0{});
                }
                if (!(alive = claim(j + 1))) break;
                put(j + 1, vb, I0_0{});
                done(j + 1);
            }
        } else {
            // a tile's loads in two halves (two whole tiles would not fit in registers):
            // the second half of tile j is in flight while the first is stored, and the
            // first half of tile j+1 while the second is stored
            constexpr int kA = (kLoads + 1) / 2;
            using I0_A = std::integral_constant<int, kA>;
            uint4 ra[kA], rb[kLoads - kA];
            if (alive && (alive = publish(0))) issue(0, ra, I0_0{});
            for (int j = 0; alive && j < n_tiles; ++j) {
                issue(j, rb, I0_A{});
                if (!(alive = claim(j))) break;
                put(j, ra, I0_0{});
                if (j + 1 < n_tiles) {
                    if (!(alive = publish(j + 1))) break;
                    issue(j + 1, ra, I0_0{});
                }
                put(j, rb, I0_A{});
                done(j);
            }
        }
        // the releases of the last two stages are the last commits aimed at the gather's
        // barriers: wait for them, so that no arrival lands after this CTA has gone
        for (int j = max(0, n_tiles - 2); alive && j < n_tiles; ++j)
            alive = mbar_wait_warp(&sempty[j & 1], (j >> 1) & 1, p.check);
        if (range) report(p.check, kCheckFp16Range);
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        if (rank == 0 && n_tiles > 0 && elect_one()) {
            bool alive = mbar_wait_cl(qready, 0, p.check);
            tc_fence_after();
            const uint32_t idesc_s = instr_desc(0, 0, 0, 0, kTile, kHeads);   // fp16 x fp16, N=64
            const uint32_t idesc_v = instr_desc(0, 0, 0, 1, 256, kHeads);     // V MN-major, N=256
            // S_j = Q . K_j^T: 36 K-steps of 16 dims, dims 0..383 with A in TMEM
            auto issue_s = [&](int jt) {
                const uint32_t kb = sb + kOffStage + (jt & 1) * kStageBytes;
                const uint32_t d = tmem + kColS + 32 * (jt & 1);
#pragma unroll
                for (int s = 0; s < 36; ++s) {
                    const uint64_t bdesc = smem_desc(kb + (s >> 2) * 4096 + (s & 3) * 32, 16, 1024,
                                                     kLayoutSw128);
                    if (s < kQtSteps)
                        mma2_ts(d, tmem + kColQ + 8 * s, bdesc, idesc_s, s > 0 ? 1u : 0u);
                    else
                        mma2_ss(d, smem_desc(sb + kOffQs + ((s - kQtSteps) >> 2) * 8192 + (s & 3) * 32,
                                             16, 1024, kLayoutSw128),
                                bdesc, idesc_s, 1u);
                }
                commit_pair(&sfull[jt & 1]);
            };
            // O += P_j . V_j: two N=256 halves of the 512 V dims, four K-steps of 16 keys
            auto issue_pv = [&](int jt) {
                const uint32_t vb = sb + kOffStage + (jt & 1) * kStageBytes + kSbufBytes;
                const uint32_t pa = sb + kOffP + (jt & 1) * kPBytes;
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma2_ss(tmem + kColO + 128 * m,
                                smem_desc(pa + kk * 32, 16, 1024, kLayoutSw128),
                                smem_desc(vb + 2 * m * 8192 + kk * 2048, 8192, 1024, kLayoutSw128),
                                idesc_v, (jt > 0 || kk > 0) ? 1u : 0u);
                commit_pair(&sempty[jt & 1]);
                commit_pair(&pvdone[jt & 1]);
            };
            // S_js once tile js is gathered in both CTAs and its score buffer js%2 is free
            // (P_{js-2}.V issued: the softmax of tile js-2 has read the buffer); P_jp.V once
            // P_jp is written in both CTAs.  P.V goes first when both are ready: it frees
            // a stage for the gather.
            int js = 0, jp = 0;
            long long t0 = clock64();
            while (alive && jp < n_tiles) {
                if (jp < js && mbar_test_cl(&pfull[jp & 1], (jp >> 1) & 1)) {
                    tc_fence_after();
                    issue_pv(jp++);
                    t0 = clock64();
                } else if (js < n_tiles && js < jp + 2 && mbar_test_cl(&full[js & 1], (js >> 1) & 1)) {
                    tc_fence_after();
                    issue_s(js++);
                    t0 = clock64();
                } else if (clock64() - t0 > kWaitLimitCycles) {
                    report(p.check, kCheckTimeout);
                    alive = false;
                }
            }
            commit_pair(mmadone);     // after everything issued above, finished or not
        }
        __syncwarp();
        if (n_tiles > 0) mbar_wait_warp(mmadone, 0, p.check);
    } else {
        // ============================================================ softmax
        const int L = threadIdx.x;                    // TMEM lane
        const int hl = L & 63, kh = L >> 6;           // head of this CTA, key half
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        uint32_t range = 0;
        bool alive = n_tiles > 0;
        if (alive) {
            // query row hl: dims 0..383 from the staging tiles into TMEM (fp16 pairs; both
            // lanes of the head write the same row), dims 384..575 converted in place
            alive = mbar_wait_warp(qload, 0, p.check);
#pragma unroll 1
            for (int r = 0; r < 6; ++r) {
                uint32_t w[32];
                const uint32_t src = sb + kOffStage + r * 8192;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 f = bf16x8_to_f16x8(lds16(src + sw128(hl, c)), range);
                    w[4 * c] = f.x;
                    w[4 * c + 1] = f.y;
                    w[4 * c + 2] = f.z;
                    w[4 * c + 3] = f.w;
                }
                tmem_st32(lane_base + kColQ + 32 * r, w);
            }
#pragma unroll 4
            for (int u = 0; u < 12; ++u) {
                const int unit = L + 128 * u, r = unit >> 9, row = (unit >> 3) & 63, c = unit & 7;
                const uint32_t a = sb + kOffQs + r * 8192 + sw128(row, c);
                sts16(a, bf16x8_to_f16x8(lds16(a), range));
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                arrive_leader(qready);
                mbar_arrive(qfree);
            }
        }
        float m_run = -INFINITY, l_run = 0.f;
        for (int j = 0; alive && j < n_tiles; ++j) {
            const int stage = j & 1;
            // ---- this thread's 32 keys of tile j: validity bits and (fp8) scales, read
            // before the scores (the tile's slots and scales are published before its S
            // is issued, so this wait never delays the one for S)
            if (!mbar_wait_warp(&meta[stage], (j >> 1) & 1, p.check)) { alive = false; break; }
            uint32_t valid = 0u;
            float tsc[kFp8 ? 32 : 1];
            {
                const int4* s4 = reinterpret_cast<const int4*>(srow + stage * 64 + 32 * kh);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int4 v = s4[q];
                    valid |= (v.x >= 0 ? 1u : 0u) << (4 * q) | (v.y >= 0 ? 2u : 0u) << (4 * q) |
                             (v.z >= 0 ? 4u : 0u) << (4 * q) | (v.w >= 0 ? 8u : 0u) << (4 * q);
                }
                if constexpr (kFp8) {
                    const float4* c4 = reinterpret_cast<const float4*>(kscale + stage * 64 + 32 * kh);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 f = c4[q];
                        tsc[4 * q] = f.x;
                        tsc[4 * q + 1] = f.y;
                        tsc[4 * q + 2] = f.z;
                        tsc[4 * q + 3] = f.w;
                    }
                }
            }
            float x[32];
            {   // ---- scores of tile j: keys 32*kh .. 32*kh+31 of head hl
                if (!mbar_wait_warp(&sfull[j & 1], (j >> 1) & 1, p.check)) { alive = false; break; }
                tc_fence_after();
                uint32_t a[32];
                tmem_ld32(lane_base + kColS + 32 * (j & 1), a);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(a[i]);
            }
            float sc = p.sc_log2;
            {   // invalid entries (skipped or bad indices) score -inf; fp8 rows x scale.
                // A warp's lanes share the tile's 32 keys (only the head differs), so
                // `valid` is warp-uniform and full tiles skip the masking
                if (valid != 0xFFFFFFFFu) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (!((valid >> i) & 1u)) x[i] = -INFINITY;
                }
                if constexpr (kFp8) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] *= p.sc_log2 * tsc[i];
                    sc = 1.0f;
                }
            }
            float mx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mx[i] = fmaxf(fmaxf(fmaxf(x[8 * i], x[8 * i + 1]), fmaxf(x[8 * i + 2], x[8 * i + 3])),
                              fmaxf(fmaxf(x[8 * i + 4], x[8 * i + 5]), fmaxf(x[8 * i + 6], x[8 * i + 7])));
            // the other half of the head's row max (lane L ^ 64, two warps away); the
            // buffer of tile j is rewritten two tiles later, after every warp has
            // published tile j+1 and so finished reading tile j
            float* rb = red + (j & 1) * 128;
            rb[L] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            __syncwarp();
            if (lane == 0) mbar_arrive(&redfull[j & 1]);
            if (!mbar_wait_warp(&redfull[j & 1], (j >> 1) & 1, p.check)) { alive = false; break; }
            const float m_tile = sc * fmaxf(rb[L], rb[L ^ 64]);
            const float m_new = fmaxf(m_run, m_tile);
            const bool need = m_new > m_run + 8.0f;           // rescale only past 2^8 growth
            const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
            if (need) m_run = m_new;
            const bool warp_rescale = __any_sync(0xffffffffu, need) && j > 0;
            const float msub = m_run == -INFINITY ? 0.f : m_run;   // exp2(-inf) = +0
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float e0 = fast_exp2(fmaf(x[i], sc, -msub));
                const float e1 = fast_exp2(fmaf(x[i + 1], sc, -msub));
                ls[(i >> 1) & 3] += e0 + e1;
                if constexpr (kFp8) pk[i / 2] = pack_f16(e0 * tsc[i], e1 * tsc[i + 1]);
                else pk[i / 2] = pack_f16(e0, e1);
            }
            l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            // ---- P_j into P buffer j%2 once P_{j-2}.V has read it
            if (j >= 2 && !mbar_wait_warp(&pvdone[j & 1], ((j - 2) >> 1) & 1, p.check)) {
                alive = false;
                break;
            }
            {
                const uint32_t pb = sb + kOffP + (j & 1) * kPBytes;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    sts16(pb + sw128(hl, 4 * kh + q),
                          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]));
            }
            // ---- O may be rescaled only once P_{j-1}.V has finished
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
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&pfull[j & 1]);
        }
        // ---- epilogue: O / l and lse (after the predecessor kernel: an earlier kernel of
        // the stream may still read the output or partial buffers)
        pdl_wait();
        const bool have = alive && n_tiles > 0 &&
                          mbar_wait_warp(&pvdone[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p.check);
        tc_fence_after();
        // the head's l is the sum of its two threads' partial sums
        float* rl = red + 2 * 128;
        rl[L] = l_run;
        __syncwarp();
        if (lane == 0) mbar_arrive(lfull);
        const bool lsum = mbar_wait_warp(lfull, 0, p.check);
        const float l_tot = l_run + (lsum ? rl[L ^ 64] : 0.f);
        const float inv = (have && l_tot > 0.f) ? 1.0f / l_tot : 0.f;
        const float lse_v = (have && l_tot > 0.f) ? (m_run + log2f(l_tot)) * 0.69314718055994531f
                                                  : -INFINITY;
        const int head = 64 * rank + hl;
        // this lane's O columns: c < 128 -> dim 128*kh + c, c >= 128 -> 256 + 128*kh + (c-128)
        if (p.nsplit == 1) {
            __nv_bfloat16* orow = p.out + ((long long)t * kHeads + head) * 512;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t o[32];
                if (have) {
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + (cc >> 2) * 256 + 128 * kh + (cc & 3) * 32);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 w = make_uint4(0u, 0u, 0u, 0u);
                    if (have) {
                        w.x = pack_bf16(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                    }
                    dst[q4] = w;
                }
            }
            if (kh == 0 && p.lse) p.lse[(long long)t * kHeads + head] = lse_v;
        } else {
            const long long pbase = ((long long)t * p.nsplit + split) * kHeads + head;
            __half* orow = p.o_part + pbase * 512;
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t o[32];
                if (have) {
                    tmem_ld32(lane_base + kColO + cc * 32, o);
                    tmem_ld_wait();
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + (cc >> 2) * 256 + 128 * kh + (cc & 3) * 32);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 w = make_uint4(0u, 0u, 0u, 0u);
                    if (have) {
                        w.x = pack_f16(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                        w.y = pack_f16(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                        w.z = pack_f16(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                        w.w = pack_f16(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                    }
                    dst[q4] = w;
                }
            }
            if (kh == 0) p.lse_part[pbase] = lse_v;
        }
        if (range) report(p.check, kCheckFp16Range);
    }

    tc_fence_before();
    cluster_sync();          // neither CTA leaves while the pair's MMAs or arrivals may touch it
    tc_fence_after();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace

cudaError_t launch_mla_tc(const void* q, float scale, const CacheView& kv, const BatchView& bv,
                          const int* idx, int k, int nsplit, void* out, float* lse, void* o_part,
                          float* lse_part, int* check, cudaStream_t st, bool pdl) {
    Params p;
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
                                        (unsigned long long)bv.total_q * kHeads, 1152, 64, 64,
                                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (me != cudaSuccess) return me;
    const bool fp8 = kv.dtype == kE4M3;
    auto kern = fp8 ? mla_pair_kernel<true> : mla_pair_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * bv.total_q * nsplit);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm_q, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dsa
