// indexer_tc.cu -- Lightning Indexer scores on sm_100a tensor cores (fp8 e4m3).
//
// I[t,s] = k_scale[s] * q_scale[t] * sum_j w[t,j] * ReLU(q[t,j,:] . k[s,:]),  s <= pos(t)
// The indexer is the light FP8 scorer of "SGLang Day-0 support for
// DeepSeek-V3.2", section "DeepSeek Sparse Attention"; its key & key_scale cache
// uses page size 64 (same section); the deployment guide (m.nxbn.cn, section 3.1)
// runs it in FP8.
//
// Mapping.  One tile = 128 keys (two 64-token pages) x (r query rows x 64 heads):
//   D[key, (row, head)] = K_tile (128 x 128 fp8, K-major) . Q_rows^T (64r x 128 fp8)
// is one tcgen05 kind::f8f6f4 MMA chain (M = 128, N = 64r, K = 4 x 32) into a TMEM
// accumulator.  Each epilogue thread owns one key (one TMEM lane) and reduces its
// row: sum_h w[row,h] * max(D, 0), then applies the key's and the query's scale.
//
// Roles: warp 0 issues TMA loads (pages through the block table into a 4-stage ring
// of 128-byte-swizzled tiles), warp 1 allocates TMEM and issues the MMAs (double-
// buffered accumulators), the epilogue warps drain TMEM and write the logits: one
// warpgroup for one or two query rows per CTA (2 CTAs per SM), two warpgroups for
// three rows and four for four (1 CTA per SM: the accumulators fill TMEM).  With four,
// each accumulator buffer has its own two warpgroups of two rows each, a tile apart.
//
// Grid: x = groups of G consecutive query rows (G = 1 for one query per sequence,
// 2 or 3 for multi-token decode, 4 otherwise; a group that spans sequences is
// processed as per-sequence runs),
// y = chunks of the key tiles, so that short batches still cover all SMs.
#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kHeads = 64;
constexpr int kDim = 128;
constexpr int kTileKeys = 128;
constexpr int kStages = 4;
constexpr int kTileBytes = kTileKeys * kDim;       // 16 KB
constexpr int kRowBytes = kHeads * kDim;            // one query row: 8 KB
// 2 producer warps + EPI epilogue warpgroups: EPI = 1 for one or two query rows per
// CTA (64 or 128 accumulator columns, 2 CTAs per SM), EPI = 2 for three or four rows
// (the double-buffered accumulator fills TMEM: 1 CTA per SM, and each warpgroup
// reduces two of the rows of every tile).
template <int EPI>
constexpr int threads_for() { return 64 + 128 * EPI; }
// With four epilogue warpgroups, warpgroups 0-1 reduce the even tiles (accumulator
// buffer 0) and 2-3 the odd ones, two rows each: the two halves then work a tile apart,
// so one half's waits and loads overlap the other half's arithmetic (all four on every
// tile, one row each, move in lockstep and leave the SM's ALUs idle half the time).
template <int EPI>
constexpr int kEpiWarpsPerBuf = EPI == 4 ? 8 : 4 * EPI;

struct Params {
    const float* w;
    const float* q_scale;
    const float* k_scale;
    const int* table;
    long long num_pages;
    int bt_stride;
    BatchView bv;
    float* logits;
    long long ld;
    int G;          // query rows per CTA
    int C;          // key tiles per chunk
    int row0;       // first query row of the launch; logits row t is at (t - row0) * ld
    int* check;
};

struct Run {        // a run of query rows of one sequence (j0 == j1: nothing to do)
    int b, t0, r, pos_lo, j0, j1;
};

// The r-th per-sequence run of the CTA's row group, restricted to its key chunk.
// Returns false when there is no such run.
__device__ __forceinline__ bool get_run(const Params& p, int k, Run* out, bool skip) {
    const int t_begin = p.row0 + blockIdx.x * p.G;
    const int t_end = min(p.bv.total_q, t_begin + p.G);
    int t = t_begin;
    for (int i = 0; t < t_end; ++i) {
        const int b = find_seq(p.bv.cu_q, p.bv.num_seqs, t);
        const int q0 = __ldg(p.bv.cu_q + b), q1 = __ldg(p.bv.cu_q + b + 1);
        const int L = __ldg(p.bv.seq_lens + b);
        const int r = min(t_end, q1) - t;
        if (i == k) {
            out->b = b;
            out->t0 = t;
            out->r = r;
            out->pos_lo = L - (q1 - q0) + (t - q0);
            const bool ok = (q1 - q0) <= L && L <= p.bv.max_seq_len && out->pos_lo >= 0;
            const int pos_hi = out->pos_lo + r - 1;
            const int tiles = ok ? (pos_hi + kTileKeys) / kTileKeys : 0;
            out->j0 = blockIdx.y * p.C;
            out->j1 = skip ? out->j0 : min(tiles, out->j0 + p.C);
            return true;
        }
        t += r;
    }
    return false;
}

// acc += a * b on a pair of floats with one packed instruction (two IEEE fp32 FMAs,
// each rounded as fmaf would).
__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) {
    acc = __ffma2_rn(a, b, acc);
}

template <int EPI>
__global__ void __launch_bounds__(threads_for<EPI>(), EPI == 1 ? 2 : 1)
indexer_fp8_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_q, Params p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned carve-up: stages | Q (G rows) | w | barriers
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a_tiles = base;
    uint8_t* q_tile = a_tiles + kStages * kTileBytes;
    float* w_s = reinterpret_cast<float*>(q_tile + p.G * kRowBytes);   // [G][64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(w_s + p.G * kHeads);
    uint64_t* full = bars;                    // [kStages] TMA -> MMA
    uint64_t* empty = bars + kStages;         // [kStages] MMA -> TMA
    uint64_t* tfull = bars + 2 * kStages;     // [2] MMA -> epilogue
    uint64_t* tempty = tfull + 2;             // [2] epilogue -> MMA
    uint64_t* qfull = tempty + 2;             // Q rows landed
    uint64_t* qempty = qfull + 1;             // MMAs of a run done with Q
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    const int ncols_buf = p.G * kHeads;                     // accumulator columns per buffer
    const uint32_t tmem_cols = ncols_buf * 2 <= 128 ? 128u : (ncols_buf * 2 <= 256 ? 256u : 512u);

    __shared__ int s_skip;
    if (threadIdx.x == 0) {
        s_skip = timed_out_before(p.check) ? 1 : 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kEpiWarpsPerBuf<EPI>);   // one arrive per warp that reads it
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_q);
    }
    pdl_wait();   // launched as a dependent: every input may come from the previous kernel
    {   // head weights of the CTA's rows, loaded once (no per-run barrier needed)
        const int t_begin = p.row0 + blockIdx.x * p.G;
        const int nrow = min(p.G, p.bv.total_q - t_begin);
        for (int i = threadIdx.x; i < nrow * kHeads; i += threads_for<EPI>())
            w_s[i] = __ldg(p.w + (long long)t_begin * kHeads + i);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = s_skip != 0;   // an earlier CTA timed out: do no work

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (elect_one()) {
            int it = 0, runs_issued = 0;
            bool alive = true;
            Run run;
            for (int k = 0; alive && get_run(p, k, &run, skip); ++k) {
                if (run.j0 >= run.j1) continue;
                if (runs_issued > 0) {
                    // the previous run's MMAs must be done reading Q
                    if (!mbar_wait(qempty, (runs_issued - 1) & 1, p.check)) { alive = false; break; }
                }
                ++runs_issued;
                mbar_arrive_expect_tx(qfull, p.G * kRowBytes);
                tma_load_2d(q_tile, &tm_q, 0, run.t0 * kHeads, qfull);
                const int pos_hi = run.pos_lo + run.r - 1;
                // block-table entries of the run's tiles, loaded four tiles at a time and
                // one group ahead of their use (a lookup right before each TMA would put a
                // global-load latency on every tile)
                const int* trow = p.table + (long long)run.b * p.bt_stride;
                auto load_pages = [&](int jt, int (&pg)[8]) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int s0 = (jt + u) * kTileKeys;
                        const bool in = jt + u < run.j1;
                        pg[2 * u] = in ? __ldg(trow + s0 / 64) : 0;
                        pg[2 * u + 1] = (in && s0 + 64 <= pos_hi) ? __ldg(trow + s0 / 64 + 1) : 0;
                    }
                };
                int cur[8], nxt[8];
                load_pages(run.j0, cur);
                load_pages(run.j0 + 4, nxt);
                for (int j4 = run.j0; alive && j4 < run.j1; j4 += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = j4 + u;
                        if (j >= run.j1) break;
                        const int stage = it % kStages;
                        const uint32_t ph = (it / kStages) & 1;
                        if (!mbar_wait(&empty[stage], ph ^ 1, p.check)) { alive = false; break; }
                        const bool two = j * kTileKeys + 64 <= pos_hi;
                        int p0 = cur[2 * u], p1 = cur[2 * u + 1];
                        const bool bad0 = p0 < 0 || (long long)p0 >= p.num_pages;
                        const bool bad1 = two && (p1 < 0 || (long long)p1 >= p.num_pages);
                        if (bad0 | bad1) report(p.check, kCheckBadPage);
                        if (bad0) p0 = 0;
                        if (bad1) p1 = 0;
                        mbar_arrive_expect_tx(&full[stage], two ? kTileBytes : kTileBytes / 2);
                        uint8_t* dst = a_tiles + stage * kTileBytes;
                        tma_load_2d(dst, &tm_k, 0, p0 * 64, &full[stage]);
                        if (two) tma_load_2d(dst + kTileBytes / 2, &tm_k, 0, p1 * 64, &full[stage]);
                        ++it;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
                    load_pages(j4 + 8, nxt);
                }
            }
            // drain: every issued copy has landed (full phase; also after a timeout, so
            // that no TMA write into this CTA's shared memory is in flight when it exits)
            // and, on the normal path, every stage has been consumed (empty phase)
            const int n = it < kStages ? it : kStages;
            bool landed = true;
            for (int i = 0; i < n && landed; ++i) {
                const int itx = it - 1 - i;
                landed = mbar_wait(&full[itx % kStages], (itx / kStages) & 1, p.check);
            }
            if (runs_issued > 0 && landed) mbar_wait(qfull, (runs_issued - 1) & 1, p.check);
            for (int i = 0; i < n && alive; ++i) {
                const int itx = it - 1 - i;
                if (!mbar_wait(&empty[itx % kStages], (itx / kStages) & 1, p.check)) break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            int it = 0, runs_done = 0;
            bool alive = true;
            Run run;
            const uint32_t q_addr = smem_u32(q_tile);
            for (int k = 0; alive && get_run(p, k, &run, skip); ++k) {
                if (run.j0 >= run.j1) continue;
                if (!mbar_wait(qfull, runs_done & 1, p.check)) { alive = false; break; }
                tc_fence_after();
                const uint32_t idesc = instr_desc(0, 0, 0, 0, run.r * kHeads, kTileKeys);
                const uint64_t bdesc = smem_desc(q_addr, 16, 1024, kLayoutSw128);
                for (int j = run.j0; j < run.j1; ++j, ++it) {
                    const int stage = it % kStages;
                    const int buf = it & 1;
                    if (!mbar_wait(&tempty[buf], ((it >> 1) & 1) ^ 1, p.check)) { alive = false; break; }
                    if (!mbar_wait(&full[stage], (it / kStages) & 1, p.check)) { alive = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * ncols_buf;
                    const uint64_t adesc =
                        smem_desc(smem_u32(a_tiles + stage * kTileBytes), 16, 1024, kLayoutSw128);
#pragma unroll
                    for (int kk = 0; kk < kDim / 32; ++kk)   // 32 fp8 = 32 bytes per K step
                        mma_f8(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    mma_commit(&empty[stage]);
                    mma_commit(&tfull[buf]);
                }
                ++runs_done;
                // free Q for a following run (not after the last one)
                Run nxt;
                bool more = false;
                for (int k2 = k + 1; get_run(p, k2, &nxt, skip); ++k2)
                    if (nxt.j0 < nxt.j1) { more = true; break; }
                if (more) mma_commit(qempty);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;          // key row within the tile
        const int wg = (warp - 2) >> 2;               // epilogue warpgroup
        constexpr int kRows = EPI == 1 ? 4 : 2;       // query rows of this warp:
        const int q_lo = EPI == 1 ? 0 : EPI == 2 ? 2 * wg : 2 * (wg & 1);   // q_lo .. q_lo + kRows - 1
        // tiles this warp reduces: all, or (four warpgroups) those of its buffer parity
        constexpr int kStep = EPI == 4 ? 2 : 1;
        const int parity = EPI == 4 ? wg >> 1 : 0;
        // rows whose TMEM loads are issued before one wait (EPI = 4 has no registers for two)
        constexpr int kPair = EPI == 4 ? 1 : 2;
        int it = 0;
        bool alive = true;
        Run run;
        for (int k = 0; alive && get_run(p, k, &run, skip); ++k) {
            if (run.j0 >= run.j1) continue;
            const int it0 = it;
            it += run.j1 - run.j0;
            const int jf = run.j0 + (kStep == 2 ? ((parity - it0) & 1) : 0);   // first tile of this warp
            const float* w_run = w_s + (run.t0 - p.row0 - blockIdx.x * p.G) * kHeads;
            // this warp's rows of the run: logits row, query scale, position (registers,
            // indexed by the unrolled row number)
            float* rowp[kRows];
            float qsc[kRows];
            int posr[kRows];
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                const int qi = q_lo + u;
                rowp[u] = p.logits + (long long)(run.t0 + qi - p.row0) * p.ld;
                qsc[u] = (qi < run.r && p.q_scale) ? __ldg(p.q_scale + run.t0 + qi) : 1.0f;
                posr[u] = run.pos_lo + qi;
            }
            const int pos_hi = run.pos_lo + run.r - 1;
            // this key's block-table entry two tiles ahead and its scale one tile ahead
            // (a table -> scale load chain per tile would stall every tile)
            const int* trow = p.table + (long long)run.b * p.bt_stride;
            auto tbl = [&](int jt) -> int {
                const int sk = jt * kTileKeys + row;
                return (jt < run.j1 && sk <= pos_hi) ? __ldg(trow + sk / 64) : 0;
            };
            auto scl = [&](int jt, int pg) -> float {
                const int sk = jt * kTileKeys + row;
                if (jt >= run.j1 || sk > pos_hi || pg < 0 || (long long)pg >= p.num_pages) return 0.f;
                return p.k_scale ? __ldg(p.k_scale + (long long)pg * 64 + (sk & 63)) : 1.0f;
            };
            int pg1 = tbl(jf), pg2 = tbl(jf + kStep);
            float ks1 = scl(jf, pg1);
            for (int j = jf; j < run.j1; j += kStep) {
                const int itj = it0 + (j - run.j0);
                const int buf = itj & 1;
                const int s = j * kTileKeys + row;
                const int page = pg1;
                const float ks = ks1;
                const int bad = (s <= pos_hi && (page < 0 || (long long)page >= p.num_pages)) ? 1 : 0;
                pg1 = pg2;
                pg2 = tbl(j + 2 * kStep);
                ks1 = scl(j + kStep, pg1);
                if (!mbar_wait_warp(&tfull[buf], (itj >> 1) & 1, p.check)) { alive = false; break; }
                tc_fence_after();
                float res[kRows];
#pragma unroll
                for (int u = 0; u < kRows; ++u) res[u] = 0.f;
                const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * ncols_buf;
                // the accumulator buffer is handed back to the MMA as soon as this warp's last
                // TMEM load of the tile has completed: the arithmetic on those values then
                // overlaps the next MMA into the buffer
                const int my_rows = max(0, min(kRows, run.r - q_lo));
                auto release = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                };
                if (my_rows == 0) release();
                // the warp's rows kPair at a time: all their 32-head TMEM loads are issued
                // before one wait (a TMEM load takes a few hundred cycles; issued one after
                // another they would serialise that latency)
                // one row at a time (four warpgroups: no registers for two): each half-row's
                // 32 accumulator columns and its 32 head weights are loaded together, so
                // the weights' shared-memory latency overlaps the TMEM load
                if constexpr (kPair == 1) {
#pragma unroll
                    for (int u = 0; u < kRows; ++u) {
                        if (u >= my_rows) break;
                        const int qi = q_lo + u;
                        const uint32_t c0 = tbase + qi * kHeads;
                        const uint32_t w_sa = smem_u32(w_run + qi * kHeads);
                        float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t v[32];
                            float4 wq[8];
                            tmem_ld32(c0 + 32 * half, v);
#pragma unroll
                            for (int q = 0; q < 8; ++q)   // volatile: see below
                                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                             : "=f"(wq[q].x), "=f"(wq[q].y), "=f"(wq[q].z), "=f"(wq[q].w)
                                             : "r"(w_sa + 128 * half + 16 * q));
                            tmem_ld_wait();
                            if (half == 1 && u + 1 >= my_rows) release();
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float2 r0 = make_float2(fmaxf(__uint_as_float(v[4 * q + 0]), 0.f),
                                                              fmaxf(__uint_as_float(v[4 * q + 1]), 0.f));
                                const float2 r1 = make_float2(fmaxf(__uint_as_float(v[4 * q + 2]), 0.f),
                                                              fmaxf(__uint_as_float(v[4 * q + 3]), 0.f));
                                ffma2(acc[(2 * q) & 3], make_float2(wq[q].x, wq[q].y), r0);
                                ffma2(acc[(2 * q + 1) & 3], make_float2(wq[q].z, wq[q].w), r1);
                            }
                        }
                        res[u] = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                                 ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
                    }
                } else {
#pragma unroll
                for (int u0 = 0; u0 < kRows; u0 += kPair) {
                    const int nr = min(kPair, my_rows - u0);   // rows of this group
                    if (nr <= 0) break;
                    uint32_t v[kPair][64];
#pragma unroll
                    for (int u = 0; u < kPair; ++u) {
                        if (u < nr) {
                            const uint32_t c0 = tbase + (q_lo + u0 + u) * kHeads;
                            tmem_ld32(c0, *reinterpret_cast<uint32_t(*)[32]>(&v[u][0]));
                            tmem_ld32(c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[u][32]));
                        }
                    }
                    tmem_ld_wait();
                    if (u0 + kPair >= my_rows) release();
#pragma unroll
                    for (int u = 0; u < kPair; ++u) {
                        if (u >= nr) break;
                        const int qi = q_lo + u0 + u;
                        // sum_h w_h * ReLU(D_h): ReLU per head, then packed pairs of FMAs
                        // into four pair accumulators (eight independent partial sums)
                        const uint32_t w_sa = smem_u32(w_run + qi * kHeads);
                        float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                        for (int h4 = 0; h4 < 16; ++h4) {
                            // volatile: executed only where control reaches it (a
                            // speculated load of a row this CTA does not have would
                            // read past its shared memory)
                            float4 wv;
                            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                         : "=f"(wv.x), "=f"(wv.y), "=f"(wv.z), "=f"(wv.w)
                                         : "r"(w_sa + 16 * h4));
                            const float2 r0 = make_float2(fmaxf(__uint_as_float(v[u][4 * h4 + 0]), 0.f),
                                                          fmaxf(__uint_as_float(v[u][4 * h4 + 1]), 0.f));
                            const float2 r1 = make_float2(fmaxf(__uint_as_float(v[u][4 * h4 + 2]), 0.f),
                                                          fmaxf(__uint_as_float(v[u][4 * h4 + 3]), 0.f));
                            ffma2(acc[(2 * h4) & 3], make_float2(wv.x, wv.y), r0);
                            ffma2(acc[(2 * h4 + 1) & 3], make_float2(wv.z, wv.w), r1);
                        }
                        res[u0 + u] = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                                      ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
                    }
                }
                }
#pragma unroll
                for (int u = 0; u < kRows; ++u) {
                    if (q_lo + u >= run.r) break;
                    float* dst = rowp[u] + s;
                    if (s <= posr[u]) *dst = bad ? -INFINITY : res[u] * ks * qsc[u];
                    else if (s < p.ld) *dst = -INFINITY;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// 2-D byte matrix [rows][128] with a 128 x box_rows box, 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, unsigned long long rows, uint32_t box_rows) {
    return make_tensor_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, rows, 128, 128,
                              box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_indexer_fp8_tc(const void* q, const float* q_scale, const float* w,
                                  const CacheView& k, const BatchView& bv, float* logits,
                                  long long ld, int* check, cudaStream_t st, bool pdl, int row0) {
    // Rows per CTA: one per sequence in decode; 2 or 3 when the batch averages that
    // many query tokens per sequence (multi-token verify), so that each sequence's
    // keys are read once for all its rows; 4 for prefill-sized batches.  The launch
    // covers rows [row0, bv.total_q).
    const int T = bv.total_q - row0, B = bv.num_seqs;
    const int G = T <= B ? 1 : T <= 2 * B ? 2 : T <= 3 * B ? 3 : 4;
    const int groups = (T + G - 1) / G;
    const int tiles_max = (bv.max_seq_len + kTileKeys - 1) / kTileKeys;
    // About 4 CTAs per SM (2 resident) balance long, uneven rows; when that would
    // leave fewer than 16 key tiles per CTA, one wave of 2 CTAs per SM is used
    // instead, so that the per-CTA setup is paid once per SM slot.
    const int target = 4 * kNumSMs, slots = (G <= 2 ? 2 : 1) * kNumSMs;
    int chunks = groups >= target / 2 ? 1 : (target + groups - 1) / groups;
    if (groups < slots && tiles_max / chunks < 16) chunks = slots / groups;
    if (chunks < 1) chunks = 1;
    if (chunks > tiles_max) chunks = tiles_max;
    const int C = (tiles_max + chunks - 1) / chunks;
    chunks = (tiles_max + C - 1) / C;

    CUtensorMap tm_k, tm_q;
    cudaError_t e = make_map(&tm_k, k.data, (unsigned long long)k.num_pages * 64, 64);
    if (e != cudaSuccess) return e;
    e = make_map(&tm_q, q, (unsigned long long)bv.total_q * kHeads, G * kHeads);
    if (e != cudaSuccess) return e;

    Params p{w, q_scale, k.scale, k.table, k.num_pages, k.bt_stride, bv, logits, ld, G, C, row0, check};
    const size_t smem = 1024 + kStages * kTileBytes + (size_t)G * kRowBytes +
                        (size_t)G * kHeads * sizeof(float) + 16 * sizeof(uint64_t) + 16;
    dim3 grid(groups, chunks);
    if (G <= 2) {
        e = cudaFuncSetAttribute(indexer_fp8_tc_kernel<1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_kernel(indexer_fp8_tc_kernel<1>, grid, dim3(threads_for<1>()), smem, st, pdl,
                          tm_k, tm_q, p);
        if (e != cudaSuccess) return e;
    } else if (G == 3) {
        e = cudaFuncSetAttribute(indexer_fp8_tc_kernel<2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_kernel(indexer_fp8_tc_kernel<2>, grid, dim3(threads_for<2>()), smem, st, pdl,
                          tm_k, tm_q, p);
        if (e != cudaSuccess) return e;
    } else {
        e = cudaFuncSetAttribute(indexer_fp8_tc_kernel<4>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_kernel(indexer_fp8_tc_kernel<4>, grid, dim3(threads_for<4>()), smem, st, pdl,
                          tm_k, tm_q, p);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace dsa
