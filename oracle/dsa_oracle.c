/*
 * dsa_oracle.c -- plain, slow CPU definition of the DeepSeek Sparse Attention
 * (DSA) hot path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * CPU-baseline leg of the benchmark call it; the library never does.
 *
 * What DSA computes (sources, by page title and section):
 *   - "SGLang Day-0 support for DeepSeek-V3.2" (winzheng.jp review), section
 *     "DeepSeek Sparse Attention": a Lightning Indexer (a light FP8 scorer)
 *     scores, for each query, the tokens before it; a top-k token selection then
 *     keeps only the most relevant key/value entries; core attention runs on
 *     those entries, cutting O(L^2) to O(Lk).  Same section: the indexer's
 *     key & key_scale cache uses page size 64, the token-level sparse operator
 *     page size 1.
 *   - "DeepSeek-V3.2-Exp DSA deployment guide" (m.nxbn.cn), section 1: the
 *     indexer scores the preceding tokens, top-k entries join attention;
 *     section 3.1: topk 2048, FP8 indexer, fp8_e4m3 KV cache; section 5.1: when
 *     the sequence is shorter than topk, DSA degenerates to dense attention.
 *   - "DeepSeek V3.2 usage guide" (SGLang docs), attention-kernel section: the
 *     sparse MLA kernels take bf16 q with a bf16 or FP8 KV cache.
 * The pages print no formula.  The problem statement this library implements
 * fixes the indexer score as
 *     I[t,s] = k_scale[s] * q_scale[t] * sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:])
 * for causal s <= pos(t), the MLA shapes (576 = 512 latent + 64 rope, V = first
 * d_v columns) and the softmax scale.
 *
 * Every function here follows the definition literally, accumulates in double,
 * and rounds once at the end.  Query rows are independent, so rows are spread
 * over threads with OpenMP; nothing inside a row is blocked, fused or
 * reordered.
 *
 * Batch convention: sequence b owns query rows cu_q[b] .. cu_q[b+1]-1; they are
 * its LAST nq_b = cu_q[b+1]-cu_q[b] tokens, so query i of sequence b sits at
 * position pos = L_b - nq_b + i and sees keys 0..pos (causal, s = t included).
 *
 * Dtype codes: 0 = fp32, 1 = bf16, 2 = fp8 e4m3 (OCP).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_E4M3 2

/* OCP FP8 e4m3, written from its bit definition: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, exponent 0
 * encodes subnormals m * 2^-9. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bf16 is the top half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, int dtype, int64_t i) {
    switch (dtype) {
    case OR_F32: return (double)((const float*)base)[i];
    case OR_BF16: return oracle_bf16_to_double(((const uint16_t*)base)[i]);
    case OR_E4M3: return oracle_e4m3_to_double(((const uint8_t*)base)[i]);
    default: return NAN;
    }
}

/* Finds the sequence of query row t and its position.  Returns 0 on success. */
static int row_info(int num_seqs, const int32_t* cu_q, const int32_t* seq_lens, int64_t t,
                    int* b_out, int64_t* pos_out) {
    for (int b = 0; b < num_seqs; ++b) {
        if (t >= cu_q[b] && t < cu_q[b + 1]) {
            int64_t nq = cu_q[b + 1] - cu_q[b];
            int64_t i = t - cu_q[b];
            *b_out = b;
            *pos_out = (int64_t)seq_lens[b] - nq + i;
            return 0;
        }
    }
    return -1;
}

/* Address (element index) of logical token s of sequence b in a paged cache. */
static int64_t cache_row(const int32_t* table, int bt_stride, int page_size, int b, int64_t s) {
    int64_t page = table[(int64_t)b * bt_stride + s / page_size];
    return page * page_size + s % page_size;
}

/*
 * Lightning Indexer logits for the listed query rows.
 *   q      [T][heads][dim]  (q_dtype)      q_scale [T] or NULL (= 1)
 *   w      [T][heads] fp32
 *   k_data [pages][page_size][dim] (k_dtype), k_scale [pages][page_size] or NULL
 * out[r][s] = I[rows[r], s] for s <= pos, -inf for pos < s < ld_out.
 * Returns 0, or -1 on a malformed row or table entry.
 */
int oracle_indexer_logits(const void* q, int q_dtype, const float* q_scale, const float* w,
                          int heads, int dim, const void* k_data, int k_dtype,
                          const float* k_scale, int page_size, const int32_t* block_table,
                          int bt_stride, int num_seqs, const int32_t* cu_q,
                          const int32_t* seq_lens, const int64_t* rows, int64_t nrows,
                          float* out, int64_t ld_out) {
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        int b;
        int64_t pos;
        float* o = out + r * ld_out;
        for (int64_t s = 0; s < ld_out; ++s) o[s] = -INFINITY;
        if (row_info(num_seqs, cu_q, seq_lens, t, &b, &pos) != 0 || pos >= ld_out) {
            bad |= 1;
            continue;
        }
        double qs = q_scale ? (double)q_scale[t] : 1.0;
        for (int64_t s = 0; s <= pos; ++s) {
            int64_t krow = cache_row(block_table, bt_stride, page_size, b, s);
            double acc = 0.0;
            for (int j = 0; j < heads; ++j) {
                double dot = 0.0;
                for (int d = 0; d < dim; ++d)
                    dot += load_elem(q, q_dtype, (t * heads + j) * (int64_t)dim + d) *
                           load_elem(k_data, k_dtype, krow * dim + d);
                double relu = dot > 0.0 ? dot : 0.0;
                acc += (double)w[t * heads + j] * relu;
            }
            double ks = k_scale ? (double)k_scale[krow] : 1.0;
            o[s] = (float)(ks * qs * acc);
        }
    }
    return bad ? -1 : 0;
}

/* Candidate order of the top-k definition: larger score first, lower index on
 * equal scores. */
typedef struct {
    float v;
    int32_t s;
} cand_t;

static int cand_cmp(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

static int int_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Top-k selection for the listed rows.  logits[r][s] holds the scores of row
 * rows[r] (only s <= pos is read).  idx[r][0..k) receives the min(k, pos+1)
 * selected positions in ascending order, then -1 padding.  When pos+1 <= k every
 * causal position is kept: attention over them is dense causal attention.
 */
int oracle_topk(const float* logits, int64_t ld, int num_seqs, const int32_t* cu_q,
                const int32_t* seq_lens, const int64_t* rows, int64_t nrows, int k,
                int32_t* idx) {
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int b;
        int64_t pos;
        int32_t* out = idx + r * (int64_t)k;
        for (int i = 0; i < k; ++i) out[i] = -1;
        if (row_info(num_seqs, cu_q, seq_lens, rows[r], &b, &pos) != 0 || pos >= ld) {
            bad |= 1;
            continue;
        }
        int64_t n = pos + 1;
        cand_t* c = (cand_t*)malloc((size_t)n * sizeof(cand_t));
        for (int64_t s = 0; s < n; ++s) {
            c[s].v = logits[r * ld + s];
            c[s].s = (int32_t)s;
        }
        qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
        int64_t m = n < k ? n : k;
        for (int64_t i = 0; i < m; ++i) out[i] = c[i].s;
        qsort(out, (size_t)m, sizeof(int32_t), int_cmp);
        free(c);
    }
    return bad ? -1 : 0;
}

/*
 * Sparse MLA over the selected latent-KV rows, for the listed query rows.
 *   q   [T][heads][d_qk] (q_dtype)
 *   kv  [pages][page_size][d_qk] (kv_dtype), kv_scale [pages][page_size] or NULL;
 *       the value vector is the first d_v columns of the same row.
 *   idx [nrows][k] logical positions, -1 entries are skipped.
 * For each head h:  z_s = softmax_scale * q[t,h,:] . kv_s   (kv_s dequantised as
 * code * kv_scale),  p = softmax over the selected s,  o = sum_s p_s kv_s[0:d_v],
 * lse = max z + log sum exp(z - max z).  out [nrows][heads][d_v], lse
 * [nrows][heads] (lse may be NULL).  A row with no valid index gets o = 0,
 * lse = -inf.  Returns -1 if an index is out of [−1, pos].
 */
int oracle_sparse_mla(const void* q, int q_dtype, int heads, int d_qk, int d_v,
                      double softmax_scale, const void* kv, int kv_dtype,
                      const float* kv_scale, int page_size, const int32_t* block_table,
                      int bt_stride, int num_seqs, const int32_t* cu_q,
                      const int32_t* seq_lens, const int32_t* idx, int k, const int64_t* rows,
                      int64_t nrows, float* out, float* lse) {
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        int b;
        int64_t pos;
        const int32_t* sel = idx + r * (int64_t)k;
        float* o_row = out + r * (int64_t)heads * d_v;
        if (row_info(num_seqs, cu_q, seq_lens, t, &b, &pos) != 0) {
            bad |= 1;
            continue;
        }
        double* z = (double*)malloc((size_t)k * sizeof(double));
        int64_t* kr = (int64_t*)malloc((size_t)k * sizeof(int64_t));
        double* acc = (double*)malloc((size_t)d_v * sizeof(double));
        int nsel = 0;
        for (int i = 0; i < k; ++i) {
            int32_t s = sel[i];
            if (s < 0) continue;
            if (s > pos) {
                bad |= 1;
                continue;
            }
            kr[nsel++] = cache_row(block_table, bt_stride, page_size, b, s);
        }
        for (int h = 0; h < heads; ++h) {
            int64_t qoff = (t * heads + h) * (int64_t)d_qk;
            double zmax = -INFINITY;
            for (int i = 0; i < nsel; ++i) {
                double ks = kv_scale ? (double)kv_scale[kr[i]] : 1.0;
                double dot = 0.0;
                for (int d = 0; d < d_qk; ++d)
                    dot += load_elem(q, q_dtype, qoff + d) *
                           (load_elem(kv, kv_dtype, kr[i] * d_qk + d) * ks);
                z[i] = softmax_scale * dot;
                if (z[i] > zmax) zmax = z[i];
            }
            for (int d = 0; d < d_v; ++d) acc[d] = 0.0;
            double denom = 0.0;
            for (int i = 0; i < nsel; ++i) {
                double p = exp(z[i] - zmax);
                double ks = kv_scale ? (double)kv_scale[kr[i]] : 1.0;
                denom += p;
                for (int d = 0; d < d_v; ++d)
                    acc[d] += p * (load_elem(kv, kv_dtype, kr[i] * d_qk + d) * ks);
            }
            for (int d = 0; d < d_v; ++d)
                o_row[(int64_t)h * d_v + d] = nsel ? (float)(acc[d] / denom) : 0.0f;
            if (lse) lse[r * heads + h] = nsel ? (float)(zmax + log(denom)) : -INFINITY;
        }
        free(z);
        free(kr);
        free(acc);
    }
    return bad ? -1 : 0;
}

int oracle_num_threads(void) { return omp_get_max_threads(); }

/* ------------------------------------------------------------ cache writes
 * The caches the indexer and the attention read are filled token by token:
 * "SGLang Day-0 support for DeepSeek-V3.2" (winzheng.jp review), section
 * "DeepSeek Sparse Attention" -- the indexer keeps a key & key_scale cache
 * (page size 64) and the sparse operator a token-level cache (page size 1);
 * its "Future work" section and its launch line's KV_CACHE_STORE_FP8 switch:
 * the KV cache may be stored in FP8, halving the bytes attention reads;
 * "DeepSeek-V3.2-Exp DSA deployment guide" (m.nxbn.cn), section 3.1:
 * fp8_e4m3 KV cache.  The problem fixes the FP8 scaling: one fp32 scale per
 * token, amax / 448 (448 = the largest finite e4m3 magnitude).
 */

/* fp32 -> OCP e4m3, round to nearest (ties to even), magnitudes that round
 * above 448 saturate to 448, the sign is kept (also on zero), NaN -> 0x7F.
 * Written from the bit layout: normal codes are (1 + m/8) * 2^(E-7) for
 * E = 1..15 (E = 15, m = 7 is NaN), subnormal codes m * 2^-9. */
uint8_t oracle_f32_to_e4m3(float f) {
    if (isnan(f)) return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);          /* a = fr * 2^e2, fr in [0.5, 1): floor(log2 a) = e2 - 1 */
    int ex = e2 - 1;
    if (ex < -6) ex = -6;   /* below 2^-6 the spacing stays 2^-9 (subnormals) */
    double quantum = ldexp(1.0, ex - 3);
    double n = nearbyint(a / quantum);   /* a / quantum is exact; default mode = ties to even */
    double v = n * quantum;
    if (v > 448.0) v = 448.0;
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6))
        return sign | (uint8_t)(v / ldexp(1.0, -9));              /* subnormal: m in 1..7 */
    frexp(v, &e2);
    ex = e2 - 1;                                                   /* -6 .. 8 */
    int m = (int)(v / ldexp(1.0, ex - 3)) - 8;                     /* 0 .. 7 */
    return sign | (uint8_t)(((ex + 7) << 3) | m);
}

/* fp32 -> bf16 bits, round to nearest even (NaN keeps a quiet NaN). */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lower = u & 0xFFFF, upper = u >> 16;
    if (lower > 0x8000 || (lower == 0x8000 && (upper & 1))) upper += 1;
    return (uint16_t)upper;
}

/*
 * Writes n tokens into a cache seen as num_rows rows of dim elements.
 *   x             [n][dim] of x_dtype (fp32 or bf16)
 *   slot_mapping  [n]: cache row of token i (page * page_size + row in page);
 *                 a negative entry skips the token
 *   cache_data    [num_rows][dim] of cache_dtype; cache_scale [num_rows] fp32
 * FP8 cache: amax = max_e |x_e| (fp32), scale = amax / 448 rounded to fp32 (1
 * when amax = 0 or the quotient underflows to 0); code_e = e4m3(x_e / scale),
 * the quotient an IEEE fp32 division, then rounded to e4m3 (nearest even,
 * saturating at +-448).  Dequantisation is code * scale, so the codes are x in
 * units of the scale.  BF16 cache: x rounded to bf16.  FP32 cache: x as is.  The scale
 * of a non-FP8 cache is left untouched.  Returns -1 (after writing the valid
 * tokens) if a slot is >= num_rows.
 */
int oracle_cache_store(const void* x, int x_dtype, int64_t n, int dim,
                       const int64_t* slot_mapping, void* cache_data, int cache_dtype,
                       float* cache_scale, int64_t num_rows) {
    int bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= num_rows) {
            bad = 1;
            continue;
        }
        float* row = (float*)malloc((size_t)dim * sizeof(float));
        for (int d = 0; d < dim; ++d) row[d] = (float)load_elem(x, x_dtype, i * dim + d);
        if (cache_dtype == OR_E4M3) {
            float amax = 0.0f;
            for (int d = 0; d < dim; ++d)
                if (fabsf(row[d]) > amax) amax = fabsf(row[d]);
            volatile float scale = amax / 448.0f;
            if (!(scale > 0.0f)) scale = 1.0f;            /* amax = 0 or underflow */
            uint8_t* dst = (uint8_t*)cache_data + slot * dim;
            for (int d = 0; d < dim; ++d) {
                volatile float quotient = row[d] / scale;
                dst[d] = oracle_f32_to_e4m3(quotient);
            }
            cache_scale[slot] = scale;
        } else if (cache_dtype == OR_BF16) {
            uint16_t* dst = (uint16_t*)cache_data + slot * dim;
            for (int d = 0; d < dim; ++d) dst[d] = oracle_f32_to_bf16(row[d]);
        } else {
            float* dst = (float*)cache_data + slot * dim;
            for (int d = 0; d < dim; ++d) dst[d] = row[d];
        }
        free(row);
    }
    return bad ? -1 : 0;
}
