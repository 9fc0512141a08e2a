/*
 * pivot_oracle.c -- plain, slow CPU oracle for the PIVOT indexer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * path.
 *
 * Sources (cited by page title and section):
 *  [ABS]  "PIVOT: Efficient Query-Group Indexing for Token-Level Sparse
 *         Attention", arXiv 2607.24593, English abstract (arxivdaily.com
 *         entry).  Grouping of nearby queries, the averaged proxy query, one
 *         full-prefix scan per group giving a candidate set, PIVOT-Reuse
 *         (the proxy's top-k shared by the group) and PIVOT-Refine (each
 *         member re-scores the candidate set with its own indexer and takes
 *         its own top-k); prefill groups are consecutive queries, decode
 *         groups are the tokens of one MTP step.
 *  [BLOG] "PIVOT 설명: 논문에서 작동하는 코드로 10분 만에 구현하기"
 *         (molayo1419.me), section "작동 방식 (How It Works)": the proxy is
 *         the mean of the group; O(L^2) -> O(L^2/g).
 *  [TUT]  "Sparse Attention의 Indexer: 내용에 따라 읽을 위치 고르기"
 *         (ai-systems-engineering.com), Fig. 1 (selection score = indexer
 *         query . indexer key, top-k returns positions only), Fig. 2 (the
 *         query at p_t may pick positions 0..t, itself included), Fig. 3
 *         (union with a recent window, deduplicated).
 *  The score with several heads, I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]),
 *  is the DeepSeek-style lightning-indexer form; [TUT] "선택용 Query와
 *  Key로 위치 고르기" says the real indexer uses several heads, and with one
 *  head, w = 1 and non-negative dot products the form reduces to Fig. 1's
 *  plain dot product.
 *
 * Readings where the pages are silent:
 *  - causal prefix is inclusive: query t sees s in [0, t]        ([TUT] Fig. 2)
 *  - selection: the k highest scores, equal scores lower position first;
 *    -0 == +0; the selected positions are listed in ascending order (the
 *    tutorial's Fig. 1 lists the picked positions by position)
 *  - a candidate row lists the proxy's top-k first, then the rest of its
 *    top-C, each ascending (Reuse shares the proxy's top-k)
 *  - fewer eligible positions than k: return them all, pad with -1
 *  - a group's full prefix runs through its last member e_j
 *  - the proxy averages both q and w, per head; a last partial group
 *    averages over its actual members; a one-member group is copied as is
 *  - FP8 proxy: average the dequantised values in fp32, then requantise with
 *    one scale amax/448 per proxy, e4m3 round-to-nearest-even, saturating
 *  - Reuse masks in-group future positions and pads with -1 (no backfill)
 *  - decode member m of Gm sees [0, cache_len - Gm + m]; the proxy scan
 *    sees [0, cache_len - 1]
 *
 * Arithmetic: scores in fp64 from the decoded input values; the proxy in
 * fp32, sequential in member order, compiled without FMA contraction, since
 * that is the precision the stored proxy has.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

/* ------------------------------------------------------------------------ */
/* Number formats, written from their definitions.                           */
/* ------------------------------------------------------------------------ */

/* OCP 8-bit float E4M3 ("fn" variant): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite
 * value 1.75 * 2^8 = 448, subnormals m/8 * 2^-6. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round |x| to the nearest value with `bits` significant bits and minimum
 * exponent `emin` (below it the quantum stays 2^(emin-bits+1)), ties to
 * even.  Exact in double for fp32 inputs. */
static double round_sig_rne(double a, int bits, int emin) {
    if (a == 0.0) return 0.0;
    int E;
    frexp(a, &E);            /* a = f * 2^E, f in [0.5,1): leading bit 2^(E-1) */
    int lead = E - 1;
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - (bits - 1));
    double n = nearbyint(a / quantum);   /* default mode: ties to even */
    return n * quantum;
}

uint8_t oracle_double_to_e4m3_satfinite(double x) {
    if (isnan(x)) return 0x7F;
    int sign = signbit(x) ? 1 : 0;
    double a = fabs(x);
    double r = round_sig_rne(a, 4, -6);
    if (r > 448.0) r = 448.0;
    uint8_t code;
    if (r == 0.0) {
        code = 0;
    } else if (r < ldexp(1.0, -6)) {
        code = (uint8_t)(r / ldexp(1.0, -9));          /* subnormal */
    } else {
        int E;
        double f = frexp(r, &E);                       /* r = (2f) * 2^(E-1) */
        int ef = E - 1 + 7;
        int m = (int)((2.0 * f - 1.0) * 8.0);
        code = (uint8_t)((ef << 3) | m);
    }
    return (uint8_t)(code | (sign << 7));
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* binary32 -> bfloat16, round to nearest even: 8 significant bits, same
 * exponent range as binary32 (minimum normal exponent -126). */
uint16_t oracle_float_to_bf16_rne(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x40);
    int sign = signbit(x) ? 1 : 0;
    double r = round_sig_rne(fabs((double)x), 8, -126);
    float rf = (float)r;                               /* exact: 8 bits */
    if (isinf(r) || r > 3.3895313892515355e38) rf = INFINITY;
    uint32_t v;
    memcpy(&v, &rf, 4);
    return (uint16_t)((v >> 16) | (sign << 15));
}

/* One stored element as a double (without any scale). */
static double decode(int dtype, const void* p, size_t i) {
    switch (dtype) {
    case OR_F32: return (double)((const float*)p)[i];
    case OR_BF16: return oracle_bf16_to_double(((const uint16_t*)p)[i]);
    default: return oracle_e4m3_to_double(((const uint8_t*)p)[i]);
    }
}

/* ------------------------------------------------------------------------ */
/* The indexer score and top-k ([TUT] Fig. 1, Fig. 2; multi-head form).      */
/* ------------------------------------------------------------------------ */

/* Indexer score of one query row against one key:
 *   I = sum_h w[h] * max(0, sum_d qx[h,d] * kx[d])
 * where qx = stored q value * q scale and kx = stored k value * k scale.
 * qd is the query row decoded to doubles [H*D], kd one key [D]. */
static double indexer_score(int H, int D, const double* qd, const float* wrow,
                            const double* kd) {
    double total = 0.0;
    for (int h = 0; h < H; ++h) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qd[(size_t)h * D + d] * kd[d];
        double relu = dot > 0.0 ? dot : 0.0;
        total += (double)wrow[h] * relu;
    }
    return total + 0.0;   /* -0 becomes +0 */
}

typedef struct { double score; int32_t pos; } entry_t;

/* Higher score first; equal scores by lower position. */
static int entry_cmp(const void* a, const void* b) {
    const entry_t* x = (const entry_t*)a;
    const entry_t* y = (const entry_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

/* Ascending position. */
static int pos_cmp(const void* a, const void* b) {
    const entry_t* x = (const entry_t*)a;
    const entry_t* y = (const entry_t*)b;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

/* Select the min(k, n) best entries (rank order: higher score, then lower
 * position) and write their positions (and scores) in ascending position
 * order -- the first min(split, k, n) best first, then the rest, when split
 * is in (0, k); pad the rest of the k slots with -1 (and -inf). */
static void take_topk_split(entry_t* e, int n, int k, int split, int32_t* out_idx,
                            double* out_score) {
    qsort(e, (size_t)n, sizeof(entry_t), entry_cmp);
    int m = n < k ? n : k;
    int s = (split > 0 && split < m) ? split : 0;
    if (s) {
        qsort(e, (size_t)s, sizeof(entry_t), pos_cmp);
        qsort(e + s, (size_t)(m - s), sizeof(entry_t), pos_cmp);
    } else {
        qsort(e, (size_t)m, sizeof(entry_t), pos_cmp);
    }
    for (int i = 0; i < k; ++i) {
        if (i < n) {
            out_idx[i] = e[i].pos;
            if (out_score) out_score[i] = e[i].score;
        } else {
            out_idx[i] = -1;
            if (out_score) out_score[i] = -INFINITY;
        }
    }
}

static void take_topk(entry_t* e, int n, int k, int32_t* out_idx, double* out_score) {
    take_topk_split(e, n, k, 0, out_idx, out_score);
}

/* Decode a query row (H*D values, times its scale) into qd. */
static void decode_qrow(int dtype, const void* q, const float* q_scale, size_t row,
                        int H, int D, double* qd) {
    double s = q_scale ? (double)q_scale[row] : 1.0;
    size_t base = row * (size_t)H * D;
    for (size_t i = 0; i < (size_t)H * D; ++i) qd[i] = decode(dtype, q, base + i) * s;
}

/* Decode keys [0, n) of a key array (row stride D) into kd[n*D]. */
static double* decode_keys(int dtype, const void* k, const float* k_scale, int n, int D) {
    double* kd = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    for (int s = 0; s < n; ++s) {
        double sc = k_scale ? (double)k_scale[s] : 1.0;
        for (int d = 0; d < D; ++d)
            kd[(size_t)s * D + d] = decode(dtype, k, (size_t)s * D + d) * sc;
    }
    return kd;
}

/* Top-k of one query row over keys [0, lim] (lim inclusive); with split in
 * (0, k) the best `split` are listed first. */
static void row_topk_prefix(int H, int D, const double* qd, const float* wrow,
                            const double* kd, int lim, int k, int split,
                            int32_t* out_idx, double* out_score) {
    int n = lim + 1;
    entry_t* e = (entry_t*)malloc(sizeof(entry_t) * (size_t)(n > 0 ? n : 1));
    for (int s = 0; s < n; ++s) {
        e[s].pos = s;
        e[s].score = indexer_score(H, D, qd, wrow, kd + (size_t)s * D);
    }
    take_topk_split(e, n, k, split, out_idx, out_score);
    free(e);
}

/* Scores of one query row against explicit key positions (no sorting),
 * for the tests' brute-force checks. out[i] = I(row, pos[i]); L here is the
 * number of keys (positions outside [0, L) give NaN). */
int oracle_score_positions(int dtype, int L, int H, int D, const void* q,
                           const float* q_scale, const float* w, const void* k,
                           const float* k_scale, int row, int npos,
                           const int32_t* pos, double* out) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
    double* kd = (double*)malloc(sizeof(double) * (size_t)D);
    decode_qrow(dtype, q, q_scale, (size_t)row, H, D, qd);
    for (int i = 0; i < npos; ++i) {
        int s = pos[i];
        if (s < 0 || s >= L) { out[i] = NAN; continue; }
        double sc = k_scale ? (double)k_scale[s] : 1.0;
        for (int d = 0; d < D; ++d) kd[d] = decode(dtype, k, (size_t)s * D + d) * sc;
        out[i] = indexer_score(H, D, qd, w + (size_t)row * H, kd);
    }
    free(qd);
    free(kd);
    return 0;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Dense indexer for the listed query rows: row t takes the top-k of
 * I(t, s) over s in [0, t].  out_idx / out_score are [nrows, k]. */
int oracle_dense_index(int dtype, int L, int H, int D, const void* q,
                       const float* q_scale, const float* w, const void* k,
                       const float* k_scale, int topk, int nrows,
                       const int32_t* rows, int32_t* out_idx, double* out_score,
                       int nthreads) {
    set_threads(nthreads);
    double* kd = decode_keys(dtype, k, k_scale, L, D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r];
        double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
        decode_qrow(dtype, q, q_scale, (size_t)t, H, D, qd);
        row_topk_prefix(H, D, qd, w + (size_t)t * H, kd, t, topk, 0,
                        out_idx + (size_t)r * topk,
                        out_score ? out_score + (size_t)r * topk : NULL);
        free(qd);
    }
    free(kd);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Proxy query ([BLOG] "How It Works": mean of the group; [ABS]).            */
/* ------------------------------------------------------------------------ */

/* Proxy of the members [t0, t0 + n) of one group, in fp32:
 *   x_m        = q value * q scale (one fp32 multiply; no scale: the value)
 *   qbar[h,d]  = (x_0 + x_1 + ... + x_{n-1}) / n    (left to right, fp32)
 *   wbar[h]    = (w_0 + ... + w_{n-1}) / n          (same)
 * then stored in the input's format: f32 as is; bf16 rounded to nearest
 * even; e4m3 with one scale s = amax/448 (s = 1 when amax = 0) and codes
 * e4m3(qbar / s), rounded to nearest even, saturating.  A group of one
 * member is that member, copied without requantisation. */
static void proxy_one(int dtype, int H, int D, const void* q, const float* q_scale,
                      const float* w, int t0, int n, void* pq_row,
                      float* pq_scale_out, float* pw_row) {
    size_t HD = (size_t)H * D;
    if (n == 1) {
        size_t esz = dtype == OR_F32 ? 4 : dtype == OR_BF16 ? 2 : 1;
        memcpy(pq_row, (const char*)q + (size_t)t0 * HD * esz, HD * esz);
        if (pq_scale_out) *pq_scale_out = q_scale ? q_scale[t0] : 1.0f;
        memcpy(pw_row, w + (size_t)t0 * H, sizeof(float) * H);
        return;
    }
    float* qbar = (float*)malloc(sizeof(float) * HD);
    for (size_t i = 0; i < HD; ++i) {
        float acc = 0.0f;
        for (int m = 0; m < n; ++m) {
            size_t row = (size_t)(t0 + m);
            float x = (float)decode(dtype, q, row * HD + i);  /* exact in fp32 */
            if (dtype == OR_E4M3) x = x * q_scale[row];
            acc = (m == 0) ? x : acc + x;
        }
        qbar[i] = acc / (float)n;
    }
    for (int h = 0; h < H; ++h) {
        float acc = 0.0f;
        for (int m = 0; m < n; ++m) {
            float x = w[(size_t)(t0 + m) * H + h];
            acc = (m == 0) ? x : acc + x;
        }
        pw_row[h] = acc / (float)n;
    }
    if (dtype == OR_F32) {
        memcpy(pq_row, qbar, sizeof(float) * HD);
    } else if (dtype == OR_BF16) {
        for (size_t i = 0; i < HD; ++i) ((uint16_t*)pq_row)[i] = oracle_float_to_bf16_rne(qbar[i]);
    } else {
        float amax = 0.0f;
        for (size_t i = 0; i < HD; ++i) {
            float a = fabsf(qbar[i]);
            if (a > amax) amax = a;
        }
        float s = amax > 0.0f ? amax / 448.0f : 1.0f;
        for (size_t i = 0; i < HD; ++i) {
            float y = qbar[i] / s;
            ((uint8_t*)pq_row)[i] = oracle_double_to_e4m3_satfinite((double)y);
        }
        *pq_scale_out = s;
    }
    free(qbar);
}

/* Prefill groups: group j holds queries [j*g, min(L, (j+1)*g)).  Writes the
 * proxies of the listed groups, compactly: pq [ngroups, H, D] in the input
 * format, pq_scale [ngroups] (e4m3 only, else may be NULL), pw [ngroups, H]. */
int oracle_proxy_reduce(int dtype, int L, int H, int D, const void* q,
                        const float* q_scale, const float* w, int g, int ngroups,
                        const int32_t* groups, void* pq, float* pq_scale, float* pw) {
    size_t esz = dtype == OR_F32 ? 4 : dtype == OR_BF16 ? 2 : 1;
    for (int r = 0; r < ngroups; ++r) {
        int j = groups[r];
        int t0 = j * g;
        int n = (L - t0) < g ? (L - t0) : g;
        proxy_one(dtype, H, D, q, q_scale, w, t0, n,
                  (char*)pq + (size_t)r * H * D * esz,
                  pq_scale ? pq_scale + r : NULL, pw + (size_t)r * H);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* One full-prefix proxy scan per group ([ABS]; [BLOG] O(L^2/g)).             */
/* ------------------------------------------------------------------------ */

/* For each listed group j: the indexer score of proxy j (rows of pq / pw /
 * pq_scale indexed by j, full [G, ...] arrays) over the prefix [0, e_j],
 * e_j = min(L, (j+1)g) - 1, and its top-C -> cand [ngroups, C]: the top
 * `topk` by position, then the rest by position. */
int oracle_proxy_scan(int dtype, int L, int H, int D, const void* pq,
                      const float* pq_scale, const float* pw, const void* k,
                      const float* k_scale, int g, int C, int topk, int ngroups,
                      const int32_t* groups, int32_t* cand, double* cand_score,
                      int nthreads) {
    set_threads(nthreads);
    double* kd = decode_keys(dtype, k, k_scale, L, D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < ngroups; ++r) {
        int j = groups[r];
        int e = ((j + 1) * g < L ? (j + 1) * g : L) - 1;
        double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
        decode_qrow(dtype, pq, pq_scale, (size_t)j, H, D, qd);
        row_topk_prefix(H, D, qd, pw + (size_t)j * H, kd, e, C, topk,
                        cand + (size_t)r * C, cand_score ? cand_score + (size_t)r * C : NULL);
        free(qd);
    }
    free(kd);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* PIVOT-Reuse ([ABS]): the proxy's top-k, shared by every member.           */
/* ------------------------------------------------------------------------ */

/* Member t of group j = t / g: the first k entries of cand[j] (the proxy's
 * top-k), keeping only positions <= t in their order, padded with -1.
 * cand is the full [G, C]; out is [nrows, k]. */
int oracle_reuse(int L, int g, const int32_t* cand, int C, int topk, int nrows,
                 const int32_t* rows, int32_t* out_idx) {
    (void)L;
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r];
        int j = t / g;
        int32_t* o = out_idx + (size_t)r * topk;
        int n = 0;
        for (int i = 0; i < topk && i < C; ++i) {
            int32_t s = cand[(size_t)j * C + i];
            if (s >= 0 && s <= t) o[n++] = s;
        }
        for (; n < topk; ++n) o[n] = -1;
    }
    return 0;
}

/* Reuse with backfill (a reading the pages leave open: [BLOG] "How It Works"
 * says only that members share the proxy's choice).  Member t of group j
 * takes, among the entries of cand[j] at positions <= t, the k with the
 * highest proxy score (cand_score[j], lower position first on ties): the
 * proxy's top-k where none of it is masked, else the next-ranked candidates
 * fill the masked slots.  Ascending positions, -1 padding. */
int oracle_reuse_backfill(int L, int g, const int32_t* cand, const double* cand_score, int C,
                          int topk, int nrows, const int32_t* rows, int32_t* out_idx) {
    (void)L;
    entry_t* e = (entry_t*)malloc(sizeof(entry_t) * (size_t)(C > 0 ? C : 1));
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r];
        int j = t / g;
        int n = 0;
        for (int i = 0; i < C; ++i) {
            int32_t s = cand[(size_t)j * C + i];
            if (s >= 0 && s <= t) {
                e[n].score = cand_score[(size_t)j * C + i];
                e[n].pos = s;
                ++n;
            }
        }
        take_topk(e, n, topk, out_idx + (size_t)r * topk, NULL);
    }
    free(e);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* PIVOT-Refine ([ABS]): each member re-scores the candidate set.            */
/* ------------------------------------------------------------------------ */

/* Member t of group j: I(t, s) with t's own q, w for every s in cand[j]
 * with 0 <= s <= t, then the top-k.  cand is the full [G, C]. */
int oracle_refine(int dtype, int L, int H, int D, const void* q,
                  const float* q_scale, const float* w, const void* k,
                  const float* k_scale, int g, const int32_t* cand, int C, int topk,
                  int nrows, const int32_t* rows, int32_t* out_idx,
                  double* out_score, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r];
        int j = t / g;
        double* qd = (double*)malloc(sizeof(double) * (size_t)H * D);
        double* kd = (double*)malloc(sizeof(double) * (size_t)D);
        entry_t* e = (entry_t*)malloc(sizeof(entry_t) * (size_t)C);
        decode_qrow(dtype, q, q_scale, (size_t)t, H, D, qd);
        int n = 0;
        for (int i = 0; i < C; ++i) {
            int32_t s = cand[(size_t)j * C + i];
            if (s < 0 || s > t || s >= L) continue;
            double sc = k_scale ? (double)k_scale[s] : 1.0;
            for (int d = 0; d < D; ++d) kd[d] = decode(dtype, k, (size_t)s * D + d) * sc;
            e[n].pos = s;
            e[n].score = indexer_score(H, D, qd, w + (size_t)t * H, kd);
            ++n;
        }
        take_topk(e, n, topk, out_idx + (size_t)r * topk,
                  out_score ? out_score + (size_t)r * topk : NULL);
        free(e);
        free(kd);
        free(qd);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode ([ABS]: the Gm tokens of one MTP step form one group).              */
/* ------------------------------------------------------------------------ */

/* One decode step for B sequences.  q [B, Gm, H, D], q_scale [B, Gm] (e4m3),
 * w [B, Gm, H]; key cache kc [B, maxlen, D], kc_scale [B, maxlen] (e4m3);
 * cache_len [B] counts the Gm new tokens' keys, already appended.
 * Member m sees [0, cache_len - Gm + m]; the proxy sees [0, cache_len - 1].
 * mode 0 = dense, 1 = Reuse, 2 = Refine.  out_idx [B, Gm, k]; cand_out
 * [B, C] (modes 1, 2; may be NULL), laid out as in the proxy scan.  Sequences are processed one at a time
 * with the same steps as prefill. */
int oracle_decode(int dtype, int B, int Gm, int H, int D, const void* q,
                  const float* q_scale, const float* w, const void* kc,
                  const float* kc_scale, int maxlen, const int32_t* cache_len,
                  int mode, int C, int topk, int32_t* out_idx, int32_t* cand_out,
                  double* out_score, int nthreads) {
    set_threads(nthreads);
    size_t esz = dtype == OR_F32 ? 4 : dtype == OR_BF16 ? 2 : 1;
    size_t HD = (size_t)H * D;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int n = cache_len[b];
        const void* kb = (const char*)kc + (size_t)b * maxlen * D * esz;
        const float* kbs = kc_scale ? kc_scale + (size_t)b * maxlen : NULL;
        double* kd = decode_keys(dtype, kb, kbs, n, D);
        double* qd = (double*)malloc(sizeof(double) * HD);
        const void* qb = (const char*)q + (size_t)b * Gm * HD * esz;
        const float* qbs = q_scale ? q_scale + (size_t)b * Gm : NULL;
        const float* wb = w + (size_t)b * Gm * H;
        int32_t* ob = out_idx + (size_t)b * Gm * topk;
        double* osb = out_score ? out_score + (size_t)b * Gm * topk : NULL;
        if (mode == 0) {
            for (int m = 0; m < Gm; ++m) {
                decode_qrow(dtype, qb, qbs, (size_t)m, H, D, qd);
                row_topk_prefix(H, D, qd, wb + (size_t)m * H, kd, n - Gm + m, topk, 0,
                                ob + (size_t)m * topk, osb ? osb + (size_t)m * topk : NULL);
            }
        } else {
            void* pq = malloc(HD * esz);
            float pqs = 1.0f;
            float* pw = (float*)malloc(sizeof(float) * H);
            int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * C);
            proxy_one(dtype, H, D, qb, qbs, wb, 0, Gm, pq, &pqs, pw);
            decode_qrow(dtype, pq, dtype == OR_E4M3 ? &pqs : NULL, 0, H, D, qd);
            row_topk_prefix(H, D, qd, pw, kd, n - 1, C, topk, cand, NULL);
            if (cand_out) memcpy(cand_out + (size_t)b * C, cand, sizeof(int32_t) * C);
            for (int m = 0; m < Gm; ++m) {
                int lim = n - Gm + m;
                int32_t* o = ob + (size_t)m * topk;
                if (mode == 1) {
                    int c = 0;
                    for (int i = 0; i < topk && i < C; ++i)
                        if (cand[i] >= 0 && cand[i] <= lim) o[c++] = cand[i];
                    for (; c < topk; ++c) o[c] = -1;
                } else {
                    entry_t* e = (entry_t*)malloc(sizeof(entry_t) * (size_t)C);
                    decode_qrow(dtype, qb, qbs, (size_t)m, H, D, qd);
                    int c = 0;
                    for (int i = 0; i < C; ++i) {
                        int32_t s = cand[i];
                        if (s < 0 || s > lim) continue;
                        e[c].pos = s;
                        e[c].score = indexer_score(H, D, qd, wb + (size_t)m * H,
                                                   kd + (size_t)s * D);
                        ++c;
                    }
                    take_topk(e, c, topk, o, osb ? osb + (size_t)m * topk : NULL);
                    free(e);
                }
            }
            free(cand);
            free(pw);
            free(pq);
        }
        free(qd);
        free(kd);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Window union ([TUT] Fig. 3): a helper for the worked example only.        */
/* ------------------------------------------------------------------------ */

/* Union of the selected positions with the window [t - win + 1, t],
 * deduplicated, ascending.  Returns the count written to out. */
int oracle_window_union(const int32_t* sel, int nsel, int t, int win, int32_t* out) {
    int n = 0;
    int lo = t - win + 1 < 0 ? 0 : t - win + 1;
    for (int p = 0; p <= t; ++p) {
        int take = (p >= lo);
        for (int i = 0; i < nsel && !take; ++i) take = (sel[i] == p);
        if (take) out[n++] = p;
    }
    return n;
}
