/*
 * DSA oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU implementation of the DeepSeek-Sparse-Attention hot path used to
 * check the CUDA library.  Only the tests, the package smoke check and the benchmark's CPU
 * baseline may load it.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes, for a query token at absolute position t (keys s = 0..t, causal, self
 * included):
 *
 *  1. Lightning-indexer scores
 *       score(t, s) = sum_h w[t,h] * max(0, sum_d qI[t,h,d] * kI[s,d])
 *     The pages describe a light "scout" module with one MQA-shared key per position that
 *     scans every position and scores it for the current token (page "快手开源大模型
 *     Keye-VL-2.0：一个能“看懂“两小时视频AI", gsyq.cn, section 一).  They give no formula;
 *     this is the formula the library adopts: no scale, no bias, w used as is (it may be
 *     negative).
 *  2. Top-k selection
 *       S_t = the first min(k, t+1) keys of 0..t ordered by (score descending, index
 *       ascending)
 *     (same page, section 一: keep the 2048 most relevant positions per token; page
 *     "从“看”到“想”多模态大模型推理能力的瓶颈与突破", wmrh.cn, section 2, step 2:
 *     keep only the k best-scored key/value pairs).  Ties go to the lower index.
 *  3. Sparse scaled-dot-product attention over S_t, one set shared by every KV group
 *     (GQA: query head h reads KV head g = h / (Hq/Hkv))
 *       z_s = scale * sum_d q[t,h,d] * k[s,g,d],  p_s = exp(z_s - max z) / sum exp(...)
 *       out[t,h,:] = sum_s p_s v[s,g,:],          lse[t,h] = max z + log(sum exp(...))
 *     (wmrh.cn page, section 2, step 3: standard scaled dot-product attention on the
 *     selected candidates; gsyq.cn page, section 一: GQA adaptation of DSA).
 *
 *  4. Indexer warm-up target (forward only; the pages' training stage 1 fits the scout to the
 *     full attention distribution by minimising a KL divergence: gsyq.cn page, section 一, the
 *     "dense warm-up" paragraph; the pages give no formula, this is the plainest reading):
 *       P_t(s) = (1/Hq) sum_h softmax_s(scale * q[t,h] . k[s,g(h)])   over s = 0..t (dense)
 *       Q_t(s) = softmax_s(score(t, s))                                over s = 0..t
 *       KL_t   = sum_s P_t(s) * (log P_t(s) - log Q_t(s))   (a term with P_t(s) = 0 adds 0)
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.  Every product
 * of two bf16 values is exact in double, so the scores are the true scores up to the
 * rounding of the fp64 sums.  Rows are independent: OpenMP splits them over host cores.
 * Index entries of -1 (rows with fewer than k causal keys) are skipped in step 3.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Step 1 for one query row: scores[s] for s = 0..n_keys-1. */
static void index_row(const uint16_t *qI_row, const uint16_t *w_row, const uint16_t *kI, int64_t n_keys,
                      int HI, int dI, double *scores) {
    for (int64_t s = 0; s < n_keys; ++s) {
        const uint16_t *ks = kI + s * dI;
        double total = 0.0;
        for (int h = 0; h < HI; ++h) {
            const uint16_t *qh = qI_row + (int64_t)h * dI;
            double dot = 0.0;
            for (int d = 0; d < dI; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(ks[d]);
            double relu = dot > 0.0 ? dot : 0.0;
            total += bf16_to_double(w_row[h]) * relu;
        }
        scores[s] = total;
    }
}

typedef struct {
    double score;
    int32_t idx;
} scored_key;

/* Order for step 2: larger score first; equal scores, lower index first. */
static int by_score_then_index(const void *pa, const void *pb) {
    const scored_key *a = (const scored_key *)pa, *b = (const scored_key *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

/* Step 2 for one row, keys lo..n-1 competing: idx[0..k) = first min(k, n-lo) of them in that
 * order, then -1.  Returns the score of the last selected key (the k-th score when n-lo >= k). */
static double topk_row(const double *scores, int64_t lo, int64_t n, int k, int32_t *idx) {
    int64_t c = n - lo;
    scored_key *buf = (scored_key *)malloc((size_t)(c > 0 ? c : 1) * sizeof(scored_key));
    for (int64_t s = lo; s < n; ++s) {
        buf[s - lo].score = scores[s];
        buf[s - lo].idx = (int32_t)s;
    }
    qsort(buf, (size_t)c, sizeof(scored_key), by_score_then_index);
    int64_t m = c < k ? c : k;
    for (int64_t j = 0; j < m; ++j) idx[j] = buf[j].idx;
    for (int64_t j = m; j < k; ++j) idx[j] = -1;
    double tau = m > 0 ? buf[m - 1].score : 0.0;
    free(buf);
    return tau;
}

/* Step 3 for one row and all heads. kc, vc: [Lk, Hkv, D]. */
static void attend_row(const uint16_t *q_row, const uint16_t *kc, const uint16_t *vc, const int32_t *idx, int k,
                       int Hq, int Hkv, int D, double scale, double *out_row, double *lse_row) {
    int G = Hq / Hkv;
    double *z = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof(double));
    for (int h = 0; h < Hq; ++h) {
        int g = h / G;
        const uint16_t *qh = q_row + (int64_t)h * D;
        double zmax = -INFINITY;
        int used = 0;
        for (int j = 0; j < k; ++j) {
            if (idx[j] < 0) {
                z[j] = -INFINITY;
                continue;
            }
            const uint16_t *ks = kc + ((int64_t)idx[j] * Hkv + g) * D;
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(ks[d]);
            z[j] = scale * dot;
            if (z[j] > zmax) zmax = z[j];
            ++used;
        }
        double *o = out_row + (int64_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (used == 0) {
            if (lse_row) lse_row[h] = -INFINITY;
            continue;
        }
        double denom = 0.0;
        for (int j = 0; j < k; ++j) {
            if (idx[j] < 0) continue;
            double p = exp(z[j] - zmax);
            denom += p;
            const uint16_t *vs = vc + ((int64_t)idx[j] * Hkv + g) * D;
            for (int d = 0; d < D; ++d) o[d] += p * bf16_to_double(vs[d]);
        }
        for (int d = 0; d < D; ++d) o[d] /= denom;
        if (lse_row) lse_row[h] = zmax + log(denom);
    }
    free(z);
}

/* Step 4 for one query row with n = t + 1 keys. */
static double kl_row(const uint16_t *q_row, const uint16_t *kc, const uint16_t *qI_row, const uint16_t *w_row,
                     const uint16_t *kI, int64_t n, int Hq, int Hkv, int D, int HI, int dI, double scale) {
    int G = Hq / Hkv;
    double *z = (double *)malloc((size_t)n * sizeof(double));
    double *P = (double *)calloc((size_t)n, sizeof(double));
    double *I = (double *)malloc((size_t)n * sizeof(double));
    /* P: the dense attention distribution of every head, averaged over heads */
    for (int h = 0; h < Hq; ++h) {
        int g = h / G;
        const uint16_t *qh = q_row + (int64_t)h * D;
        double zmax = -INFINITY;
        for (int64_t s = 0; s < n; ++s) {
            const uint16_t *ks = kc + (s * Hkv + g) * D;
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(ks[d]);
            z[s] = scale * dot;
            if (z[s] > zmax) zmax = z[s];
        }
        double denom = 0.0;
        for (int64_t s = 0; s < n; ++s) denom += exp(z[s] - zmax);
        for (int64_t s = 0; s < n; ++s) P[s] += exp(z[s] - zmax) / denom / (double)Hq;
    }
    /* log Q: log-softmax of the indexer scores */
    index_row(qI_row, w_row, kI, n, HI, dI, I);
    double imax = -INFINITY;
    for (int64_t s = 0; s < n; ++s) imax = I[s] > imax ? I[s] : imax;
    double isum = 0.0;
    for (int64_t s = 0; s < n; ++s) isum += exp(I[s] - imax);
    double lse_i = imax + log(isum);
    double kl = 0.0;
    for (int64_t s = 0; s < n; ++s)
        if (P[s] > 0.0) kl += P[s] * (log(P[s]) - (I[s] - lse_i));
    free(z);
    free(P);
    free(I);
    return kl;
}

/* ------------------------------------------------------------------------------------- */
/* Exported entry points.  Row r of every per-row array belongs to query position t_rows[r]. */

/* Step 1.  qI: [nr, HI, dI], w: [nr, HI], kI: [>= max t + 1, dI].
 * scores[r * ld + s] for s <= t_rows[r]; other entries are not written. */
void oracle_index_rows(const uint16_t *qI, const uint16_t *w, const uint16_t *kI, const int64_t *t_rows,
                       int64_t nr, int HI, int dI, double *scores, int64_t ld) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r)
        index_row(qI + r * HI * dI, w + r * HI, kI, t_rows[r] + 1, HI, dI, scores + r * ld);
}

/* Step 2.  n_valid[r] keys per row (t + 1 for a causal row); with first[r] (nullable) only keys
 * first[r] .. n_valid[r]-1 compete (a sliding window).  tau[r] (nullable) receives the score of
 * the last selected key. */
void oracle_topk_rows(const double *scores, int64_t ld, const int64_t *n_valid, const int64_t *first, int64_t nr,
                      int k, int32_t *idx, double *tau) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r) {
        double t = topk_row(scores + r * ld, first ? first[r] : 0, n_valid[r], k, idx + r * k);
        if (tau) tau[r] = t;
    }
}

/* Step 3.  q: [nr, Hq, D]; kc, vc: [Lk, Hkv, D]; idx: [nr, k].  out: [nr, Hq, D]; lse: [nr, Hq]
 * (nullable). */
void oracle_sparse_attn_rows(const uint16_t *q, const uint16_t *kc, const uint16_t *vc, const int32_t *idx,
                             int64_t nr, int k, int Hq, int Hkv, int D, double scale, double *out, double *lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r)
        attend_row(q + r * Hq * D, kc, vc, idx + r * k, k, Hq, Hkv, D, scale, out + r * Hq * D,
                   lse ? lse + r * Hq : NULL);
}

/* Steps 1-3 for a set of rows of one causal sequence, without keeping more than one score row
 * per thread.  window > 0: only keys t-window+1 .. t compete in step 2 (sliding-window DSA,
 * page "DSA注意力机制：多模态学习中的强化推理新范式", showapi.com, section 1.4).  scores (nullable) [nr, ld] keeps the score rows; tau [nr] (nullable); absmax[nr]
 * (nullable) receives max_s |score(t, s)|. */
void oracle_dsa_rows(const uint16_t *q, const uint16_t *qI, const uint16_t *w, const uint16_t *kc,
                     const uint16_t *vc, const uint16_t *kI, const int64_t *t_rows, int64_t nr, int Hq, int Hkv,
                     int D, int HI, int dI, int k, int64_t window, double scale, int32_t *idx, double *out,
                     double *lse, double *scores, int64_t ld, double *tau, double *absmax) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r) {
        int64_t n = t_rows[r] + 1;
        double *row = scores ? scores + r * ld : (double *)malloc((size_t)n * sizeof(double));
        index_row(qI + r * HI * dI, w + r * HI, kI, n, HI, dI, row);
        if (absmax) {
            double m = 0.0;
            for (int64_t s = 0; s < n; ++s) m = fabs(row[s]) > m ? fabs(row[s]) : m;
            absmax[r] = m;
        }
        int64_t lo = (window > 0 && n > window) ? n - window : 0;
        double t = topk_row(row, lo, n, k, idx + r * k);
        if (tau) tau[r] = t;
        attend_row(q + r * Hq * D, kc, vc, idx + r * k, k, Hq, Hkv, D, scale, out + r * Hq * D,
                   lse ? lse + r * Hq : NULL);
        if (!scores) free(row);
    }
}

/* Step 4.  q: [nr, Hq, D], qI: [nr, HI, dI], w: [nr, HI]; k: [>= max t + 1, Hkv, D], kI: [>= max t + 1, dI].
 * kl[r] = KL(P_t || Q_t) for t = t_rows[r]. */
void oracle_kl_rows(const uint16_t *q, const uint16_t *kc, const uint16_t *qI, const uint16_t *w, const uint16_t *kI,
                    const int64_t *t_rows, int64_t nr, int Hq, int Hkv, int D, int HI, int dI, double scale,
                    double *kl) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r)
        kl[r] = kl_row(q + r * Hq * D, kc, qI + r * HI * dI, w + r * HI, kI, t_rows[r] + 1, Hq, Hkv, D, HI, dI,
                       scale);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
