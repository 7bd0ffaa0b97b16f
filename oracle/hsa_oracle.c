/*
 * hsa_oracle.c -- plain CPU float64 restatement of hierarchical chunk-sparse
 * landmark attention (HSA / HiLS / DHSA forward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle the CUDA path is checked
 * against.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load it; the library's product path never does.  It shares
 * no source, header, table or helper with the CUDA code.
 *
 * Everything is computed in double, one step after another, in the order the
 * method states them.  No blocking, fusion or reordering: a reader should be
 * able to check each step against the sources by eye.
 *
 * Sources (web pages) and the step each one defines:
 *  - HiLS Attention abstract (mlsift "length extrapolation" tag page): each
 *    query attends independently inside every retrieved chunk, and the chunk
 *    outputs are fused with weights given by the chunk retrieval scores.
 *  - Understanding and Improving Length Generalization in Hierarchical Sparse
 *    Attention Models (ai.info summary), "Methodology in Plain English": the
 *    sequence is cut into chunks of 64 tokens, each chunk has one landmark,
 *    the top-K (K = 8) chunks are retrieved per token ("Main Findings":
 *    per-token retrieval); upper layers combine local attention with the
 *    retrieved chunks.
 *  - Dynamic Hierarchical Sparse Attention (pith.science review), "What
 *    carries the argument": a chunk's key representation is sqrt(|C|) times
 *    the mean of its keys; TopK keeps the best-scoring ones.
 *
 * Readings taken where the pages leave a step open (each one is listed with
 * its reason in the design notes of the repository):
 *  R1  score = scale * q . l with scale = 1/sqrt(d) unless given; the same
 *      scale is used for the in-chunk logits.
 *  R2  fusion weights are a softmax over the *selected* chunks of the same
 *      per-head landmark scores.
 *  R3  selection is shared by the G query heads of a KV group; the group
 *      score is the mean of the heads' scores = scale * qbar . l.
 *  R4  query t may select only chunks that end before its own chunk
 *      c_t = floor(t / S); with own_chunk = 1 the causal attention over keys
 *      c_t*S .. t is added with weight 1.
 *  R5  fewer than K visible chunks: all of them are taken, indices padded
 *      with -1 and weights with 0.
 *  R6  order: higher score first, equal scores broken by lower chunk index.
 *  R12 decode: the query sits at position Lc, every one of the Lc/S chunks is
 *      visible, and there is no own-chunk term.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

/* One candidate chunk during selection. */
typedef struct {
    double score;
    int64_t index;
} candidate_t;

/* R6: higher score first; equal scores ordered by lower chunk index. */
static int candidate_order(const void *pa, const void *pb)
{
    const candidate_t *a = (const candidate_t *)pa;
    const candidate_t *b = (const candidate_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

static double dot(const double *x, const double *y, int n)
{
    double acc = 0.0;
    for (int j = 0; j < n; ++j) acc += x[j] * y[j];
    return acc;
}

/* Magnitude of the terms of the dot product x . y: sum_j |x_j * y_j|.  A
 * score computed in finite precision carries rounding errors relative to this
 * sum, not to the (possibly cancelled) value of the score itself; the near-tie
 * rule of the parity checks measures score gaps against it. */
static double abs_dot(const double *x, const double *y, int n)
{
    double acc = 0.0;
    for (int j = 0; j < n; ++j) acc += fabs(x[j] * y[j]);
    return acc;
}

/*
 * Ordinary softmax attention of one query over n consecutive key/value rows
 * (HiLS: attention "independently with each retrieved chunk").
 *   out = sum_j softmax_j(scale * q . k_j) * v_j
 * The maximum logit is subtracted before exponentiating, which leaves the
 * softmax unchanged.  logit is caller scratch of length >= n.
 */
static void chunk_attention(const double *q, const double *k, const double *v,
                            int64_t n, int d, double scale, double *logit, double *out)
{
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (n <= 0) return;
    double m = -INFINITY;
    for (int64_t r = 0; r < n; ++r) {
        logit[r] = scale * dot(q, k + r * d, d);
        if (logit[r] > m) m = logit[r];
    }
    double denom = 0.0;
    for (int64_t r = 0; r < n; ++r) {
        logit[r] = exp(logit[r] - m);
        denom += logit[r];
    }
    for (int64_t r = 0; r < n; ++r) {
        double p = logit[r] / denom;
        for (int j = 0; j < d; ++j) out[j] += p * v[r * d + j];
    }
}

/* softmax of n logits in place (R2). */
static void softmax_inplace(double *x, int n)
{
    if (n <= 0) return;
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) if (x[i] > m) m = x[i];
    double denom = 0.0;
    for (int i = 0; i < n; ++i) { x[i] = exp(x[i] - m); denom += x[i]; }
    for (int i = 0; i < n; ++i) x[i] /= denom;
}

/*
 * DHSA landmark (review, "What carries the argument"): the representation of
 * chunk C is sqrt(|C|) times the mean of its keys.  Only complete chunks
 * (Nc = floor(L / S)) have a landmark.
 *   k   [B, Hkv, L, d]
 *   out [B, Hkv, Nc, d]
 */
int hsa_oracle_landmarks(const double *k, int B, int Hkv, int64_t L, int d, int S, double *out)
{
    if (!k || !out || B < 1 || Hkv < 1 || L < 0 || d < 1 || S < 1) return ORACLE_BAD_ARG;
    const int64_t Nc = L / S;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg) {
        for (int64_t i = 0; i < Nc; ++i) {
            const double *kc = k + (bg * L + i * S) * d;
            double *l = out + (bg * Nc + i) * d;
            for (int j = 0; j < d; ++j) {
                double sum = 0.0;
                for (int r = 0; r < S; ++r) sum += kc[(int64_t)r * d + j];
                double mean = sum / (double)S;
                l[j] = sqrt((double)S) * mean;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Prefill forward for a list of query rows.
 *
 *   q          [n_rows, H, d]   the queries of the requested rows
 *   rows       [n_rows]         flattened position b*L + t of each row
 *   k, v       [B, Hkv, L, d]
 *   lm         [B, Hkv, Nc, d]  landmark input, or NULL for the DHSA form
 *                               computed here from k (Nc = floor(L/S))
 *   forced_idx [n_rows, Hkv, topk] or NULL: use these chunk indices (-1 pads)
 *                               instead of selecting; used to recompute a row
 *                               with another selection.
 * Outputs (any may be NULL except O):
 *   O          [n_rows, H, d]
 *   idx        [n_rows, Hkv, topk]  selected chunks in rank order, -1 padded
 *   w          [n_rows, H, topk]    fusion weights, 0 padded
 *   sbar       [n_rows, Hkv, topk]  group scores of the selected chunks
 *   gap        [n_rows, Hkv]        score(K-th) - score(K+1-th) of the group
 *                                   ranking, +inf when at most K chunks are
 *                                   visible, NaN with forced_idx
 *   smag       [n_rows, Hkv, topk+1] magnitude scale * sum_j |qbar_j l_ij| of
 *                                   the group score of each selected chunk in
 *                                   rank order (0 padded), and in the last
 *                                   slot that of the (K+1)-th ranked chunk
 *                                   (0 when there is none or with forced_idx)
 */
int hsa_oracle_prefill(const double *q, const int64_t *rows, int64_t n_rows,
                       const double *k, const double *v, const double *lm,
                       int B, int H, int Hkv, int64_t L, int d, int S, int topk,
                       int own_chunk, double scale, const int32_t *forced_idx,
                       double *O, int32_t *idx, double *w, double *sbar, double *gap,
                       double *smag)
{
    if (!q || !rows || !k || !v || !O) return ORACLE_BAD_ARG;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || L < 1 || d < 1 || S < 1 || topk < 1)
        return ORACLE_BAD_ARG;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * L) return ORACLE_BAD_ARG;
    const int G = H / Hkv;
    const int64_t Nc = L / S;
    if (scale == 0.0) scale = 1.0 / sqrt((double)d);

    double *lm_dhsa = NULL;
    if (!lm) {
        lm_dhsa = (double *)malloc(sizeof(double) * (size_t)B * Hkv * (Nc > 0 ? Nc : 1) * d);
        if (!lm_dhsa) return ORACLE_NO_MEMORY;
        hsa_oracle_landmarks(k, B, Hkv, L, d, S, lm_dhsa);
        lm = lm_dhsa;
    }
    int status = ORACLE_OK;

#pragma omp parallel
    {
        candidate_t *cand = (candidate_t *)malloc(sizeof(candidate_t) * (size_t)(Nc > 0 ? Nc : 1));
        double *qbar = (double *)malloc(sizeof(double) * d);
        double *logit = (double *)malloc(sizeof(double) * (size_t)(S > topk ? S : topk));
        double *o_part = (double *)malloc(sizeof(double) * d);
        double *o_row = (double *)malloc(sizeof(double) * d);
        double *wk = (double *)malloc(sizeof(double) * topk);
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * topk);
        if (!cand || !qbar || !logit || !o_part || !o_row || !wk || !sel) {
#pragma omp atomic write
            status = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t rg = 0; rg < n_rows * Hkv; ++rg) {
            if (status != ORACLE_OK) continue;
            const int64_t r = rg / Hkv;
            const int g = (int)(rg % Hkv);
            const int64_t b = rows[r] / L;
            const int64_t t = rows[r] % L;
            const int64_t c = t / S;        /* own chunk of t */
            const int64_t nvis = c;         /* R4: chunks 0..c-1 end before t's chunk */
            const double *q_row = q + r * H * d;
            const double *lm_bg = lm + ((b * Hkv + g) * Nc) * d;
            const double *k_bg = k + ((b * Hkv + g) * L) * d;
            const double *v_bg = v + ((b * Hkv + g) * L) * d;

            /* R3: group query qbar = mean over the G heads of the group. */
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int h = 0; h < G; ++h) acc += q_row[(int64_t)(g * G + h) * d + j];
                qbar[j] = acc / (double)G;
            }

            /* Selection: top-K of the group scores over the visible chunks. */
            int64_t nsel = 0;
            double gap_val;
            if (forced_idx) {
                const int32_t *f = forced_idx + (r * Hkv + g) * topk;
                for (int kk = 0; kk < topk; ++kk)
                    if (f[kk] >= 0 && f[kk] < nvis) sel[nsel++] = f[kk];
                gap_val = NAN;
            } else {
                for (int64_t i = 0; i < nvis; ++i) {
                    cand[i].score = scale * dot(qbar, lm_bg + i * d, d);
                    cand[i].index = i;
                }
                qsort(cand, (size_t)nvis, sizeof(candidate_t), candidate_order);
                nsel = nvis < topk ? nvis : topk;               /* R5 */
                for (int64_t kk = 0; kk < nsel; ++kk) sel[kk] = cand[kk].index;
                gap_val = nvis > topk ? cand[topk - 1].score - cand[topk].score : INFINITY;
            }
            if (idx)
                for (int kk = 0; kk < topk; ++kk)
                    idx[(r * Hkv + g) * topk + kk] = kk < nsel ? (int32_t)sel[kk] : -1;
            if (sbar)
                for (int kk = 0; kk < topk; ++kk)
                    sbar[(r * Hkv + g) * topk + kk] =
                        kk < nsel ? scale * dot(qbar, lm_bg + sel[kk] * d, d) : 0.0;
            if (gap) gap[r * Hkv + g] = gap_val;
            if (smag) {
                double *m = smag + (r * Hkv + g) * (topk + 1);
                for (int kk = 0; kk < topk; ++kk)
                    m[kk] = kk < nsel ? scale * abs_dot(qbar, lm_bg + sel[kk] * d, d) : 0.0;
                m[topk] = (!forced_idx && nvis > topk)
                              ? scale * abs_dot(qbar, lm_bg + cand[topk].index * d, d) : 0.0;
            }

            for (int h = 0; h < G; ++h) {
                const int hh = g * G + h;
                const double *q_h = q_row + (int64_t)hh * d;
                /* R2: fusion weights = softmax over the selected chunks of the
                 * head's own landmark scores. */
                for (int64_t kk = 0; kk < nsel; ++kk)
                    wk[kk] = scale * dot(q_h, lm_bg + sel[kk] * d, d);
                softmax_inplace(wk, (int)nsel);

                for (int j = 0; j < d; ++j) o_row[j] = 0.0;
                /* HiLS: attend inside each selected chunk, then fuse. */
                for (int64_t kk = 0; kk < nsel; ++kk) {
                    const int64_t first = sel[kk] * S;
                    chunk_attention(q_h, k_bg + first * d, v_bg + first * d, S, d, scale,
                                    logit, o_part);
                    for (int j = 0; j < d; ++j) o_row[j] += wk[kk] * o_part[j];
                }
                /* R4: causal attention inside the own chunk, weight 1. */
                if (own_chunk) {
                    const int64_t first = c * S;
                    chunk_attention(q_h, k_bg + first * d, v_bg + first * d, t - first + 1, d,
                                    scale, logit, o_part);
                    for (int j = 0; j < d; ++j) o_row[j] += o_part[j];
                }
                memcpy(O + (r * H + hh) * d, o_row, sizeof(double) * d);
                if (w)
                    for (int kk = 0; kk < topk; ++kk)
                        w[(r * H + hh) * topk + kk] = kk < nsel ? wk[kk] : 0.0;
            }
        }
        free(cand); free(qbar); free(logit); free(o_part); free(o_row); free(wk); free(sel);
    }
    free(lm_dhsa);
    return status;
}

/*
 * Prefill forward of the retrieval variants, for a list of query rows.
 *
 * Retrieval interval (HSA summary, "Main Findings": per-token retrieval
 * against per-8-token retrieval).  Tokens are cut into blocks of `interval`
 * consecutive tokens starting at 0 (interval divides S, so a block never
 * straddles a chunk boundary and all its tokens see the same chunks).  One
 * selection serves every token of a block; its group query is
 *   pool_mean = 0: the group query of the block's first token (it is known
 *                  when the block starts: the causal reading);
 *   pool_mean = 1: the mean over the block's tokens of their group queries
 *                  (the DHSA chunk-level query: sqrt(|C|) times the mean of
 *                  the chunk's queries, "What carries the argument", when
 *                  interval = S; the positive factor sqrt(|C|) does not change
 *                  the ranking and is left out).
 * The visible chunks are those before the block's chunk.  interval = 1 is
 * the per-token retrieval of hsa_oracle_prefill.
 *
 * Fusion:
 *   union_softmax = 0: softmax inside each selected chunk, outputs fused by
 *                      the softmax over the selection of the head's landmark
 *                      scores (HiLS Attention abstract), own chunk added;
 *   union_softmax = 1: one softmax over the keys of all selected chunks and,
 *                      with own_chunk, the causal own-chunk keys (Dynamic
 *                      Hierarchical Sparse Attention review, "What carries the
 *                      argument": attention under the selected-chunk mask).
 *
 * Variable-length chunks (Dynamic Hierarchical Sparse Attention review, "What
 * carries the argument": chunks of varying size, represented by sqrt(|C|)
 * times the mean of their keys): with bounds = {0 = c_0 < c_1 < ... < c_n = L}
 * chunk i holds tokens c_i .. c_{i+1} - 1, its landmark (lm == NULL) is
 * sqrt(|C_i|) * mean of its keys, the visible chunks of token t are those
 * before the chunk holding t, and the own chunk starts at that chunk's first
 * token.  bounds == NULL: chunks of S tokens (the last may be partial and has
 * no landmark).  interval must be 1 with bounds.
 *
 *   Q    [B, L, H, d]  all queries (pooling reads the block's other tokens)
 *   rows [n_rows]      flattened positions b*L + t to compute
 * Outputs O [n_rows, H, d], idx [n_rows, Hkv, topk] (may be NULL),
 * w [n_rows, H, topk] (may be NULL; the fusion weights of the HiLS form,
 * zero with union_softmax), and, as for hsa_oracle_prefill, the block
 * selection's group scores sbar [n_rows, Hkv, topk], gap [n_rows, Hkv] and
 * score-term magnitudes smag [n_rows, Hkv, topk+1] (all may be NULL).
 */
int hsa_oracle_prefill_variant(const double *Q, const int64_t *rows, int64_t n_rows,
                               const double *k, const double *v, const double *lm,
                               int B, int H, int Hkv, int64_t L, int d, int S, int topk,
                               int own_chunk, double scale, int interval, int pool_mean,
                               int union_softmax, const int64_t *bounds, int64_t n_chunks,
                               double *O, int32_t *idx, double *w,
                               double *sbar, double *gap, double *smag)
{
    if (!Q || !rows || !k || !v || !O) return ORACLE_BAD_ARG;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || L < 1 || d < 1 || S < 1 || topk < 1)
        return ORACLE_BAD_ARG;
    if (interval < 1 || S % interval != 0) return ORACLE_BAD_ARG;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * L) return ORACLE_BAD_ARG;
    int64_t maxlen = S;                    /* longest chunk */
    if (bounds) {
        if (interval != 1 || n_chunks < 1 || bounds[0] != 0 || bounds[n_chunks] != L)
            return ORACLE_BAD_ARG;
        maxlen = 0;
        for (int64_t i = 0; i < n_chunks; ++i) {
            if (bounds[i + 1] <= bounds[i]) return ORACLE_BAD_ARG;
            if (bounds[i + 1] - bounds[i] > maxlen) maxlen = bounds[i + 1] - bounds[i];
        }
    }
    const int G = H / Hkv;
    /* chunks with a landmark: every varlen chunk, the complete ones of fixed S */
    const int64_t Nc = bounds ? n_chunks : L / S;
    if (scale == 0.0) scale = 1.0 / sqrt((double)d);

    double *lm_dhsa = NULL;
    if (!lm) {
        lm_dhsa = (double *)malloc(sizeof(double) * (size_t)B * Hkv * (Nc > 0 ? Nc : 1) * d);
        if (!lm_dhsa) return ORACLE_NO_MEMORY;
        if (!bounds) {
            hsa_oracle_landmarks(k, B, Hkv, L, d, S, lm_dhsa);
        } else {
            /* sqrt(|C_i|) * mean of chunk i's keys */
            for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg)
                for (int64_t i = 0; i < Nc; ++i) {
                    const int64_t n = bounds[i + 1] - bounds[i];
                    for (int j = 0; j < d; ++j) {
                        double sum = 0.0;
                        for (int64_t r = bounds[i]; r < bounds[i + 1]; ++r)
                            sum += k[(bg * L + r) * d + j];
                        lm_dhsa[(bg * Nc + i) * d + j] = sqrt((double)n) * (sum / (double)n);
                    }
                }
        }
        lm = lm_dhsa;
    }
    int status = ORACLE_OK;
    const int64_t maxkeys = (int64_t)topk * maxlen + maxlen;

#pragma omp parallel
    {
        candidate_t *cand = (candidate_t *)malloc(sizeof(candidate_t) * (size_t)(Nc > 0 ? Nc : 1));
        double *qbar = (double *)malloc(sizeof(double) * d);
        double *logit = (double *)malloc(sizeof(double) * (size_t)(maxkeys > topk ? maxkeys : topk));
        double *o_part = (double *)malloc(sizeof(double) * d);
        double *o_row = (double *)malloc(sizeof(double) * d);
        double *wk = (double *)malloc(sizeof(double) * topk);
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * topk);
        int64_t *keyrow = (int64_t *)malloc(sizeof(int64_t) * (size_t)maxkeys);
        if (!cand || !qbar || !logit || !o_part || !o_row || !wk || !sel || !keyrow) {
#pragma omp atomic write
            status = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t rg = 0; rg < n_rows * Hkv; ++rg) {
            if (status != ORACLE_OK) continue;
            const int64_t r = rg / Hkv;
            const int g = (int)(rg % Hkv);
            const int64_t b = rows[r] / L;
            const int64_t t = rows[r] % L;
            const int64_t t0 = (t / interval) * interval;      /* the block's first token */
            const int64_t t1 = t0 + interval < L ? t0 + interval : L;
            /* own chunk (t0's): the chunk holding t; chunks before it are visible */
            int64_t c = t / S;
            if (bounds) {
                c = 0;
                while (bounds[c + 1] <= t) ++c;
            }
            const int64_t nvis = c;
            const int64_t own_first = bounds ? bounds[c] : c * S;
            const double *lm_bg = lm + ((b * Hkv + g) * Nc) * d;
            const double *k_bg = k + ((b * Hkv + g) * L) * d;
            const double *v_bg = v + ((b * Hkv + g) * L) * d;

            /* the block's group query: first token's, or the mean over its tokens */
            const int64_t u1 = pool_mean ? t1 : t0 + 1;
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t u = t0; u < u1; ++u)
                    for (int h = 0; h < G; ++h) acc += Q[((b * L + u) * H + g * G + h) * d + j];
                qbar[j] = acc / ((double)G * (double)(u1 - t0));
            }
            for (int64_t i = 0; i < nvis; ++i) {
                cand[i].score = scale * dot(qbar, lm_bg + i * d, d);
                cand[i].index = i;
            }
            qsort(cand, (size_t)nvis, sizeof(candidate_t), candidate_order);
            const int64_t nsel = nvis < topk ? nvis : topk;
            for (int64_t kk = 0; kk < nsel; ++kk) sel[kk] = cand[kk].index;
            if (idx)
                for (int kk = 0; kk < topk; ++kk)
                    idx[(r * Hkv + g) * topk + kk] = kk < nsel ? (int32_t)sel[kk] : -1;
            if (sbar)
                for (int kk = 0; kk < topk; ++kk)
                    sbar[(r * Hkv + g) * topk + kk] = kk < nsel ? cand[kk].score : 0.0;
            if (gap)
                gap[r * Hkv + g] = nvis > topk ? cand[topk - 1].score - cand[topk].score : INFINITY;
            if (smag) {
                double *m = smag + (r * Hkv + g) * (topk + 1);
                for (int kk = 0; kk < topk; ++kk)
                    m[kk] = kk < nsel ? scale * abs_dot(qbar, lm_bg + sel[kk] * d, d) : 0.0;
                m[topk] = nvis > topk ? scale * abs_dot(qbar, lm_bg + cand[topk].index * d, d) : 0.0;
            }

            for (int h = 0; h < G; ++h) {
                const int hh = g * G + h;
                const double *q_h = Q + ((b * L + t) * H + hh) * d;
                for (int j = 0; j < d; ++j) o_row[j] = 0.0;
                for (int kk = 0; kk < topk; ++kk) wk[kk] = 0.0;
                if (!union_softmax) {
                    /* HiLS form: each token's own landmark scores weight the chunks */
                    for (int64_t kk = 0; kk < nsel; ++kk)
                        wk[kk] = scale * dot(q_h, lm_bg + sel[kk] * d, d);
                    softmax_inplace(wk, (int)nsel);
                    for (int64_t kk = 0; kk < nsel; ++kk) {
                        const int64_t first = bounds ? bounds[sel[kk]] : sel[kk] * S;
                        const int64_t len = bounds ? bounds[sel[kk] + 1] - first : S;
                        chunk_attention(q_h, k_bg + first * d, v_bg + first * d, len, d, scale,
                                        logit, o_part);
                        for (int j = 0; j < d; ++j) o_row[j] += wk[kk] * o_part[j];
                    }
                    if (own_chunk) {
                        chunk_attention(q_h, k_bg + own_first * d, v_bg + own_first * d,
                                        t - own_first + 1, d, scale, logit, o_part);
                        for (int j = 0; j < d; ++j) o_row[j] += o_part[j];
                    }
                } else {
                    /* DHSA form: one softmax over the union of the selected keys */
                    int64_t nk = 0;
                    for (int64_t kk = 0; kk < nsel; ++kk) {
                        const int64_t first = bounds ? bounds[sel[kk]] : sel[kk] * S;
                        const int64_t len = bounds ? bounds[sel[kk] + 1] - first : S;
                        for (int64_t jj = 0; jj < len; ++jj) keyrow[nk++] = first + jj;
                    }
                    if (own_chunk)
                        for (int64_t jj = own_first; jj <= t; ++jj) keyrow[nk++] = jj;
                    if (nk > 0) {
                        double m = -INFINITY;
                        for (int64_t e = 0; e < nk; ++e) {
                            logit[e] = scale * dot(q_h, k_bg + keyrow[e] * d, d);
                            if (logit[e] > m) m = logit[e];
                        }
                        double den = 0.0;
                        for (int64_t e = 0; e < nk; ++e) {
                            logit[e] = exp(logit[e] - m);
                            den += logit[e];
                        }
                        for (int64_t e = 0; e < nk; ++e) {
                            const double p = logit[e] / den;
                            for (int j = 0; j < d; ++j) o_row[j] += p * v_bg[keyrow[e] * d + j];
                        }
                    }
                }
                memcpy(O + (r * H + hh) * d, o_row, sizeof(double) * d);
                if (w)
                    for (int kk = 0; kk < topk; ++kk) w[(r * H + hh) * topk + kk] = wk[kk];
            }
        }
        free(cand); free(qbar); free(logit); free(o_part); free(o_row); free(wk); free(sel);
        free(keyrow);
    }
    free(lm_dhsa);
    return status;
}

/*
 * Decode, step 1: selection for one new query per sequence at position Lc
 * (R12: all Nc = Lc/S chunks visible).
 *   q    [B, H, d]
 *   lm   [B, Hkv, Nc, d]
 *   idx  [B, Hkv, topk]  (-1 padded when Nc < topk)
 *   sbar [B, Hkv, topk]  group scores of the selected chunks (may be NULL)
 *   gap  [B, Hkv]        score(K-th) - score(K+1-th), +inf if Nc <= K (may be NULL)
 *   smag [B, Hkv, topk+1] magnitudes scale * sum_j |qbar_j l_ij| of the selected
 *                        chunks' scores and, last, of the (K+1)-th (may be NULL)
 */
int hsa_oracle_decode_select(const double *q, const double *lm, int B, int H, int Hkv,
                             int64_t Nc, int d, int topk, double scale,
                             int32_t *idx, double *sbar, double *gap, double *smag)
{
    if (!q || !lm || !idx) return ORACLE_BAD_ARG;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || Nc < 0 || d < 1 || topk < 1)
        return ORACLE_BAD_ARG;
    const int G = H / Hkv;
    if (scale == 0.0) scale = 1.0 / sqrt((double)d);
    int status = ORACLE_OK;
    for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg) {
        const int64_t b = bg / Hkv;
        const int g = (int)(bg % Hkv);
        double *qbar = (double *)malloc(sizeof(double) * d);
        candidate_t *cand = (candidate_t *)malloc(sizeof(candidate_t) * (size_t)(Nc > 0 ? Nc : 1));
        if (!qbar || !cand) { free(qbar); free(cand); return ORACLE_NO_MEMORY; }
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int h = 0; h < G; ++h) acc += q[(b * H + g * G + h) * d + j];
            qbar[j] = acc / (double)G;
        }
        const double *lm_bg = lm + bg * Nc * d;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < Nc; ++i) {
            cand[i].score = scale * dot(qbar, lm_bg + i * d, d);
            cand[i].index = i;
        }
        qsort(cand, (size_t)Nc, sizeof(candidate_t), candidate_order);
        const int64_t nsel = Nc < topk ? Nc : topk;
        for (int kk = 0; kk < topk; ++kk) {
            idx[bg * topk + kk] = kk < nsel ? (int32_t)cand[kk].index : -1;
            if (sbar) sbar[bg * topk + kk] = kk < nsel ? cand[kk].score : 0.0;
        }
        if (gap) gap[bg] = Nc > topk ? cand[topk - 1].score - cand[topk].score : INFINITY;
        if (smag) {
            double *m = smag + bg * (topk + 1);
            for (int kk = 0; kk <= topk; ++kk)
                m[kk] = kk < Nc ? scale * abs_dot(qbar, lm_bg + cand[kk].index * d, d) : 0.0;
        }
        free(qbar);
        free(cand);
    }
    return status;
}

/*
 * Decode, step 2: attention inside the selected chunks and score-weighted
 * fusion (HiLS), for one query per sequence.
 *   q      [B, H, d]
 *   lm     [B, Hkv, Nc, d]
 *   kg, vg [B, Hkv, topk, S, d]  keys/values of chunk idx[b,g,kk] (rows of
 *                                padded slots are ignored)
 *   idx    [B, Hkv, topk]
 *   O      [B, H, d];  w [B, H, topk] (may be NULL)
 */
int hsa_oracle_decode_attend(const double *q, const double *lm, const double *kg,
                             const double *vg, const int32_t *idx, int B, int H, int Hkv,
                             int64_t Nc, int d, int S, int topk, double scale,
                             double *O, double *w)
{
    if (!q || !lm || !kg || !vg || !idx || !O) return ORACLE_BAD_ARG;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || Nc < 0 || d < 1 || S < 1 || topk < 1)
        return ORACLE_BAD_ARG;
    const int G = H / Hkv;
    if (scale == 0.0) scale = 1.0 / sqrt((double)d);
    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(S > topk ? S : topk));
        double *o_part = (double *)malloc(sizeof(double) * d);
        double *wk = (double *)malloc(sizeof(double) * topk);
        int64_t *sel = (int64_t *)malloc(sizeof(int64_t) * topk);
        int *slot = (int *)malloc(sizeof(int) * topk);
        if (!logit || !o_part || !wk || !sel || !slot) {
#pragma omp atomic write
            status = ORACLE_NO_MEMORY;
        }
#pragma omp for schedule(static)
        for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
            if (status != ORACLE_OK) continue;
            const int64_t b = bh / H;
            const int hh = (int)(bh % H);
            const int g = hh / G;
            const int64_t bg = b * Hkv + g;
            const double *q_h = q + bh * d;
            int nsel = 0;
            for (int kk = 0; kk < topk; ++kk) {
                const int32_t i = idx[bg * topk + kk];
                if (i >= 0 && i < Nc) { sel[nsel] = i; slot[nsel] = kk; ++nsel; }
            }
            for (int n = 0; n < nsel; ++n) wk[n] = scale * dot(q_h, lm + (bg * Nc + sel[n]) * d, d);
            softmax_inplace(wk, nsel);
            double *o_row = O + bh * d;
            for (int j = 0; j < d; ++j) o_row[j] = 0.0;
            for (int n = 0; n < nsel; ++n) {
                const int64_t base = ((bg * topk + slot[n]) * S) * d;
                chunk_attention(q_h, kg + base, vg + base, S, d, scale, logit, o_part);
                for (int j = 0; j < d; ++j) o_row[j] += wk[n] * o_part[j];
            }
            if (w) {
                for (int kk = 0; kk < topk; ++kk) w[bh * topk + kk] = 0.0;
                for (int n = 0; n < nsel; ++n) w[bh * topk + slot[n]] = wk[n];
            }
        }
        free(logit); free(o_part); free(wk); free(sel); free(slot);
    }
    return status;
}

int hsa_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
