/*
 * hsa_oracle.c -- plain, slow, fp64 CPU oracle for Hierarchical Sparse
 * Attention (HSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: it exists so that tests (and the timed CPU baseline of the
 * benchmark) can check the CUDA library against an independent statement of
 * what the method computes.  It shares no code, header, table or constant with
 * the CUDA sources.
 *
 * Sources (cited by title and section):
 *   [P1] "Hardware-aligned Hierarchical Sparse Attention for Efficient
 *        Long-term Memory Access" -- paper notes (papernotes.org), sections
 *        "层次化稀疏注意力（HSA）" (HSA), "硬件对齐 Kernel" (kernel) and
 *        "训练与推理优化" (training / inference).
 *   [P3] "Hardware-aligned Hierarchical Sparse Attention for Efficient
 *        Long-term Memory Access" -- AI summary (atlas.scime.ai), "Approach".
 *
 * The pages give the method in prose only.  Where they leave a step open this
 * file uses the following conventions (each is repeated at its use site):
 *   C1  chunk c (tokens cS .. cS+S-1) is eligible for token t iff c < floor(t/S):
 *       it ends at or before the start of t's own chunk.  Only complete chunks
 *       (c < floor(L/S)) exist in the chunk index.
 *   C2  selection score s = q_slc . kbar_c / sqrt(d), one selection query per
 *       (token, KV group); kbar is the fp32 mean-pooled key of the chunk.
 *   C3  top-K by score, ties broken toward the higher chunk index; fewer than
 *       K eligible chunks -> take all of them; empty slots get idx=-1, w=0.
 *   C4  the selected list is ordered most-recent-first (descending index).
 *   C5  stick-breaking weights w_k = sig(s_k) * prod_{j<k} (1 - sig(s_j)).
 *   C6  softmax-off-by-one p_i = exp(x_i) / (1 + sum_j exp(x_j)),
 *       x_i = q . k_i / sqrt(d); computed with m = max(0, max_j x_j).
 *   C7  query head h belongs to KV group floor(h / (h_q/h_kv)).
 *   C8  tokens of chunk 0 (no eligible chunk) output zero.
 *
 * Layouts (row-major, all fp64 unless stated):
 *   q, o, dO, dq      [B, L, h_q, d]
 *   q_slc, dq_slc     [B, L, h_kv, d]
 *   k, v, dk, dv      [B, h_kv, L, d]
 *   kbar (fp32), dkbar [B, h_kv, n_c, d]      n_c = floor(L/S)
 *   idx (int32), w    [B, L, h_kv, K]
 *   lse               [B, L, h_q, K]
 *
 * All functions return 0 on success, a negative number on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_MAX_K 64

/* ------------------------------------------------------------------------- */
/* Step 1: mean-pooled chunk keys.                                           */
/* [P1 §HSA, "Chunk Selection"]: each chunk is represented for selection by  */
/* the mean of its keys; [P1 §training/inference, "KV Cache Offloading"]:    */
/* the chunk-level index holds floor(L/S) rows of width d.                   */
/* The mean is taken in fp64 and the index is then stored as fp32; the       */
/* stored fp32 value is the definition every later step reads.               */
/* ------------------------------------------------------------------------- */
int or_pool(int B, int h_kv, int L, int d, int S, const double *k, float *kbar)
{
    if (B < 0 || h_kv < 1 || L < 0 || d < 1 || S < 1 || (!k && L > 0) || !kbar)
        return -1;
    const int n_c = L / S;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < h_kv; ++g)
            for (int c = 0; c < n_c; ++c)
                for (int j = 0; j < d; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < S; ++i)
                        acc += k[(((int64_t)b * h_kv + g) * L + (int64_t)c * S + i) * d + j];
                    kbar[(((int64_t)b * h_kv + g) * n_c + c) * d + j] = (float)(acc / S);
                }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Step 2/3/4: score, top-K, order, stick-breaking weights for one row.      */
/* ------------------------------------------------------------------------- */
typedef struct {
    double s;
    int c;
} cand_t;

/* better-first: higher score first; equal scores -> higher chunk index first (C3) */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->c > y->c) ? -1 : (x->c < y->c) ? 1 : 0;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Selection for one (b, t, g) row.
 *   qs    : q_slc row (d values)
 *   kb    : kbar block of group g, [n_c, d] fp32
 *   n_elig: number of eligible chunks (C1)
 * Writes idx[K], w[K], s_out[K] (score of each slot) and *gap.
 * cand is caller-provided scratch of n_elig entries.
 */
static void select_row(int d, int K, const double *qs, const float *kb, int n_elig,
                       cand_t *cand, int32_t *idx, double *w, double *s_out, double *gap)
{
    const double scale = 1.0 / sqrt((double)d);
    /* [P1 §HSA, "Chunk Selection"]: dot product of the token's selection
       query with each chunk's pooled key (scale: C2). */
    for (int c = 0; c < n_elig; ++c) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += qs[j] * (double)kb[(int64_t)c * d + j];
        cand[c].s = acc * scale;
        cand[c].c = c;
    }
    /* top-K: full sort, best first (C3) */
    qsort(cand, (size_t)n_elig, sizeof(cand_t), cand_cmp);
    const int n_sel = n_elig < K ? n_elig : K;
    *gap = (n_elig > K) ? cand[K - 1].s - cand[K].s : INFINITY;

    /* order the chosen chunks most-recent-first (C4): sort the first n_sel by
       descending chunk index (insertion sort; n_sel <= K is tiny). */
    cand_t chosen[OR_MAX_K];
    for (int i = 0; i < n_sel; ++i) chosen[i] = cand[i];
    for (int i = 1; i < n_sel; ++i) {
        cand_t x = chosen[i];
        int j = i - 1;
        while (j >= 0 && chosen[j].c < x.c) { chosen[j + 1] = chosen[j]; --j; }
        chosen[j + 1] = x;
    }
    /* [P1 §HSA, second stage]: stick-breaking weights from the sigmoid of the
       relevance score only, no positional term (C5). */
    double remaining = 1.0;
    for (int i = 0; i < K; ++i) {
        if (i < n_sel) {
            const double sg = sigmoid(chosen[i].s);
            idx[i] = chosen[i].c;
            s_out[i] = chosen[i].s;
            w[i] = sg * remaining;
            remaining *= (1.0 - sg);
        } else {
            idx[i] = -1;
            s_out[i] = 0.0;
            w[i] = 0.0;
        }
    }
}

static int row_of(const int64_t *rows, int64_t i) { return rows ? (int)rows[i] : (int)i; }

int or_select(int B, int L, int h_kv, int d, int S, int K, const double *q_slc, const float *kbar,
              const int64_t *rows, int64_t nrows, int32_t *idx, double *w, double *s, double *gap)
{
    if (B < 0 || L < 0 || h_kv < 1 || d < 1 || S < 1 || K < 1 || K > OR_MAX_K) return -1;
    if (!rows) nrows = (int64_t)B * L;
    const int n_c = L / S;
    for (int64_t i = 0; i < nrows; ++i) {
        const int r = row_of(rows, i);
        if (r < 0 || r >= B * L) return -2;
    }
    int err = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_c > 0 ? n_c : 1));
        if (!cand) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < nrows; ++i) {
                const int r = row_of(rows, i);
                const int b = r / L, t = r % L;
                int n_elig = t / S; /* C1 */
                if (n_elig > n_c) n_elig = n_c;
                for (int g = 0; g < h_kv; ++g) {
                    const int64_t o = (i * h_kv + g) * K;
                    double gp;
                    select_row(d, K, q_slc + ((int64_t)r * h_kv + g) * d,
                               kbar + ((int64_t)b * h_kv + g) * n_c * d, n_elig, cand,
                               idx + o, w + o, s + o, &gp);
                    if (gap) gap[i * h_kv + g] = gp;
                }
            }
            free(cand);
        }
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Step 5: softmax-off-by-one attention inside one chunk.                    */
/* [P1 §HSA, first stage]: ordinary attention inside each selected chunk     */
/* gives a chunk-level output O_{t,k}; [P1 §kernel]: the softmax carries an  */
/* extra 1 in its denominator so a token can ignore the retrieved tokens     */
/* (C6).  No mask is needed inside the chunk: it lies wholly in t's past.    */
/* Writes O (d values) and returns lse = log(1 + sum_i exp(x_i)).            */
/* ------------------------------------------------------------------------- */
static double chunk_attend(int d, int S, const double *qh, const double *kc, const double *vc,
                           double *x /* scratch S */, double *O)
{
    const double scale = 1.0 / sqrt((double)d);
    double m = 0.0; /* max(0, max_i x_i) */
    for (int i = 0; i < S; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += qh[j] * kc[(int64_t)i * d + j];
        x[i] = acc * scale;
        if (x[i] > m) m = x[i];
    }
    double Z = exp(-m);
    for (int i = 0; i < S; ++i) {
        x[i] = exp(x[i] - m);
        Z += x[i];
    }
    for (int j = 0; j < d; ++j) O[j] = 0.0;
    for (int i = 0; i < S; ++i) {
        const double p = x[i] / Z;
        for (int j = 0; j < d; ++j) O[j] += p * vc[(int64_t)i * d + j];
    }
    return m + log(Z);
}

/* Attention and fusion of one token row for a given selection (idx_row, w_row
   per group).  [P1 §kernel]: per token, the output accumulator starts at zero
   and each selected chunk adds w times its chunk output.  */
static void attend_row(int L, int h_q, int h_kv, int d, int S, int K, int b, const double *q_row,
                       const double *k, const double *v, const int32_t *idx_row, const double *w_row,
                       double *x, double *Ok, double *o_row, double *lse_row)
{
    const int G = h_q / h_kv; /* C7 */
    for (int h = 0; h < h_q; ++h) {
        const int g = h / G;
        double *oh = o_row + (int64_t)h * d;
        for (int j = 0; j < d; ++j) oh[j] = 0.0; /* C8 when nothing is selected */
        for (int kk = 0; kk < K; ++kk) {
            const int c = idx_row[g * K + kk];
            if (c < 0) {
                if (lse_row) lse_row[h * K + kk] = 0.0;
                continue;
            }
            const int64_t base = (((int64_t)b * h_kv + g) * L + (int64_t)c * S) * d;
            const double l = chunk_attend(d, S, q_row + (int64_t)h * d, k + base, v + base, x, Ok);
            if (lse_row) lse_row[h * K + kk] = l;
            const double wk = w_row[g * K + kk];
            for (int j = 0; j < d; ++j) oh[j] += wk * Ok[j];
        }
    }
}

/* One token row of the forward pass: selection per group, then attention and
   fusion per query head.  */
static void fwd_row(int L, int h_q, int h_kv, int d, int S, int K, int b, int t, int n_c,
                    const double *q_row /* [h_q,d] */, const double *k, const double *v,
                    const double *qs_row /* [h_kv,d] */, const float *kbar, cand_t *cand,
                    double *x, double *Ok, double *o_row /* [h_q,d] */, double *lse_row /* [h_q,K] */,
                    int32_t *idx_row /* [h_kv,K] */, double *w_row /* [h_kv,K] */,
                    double *gap_row /* [h_kv] or NULL */)
{
    int n_elig = t / S;       /* C1 */
    if (n_elig > n_c) n_elig = n_c;
    double s_tmp[OR_MAX_K], gp;
    for (int g = 0; g < h_kv; ++g)
        select_row(d, K, qs_row + (int64_t)g * d, kbar + ((int64_t)b * h_kv + g) * n_c * d, n_elig,
                   cand, idx_row + g * K, w_row + g * K, s_tmp, gap_row ? gap_row + g : &gp);
    attend_row(L, h_q, h_kv, d, S, K, b, q_row, k, v, idx_row, w_row, x, Ok, o_row, lse_row);
}

int or_fwd(int B, int L, int h_q, int h_kv, int d, int S, int K, const double *q, const double *k,
           const double *v, const double *q_slc, const float *kbar, const int64_t *rows,
           int64_t nrows, double *o, double *lse, int32_t *idx, double *w)
{
    if (B < 0 || L < 0 || h_q < 1 || h_kv < 1 || h_q % h_kv || d < 1 || S < 1 || K < 1 ||
        K > OR_MAX_K || !o || !idx || !w)
        return -1;
    if (!rows) nrows = (int64_t)B * L;
    const int n_c = L / S;
    for (int64_t i = 0; i < nrows; ++i) {
        const int r = row_of(rows, i);
        if (r < 0 || r >= B * L) return -2;
    }
    int err = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_c > 0 ? n_c : 1));
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        double *Ok = (double *)malloc(sizeof(double) * (size_t)d);
        if (!cand || !x || !Ok) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < nrows; ++i) {
                const int r = row_of(rows, i);
                fwd_row(L, h_q, h_kv, d, S, K, r / L, r % L, n_c, q + (int64_t)r * h_q * d, k, v,
                        q_slc + (int64_t)r * h_kv * d, kbar, cand, x, Ok, o + i * h_q * d,
                        lse ? lse + i * h_q * K : NULL, idx + i * h_kv * K, w + i * h_kv * K, NULL);
            }
        }
        free(cand);
        free(x);
        free(Ok);
    }
    return err;
}

/* Attention and fusion for a caller-given selection.  [P1 §training/inference]:
   one chunk retrieval per step is shared by all HSA layers, so a later layer
   attends with its own q, k, v over the chunks (and weights) that the shared
   selection chose.  idx, w [nrows, h_kv, K] hold the selection of each listed
   row; -1 marks an empty slot.  An entry outside 0 <= c < min(t/S, n_c) is
   not a causal complete chunk and makes the call fail (-4). */
int or_attend(int B, int L, int h_q, int h_kv, int d, int S, int K, const double *q, const double *k,
              const double *v, const int32_t *idx, const double *w, const int64_t *rows, int64_t nrows,
              double *o, double *lse)
{
    if (B < 0 || L < 0 || h_q < 1 || h_kv < 1 || h_q % h_kv || d < 1 || S < 1 || K < 1 || !idx ||
        !w || !o)
        return -1;
    if (!rows) nrows = (int64_t)B * L;
    const int n_c = L / S;
    for (int64_t i = 0; i < nrows; ++i) {
        const int r = row_of(rows, i);
        if (r < 0 || r >= B * L) return -2;
        const int n_elig = (r % L) / S < n_c ? (r % L) / S : n_c;
        for (int e = 0; e < h_kv * K; ++e) {
            const int c = idx[i * h_kv * K + e];
            if (c >= n_elig) return -4;
        }
    }
    int err = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        double *Ok = (double *)malloc(sizeof(double) * (size_t)d);
        if (!x || !Ok) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < nrows; ++i) {
                const int r = row_of(rows, i);
                attend_row(L, h_q, h_kv, d, S, K, r / L, q + (int64_t)r * h_q * d, k, v,
                           idx + i * h_kv * K, w + i * h_kv * K, x, Ok, o + i * h_q * d,
                           lse ? lse + i * h_q * K : NULL);
            }
        }
        free(x);
        free(Ok);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Decode step.  [P1 §training/inference, "KV Cache Offloading"]: at         */
/* inference the GPU keeps only the chunk-level index; each step selects     */
/* chunks against it and reads only the selected chunks' K/V.  The new token */
/* sits at position P, so every complete cached chunk c < floor(P/S) is      */
/* eligible (C1).  This is exactly forward row t = P of the prompt plus one. */
/* ------------------------------------------------------------------------- */
int or_decode(int B, int P, int h_q, int h_kv, int d, int S, int K, const double *q,
              const double *q_slc, const double *k_cache, const double *v_cache, const float *kbar,
              double *o, int32_t *idx, double *w, double *gap)
{
    if (B < 0 || P < 0 || h_q < 1 || h_kv < 1 || h_q % h_kv || d < 1 || S < 1 || K < 1 ||
        K > OR_MAX_K || !o)
        return -1;
    const int n_c = P / S;
    int err = 0;
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_c > 0 ? n_c : 1));
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        double *Ok = (double *)malloc(sizeof(double) * (size_t)d);
        int32_t *idx_l = (int32_t *)malloc(sizeof(int32_t) * (size_t)h_kv * K);
        double *w_l = (double *)malloc(sizeof(double) * (size_t)h_kv * K);
        if (!cand || !x || !Ok || !idx_l || !w_l) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int b = 0; b < B; ++b) {
                /* cache length P: the caches are [B, h_kv, P, d] */
                fwd_row(P, h_q, h_kv, d, S, K, b, P, n_c, q + (int64_t)b * h_q * d, k_cache,
                        v_cache, q_slc + (int64_t)b * h_kv * d, kbar, cand, x, Ok,
                        o + (int64_t)b * h_q * d, NULL, idx_l, w_l, gap ? gap + (int64_t)b * h_kv : NULL);
                if (idx) memcpy(idx + (int64_t)b * h_kv * K, idx_l, sizeof(int32_t) * h_kv * K);
                if (w) memcpy(w + (int64_t)b * h_kv * K, w_l, sizeof(double) * h_kv * K);
            }
        }
        free(cand);
        free(x);
        free(Ok);
        free(idx_l);
        free(w_l);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Backward.  [P1 §kernel]: gradients are taken in two phases, first those   */
/* of Q and of the chunk weights w per token, then those of K and V per      */
/* chunk.  [P1 §HSA, "end-to-end learning"]: the chunk weight receives the   */
/* gradient of the whole chunk's contribution, and through w it reaches the  */
/* selection score (hence q_slc and the pooled keys).  The top-K choice is   */
/* piecewise constant and carries no gradient.                               */
/*                                                                           */
/* This oracle walks tokens one at a time (per-token loops, not per-chunk    */
/* lists) and accumulates dk, dv, dkbar directly, so that any error in a     */
/* per-chunk inversion on the other side shows up as a mismatch.             */
/*                                                                           */
/* Derivation, per token t, head h in group g, slot k (chunk c, weight w_k): */
/*   O_k = sum_i p_i v_i,  p = softmax-off-by-one(x),  x_i = q.k_i/sqrt(d)   */
/*   o   = sum_k w_k O_k                                                     */
/*   dw_k   += dO . O_k                       (summed over h in g)           */
/*   dp_i    = w_k dO . v_i                                                  */
/*   dx_i    = p_i (dp_i - sum_j p_j dp_j) = w_k p_i (dO.v_i - dO.O_k)       */
/*   dq     += dx_i k_i / sqrt(d);  dk_i += dx_i q / sqrt(d)                 */
/*   dv_i   += w_k p_i dO                                                    */
/* stick-breaking (C5): dw_j/ds_j chain with sig_j = sigmoid(s_j):           */
/*   ds_j = dw_j w_j (1 - sig_j) - sig_j sum_{k>j} dw_k w_k                  */
/* then s_j = q_slc . kbar_{c_j}/sqrt(d):                                    */
/*   dq_slc += ds_j kbar_{c_j}/sqrt(d);  dkbar_{c_j} += ds_j q_slc/sqrt(d)   */
/* and the pooling kbar_c = mean of its S keys gives dk += dkbar_c / S.      */
/* ------------------------------------------------------------------------- */
int or_bwd(int B, int L, int h_q, int h_kv, int d, int S, int K, const double *q, const double *k,
           const double *v, const double *q_slc, const float *kbar, const double *dO,
           const uint8_t *tok_mask, double *dq, double *dk, double *dv, double *dq_slc,
           double *dkbar)
{
    if (B < 0 || L < 0 || h_q < 1 || h_kv < 1 || h_q % h_kv || d < 1 || S < 1 || K < 1 ||
        K > OR_MAX_K || !dq || !dk || !dv || !dq_slc || !dkbar)
        return -1;
    const int G = h_q / h_kv;
    const int n_c = L / S;
    const double scale = 1.0 / sqrt((double)d);
    memset(dq, 0, sizeof(double) * (size_t)B * L * h_q * d);
    memset(dq_slc, 0, sizeof(double) * (size_t)B * L * h_kv * d);
    memset(dk, 0, sizeof(double) * (size_t)B * h_kv * L * d);
    memset(dv, 0, sizeof(double) * (size_t)B * h_kv * L * d);
    memset(dkbar, 0, sizeof(double) * (size_t)B * h_kv * (n_c > 0 ? n_c : 0) * d);
    int err = 0;
    /* parallel over (b, g): each owns its slice of dk, dv, dkbar */
#pragma omp parallel
    {
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_c > 0 ? n_c : 1));
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        double *p = (double *)malloc(sizeof(double) * (size_t)S);
        double *Ok = (double *)malloc(sizeof(double) * (size_t)d);
        if (!cand || !x || !p || !Ok) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1) collapse(2)
            for (int b = 0; b < B; ++b)
                for (int g = 0; g < h_kv; ++g) {
                    const float *kb = kbar + ((int64_t)b * h_kv + g) * n_c * d;
                    for (int t = 0; t < L; ++t) {
                        if (tok_mask && !tok_mask[(int64_t)b * L + t]) continue;
                        int n_elig = t / S;
                        if (n_elig > n_c) n_elig = n_c;
                        const int64_t r = (int64_t)b * L + t;
                        const double *qs = q_slc + (r * h_kv + g) * d;
                        int32_t idx[OR_MAX_K];
                        double w[OR_MAX_K], s[OR_MAX_K], dw[OR_MAX_K], gp;
                        select_row(d, K, qs, kb, n_elig, cand, idx, w, s, &gp);
                        for (int kk = 0; kk < K; ++kk) dw[kk] = 0.0;
                        for (int h = g * G; h < (g + 1) * G; ++h) {
                            const double *qh = q + (r * h_q + h) * d;
                            const double *dOh = dO + (r * h_q + h) * d;
                            double *dqh = dq + (r * h_q + h) * d;
                            for (int kk = 0; kk < K; ++kk) {
                                const int c = idx[kk];
                                if (c < 0) continue;
                                const int64_t base = (((int64_t)b * h_kv + g) * L + (int64_t)c * S) * d;
                                const double *kc = k + base, *vc = v + base;
                                /* recompute p and O_k */
                                double m = 0.0;
                                for (int i = 0; i < S; ++i) {
                                    double acc = 0.0;
                                    for (int j = 0; j < d; ++j) acc += qh[j] * kc[(int64_t)i * d + j];
                                    x[i] = acc * scale;
                                    if (x[i] > m) m = x[i];
                                }
                                double Z = exp(-m);
                                for (int i = 0; i < S; ++i) { p[i] = exp(x[i] - m); Z += p[i]; }
                                for (int i = 0; i < S; ++i) p[i] /= Z;
                                for (int j = 0; j < d; ++j) Ok[j] = 0.0;
                                for (int i = 0; i < S; ++i)
                                    for (int j = 0; j < d; ++j) Ok[j] += p[i] * vc[(int64_t)i * d + j];
                                double delta = 0.0; /* dO . O_k */
                                for (int j = 0; j < d; ++j) delta += dOh[j] * Ok[j];
                                dw[kk] += delta;
                                const double wk = w[kk];
                                for (int i = 0; i < S; ++i) {
                                    double dov = 0.0;
                                    for (int j = 0; j < d; ++j) dov += dOh[j] * vc[(int64_t)i * d + j];
                                    const double dxi = wk * p[i] * (dov - delta);
                                    double *dki = dk + base + (int64_t)i * d;
                                    double *dvi = dv + base + (int64_t)i * d;
                                    for (int j = 0; j < d; ++j) {
                                        dqh[j] += dxi * kc[(int64_t)i * d + j] * scale;
                                        dki[j] += dxi * qh[j] * scale;
                                        dvi[j] += wk * p[i] * dOh[j];
                                    }
                                }
                            }
                        }
                        /* stick-breaking backward over the ordered list */
                        double *dqs = dq_slc + (r * h_kv + g) * d;
                        for (int jj = 0; jj < K; ++jj) {
                            if (idx[jj] < 0) continue;
                            const double sg = sigmoid(s[jj]);
                            double tail = 0.0;
                            for (int kk = jj + 1; kk < K; ++kk)
                                if (idx[kk] >= 0) tail += dw[kk] * w[kk];
                            const double ds = dw[jj] * w[jj] * (1.0 - sg) - sg * tail;
                            const float *kbc = kb + (int64_t)idx[jj] * d;
                            double *dkbc = dkbar + (((int64_t)b * h_kv + g) * n_c + idx[jj]) * d;
                            for (int j = 0; j < d; ++j) {
                                dqs[j] += ds * (double)kbc[j] * scale;
                                dkbc[j] += ds * qs[j] * scale;
                            }
                        }
                    }
                    /* pooling path: dk of every key of chunk c gains dkbar_c / S */
                    for (int c = 0; c < n_c; ++c) {
                        const double *dkbc = dkbar + (((int64_t)b * h_kv + g) * n_c + c) * d;
                        for (int i = 0; i < S; ++i) {
                            double *dki = dk + (((int64_t)b * h_kv + g) * L + (int64_t)c * S + i) * d;
                            for (int j = 0; j < d; ++j) dki[j] += dkbc[j] / S;
                        }
                    }
                }
        }
        free(cand);
        free(x);
        free(p);
        free(Ok);
    }
    return err;
}

int or_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
