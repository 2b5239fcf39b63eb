/*
 * oracle.c - plain, slow, fp64 CPU reference for exact maximum-inner-product
 * search (brute-force top-k by dot product over an L2-normalised corpus).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. The product path (the
 * CUDA library under exact_inner_product_b200/) shares no code, header, table
 * or helper with this file, and neither side includes or links the other.
 *
 * What it computes, and where each step comes from:
 *   - Row normalisation: v / sqrt(max(sum_i v_i^2, 1e-12)).
 *     x-algorithm recsys_two_tower_model.py, `_l2_normalize_candidates`
 *     (EPS = 1e-12 clamps the squared norm); the same formula is applied to
 *     the user vector in `RecsysTwoTowerModel.__call__` before retrieval.
 *   - Score: s_bj = (u_b . v_j) / tau. recsys_two_tower_model.py `forward`,
 *     inner `compute_top_k` (user x post_embeddings^T); "Two-Tower Retrieval
 *     at Industrial Scale", TwoTower.score (u @ v.t() / tau).
 *     With the corpus kept raw ("fused" normalisation), s_bj is divided by the
 *     row norm of v_j as well: s_bj = (u_b . v_j) / norm_j / tau.
 *   - Exclusion: candidates whose exclusion bit is set never appear
 *     (recsys_two_tower_model.py `mask_and_top_k`, masked scores pushed to the
 *     bottom; here they are removed outright and the list is padded).
 *   - Top-k: sort every eligible (score, id) pair by score descending, ties by
 *     ascending id, and keep the first k; pad with (id -1, score -inf) when
 *     fewer than k are eligible. mhtirogla.ai "Two-tower retrieval", Code
 *     section, `Towers::top_k` (score every item, stable sort descending, take
 *     k: a stable sort keeps the lower index first on equal scores).
 *
 * int8 scoring (recsys_two_tower_model.py `forward`, inner
 * `compute_top_k_int8`): each query row u is quantised symmetrically in fp32,
 * us = max(max_i |u_i| / 127, 1e-12), u8_i = clip(round(u_i / us), -127, 127)
 * (round half to even), and the candidate rows arrive as int8 codes with one
 * fp32 scale each; the score is the int32 dot product of the codes times
 * us times the candidate's scale. The pages do not show how the candidate
 * codes are made; they are taken to be the same scheme applied to the
 * L2-normalised candidate row (held in fp32). Here the score is the fp64
 * value of the dequantised vectors, (sum_i u8_i v8_ij) * us * scale_j / tau,
 * whose integer sum is exact.
 *
 * In-batch sampled softmax (training loss): users u_i (i < b) against the
 * candidate rows v_j (j < nc, nc >= b); row i's positive is candidate i and
 * the rest of the columns are its negatives ("Two-Tower Retrieval at
 * Industrial Scale", section 3, In-batch sampled softmax, `in_batch_loss`;
 * columns j >= b are negatives shared by every row, like the global
 * negatives of x-algorithm recsys_two_tower_model.py
 * `compute_retrieval_loss`). The corrected logit is
 * l_ij = (u_i . v_j) / tau - logq_j, with the correction on every column,
 * the positive included (same article, section 4, The LogQ Correction,
 * `corrected_in_batch_loss`). Column j enters row i's denominator when it is
 * valid and is not an accidental hit: a column j != i whose item id equals
 * item i's (`corrected_in_batch_loss`, masked with -inf; mhtirogla.ai
 * "Two-tower retrieval", Code section, `step`). Then
 * lse_i = log sum_j exp(l_ij) over that set, loss_i = lse_i - l_ii for a
 * valid row (0 for an invalid one), and the loss is the mean of loss_i over
 * the valid rows, 0 when there are none (`compute_retrieval_loss`:
 * neg_log_probs = log_denominator - numerator_logits, averaged over valid
 * positives, then over users with one).
 *
 * Storage rounding: where the corpus or the queries are stored in bf16 or
 * fp32, the fp64 normalised value is rounded once, to nearest with ties to
 * even, to the storage type (recsys_two_tower_model.py keeps the candidate
 * index as a bf16 array; `make_post_embeddings`).
 *
 * All arithmetic is IEEE fp64 in index order; no blocking or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_I8 2
#define ORACLE_EPS 1e-12
#define ORACLE_Q8_FLOOR 1e-12f

/* ---- element access ---------------------------------------------------- */

static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void *base, int dtype, int64_t idx)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[idx];
    if (dtype == ORACLE_I8)
        return (double)((const int8_t *)base)[idx];
    return bf16_bits_to_double(((const uint16_t *)base)[idx]);
}

/* Round an fp64 value to bf16, to nearest, ties to even, in one step (no
 * intermediate fp32 rounding). bf16 keeps 8 significant bits and the fp32
 * exponent range; below 2^-126 the quantum stays 2^-133 (subnormals). */
uint16_t oracle_bf16_from_double(double x)
{
    if (x == 0.0)
        return signbit(x) ? 0x8000u : 0x0000u;
    double ax = fabs(x);
    int e2;
    frexp(ax, &e2); /* ax = f * 2^e2, f in [0.5, 1): leading bit is 2^(e2-1) */
    int lead = e2 - 1;
    if (lead < -126)
        lead = -126;
    double quantum = ldexp(1.0, lead - 7);
    double q = rint(ax / quantum); /* default rounding mode: nearest-even */
    float v = (float)(q * quantum); /* exact: at most 9 significant bits */
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    uint16_t h = (uint16_t)(u >> 16);
    if (x < 0)
        h |= 0x8000u;
    return h;
}

static void store_elem(void *base, int dtype, int64_t idx, double y)
{
    if (dtype == ORACLE_F32)
        ((float *)base)[idx] = (float)y; /* C conversion rounds to nearest-even */
    else
        ((uint16_t *)base)[idx] = oracle_bf16_from_double(y);
}

/* ---- normalisation ------------------------------------------------------ */

/* norm_j = sqrt(max(sum_i v_ji^2, EPS)) for every row j. */
void oracle_row_norms(const void *in, int in_dtype, int64_t n, int d, double *norms)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) {
            double x = load_elem(in, in_dtype, j * (int64_t)d + i);
            ss += x * x;
        }
        norms[j] = sqrt(ss > ORACLE_EPS ? ss : ORACLE_EPS);
    }
}

/* out_j = v_j / norm_j, rounded once to out_dtype. */
void oracle_normalize(const void *in, int in_dtype, int64_t n, int d, void *out, int out_dtype)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) {
            double x = load_elem(in, in_dtype, j * (int64_t)d + i);
            ss += x * x;
        }
        double norm = sqrt(ss > ORACLE_EPS ? ss : ORACLE_EPS);
        for (int i = 0; i < d; ++i) {
            double x = load_elem(in, in_dtype, j * (int64_t)d + i);
            store_elem(out, out_dtype, j * (int64_t)d + i, x / norm);
        }
    }
}

/* ---- int8 quantisation -------------------------------------------------- */

/* Symmetric per-row int8 codes, in fp32 arithmetic as written on the page:
 * row values w_i (fp32), us = max(max|w_i| / 127, 1e-12),
 * code_i = clip(round_half_even(w_i / us), -127, 127).
 * normalise != 0: w_i = fl32(v_i / norm) with the fp64 norm of
 * oracle_normalize (the L2-normalised candidate row held in fp32);
 * normalise == 0: w_i = v_i as given (a query row). */
void oracle_quantize_rows(const void *in, int in_dtype, int64_t n, int d, int normalise,
                          int8_t *codes, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        double norm = 1.0;
        if (normalise) {
            double ss = 0.0;
            for (int i = 0; i < d; ++i) {
                double x = load_elem(in, in_dtype, j * (int64_t)d + i);
                ss += x * x;
            }
            norm = sqrt(ss > ORACLE_EPS ? ss : ORACLE_EPS);
        }
        float maxabs = 0.0f;
        for (int i = 0; i < d; ++i) {
            double x = load_elem(in, in_dtype, j * (int64_t)d + i);
            float w = normalise ? (float)(x / norm) : (float)x;
            float a = fabsf(w);
            if (a > maxabs)
                maxabs = a;
        }
        float us = maxabs / 127.0f;
        if (us < ORACLE_Q8_FLOOR)
            us = ORACLE_Q8_FLOOR;
        scales[j] = us;
        for (int i = 0; i < d; ++i) {
            double x = load_elem(in, in_dtype, j * (int64_t)d + i);
            float w = normalise ? (float)(x / norm) : (float)x;
            float r = rintf(w / us); /* nearest, ties to even */
            if (r > 127.0f)
                r = 127.0f;
            if (r < -127.0f)
                r = -127.0f;
            codes[j * (int64_t)d + i] = (int8_t)r;
        }
    }
}

/* ---- scoring and top-k ------------------------------------------------- */

static int is_excluded(const uint32_t *exclude, int64_t j)
{
    if (!exclude)
        return 0;
    return (int)((exclude[j >> 5] >> (j & 31)) & 1u);
}

/* s = (q . v_j) [/ norm_j] [* qscale_q * vscale_j] / tau, summed in index
 * order (for int8 codes every partial sum is an exact integer). */
static double score_one(const void *q, int q_dtype, int64_t qrow, const void *v, int v_dtype,
                        int64_t j, int d, const double *norms, const float *qscales,
                        const float *vscales, double tau)
{
    double dot = 0.0;
    for (int i = 0; i < d; ++i)
        dot += load_elem(q, q_dtype, qrow * (int64_t)d + i) *
               load_elem(v, v_dtype, j * (int64_t)d + i);
    if (norms)
        dot = dot / norms[j];
    if (qscales)
        dot = dot * (double)qscales[qrow] * (double)vscales[j];
    return dot / tau;
}

typedef struct {
    double s;
    int64_t id;
} oracle_pair;

/* Score descending; on equal scores the lower id comes first. */
static int cmp_pair(const void *pa, const void *pb)
{
    const oracle_pair *a = (const oracle_pair *)pa;
    const oracle_pair *b = (const oracle_pair *)pb;
    if (a->s > b->s)
        return -1;
    if (a->s < b->s)
        return 1;
    if (a->id < b->id)
        return -1;
    if (a->id > b->id)
        return 1;
    return 0;
}

/* For each of the b queries: score every eligible candidate, sort all of
 * them, keep the first k. out_ids [b,k] (int32), out_scores [b,k] (fp64).
 * Returns 0, or -1 if a work buffer could not be allocated. */
static int topk_impl(const void *q, int q_dtype, int64_t b, const void *v, int v_dtype, int64_t n,
                     int d, const double *norms, const float *qscales, const float *vscales,
                     const uint32_t *exclude, double tau, int64_t k, int32_t *out_ids,
                     double *out_scores)
{
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t qi = 0; qi < b; ++qi) {
        oracle_pair *pairs = (oracle_pair *)malloc((size_t)(n > 0 ? n : 1) * sizeof(oracle_pair));
        if (!pairs) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        int64_t m = 0;
        for (int64_t j = 0; j < n; ++j) {
            if (is_excluded(exclude, j))
                continue;
            pairs[m].s = score_one(q, q_dtype, qi, v, v_dtype, j, d, norms, qscales, vscales, tau);
            pairs[m].id = j;
            ++m;
        }
        qsort(pairs, (size_t)m, sizeof(oracle_pair), cmp_pair);
        for (int64_t r = 0; r < k; ++r) {
            if (r < m) {
                out_ids[qi * k + r] = (int32_t)pairs[r].id;
                out_scores[qi * k + r] = pairs[r].s;
            } else {
                out_ids[qi * k + r] = -1;
                out_scores[qi * k + r] = -INFINITY;
            }
        }
        free(pairs);
    }
    return failed ? -1 : 0;
}

int oracle_topk(const void *q, int q_dtype, int64_t b, const void *v, int v_dtype, int64_t n,
                int d, const double *norms, const uint32_t *exclude, double tau, int64_t k,
                int32_t *out_ids, double *out_scores)
{
    return topk_impl(q, q_dtype, b, v, v_dtype, n, d, norms, NULL, NULL, exclude, tau, k, out_ids,
                     out_scores);
}

/* Top-k over int8 codes: s = (sum_i q8_i v8_ji) * qscales[q] * vscales[j] / tau. */
int oracle_topk_q8(const int8_t *q, const float *qscales, int64_t b, const int8_t *v,
                   const float *vscales, int64_t n, int d, const uint32_t *exclude, double tau,
                   int64_t k, int32_t *out_ids, double *out_scores)
{
    return topk_impl(q, ORACLE_I8, b, v, ORACLE_I8, n, d, NULL, qscales, vscales, exclude, tau, k,
                     out_ids, out_scores);
}

/* Scores of listed candidates for one query: out[t] = s(qrow, ids[t]). */
void oracle_scores(const void *q, int q_dtype, int64_t qrow, const void *v, int v_dtype, int d,
                   const double *norms, double tau, const int64_t *ids, int64_t count,
                   double *out)
{
    for (int64_t t = 0; t < count; ++t)
        out[t] = score_one(q, q_dtype, qrow, v, v_dtype, ids[t], d, norms, NULL, NULL, tau);
}

void oracle_scores_q8(const int8_t *q, const float *qscales, int64_t qrow, const int8_t *v,
                      const float *vscales, int d, double tau, const int64_t *ids, int64_t count,
                      double *out)
{
    for (int64_t t = 0; t < count; ++t)
        out[t] = score_one(q, ORACLE_I8, qrow, v, ORACLE_I8, ids[t], d, NULL, qscales, vscales, tau);
}

/* ---- in-batch sampled softmax ------------------------------------------- */

static int inbatch_in_denominator(const int64_t *item_ids, const uint8_t *valid, int64_t i,
                                  int64_t j)
{
    if (valid && !valid[j])
        return 0;
    if (item_ids && j != i && item_ids[j] == item_ids[i])
        return 0; /* accidental hit: the same item as row i's positive */
    return 1;
}

/* lse [b], loss [b], *mean: see the header comment. u [b,d] and v [nc,d] in
 * their storage types; logq [nc] (NULL: no correction); item_ids [nc] (NULL:
 * no accidental-hit mask); valid [nc] bytes (NULL: every row and column is
 * valid). Returns 0, or -1 if a work buffer could not be allocated. */
int oracle_inbatch_softmax(const void *u, int u_dtype, int64_t b, const void *v, int v_dtype,
                           int64_t nc, int d, const double *logq, const int64_t *item_ids,
                           const uint8_t *valid, double tau, double *lse, double *loss,
                           double *mean)
{
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < b; ++i) {
        double *l = (double *)malloc((size_t)(nc > 0 ? nc : 1) * sizeof(double));
        if (!l) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        double m = -INFINITY;
        for (int64_t j = 0; j < nc; ++j) {
            l[j] = score_one(u, u_dtype, i, v, v_dtype, j, d, NULL, NULL, NULL, tau);
            if (logq)
                l[j] -= logq[j];
            if (inbatch_in_denominator(item_ids, valid, i, j) && l[j] > m)
                m = l[j];
        }
        /* log sum exp, with the largest term factored out so that nothing
         * overflows: log sum_j exp(l_j) = m + log sum_j exp(l_j - m) */
        double sum = 0.0;
        for (int64_t j = 0; j < nc; ++j)
            if (inbatch_in_denominator(item_ids, valid, i, j))
                sum += exp(l[j] - m);
        lse[i] = sum > 0.0 ? m + log(sum) : -INFINITY;
        loss[i] = (!valid || valid[i]) ? lse[i] - l[i] : 0.0;
        free(l);
    }
    if (failed)
        return -1;
    double total = 0.0;
    int64_t rows = 0;
    for (int64_t i = 0; i < b; ++i)
        if (!valid || valid[i]) {
            total += loss[i];
            ++rows;
        }
    *mean = rows > 0 ? total / (double)rows : 0.0;
    return 0;
}

/* ---- threading ---------------------------------------------------------- */

void oracle_set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
