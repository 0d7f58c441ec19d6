/*
 * Reference oracle for Loki-style low-rank-key sparse decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is compiled into liboracle.so, which only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg load.
 * The product library (rank_key_top_b200/csrc) never links, includes or calls
 * it, and it shares no header, helper, table or constant with that library.
 *
 * Everything here is plain, slow, single-threaded-per-problem C in binary64.
 * Each function restates one step of the method as the pages state it, in the
 * pages' order and notation, so that a reader can check it by eye:
 *
 *   AQUA page ("AQUA: Attention via QUery mAgnitudes ..."), decode-step
 *     equations (1)-(5): cache update, scores S = q K^T, scaling by
 *     1/sqrt(d_head), softmax, context c = A V.
 *   AQUA page, information-retention paragraph: projection is the row-vector
 *     product v_hat = v P.
 *   AQUA page, related work on LoKi: an offline projection transforms query and
 *     key vectors, the trailing dimensions are sliced off (the first ones are
 *     kept), and tokens are temporarily dropped based on the resulting
 *     approximate scores.
 *   Loki page ("Loki: Low-rank Keys for Efficient Sparse Attention"), abstract:
 *     tokens are ranked and selected by attention scores computed in the
 *     low-dimensional space.
 *   aitopics page "low rank approximation", LRQK abstract: the top-k tokens
 *     plus a small fixed set of recent tokens are kept and attended exactly.
 *   AQUA page, appendix on rotation invariance: q_hat K_hat^T = q K^T for an
 *     orthogonal P (used by the tests, not here).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - group reduction for grouped-query attention: the approximate score of a
 *     token for a kv head is the SUM over the group's query heads (option MAX);
 *   - ties in the approximate score go to the lower token index;
 *   - the recent window W is forced, top-k is taken among the other tokens;
 *   - the exact logits use the full head dimension and 1/sqrt(d) by default;
 *   - softmax is renormalised over the kept set only;
 *   - AQUA's per-dimension selection for a query group ranks a dim by the
 *     magnitude of the group's summed query (SUM) or by the heads' summed
 *     squares (MAX), ties to the lower dim;
 *   - the asymmetric factors minimise the score distortion with uncentred
 *     second moments (the SAKI abstract stops before its noise correction).
 * Every function below is pinned by tests/test_oracle_pins.py against values
 * the pages or the mathematics fix (closed forms, brute force, invariants,
 * hand-derived fixtures); none is left unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Rounding of an exact binary64 value to the cache storage types.           */
/* ------------------------------------------------------------------------- */

/* Round-to-nearest-even of a binary64 value to bfloat16 (1 sign bit, 8
 * exponent bits, 7 stored mantissa bits; 8 significant bits), done in one step
 * from binary64 so that no double rounding through binary32 can occur.
 * Returned as the binary64 value of the rounded bfloat16. */
double oracle_round_bf16(double v)
{
    if (v == 0.0 || isnan(v) || isinf(v))
        return v;
    int e;
    frexp(v, &e);                 /* v = m * 2^e with 0.5 <= |m| < 1 */
    int spacing_exp = e - 8;      /* 8 significant bits in this binade */
    if (spacing_exp < -133)       /* subnormal bfloat16 spacing is 2^-133 */
        spacing_exp = -133;
    double steps = nearbyint(ldexp(v, -spacing_exp)); /* ties to even */
    double r = ldexp(steps, spacing_exp);
    const double bf16_max = ldexp(255.0, 120);         /* (2 - 2^-7) * 2^127 */
    if (fabs(r) > bf16_max)
        r = copysign(INFINITY, v);
    return r;
}

/* bfloat16 bit pattern of a value that oracle_round_bf16 returned. */
uint16_t oracle_bf16_bits(double rounded)
{
    float f = (float)rounded;     /* exact: every bfloat16 is a binary32 */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void oracle_round_bf16_array(const double* x, int64_t n, double* out, uint16_t* bits)
{
    for (int64_t i = 0; i < n; ++i) {
        out[i] = oracle_round_bf16(x[i]);
        if (bits)
            bits[i] = oracle_bf16_bits(out[i]);
    }
}

/* ------------------------------------------------------------------------- */
/* Projection into the PCA basis: row vectors, v_hat = v P.                  */
/* AQUA page, information-retention paragraph and appendix step 1            */
/* ("projecting the current query and key with P").                          */
/* ------------------------------------------------------------------------- */
void oracle_rotate(const double* x, const double* P, int64_t n, int d, double* out)
{
    for (int64_t i = 0; i < n; ++i)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int a = 0; a < d; ++a)
                acc += x[i * d + a] * P[(int64_t)a * d + c];
            out[i * d + c] = acc;
        }
}

/* Cache update of a decode step (AQUA page, equations (1)-(2)) for keys kept
 * in the PCA basis: k_tilde = round(k P) to the cache type. dtype 1 = bf16,
 * dtype 0 = binary32. */
void oracle_append(const double* k_new, const double* P, int64_t n, int d, int dtype,
                   double* out)
{
    oracle_rotate(k_new, P, n, d, out);
    for (int64_t i = 0; i < n * d; ++i)
        out[i] = dtype == 1 ? oracle_round_bf16(out[i]) : (double)(float)out[i];
}

/* ------------------------------------------------------------------------- */
/* Exact attention over a given token set T, for the g query heads of one    */
/* kv head. AQUA page, equations (3)-(5): z = q_hat k_tilde^T * scale over    */
/* the full head dimension, A = softmax(z) over T, c = A V.                   */
/* qhat: [g][d] (already in the PCA basis). Kt, V: [L][d]. out: [g][d].       */
/* scale 0 means 1/sqrt(d).                                                   */
/* weights (nullable): [g][nT], the softmax weights in the order of T.        */
/* ------------------------------------------------------------------------- */
void oracle_attend_set(const double* Kt, const double* V, const double* qhat,
                       const int32_t* T, int nT, int d, int g, double scale,
                       double* out, double* weights)
{
    if (scale == 0.0)
        scale = 1.0 / sqrt((double)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)(nT > 0 ? nT : 1));
    for (int j = 0; j < g; ++j) {
        for (int c = 0; c < d; ++c)
            out[j * d + c] = 0.0;
        if (nT == 0)
            continue;
        /* equation (3), scaled as in equation (4) */
        double zmax = -INFINITY;
        for (int i = 0; i < nT; ++i) {
            const double* k = Kt + (int64_t)T[i] * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += qhat[j * d + c] * k[c];
            z[i] = s * scale;
            if (z[i] > zmax)
                zmax = z[i];
        }
        /* softmax of equation (4), shifted by the maximum for range only */
        double denom = 0.0;
        for (int i = 0; i < nT; ++i) {
            z[i] = exp(z[i] - zmax);
            denom += z[i];
        }
        /* context vector, equation (5) */
        for (int i = 0; i < nT; ++i) {
            double a = z[i] / denom;
            if (weights)
                weights[(int64_t)j * nT + i] = a;
            const double* v = V + (int64_t)T[i] * d;
            for (int c = 0; c < d; ++c)
                out[j * d + c] += a * v[c];
        }
    }
    free(z);
}

/* ------------------------------------------------------------------------- */
/* Top-k with ties to the lower index: sort candidates by (score descending, */
/* index ascending) and keep the first k.                                    */
/* ------------------------------------------------------------------------- */
typedef struct {
    double s;
    int32_t t;
} scored_token;

static int by_score_then_index(const void* pa, const void* pb)
{
    const scored_token* a = (const scored_token*)pa;
    const scored_token* b = (const scored_token*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

static int by_index(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Step 4 of a decode: keep the k best of the ncand candidates, ties to the  */
/* lower index, in ascending order, then add the recent window (LRQK: top-k  */
/* tokens plus a fixed set of recent ones). cand is sorted in place; T has   */
/* room for ncand + w_eff entries. Returns the number kept; *kth (nullable)  */
/* gets the score of the last token kept by score, NaN if none.              */
static int keep_top_k_and_window(scored_token* cand, int ncand, int k, int w_eff, int32_t* T, double* kth)
{
    int keff = k < ncand ? k : ncand;
    qsort(cand, (size_t)ncand, sizeof(scored_token), by_score_then_index);
    if (kth)
        *kth = keff > 0 ? cand[keff - 1].s : NAN;
    for (int i = 0; i < keff; ++i)
        T[i] = cand[i].t;
    qsort(T, (size_t)keff, sizeof(int32_t), by_index);
    for (int i = 0; i < w_eff; ++i)
        T[keff + i] = ncand + i;
    return keff + w_eff;
}

/* ------------------------------------------------------------------------- */
/* One decode step of Loki-style sparse attention for one (sequence, kv      */
/* head) pair and its g query heads.                                         */
/*                                                                           */
/* Kt  [L][d]  keys as stored in the cache, already in the PCA basis          */
/* V   [L][d]  values as stored                                               */
/* q   [g][d]  unrotated queries of the group                                 */
/* P   [d][d]  projection, row-major; the PCA basis is v_hat = v P            */
/* r           number of leading rotated dimensions used for scoring          */
/* k           tokens kept by score; W recent tokens always kept              */
/* group_max   0: group score = sum over heads; 1: maximum over heads         */
/* scale       exact-logit scale; 0 means 1/sqrt(d)                           */
/* out [g][d]  attention output                                               */
/* sel [k+W]   kept token indices, ascending, -1 padded (nullable)            */
/* n_sel       number of kept tokens (nullable)                               */
/* scores [L]  approximate scores of the candidates, NaN elsewhere (nullable) */
/* kth         score of the last token kept by score, NaN if none (nullable)  */
/* Returns 0, or -1 when k = 0 and W = 0 (nothing could ever be kept).        */
/* ------------------------------------------------------------------------- */
int oracle_decode_pair(const double* Kt, const double* V, const double* q, const double* P,
                       int L, int d, int g, int r, int k, int W, int group_max, double scale,
                       double* out, int32_t* sel, int* n_sel, double* scores, double* kth)
{
    if (k < 0 || W < 0 || (k == 0 && W == 0) || r < 1 || r > d || L < 0)
        return -1;
    if (scale == 0.0)
        scale = 1.0 / sqrt((double)d);

    /* Step 1: rotate the queries into the PCA basis (AQUA appendix, step 1). */
    double* qhat = (double*)malloc(sizeof(double) * (size_t)g * d);
    oracle_rotate(q, P, g, d, qhat);

    /* Step 2: candidates are the tokens outside the forced recent window.    */
    int w_eff = W < L ? W : L;
    int ncand = L - w_eff;

    /* Step 3: approximate scores from the leading r rotated dimensions only  */
    /* (LoKi as described on the AQUA page: slice the trailing dimensions;    */
    /* Loki abstract: scores computed in the low-dimensional space).          */
    scored_token* cand = (scored_token*)malloc(sizeof(scored_token) * (size_t)(ncand > 0 ? ncand : 1));
    for (int t = 0; t < ncand; ++t) {
        const double* kt = Kt + (int64_t)t * d;
        double s = group_max ? -INFINITY : 0.0;
        for (int j = 0; j < g; ++j) {
            double sj = 0.0;
            for (int c = 0; c < r; ++c)
                sj += qhat[j * d + c] * kt[c];
            if (group_max)
                s = sj > s ? sj : s;
            else
                s += sj;
        }
        cand[t].s = s;
        cand[t].t = t;
    }
    if (scores) {
        for (int t = 0; t < L; ++t)
            scores[t] = NAN;
        for (int t = 0; t < ncand; ++t)
            scores[t] = cand[t].s;
    }

    /* Step 4: keep the k best candidates and the recent window.             */
    int32_t* T = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ncand + w_eff + 1));
    int nT = keep_top_k_and_window(cand, ncand, k, w_eff, T, kth);

    /* Step 5: exact softmax attention over the kept set (equations (3)-(5)). */
    oracle_attend_set(Kt, V, qhat, T, nT, d, g, scale, out, NULL);

    if (sel) {
        for (int i = 0; i < k + W; ++i)
            sel[i] = i < nT ? T[i] : -1;
    }
    if (n_sel)
        *n_sel = nT;
    free(T);
    free(cand);
    free(qhat);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Key index of an asymmetric score factorisation (SAKI page, abstract: a    */
/* rank-r factorisation of the query-key score operator with its own key     */
/* factor): idx = round(k A_k) to the cache type, row vectors.               */
/* k [n][d]; Ak [d][ri] row-major; out [n][ri]. dtype 1 = bf16, 0 = binary32. */
/* ------------------------------------------------------------------------- */
void oracle_index_keys(const double* k, const double* Ak, int64_t n, int d, int ri, int dtype, double* out)
{
    for (int64_t i = 0; i < n; ++i)
        for (int c = 0; c < ri; ++c) {
            double acc = 0.0;
            for (int a = 0; a < d; ++a)
                acc += k[i * d + a] * Ak[(int64_t)a * ri + c];
            out[i * ri + c] = dtype == 1 ? oracle_round_bf16(acc) : (double)(float)acc;
        }
}

/* ------------------------------------------------------------------------- */
/* One decode step whose approximate scores come from an asymmetric pair of */
/* factors (SAKI page, abstract: the score q k^T is approximated as          */
/* (q A_q)(k A_k)^T, A_q and A_k of rank r from the SVD of the covariance-   */
/* weighted query-key operator). The key index holds the stored rows         */
/* Kidx[t] = round(k_t A_k); for the candidates                               */
/*   s_t = reduce_j sum_{c < r} (q_j A_q)[c] * Kidx[t][c].                    */
/* Steps 2, 4 and 5 are those of oracle_decode_pair: the exact attention     */
/* uses q_hat = q P against the full keys Kt in the PCA basis.                */
/* Kidx [L][ri]; Aq [d][ri] row-major, its first r columns are used.         */
/* Other arguments and the return value as for oracle_decode_pair.           */
/* ------------------------------------------------------------------------- */
int oracle_decode_pair_asym(const double* Kt, const double* V, const double* Kidx, const double* q,
                            const double* P, const double* Aq, int L, int d, int ri, int g, int r, int k,
                            int W, int group_max, double scale, double* out, int32_t* sel, int* n_sel,
                            double* scores, double* kth)
{
    if (k < 0 || W < 0 || (k == 0 && W == 0) || r < 1 || r > ri || ri > d || L < 0)
        return -1;
    if (scale == 0.0)
        scale = 1.0 / sqrt((double)d);

    /* Step 1: the query in the PCA basis (exact attention) and its score    */
    /* factor q A_q (first r columns).                                       */
    double* qhat = (double*)malloc(sizeof(double) * (size_t)g * d);
    double* qt = (double*)malloc(sizeof(double) * (size_t)g * r);
    oracle_rotate(q, P, g, d, qhat);
    for (int j = 0; j < g; ++j)
        for (int c = 0; c < r; ++c) {
            double acc = 0.0;
            for (int a = 0; a < d; ++a)
                acc += q[j * d + a] * Aq[(int64_t)a * ri + c];
            qt[j * r + c] = acc;
        }

    /* Step 2: candidates are the tokens outside the forced recent window.    */
    int w_eff = W < L ? W : L;
    int ncand = L - w_eff;

    /* Step 3: approximate scores from the key index and the query factor.   */
    scored_token* cand = (scored_token*)malloc(sizeof(scored_token) * (size_t)(ncand > 0 ? ncand : 1));
    for (int t = 0; t < ncand; ++t) {
        const double* x = Kidx + (int64_t)t * ri;
        double s = group_max ? -INFINITY : 0.0;
        for (int j = 0; j < g; ++j) {
            double sj = 0.0;
            for (int c = 0; c < r; ++c)
                sj += qt[j * r + c] * x[c];
            if (group_max)
                s = sj > s ? sj : s;
            else
                s += sj;
        }
        cand[t].s = s;
        cand[t].t = t;
    }
    if (scores) {
        for (int t = 0; t < L; ++t)
            scores[t] = NAN;
        for (int t = 0; t < ncand; ++t)
            scores[t] = cand[t].s;
    }

    /* Step 4: keep the k best candidates and the recent window.             */
    int32_t* T = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ncand + w_eff + 1));
    int nT = keep_top_k_and_window(cand, ncand, k, w_eff, T, kth);

    /* Step 5: exact softmax attention over the kept set (equations (3)-(5)). */
    oracle_attend_set(Kt, V, qhat, T, nT, d, g, scale, out, NULL);

    if (sel) {
        for (int i = 0; i < k + W; ++i)
            sel[i] = i < nT ? T[i] : -1;
    }
    if (n_sel)
        *n_sel = nT;
    free(T);
    free(cand);
    free(qt);
    free(qhat);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Dense decode attention for one (sequence, kv head) pair: equations (3)-(5) */
/* over every token, written independently of the sparse path. With P = NULL */
/* the keys are used as given (the unrotated comparison); otherwise the       */
/* queries are rotated by P first and K holds keys in the PCA basis.         */
/* ------------------------------------------------------------------------- */
void oracle_dense_pair(const double* K, const double* V, const double* q, const double* P,
                       int L, int d, int g, double scale, double* out)
{
    if (scale == 0.0)
        scale = 1.0 / sqrt((double)d);
    double* qq = (double*)malloc(sizeof(double) * (size_t)g * d);
    if (P)
        oracle_rotate(q, P, g, d, qq);
    else
        memcpy(qq, q, sizeof(double) * (size_t)g * d);
    double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int j = 0; j < g; ++j) {
        double zmax = -INFINITY;
        for (int t = 0; t < L; ++t) {
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += qq[j * d + c] * K[(int64_t)t * d + c];
            z[t] = s * scale;
            zmax = z[t] > zmax ? z[t] : zmax;
        }
        double denom = 0.0;
        for (int t = 0; t < L; ++t) {
            z[t] = exp(z[t] - zmax);
            denom += z[t];
        }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < L; ++t)
                acc += z[t] / denom * V[(int64_t)t * d + c];
            out[j * d + c] = L > 0 ? acc : 0.0;
        }
    }
    free(z);
    free(qq);
}

/* ------------------------------------------------------------------------- */
/* Many independent pairs at once (the same computation as above, one pair   */
/* per OpenMP thread). Pair p reads Kt/V at p*Lmax*d, q at p*g*d, P at p*d*d */
/* and writes out at p*g*d, sel at p*(kmax+W).                                */
/* ------------------------------------------------------------------------- */
int oracle_decode_batch(int n_pairs, const double* Kt, const double* V, const double* q,
                        const double* P, const int32_t* L, int Lmax, int d, int g, int r,
                        const int32_t* k_per_pair, int kmax, int W, int group_max,
                        double scale, double* out, int32_t* sel)
{
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int p = 0; p < n_pairs; ++p) {
        int32_t* s = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k_per_pair[p] + W));
        int rc = oracle_decode_pair(Kt + (int64_t)p * Lmax * d, V + (int64_t)p * Lmax * d,
                                    q + (int64_t)p * g * d, P + (int64_t)p * d * d, L[p], d, g,
                                    r, k_per_pair[p], W, group_max, scale,
                                    out + (int64_t)p * g * d, s, NULL, NULL, NULL);
        if (rc != 0)
            bad = 1;
        if (sel)
            for (int i = 0; i < kmax + W; ++i)
                sel[(int64_t)p * (kmax + W) + i] = i < k_per_pair[p] + W ? s[i] : -1;
        free(s);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------- */
/* Offline calibration of P: the principal directions of calibration keys.   */
/* AQUA page, appendix on SVD (the basis whose leading columns hold the most */
/* variance) and Fig. 2 (P calibrated once, on other data). The covariance   */
/* is centred and normalised by 1/n (this oracle's reading; the directions   */
/* do not depend on the normalisation). The eigendecomposition itself is a   */
/* library step of the Python wrapper.                                       */
/*   C[i][j] = (1/n) sum_t (x[t][i] - mu[i]) (x[t][j] - mu[j]),              */
/*   mu[i]   = (1/n) sum_t x[t][i].                                          */
/* ------------------------------------------------------------------------- */
void oracle_covariance(const double* x, int64_t n, int d, double* C)
{
    double* mu = (double*)calloc((size_t)d, sizeof(double));
    for (int64_t t = 0; t < n; ++t)
        for (int i = 0; i < d; ++i)
            mu[i] += x[t * d + i];
    for (int i = 0; i < d; ++i)
        mu[i] /= (double)n;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) {
            double s = 0.0;
            for (int64_t t = 0; t < n; ++t)
                s += (x[t * d + i] - mu[i]) * (x[t * d + j] - mu[j]);
            C[i * d + j] = s / (double)n;
        }
    free(mu);
}

/* ------------------------------------------------------------------------- */
/* Magnitude-based choice of scoring dimensions for one (sequence, kv head)  */
/* pair (AQUA page, Algorithm 1 in prose: per decode step, the dimensions    */
/* whose projected-query magnitude is largest are the ones used to score;    */
/* information-retention paragraph: what a choice keeps is the energy of     */
/* the projected vector on it). This library's reading chooses whole slabs   */
/* of 16 consecutive dimensions among the first index_dims:                  */
/*   u = sum_j q_hat_j  (group SUM):   e_s = sum_{c in slab s} u[c]^2        */
/*   group MAX:                        e_s = sum_j sum_{c in slab s} q_hat_j[c]^2 */
/* and keeps the r/16 slabs of largest e_s, ties to the lower slab, listed   */
/* in ascending order.                                                       */
/*                                                                           */
/* q [g][d] unrotated queries; P [d][d]; slabs [r/16] (written, ascending);  */
/* energy [index_dims/16] (nullable). Returns 0, or -1 on bad sizes.         */
/* ------------------------------------------------------------------------- */
int oracle_magnitude_slabs(const double* q, const double* P, int d, int g, int index_dims, int r,
                           int group_max, int32_t* slabs, double* energy)
{
    if (d < 16 || index_dims < 16 || index_dims > d || index_dims % 16 != 0 || r < 16 || r > index_dims ||
        r % 16 != 0 || g < 1)
        return -1;
    int nsl = index_dims / 16, keep = r / 16;
    double* qhat = (double*)malloc(sizeof(double) * (size_t)g * d);
    double* e = (double*)calloc((size_t)nsl, sizeof(double));
    oracle_rotate(q, P, g, d, qhat);
    for (int s = 0; s < nsl; ++s)
        for (int c = 16 * s; c < 16 * s + 16; ++c) {
            if (group_max) {
                for (int j = 0; j < g; ++j)
                    e[s] += qhat[j * d + c] * qhat[j * d + c];
            } else {
                double u = 0.0;
                for (int j = 0; j < g; ++j)
                    u += qhat[j * d + c];
                e[s] += u * u;
            }
        }
    /* slab s is kept when fewer than r/16 slabs beat it (larger energy, or */
    /* equal energy at a lower index)                                       */
    int n = 0;
    for (int s = 0; s < nsl; ++s) {
        int beaten_by = 0;
        for (int o = 0; o < nsl; ++o)
            if (e[o] > e[s] || (e[o] == e[s] && o < s))
                ++beaten_by;
        if (beaten_by < keep)
            slabs[n++] = s;
    }
    if (energy)
        for (int s = 0; s < nsl; ++s)
            energy[s] = e[s];
    free(e);
    free(qhat);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Magnitude-based choice of single scoring dimensions for one (sequence,    */
/* kv head) pair: AQUA page, Algorithm 1 in prose (at each decode step the   */
/* indices of the top dimensions by magnitude of the projected query are     */
/* found, and the approximate scores use only those dimensions of the query  */
/* and of the key cache) and its appendix on complexity, steps 2-4 (the      */
/* element-wise absolute value of q_hat, a selection of the top indices,     */
/* the slice of those columns of the key cache, the product with the sliced  */
/* query).                                                                   */
/*                                                                           */
/* The page scores one query; for a group of g query heads that share a kv   */
/* head (the pages are silent on grouped-query attention) this oracle reads  */
/* the magnitude of dimension c as                                           */
/*   SUM: w[c] = |u[c]|, u = sum_j q_hat_j  (the query that ranks the tokens) */
/*   MAX: w[c] = sqrt(sum_j q_hat_j[c]^2)  (every head scores alone)         */
/* so that for g = 1 both are |q_hat[c]|. The r dimensions of largest w      */
/* among the first index_dims are kept, ties to the lower dimension, and are */
/* listed in ascending order.                                                */
/*                                                                           */
/* q [g][d] unrotated queries; P [d][d]; dims [r] (written, ascending);      */
/* weight [index_dims] (nullable): w. Returns 0, or -1 on bad sizes.         */
/* ------------------------------------------------------------------------- */
int oracle_magnitude_dims(const double* q, const double* P, int d, int g, int index_dims, int r,
                          int group_max, int32_t* dims, double* weight)
{
    if (d < 1 || g < 1 || index_dims < 1 || index_dims > d || r < 1 || r > index_dims)
        return -1;
    double* qhat = (double*)malloc(sizeof(double) * (size_t)g * d);
    double* w = (double*)malloc(sizeof(double) * (size_t)index_dims);
    /* appendix step 1: project the query */
    oracle_rotate(q, P, g, d, qhat);
    /* appendix step 2: element-wise magnitude */
    for (int c = 0; c < index_dims; ++c) {
        double acc = 0.0;
        if (group_max) {
            for (int j = 0; j < g; ++j)
                acc += qhat[j * d + c] * qhat[j * d + c];
            w[c] = sqrt(acc);
        } else {
            for (int j = 0; j < g; ++j)
                acc += qhat[j * d + c];
            w[c] = fabs(acc);
        }
    }
    /* appendix step 2: the indices of the r largest magnitudes. Dimension c */
    /* is kept when fewer than r dimensions beat it (a larger magnitude, or  */
    /* an equal one at a lower index).                                       */
    int n = 0;
    for (int c = 0; c < index_dims; ++c) {
        int beaten_by = 0;
        for (int o = 0; o < index_dims; ++o)
            if (w[o] > w[c] || (w[o] == w[c] && o < c))
                ++beaten_by;
        if (beaten_by < r)
            dims[n++] = c;
    }
    if (weight)
        for (int c = 0; c < index_dims; ++c)
            weight[c] = w[c];
    free(w);
    free(qhat);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* One decode step whose approximate scores use the dimensions that          */
/* oracle_magnitude_dims chooses (AQUA page, appendix on complexity, steps   */
/* 3-4: the key cache sliced to those columns, times the sliced query):      */
/*   s_t = reduce_j sum_{c in dims, ascending} q_hat_j[c] * K~[t][c].        */
/* Steps 2, 4 and 5 are those of oracle_decode_pair. index_dims bounds the   */
/* dimensions to choose from; dims_out [r] (nullable) receives the choice.   */
/* Other arguments and the return value as for oracle_decode_pair.           */
/* ------------------------------------------------------------------------- */
int oracle_decode_pair_dims(const double* Kt, const double* V, const double* q, const double* P,
                            int L, int d, int g, int index_dims, int r, int k, int W, int group_max,
                            double scale, double* out, int32_t* sel, int* n_sel, double* scores,
                            double* kth, int32_t* dims_out)
{
    if (k < 0 || W < 0 || (k == 0 && W == 0) || r < 1 || r > index_dims || index_dims > d || L < 0)
        return -1;
    if (scale == 0.0)
        scale = 1.0 / sqrt((double)d);

    /* Steps 1-2 of the appendix: the query in the PCA basis and the r       */
    /* dimensions of largest magnitude.                                      */
    int32_t* dims = (int32_t*)malloc(sizeof(int32_t) * (size_t)r);
    if (oracle_magnitude_dims(q, P, d, g, index_dims, r, group_max, dims, NULL) != 0) {
        free(dims);
        return -1;
    }
    double* qhat = (double*)malloc(sizeof(double) * (size_t)g * d);
    oracle_rotate(q, P, g, d, qhat);

    /* Candidates are the tokens outside the forced recent window.           */
    int w_eff = W < L ? W : L;
    int ncand = L - w_eff;

    /* Steps 3-4 of the appendix: scores from the chosen columns only.       */
    scored_token* cand = (scored_token*)malloc(sizeof(scored_token) * (size_t)(ncand > 0 ? ncand : 1));
    for (int t = 0; t < ncand; ++t) {
        const double* kt = Kt + (int64_t)t * d;
        double s = group_max ? -INFINITY : 0.0;
        for (int j = 0; j < g; ++j) {
            double sj = 0.0;
            for (int i = 0; i < r; ++i)
                sj += qhat[j * d + dims[i]] * kt[dims[i]];
            if (group_max)
                s = sj > s ? sj : s;
            else
                s += sj;
        }
        cand[t].s = s;
        cand[t].t = t;
    }
    if (scores) {
        for (int t = 0; t < L; ++t)
            scores[t] = NAN;
        for (int t = 0; t < ncand; ++t)
            scores[t] = cand[t].s;
    }

    /* Keep the k best candidates and the recent window, then attend exactly */
    /* over the full head dimension (equations (3)-(5)).                     */
    int32_t* T = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ncand + w_eff + 1));
    int nT = keep_top_k_and_window(cand, ncand, k, w_eff, T, kth);
    oracle_attend_set(Kt, V, qhat, T, nT, d, g, scale, out, NULL);

    if (sel) {
        for (int i = 0; i < k + W; ++i)
            sel[i] = i < nT ? T[i] : -1;
    }
    if (n_sel)
        *n_sel = nT;
    if (dims_out)
        for (int i = 0; i < r; ++i)
            dims_out[i] = dims[i];
    free(T);
    free(cand);
    free(qhat);
    free(dims);
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
