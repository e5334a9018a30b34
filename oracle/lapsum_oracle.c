/*
 * Fast LapSum soft top-k -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  The CUDA product path
 * never calls, links or includes anything from here, and nothing here comes
 * from the CUDA path: the two share no code.
 *
 * What it computes follows "Fast LapSum: Exact Differentiable Top-k at Million
 * Scale" (gist.science explainer pages):
 *   - section 2.1 "The LapSum operator": p_i = sigma((r_i - b)/t) with sigma the
 *     CDF of Laplace(0,1) (scores perturbed by Laplace(0,t) noise), and the
 *     scalar b fixed by sum_i p_i = k, solved exactly;
 *   - section 2.1, last sentence: the backward pass is an analytic VJP.  The
 *     pages print no formula; the one used is the implicit-function derivative
 *     of the budget equation, g_i = (f_i/t)(v_i - sum_j v_j f_j / sum_j f_j),
 *     f_i = 0.5 exp(-|r_i - b|/t) = sigma'((r_i-b)/t);
 *   - section 2.2 "Probabilistic bracketing", steps 1-2: a sample of
 *     Laplace-noised scores, a bracket [a_L, a_R) from binomial order
 *     statistics, and the fold of out-of-bracket scores into tail sums;
 *   - section 2.3 "Relation to DFTopK": the zero-temperature limit of the
 *     operator (the midpoint threshold, with tied boundary scores sharing the
 *     remaining budget), written out in lso_hard_topk.
 *
 * The threshold solve is the plain definition, not the paper's fast solver:
 * a full sort (used only to bound the search), then bisection on b with the
 * sign of F(b) - k taken in a cancellation-free form (exact integer count plus
 * two log-sum-exps), run to full fp64 resolution.
 *
 * Parity pins (tests/test_oracle_pins.py) tie every function here to something
 * other than itself: closed forms (n = 1, all-equal rows, the symmetric
 * two-point row), a high-precision segment-by-segment quadratic brute force on
 * tiny rows, invariants (shift, scale, permutation, mirror), the zero
 * temperature limit, central finite differences of the VJP, the published
 * SplitMix64 test vector and scipy's binomial distribution; the hard top-k by
 * worked cases and by the soft solve far below the score gaps.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define LSO_OK 0
#define LSO_EINVAL 1
#define LSO_ENONFINITE 3

int lso_abi_version(void) { return 1; }

/* CDF of Laplace(0,1): 0.5 e^x below zero, 1 - 0.5 e^-x at and above zero. */
double lso_laplace_cdf(double x) { return x < 0.0 ? 0.5 * exp(x) : 1.0 - 0.5 * exp(-x); }

/* ---------------------------------------------------------------------------
 * F(b) = sum_i sigma((r_i - b)/t), summed pairwise (recursive halving).  Used
 * for the reported budget sum; the solve itself uses the sign function below.
 * ------------------------------------------------------------------------- */
static double budget_sum_range(const double* r, int64_t lo, int64_t hi, double b, double t) {
    if (hi - lo <= 32) {
        double s = 0.0;
        for (int64_t i = lo; i < hi; ++i) s += lso_laplace_cdf((r[i] - b) / t);
        return s;
    }
    int64_t mid = lo + (hi - lo) / 2;
    return budget_sum_range(r, lo, mid, b, t) + budget_sum_range(r, mid, hi, b, t);
}

double lso_budget_sum(const double* r, int64_t n, double b, double t) {
    return budget_sum_range(r, 0, n, b, t);
}

/* ---------------------------------------------------------------------------
 * Sign of F(b) - k without cancellation.
 *   F(b) - k = c_b - 0.5 e^U + 0.5 e^L, where
 *   c_b = #{r_i >= b} - k                     (exact),
 *   U   = log sum_{r_i >= b} exp(-(r_i - b)/t),
 *   L   = log sum_{r_i <  b} exp( (r_i - b)/t).
 * When c_b == 0 the sign is the sign of L - U, which stays exact on the flat
 * stretches of F between widely spaced scores where a plain sum rounds to k.
 * Returns +1, 0 or -1.
 * ------------------------------------------------------------------------- */
int lso_budget_sign(const double* r, int64_t n, double b, double k, double t) {
    int64_t count_ge = 0;
    double max_u = -INFINITY, max_l = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double x = (r[i] - b) / t;
        if (r[i] >= b) {
            ++count_ge;
            if (-x > max_u) max_u = -x;
        } else {
            if (x > max_l) max_l = x;
        }
    }
    double su = 0.0, sl = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double x = (r[i] - b) / t;
        if (r[i] >= b) su += exp(-x - max_u);
        else sl += exp(x - max_l);
    }
    double U = count_ge > 0 ? max_u + log(su) : -INFINITY;
    double L = count_ge < n ? max_l + log(sl) : -INFINITY;
    double c = (double)count_ge - k;
    if (c == 0.0) {
        if (L > U) return 1;
        if (L < U) return -1;
        return 0;
    }
    double val = c - 0.5 * exp(U) + 0.5 * exp(L);
    return (val > 0.0) - (val < 0.0);
}

static int cmp_double(const void* a, const void* b) {
    double x = *(const double*)a, y = *(const double*)b;
    return (x > y) - (x < y);
}

/* Validation shared by the entry points: 0 < k < n, t > 0, finite scores. */
static int validate(const double* r, int64_t n, double k, double t) {
    if (r == NULL || n < 1 || !(t > 0.0) || !isfinite(t) || !(k > 0.0) || !(k < (double)n))
        return LSO_EINVAL;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(r[i])) return LSO_ENONFINITE;
    return LSO_OK;
}

/* ---------------------------------------------------------------------------
 * Exact threshold b with F(b) = k.
 *   1. sort a copy of the scores (full sort);
 *   2. closed-form outer bounds:
 *        b_hi = s_max + t max(0, ln(n/(2k)))      so F(b_hi) <= k,
 *        b_lo = s_min + t min(0, ln(2(n-k)/n))    so F(b_lo) >= k;
 *   3. binary search over the sorted scores for the last s_j with
 *      F(s_j) >= k, which narrows [b_lo, b_hi] to one gap of the sorted order;
 *   4. bisection on b with the cancellation-free sign until the midpoint
 *      equals an endpoint (full fp64 resolution) or 400 steps.
 * `iters` (may be NULL) receives the number of sign evaluations.
 * ------------------------------------------------------------------------- */
int lso_solve_b(const double* r, int64_t n, double k, double t, double* b_out, int* iters) {
    int st = validate(r, n, k, t);
    if (st != LSO_OK) return st;
    double* s = (double*)malloc((size_t)n * sizeof(double));
    if (!s) return LSO_EINVAL;
    memcpy(s, r, (size_t)n * sizeof(double));
    qsort(s, (size_t)n, sizeof(double), cmp_double);

    int evals = 0;
    double lo = s[0] + t * fmin(0.0, log(2.0 * ((double)n - k) / (double)n));
    double hi = s[n - 1] + t * fmax(0.0, log((double)n / (2.0 * k)));

    /* F is decreasing; find the largest index j with sign(F(s_j) - k) >= 0. */
    int64_t jlo = -1, jhi = n; /* invariant: F(s_jlo) >= k (or jlo = -1), F(s_jhi) < k (or jhi = n) */
    while (jhi - jlo > 1) {
        int64_t jm = jlo + (jhi - jlo) / 2;
        int sg = lso_budget_sign(s, n, s[jm], k, t);
        ++evals;
        if (sg >= 0) jlo = jm; else jhi = jm;
    }
    if (jlo >= 0 && s[jlo] > lo) lo = s[jlo];
    if (jhi < n && s[jhi] < hi) hi = s[jhi];

    double b = lo;
    for (int it = 0; it < 400; ++it) {
        double mid = lo + 0.5 * (hi - lo);
        if (!(mid > lo) || !(mid < hi)) { b = mid; break; }
        int sg = lso_budget_sign(s, n, mid, k, t);
        ++evals;
        if (sg > 0) lo = mid;
        else if (sg < 0) hi = mid;
        else { lo = hi = mid; b = mid; break; }
        b = lo + 0.5 * (hi - lo);
    }
    free(s);
    *b_out = b;
    if (iters) *iters = evals;
    return LSO_OK;
}

/* p_i = sigma((r_i - b)/t). */
void lso_emit_p(const double* r, int64_t n, double b, double t, double* p) {
    for (int64_t i = 0; i < n; ++i) p[i] = lso_laplace_cdf((r[i] - b) / t);
}

/* f_i = 0.5 exp(-|r_i - b|/t), the Laplace density at the scaled margin. */
void lso_density(const double* r, int64_t n, double b, double t, double* f) {
    for (int64_t i = 0; i < n; ++i) f[i] = 0.5 * exp(-fabs(r[i] - b) / t);
}

/* ---------------------------------------------------------------------------
 * VJP  g_i = (f_i/t)(v_i - R),  R = sum_j v_j f_j / sum_j f_j.
 * R is formed with weights w_j = exp(-(|x_j| - mu)), mu = min_j |x_j|, so it
 * never becomes 0/0 when every f_j underflows.  Outputs R and
 * sum_f = 0.5 e^-mu sum_j w_j (may be NULL).
 * ------------------------------------------------------------------------- */
void lso_vjp(const double* r, const double* v, int64_t n, double b, double t, double* g,
             double* R_out, double* sum_f_out) {
    double mu = INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double ax = fabs(r[i] - b) / t;
        if (ax < mu) mu = ax;
    }
    double sw = 0.0, swv = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(-(fabs(r[i] - b) / t - mu));
        sw += w;
        swv += w * v[i];
    }
    double R = swv / sw;
    for (int64_t i = 0; i < n; ++i) {
        double f = 0.5 * exp(-fabs(r[i] - b) / t);
        g[i] = (f / t) * (v[i] - R);
    }
    if (R_out) *R_out = R;
    if (sum_f_out) *sum_f_out = 0.5 * exp(-mu) * sw;
}

/* ---------------------------------------------------------------------------
 * Gradients of L = sum_i v_i p_i with respect to the budget k and the
 * temperature t (section 2.1's budget equation differentiated implicitly,
 * the same way as the VJP above).  With x_i = (r_i - b)/t, f_i = 0.5 e^{-|x_i|}:
 *   db/dk = -t / sum f            so  dL/dk = sum v f / sum f;
 *   db/dt = -sum f x / sum f      so  dL/dt = -(1/t) sum_i v_i f_i (x_i - xbar),
 *   xbar = sum f x / sum f.
 * The weights are shifted by min |x| as in lso_vjp; dL/dt carries the shift
 * back through 0.5 e^{-mu}.
 * ------------------------------------------------------------------------- */
void lso_vjp_kt(const double* r, const double* v, int64_t n, double b, double t, double* g_k,
                double* g_t) {
    double mu = INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double ax = fabs(r[i] - b) / t;
        if (ax < mu) mu = ax;
    }
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;  /* sums of w, w v, w x, w v x */
    for (int64_t i = 0; i < n; ++i) {
        double x = (r[i] - b) / t;
        double wt = exp(-(fabs(x) - mu));
        a0 += wt;
        a1 += wt * v[i];
        a2 += wt * x;
        a3 += wt * v[i] * x;
    }
    *g_k = a1 / a0;
    *g_t = -(1.0 / t) * 0.5 * exp(-mu) * (a3 - a1 * a2 / a0);
}

/* ---------------------------------------------------------------------------
 * Probabilistic bracketing, step 2 (fold): with a bracket [aL, aR),
 *   cnt_R = #{r >= aR},  S_R = sum_{r >= aR} exp(-(r - aR)/t),
 *   cnt_L = #{r <  aL},  S_L = sum_{r <  aL} exp( (r - aL)/t),
 *   n_band = #{aL <= r < aR}.
 * Every term is at most 1.  aR = +inf or aL = -inf give empty tails.
 * ------------------------------------------------------------------------- */
void lso_fold(const double* r, int64_t n, double aL, double aR, double t, int64_t* cnt_R,
              int64_t* cnt_L, int64_t* n_band, double* S_L, double* S_R) {
    int64_t cr = 0, cl = 0, nb = 0;
    double sr = 0.0, sl = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (r[i] >= aR) { ++cr; sr += exp(-(r[i] - aR) / t); }
        else if (r[i] < aL) { ++cl; sl += exp((r[i] - aL) / t); }
        else ++nb;
    }
    *cnt_R = cr; *cnt_L = cl; *n_band = nb; *S_L = sl; *S_R = sr;
}

/* ---------------------------------------------------------------------------
 * SplitMix64 (Steele, Lea and Flood, OOPSLA 2014), used as a counter-based
 * generator: output number c (c = 0, 1, ...) of the stream seeded with `seed`
 * is mix(seed + (c + 1) * 0x9E3779B97F4A7C15).
 * ------------------------------------------------------------------------- */
uint64_t lso_splitmix64_at(uint64_t seed, uint64_t c) {
    uint64_t z = seed + (c + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* ---------------------------------------------------------------------------
 * Probabilistic bracketing, step 1 (localization sample): sample s = 0..m-1
 *   index  I_s = floor(z1 * n / 2^64),          z1 = splitmix(seed, c0 + 2s),
 *   u_s    = ((z2 >> 40) + 0.5) 2^-24 - 0.5,    z2 = splitmix(seed, c0 + 2s + 1),
 *   eps_s  = -t sgn(u_s) ln(1 - 2|u_s|)          (inverse CDF of Laplace(0,t)),
 *   y_s    = r[I_s] + eps_s.
 * Also returns the sampled indices (may be NULL).
 * ------------------------------------------------------------------------- */
void lso_sample(const double* r, int64_t n, double t, uint64_t seed, uint64_t c0, int64_t m,
                double* y, int64_t* idx_out) {
    for (int64_t s = 0; s < m; ++s) {
        uint64_t z1 = lso_splitmix64_at(seed, c0 + 2 * (uint64_t)s);
        uint64_t z2 = lso_splitmix64_at(seed, c0 + 2 * (uint64_t)s + 1);
        int64_t I = (int64_t)(((unsigned __int128)z1 * (unsigned __int128)(uint64_t)n) >> 64);
        double u = ((double)(z2 >> 40) + 0.5) * (1.0 / 16777216.0) - 0.5;
        double eps = (u < 0.0 ? 1.0 : -1.0) * t * log(1.0 - 2.0 * fabs(u));
        y[s] = r[I] + eps;
        if (idx_out) idx_out[s] = I;
    }
}

/* ---------------------------------------------------------------------------
 * Binomial order-statistic ranks.  Each noised sample exceeds b with
 * probability q = k/n, so C = #{y_s > b} ~ Binomial(m, q).  With the samples
 * in descending order y_(1) >= y_(2) >= ...:
 *   a_R = y_(l) misses (b >= a_R) iff C < l;      l = largest with P(C < l) <= alpha,
 *   a_L = y_(h) misses (b <  a_L) iff C >= h;     h = smallest with P(C >= h) <= alpha.
 * l = 0 means a_R = +inf and h = m + 1 means a_L = -inf.
 * ------------------------------------------------------------------------- */
static double binom_logpmf(int64_t m, double q, int64_t c) {
    return lgamma((double)m + 1.0) - lgamma((double)c + 1.0) - lgamma((double)(m - c) + 1.0) +
           (double)c * log(q) + (double)(m - c) * log1p(-q);
}

void lso_binom_ranks(int64_t m, double q, double alpha, int64_t* l_out, int64_t* h_out) {
    /* lower tail: P(C <= l-1) accumulated upward from 0 */
    double cdf = 0.0;
    int64_t l = 0;
    for (int64_t c = 0; c <= m; ++c) {
        cdf += exp(binom_logpmf(m, q, c)); /* cdf = P(C <= c) */
        if (cdf <= alpha) l = c + 1;       /* P(C < c+1) <= alpha */
        else break;
    }
    /* upper tail: P(C >= h) accumulated downward from m */
    double sf = 0.0;
    int64_t h = m + 1;
    for (int64_t c = m; c >= 0; --c) {
        sf += exp(binom_logpmf(m, q, c)); /* sf = P(C >= c) */
        if (sf <= alpha) h = c;
        else break;
    }
    *l_out = l;
    *h_out = h;
}

/* Bracket from a sample: descending order statistics at ranks l and h. */
void lso_bracket_from_sample(const double* y, int64_t m, int64_t l, int64_t h, double* aL,
                             double* aR) {
    double* s = (double*)malloc((size_t)m * sizeof(double));
    memcpy(s, y, (size_t)m * sizeof(double));
    qsort(s, (size_t)m, sizeof(double), cmp_double); /* ascending: y_(j) = s[m - j] */
    *aR = (l >= 1) ? s[m - l] : INFINITY;
    *aL = (h <= m) ? s[m - h] : -INFINITY;
    free(s);
}

/* ---------------------------------------------------------------------------
 * Zero-temperature limit (hard top-k).  Section 2.3 of the pages ties the
 * method to DFTopK, whose threshold is the midpoint of the k-th and (k+1)-th
 * largest scores, as the t -> 0 limit.  The limit of the balance equation,
 * written out here for any real k in (0, n):
 *   c = the ceil(k)-th largest score, a = #{r > c}, m = #{r = c}
 *   (so a < k <= a + m);
 *   - k < a + m: b = c, and the scores equal to c share the remaining budget,
 *     p = (k - a)/m each (sigma of the common limit of (c - b)/t);
 *   - k = a + m (k an integer at a gap of the sorted order): b is the
 *     midpoint of c and d = the largest score below c, and p is the 0/1 mask
 *     of the scores above b.
 * Either way sum p = k.  The sort is plain qsort on a copy.
 * ------------------------------------------------------------------------- */
int lso_hard_topk(const double* r, int64_t n, double k, double* b_out, double* p) {
    if (r == NULL || n < 1 || !(k > 0.0) || !(k < (double)n)) return LSO_EINVAL;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(r[i])) return LSO_ENONFINITE;
    double* s = (double*)malloc((size_t)n * sizeof(double));
    if (s == NULL) return LSO_EINVAL;
    memcpy(s, r, (size_t)n * sizeof(double));
    qsort(s, (size_t)n, sizeof(double), cmp_double);  /* ascending */
    const int64_t rank = (int64_t)ceil(k);              /* 1-based, from the top */
    const double c = s[n - rank];
    int64_t a = 0, m = 0;
    double d = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        if (s[i] > c) ++a;
        else if (s[i] == c) ++m;
        else if (s[i] > d) d = s[i];
    }
    free(s);
    double b, frac;
    if (k < (double)(a + m)) {
        b = c;
        frac = (k - (double)a) / (double)m;
    } else {
        b = 0.5 * (c + d);
        frac = 1.0;  /* every score equal to c lies above b */
    }
    *b_out = b;
    if (p != NULL)
        for (int64_t i = 0; i < n; ++i)
            p[i] = r[i] > c ? 1.0 : (r[i] == c ? frac : 0.0);
    return LSO_OK;
}
