/*
 * lapsum_oracle.c -- plain, slow, obviously-correct fp64 CPU oracle for the
 * Fast LapSum exact-budget soft top-k.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline
 * leg of the benchmark call it; the product path (the CUDA library) never
 * does, and the two share no code: no header, helper, table or constant.
 *
 * What it computes (web pages on the method):
 *   [FL-2.1]  "Fast LapSum: Exact Differentiable Top-k at Million Scale",
 *             technical summary, section 2.1: p_i = F((r_i - b)/t) with F the
 *             standard Laplace CDF, the threshold b fixed by sum_i p_i = k and
 *             solved exactly, and an analytic vector-Jacobian product.
 *   [FL-2.2]  same page, section 2.2: the probabilistic-bracketing pipeline
 *             (sample of kernel-noised scores, binomial order-statistic bracket
 *             [a_L, a_R), one streaming pass, band solve, certification).
 *   [FL-abs]  "Fast LapSum", abstract: kernel-noised samples, binomial order
 *             statistic, certification pass, full-sort fallback.
 *
 * The oracle does not follow the method's fast solver: b is found from the
 * plain definition, by bisection (or safeguarded Newton) on
 *   G(b) = sum_i F((r_i - b)/t) = k,
 * with every G evaluated over all n terms, in fp64, with Neumaier-compensated
 * sums over fixed 64Ki-element chunks combined in a fixed order (so results do
 * not depend on the OpenMP thread count).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 *        (no contraction, so the restated sampler below rounds exactly as written).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_CHUNK 65536

/* ------------------------------------------------------------------ sums -- */

typedef struct { double s, c; } nsum;            /* Neumaier running sum */

static void nsum_add(nsum *a, double x)
{
    double t = a->s + x;
    if (fabs(a->s) >= fabs(x)) a->c += (a->s - t) + x;
    else                       a->c += (x - t) + a->s;
    a->s = t;
}
static double nsum_val(const nsum *a) { return a->s + a->c; }

/* ------------------------------------------------------------ operator -- */

/* Standard Laplace CDF [FL-2.1]: F(x) = e^x/2 for x < 0, 1 - e^{-x}/2 for x >= 0. */
double orc_laplace_cdf(double x)
{
    return x < 0.0 ? 0.5 * exp(x) : 1.0 - 0.5 * exp(-x);
}

/* Inverse of F: F^{-1}(q) = ln(2q) for q < 1/2, -ln(2(1-q)) otherwise. */
double orc_laplace_icdf(double q)
{
    return q < 0.5 ? log(2.0 * q) : -log(2.0 * (1.0 - q));
}

/*
 * G(b) = sum_i F((r_i - b)/t), evaluated term by term from the definition
 * [FL-2.1] and accumulated as
 *     G = #{x_i >= 0} - 1/2 sum_{x_i>=0} e^{-x_i} + 1/2 sum_{x_i<0} e^{x_i},
 * x_i = (r_i - b)/t, so no 1 - e^{-x}/2 term is ever rounded on its own.
 * Also returns sum_i f(x_i), f(x) = e^{-|x|}/2 the Laplace density.
 * Returns -1 if a score is not finite.
 */
int orc_G(const float *r, int64_t n, double b, double t, double *G_out, double *sumf_out)
{
    int64_t nch = (n + ORC_CHUNK - 1) / ORC_CHUNK;
    int64_t *cnt = calloc((size_t)(nch ? nch : 1), sizeof(int64_t));
    double *shi = calloc((size_t)(nch ? nch : 1), sizeof(double));
    double *slo = calloc((size_t)(nch ? nch : 1), sizeof(double));
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t c = 0; c < nch; ++c) {
        int64_t lo = c * ORC_CHUNK, hi = lo + ORC_CHUNK < n ? lo + ORC_CHUNK : n;
        nsum a = {0, 0}, z = {0, 0};
        int64_t m = 0;
        for (int64_t i = lo; i < hi; ++i) {
            double ri = (double)r[i];
            if (!isfinite(ri)) { bad = 1; continue; }
            double x = (ri - b) / t;
            if (x >= 0.0) { ++m; nsum_add(&a, exp(-x)); }
            else          { nsum_add(&z, exp(x)); }
        }
        cnt[c] = m; shi[c] = nsum_val(&a); slo[c] = nsum_val(&z);
    }
    int64_t m = 0;
    nsum A = {0, 0}, Z = {0, 0};
    for (int64_t c = 0; c < nch; ++c) { m += cnt[c]; nsum_add(&A, shi[c]); nsum_add(&Z, slo[c]); }
    free(cnt); free(shi); free(slo);
    double sa = nsum_val(&A), sz = nsum_val(&Z);
    if (G_out) *G_out = (double)m + (0.5 * sz - 0.5 * sa);
    if (sumf_out) *sumf_out = 0.5 * (sa + sz);
    return bad ? -1 : 0;
}

static void minmax(const float *r, int64_t n, double *mn, double *mx)
{
    double a = INFINITY, z = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        double v = (double)r[i];
        if (v < a) a = v;
        if (v > z) z = v;
    }
    *mn = a; *mx = z;
}

/*
 * The unique b with G(b) = k [FL-2.1] (G is continuous and strictly decreasing
 * from n to 0, so 0 < k < n has exactly one root).
 *
 * Bracket: with q = k/n, n F((min r - b)/t) <= G(b) <= n F((max r - b)/t), so
 *   b in [min r - t F^{-1}(q), max r - t F^{-1}(q)].
 * method 0: plain bisection until the bracket holds no representable midpoint
 *           (or 400 halvings).
 * method 1: Newton on G(b) - k with G'(b) = -sum f / t, each step kept inside
 *           the current bracket (bisection when it leaves it or stalls).
 * Returns the bracket end with the smaller |G - k|, and the number of G
 * evaluations.  Error codes: -1 bad arguments, -2 non-finite scores.
 */
int orc_solve(const float *r, int64_t n, double k, double t, int method,
              double *b_out, int *evals_out)
{
    if (n < 1 || !(k > 0.0) || !(k < (double)n) || !(t > 0.0) || !isfinite(t)) return -1;
    double mn, mx;
    minmax(r, n, &mn, &mx);
    if (!isfinite(mn) || !isfinite(mx)) return -2;
    double q = k / (double)n;
    double fi = orc_laplace_icdf(q);
    double lo = mn - t * fi, hi = mx - t * fi;
    double Glo, Ghi, sf;
    int ev = 0;
    orc_G(r, n, lo, t, &Glo, &sf); ++ev;
    orc_G(r, n, hi, t, &Ghi, &sf); ++ev;
    /* rounding of the bracket ends can put the root a hair outside: widen */
    for (int w = 0; w < 64 && Glo < k; ++w) { lo -= t * (1.0 + fabs(lo) * 1e-12); orc_G(r, n, lo, t, &Glo, &sf); ++ev; }
    for (int w = 0; w < 64 && Ghi > k; ++w) { hi += t * (1.0 + fabs(hi) * 1e-12); orc_G(r, n, hi, t, &Ghi, &sf); ++ev; }
    if (method == 0) {
        for (int it = 0; it < 400; ++it) {
            double mid = lo + 0.5 * (hi - lo);
            if (!(mid > lo && mid < hi)) break;
            double Gm;
            orc_G(r, n, mid, t, &Gm, &sf); ++ev;
            if (Gm > k) { lo = mid; Glo = Gm; }      /* G decreasing: root above mid */
            else        { hi = mid; Ghi = Gm; }
        }
    } else {
        double b = lo + 0.5 * (hi - lo);
        for (int it = 0; it < 200; ++it) {
            double Gb, sfb;
            orc_G(r, n, b, t, &Gb, &sfb); ++ev;
            if (Gb > k) { lo = b; Glo = Gb; } else { hi = b; Ghi = Gb; }
            if (Gb == k) { lo = hi = b; Glo = Ghi = Gb; break; }
            double nb = (sfb > 0.0) ? b + t * (Gb - k) / sfb : NAN;
            if (!(nb > lo && nb < hi)) nb = lo + 0.5 * (hi - lo);
            if (!(nb > lo && nb < hi)) break;               /* bracket is two adjacent doubles */
            if (fabs(nb - b) <= 4.0 * DBL_EPSILON * (fabs(b) + t)) {
                /* converged: tighten with one-sided probes instead of looping */
                double Gn; orc_G(r, n, nb, t, &Gn, &sfb); ++ev;
                if (Gn > k) { lo = nb; Glo = Gn; } else { hi = nb; Ghi = Gn; }
                break;
            }
            b = nb;
        }
    }
    *b_out = (fabs(Glo - k) <= fabs(Ghi - k)) ? lo : hi;
    if (evals_out) *evals_out = ev;
    return 0;
}

/* p_i = F((r_i - b)/t) [FL-2.1], fp64. */
void orc_p(const float *r, int64_t n, double b, double t, double *p)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) p[i] = orc_laplace_cdf(((double)r[i] - b) / t);
}

/*
 * Analytic VJP [FL-2.1].  Differentiating sum_i F((r_i - b)/t) = k gives
 * db/dr_j = f_j / sum_i f_i, and dp_i/dr_j = (f_i/t)(delta_ij - f_j/sum f), so
 *   grad_j = sum_i g_i dp_i/dr_j = (f_j/t) (g_j - <g,f>/sum f),
 * f_i = f((r_i - b)/t) = e^{-|x_i|}/2.  The ratio <g,f>/sum f is formed from
 * terms shifted by the smallest |x_i| (the shift cancels), so it stays defined
 * when every f_i underflows.  Returns <g,f> and sum f unshifted.
 */
void orc_vjp(const float *r, const float *g, int64_t n, double b, double t,
             double *grad, double *gf_out, double *sf_out)
{
    double xmin = INFINITY;
#pragma omp parallel for schedule(static) reduction(min:xmin)
    for (int64_t i = 0; i < n; ++i) {
        double ax = fabs(((double)r[i] - b) / t);
        if (ax < xmin) xmin = ax;
    }
    int64_t nch = (n + ORC_CHUNK - 1) / ORC_CHUNK;
    double *part = calloc((size_t)(4 * (nch ? nch : 1)), sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < nch; ++c) {
        int64_t lo = c * ORC_CHUNK, hi = lo + ORC_CHUNK < n ? lo + ORC_CHUNK : n;
        nsum S = {0, 0}, GF = {0, 0}, S0 = {0, 0}, GF0 = {0, 0};
        for (int64_t i = lo; i < hi; ++i) {
            double ax = fabs(((double)r[i] - b) / t);
            double fs = 0.5 * exp(-(ax - xmin));       /* shifted density */
            double f = 0.5 * exp(-ax);
            nsum_add(&S, fs); nsum_add(&GF, (double)g[i] * fs);
            nsum_add(&S0, f); nsum_add(&GF0, (double)g[i] * f);
        }
        part[4 * c + 0] = nsum_val(&S);  part[4 * c + 1] = nsum_val(&GF);
        part[4 * c + 2] = nsum_val(&S0); part[4 * c + 3] = nsum_val(&GF0);
    }
    nsum S = {0, 0}, GF = {0, 0}, S0 = {0, 0}, GF0 = {0, 0};
    for (int64_t c = 0; c < nch; ++c) {
        nsum_add(&S, part[4 * c + 0]); nsum_add(&GF, part[4 * c + 1]);
        nsum_add(&S0, part[4 * c + 2]); nsum_add(&GF0, part[4 * c + 3]);
    }
    free(part);
    double lam = nsum_val(&GF) / nsum_val(&S);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double f = 0.5 * exp(-fabs(((double)r[i] - b) / t));
        grad[i] = (f / t) * ((double)g[i] - lam);
    }
    if (gf_out) *gf_out = nsum_val(&GF0);
    if (sf_out) *sf_out = nsum_val(&S0);
}

/*
 * Tail sums of the streaming pass [FL-2.2 step 2], from their definition:
 *   S_L = sum_{r < a_L} e^{(r - a_L)/t},   S_R = sum_{r >= a_R} e^{-(r - a_R)/t}
 * (every term at most 1; an infinite end has an empty tail).  Also returns the
 * part of each sum made of terms with z = |r - a|/t > 16, the terms a fast
 * solver may form in a lower precision, so a test can bound their error.
 * Neumaier sums over fixed chunks, combined in chunk order.
 */
void orc_tail_sums(const float *r, int64_t n, float aL, float aR, double t,
                   double *SL, double *SR, double *SL_far, double *SR_far)
{
    int64_t nch = (n + ORC_CHUNK - 1) / ORC_CHUNK;
    double *part = calloc((size_t)(4 * (nch ? nch : 1)), sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < nch; ++c) {
        int64_t lo = c * ORC_CHUNK, hi = lo + ORC_CHUNK < n ? lo + ORC_CHUNK : n;
        nsum L = {0, 0}, R = {0, 0}, Lf = {0, 0}, Rf = {0, 0};
        for (int64_t i = lo; i < hi; ++i) {
            float v = r[i];
            if (!isinf(aL) && v < aL) {
                double z = ((double)aL - (double)v) / t;
                double e = exp(-z);
                nsum_add(&L, e);
                if (z > 16.0) nsum_add(&Lf, e);
            } else if (!isinf(aR) && v >= aR) {
                double z = ((double)v - (double)aR) / t;
                double e = exp(-z);
                nsum_add(&R, e);
                if (z > 16.0) nsum_add(&Rf, e);
            }
        }
        part[4 * c + 0] = nsum_val(&L);  part[4 * c + 1] = nsum_val(&R);
        part[4 * c + 2] = nsum_val(&Lf); part[4 * c + 3] = nsum_val(&Rf);
    }
    nsum L = {0, 0}, R = {0, 0}, Lf = {0, 0}, Rf = {0, 0};
    for (int64_t c = 0; c < nch; ++c) {
        nsum_add(&L, part[4 * c + 0]);  nsum_add(&R, part[4 * c + 1]);
        nsum_add(&Lf, part[4 * c + 2]); nsum_add(&Rf, part[4 * c + 3]);
    }
    free(part);
    *SL = nsum_val(&L); *SR = nsum_val(&R); *SL_far = nsum_val(&Lf); *SR_far = nsum_val(&Rf);
}

static int cmp_desc(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/* Scores as fp64, sorted descending (order statistics for the limit checks). */
void orc_sort_desc(const float *r, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (double)r[i];
    qsort(out, (size_t)n, sizeof(double), cmp_desc);
}

/* ===================================================================== *
 *  Restatement of the probabilistic bracket [FL-2.2 step 1, FL-abs], for
 *  exact (integer) comparison with the GPU path.  Random numbers come from
 *  Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *  easy as 1, 2, 3", SC'11), written here from its published definition.
 * ===================================================================== */

static void mulhilo64(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo)
{
    unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

/* Philox4x64 with 10 rounds: each round multiplies words 0 and 2 by the two
 * round multipliers, swaps the halves across the pair and xors in the key;
 * the key is bumped by the two Weyl constants between rounds. */
void orc_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4])
{
    const uint64_t M0 = 0xD2E7470EE14C6C93ULL, M1 = 0xCA5A826395121157ULL;
    const uint64_t W0 = 0x9E3779B97F4A7C15ULL, W1 = 0xBB67AE8584CAA73BULL;
    uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t h0, l0, h1, l1;
        mulhilo64(M0, x0, &h0, &l0);
        mulhilo64(M1, x2, &h1, &l1);
        uint64_t y0 = h1 ^ x1 ^ k0, y1 = l1, y2 = h0 ^ x3 ^ k1, y3 = l0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += W0; k1 += W1;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/*
 * Natural log from the identity ln m = 2 atanh((m-1)/(m+1)) after the
 * reduction x = m 2^e, m in [sqrt(1/2), sqrt(2)): atanh(s)/s = sum_j s^{2j}/(2j+1)
 * (|s| <= 0.1716, 11 terms), then ln x = e ln2 + ln m.  Only correctly-rounded
 * IEEE operations (+, *, /, fma) in a fixed order, so any platform that rounds
 * those to nearest gets the same bits.  For x > 0, finite, normal.
 */
double orc_ln(double x)
{
    uint64_t bits;
    memcpy(&bits, &x, sizeof bits);
    int64_t e = (int64_t)((bits >> 52) & 0x7FF) - 1022;           /* x = m 2^e, m in [1/2,1) */
    uint64_t mb = (bits & 0x800FFFFFFFFFFFFFULL) | (0x3FEULL << 52);
    double m;
    memcpy(&m, &mb, sizeof m);
    if (m < 0x1.6a09e667f3bcdp-1) { m = m + m; e -= 1; }           /* m in [sqrt(1/2), sqrt(2)) */
    double s = (m - 1.0) / (m + 1.0);
    double z = s * s;
    double p = 1.0 / 21.0;
    p = fma(p, z, 1.0 / 19.0);
    p = fma(p, z, 1.0 / 17.0);
    p = fma(p, z, 1.0 / 15.0);
    p = fma(p, z, 1.0 / 13.0);
    p = fma(p, z, 1.0 / 11.0);
    p = fma(p, z, 1.0 / 9.0);
    p = fma(p, z, 1.0 / 7.0);
    p = fma(p, z, 1.0 / 5.0);
    p = fma(p, z, 1.0 / 3.0);
    p = fma(p, z, 1.0);
    double lnm = (s + s) * p;
    const double LN2 = 0x1.62e42fefa39efp-1;                       /* ln 2 rounded to 53 bits */
    return fma((double)e, LN2, lnm);
}

/* Philox key word 1 of the bracketing sample (an arbitrary fixed stream tag). */
#define ORC_SAMPLE_TAG 0x4C41505355534D50ULL

/*
 * Kernel-noised sample [FL-abs, FL-2.2 step 1]: y_j = r_{I_j} + t L_j,
 * j = 0..s-1, with I_j uniform on [0, n) and L_j ~ Laplace(0,1), the same
 * noise kernel as the operator's (p_i = P(r_i + eps > b), eps ~ Laplace(0,t)),
 * so P(y_j > b) = k/n exactly.
 *   Philox4x64-10, key (seed, TAG), counter (j, row, 0, 0) -> words u0..u3;
 *   I = floor(u0 * n / 2^64);
 *   U = ((u1 >> 11) + 1) 2^-53 in (0, 1]; E = -ln U ~ Exp(1);
 *   L = E if bit 0 of u1 is set, else -E   (a random sign: Laplace(0,1));
 *   y = (double)r_I + t*L  (product rounded, then sum rounded).
 */
void orc_sample(const float *r, int64_t n, double t, uint64_t seed, int64_t row,
                int64_t s, double *y, int64_t *idx_out)
{
    const uint64_t key[2] = {seed, ORC_SAMPLE_TAG};
    for (int64_t j = 0; j < s; ++j) {
        uint64_t ctr[4] = {(uint64_t)j, (uint64_t)row, 0, 0}, u[4];
        orc_philox4x64_10(ctr, key, u);
        uint64_t hi, lo;
        mulhilo64(u[0], (uint64_t)n, &hi, &lo);
        int64_t I = (int64_t)hi;
        double U = (double)((u[1] >> 11) + 1) * 0x1p-53;
        double E = -orc_ln(U);
        double L = (u[1] & 1) ? E : -E;
        double tl = t * L;
        y[j] = (double)r[I] + tl;
        if (idx_out) idx_out[j] = I;
    }
}

/* Binomial(s, pi) log-pmf from the definition, via lgamma. */
static double binom_logpmf(int64_t s, double pi, int64_t j)
{
    return lgamma((double)s + 1.0) - lgamma((double)j + 1.0) - lgamma((double)(s - j) + 1.0)
         + (double)j * log(pi) + (double)(s - j) * log1p(-pi);
}

/*
 * Ranks of the binomial order-statistic bracket [FL-2.2 step 1, FL-abs].
 * With X = #{j : y_j > b} ~ Binomial(s, pi = k/n) and y_(1) >= ... >= y_(s):
 *   X >= jR      implies y_(jR) > b   (b below a_R = y_(jR)),
 *   X <= jL - 1  implies y_(jL) <= b  (b at or above a_L = y_(jL)),
 * so b in [a_L, a_R) except with probability P(X < jR) + P(X >= jL) <= delta.
 *   jR = the largest j with P(X < j) <= delta/2   (0: a_R = +inf),
 *   jL = the smallest j with P(X >= j) <= delta/2 (s+1: a_L = -inf).
 * Tails are summed term by term (Neumaier) from the log-pmf.
 */
int orc_binom_ranks(int64_t s, double pi, double delta, int64_t *jR, int64_t *jL)
{
    if (s < 1 || !(pi > 0.0) || !(pi < 1.0) || !(delta > 0.0) || !(delta < 1.0)) return -1;
    double half = 0.5 * delta;
    /* lower tail: P(X < j) = sum_{i<j} pmf(i), increasing in j */
    nsum lt = {0, 0};
    int64_t r = 0;
    for (int64_t j = 1; j <= s; ++j) {
        nsum_add(&lt, exp(binom_logpmf(s, pi, j - 1)));     /* now lt = P(X < j) */
        if (nsum_val(&lt) <= half) r = j; else break;
    }
    /* upper tail: P(X >= j) = sum_{i>=j} pmf(i), decreasing in j */
    nsum ut = {0, 0};
    int64_t l = s + 1;
    for (int64_t j = s; j >= 0; --j) {
        nsum_add(&ut, exp(binom_logpmf(s, pi, j)));         /* now ut = P(X >= j) */
        if (nsum_val(&ut) <= half) l = j; else break;
    }
    *jR = r; *jL = l;
    return 0;
}

/* float rounding of a double toward -inf, from the round-to-nearest cast */
static float f32_down(double y)
{
    float f = (float)y;
    if ((double)f > y) f = nextafterf(f, -INFINITY);
    return f;
}

/*
 * Bracket ends [FL-2.2 step 1], rounded outward to fp32 so the bracket can
 * only widen:  a_L = rd(y_(jL)),  a_R = nextup(rd(y_(jR)))  (> y_(jR) always);
 * a_R = +inf when jR = 0, a_L = -inf when jL = s + 1.
 * Order statistics by a full sort of the fp64 sample.
 */
int orc_bracket(const float *r, int64_t n, double k, double t, uint64_t seed, int64_t row,
                int64_t s, double delta, float *aL, float *aR, int64_t *jR_out, int64_t *jL_out)
{
    int64_t jR, jL;
    if (orc_binom_ranks(s, k / (double)n, delta, &jR, &jL) != 0) return -1;
    double *y = malloc((size_t)s * sizeof(double));
    orc_sample(r, n, t, seed, row, s, y, NULL);
    qsort(y, (size_t)s, sizeof(double), cmp_desc);
    *aR = jR >= 1 ? nextafterf(f32_down(y[jR - 1]), INFINITY) : INFINITY;
    *aL = jL <= s ? f32_down(y[jL - 1]) : -INFINITY;
    free(y);
    *jR_out = jR; *jL_out = jL;
    return 0;
}

/*
 * Bracket ends at given ranks of the same sample (outward fp32 rounding as in
 * orc_bracket): a_R = nextup(rd(y_(jR))) (+inf for jR = 0), a_L = rd(y_(jL))
 * (-inf for jL = s + 1).
 */
int orc_bracket_at_ranks(const float *r, int64_t n, double t, uint64_t seed, int64_t row, int64_t s,
                         int64_t jR, int64_t jL, float *aL, float *aR)
{
    if (s < 1 || jR < 0 || jR > s || jL < 1 || jL > s + 1) return -1;
    double *y = malloc((size_t)s * sizeof(double));
    orc_sample(r, n, t, seed, row, s, y, NULL);
    qsort(y, (size_t)s, sizeof(double), cmp_desc);
    *aR = jR >= 1 ? nextafterf(f32_down(y[jR - 1]), INFINITY) : INFINITY;
    *aL = jL <= s ? f32_down(y[jL - 1]) : -INFINITY;
    free(y);
    return 0;
}

/*
 * Ranks of the widening round ("iteratively widened" bracket, technical
 * summary section 2.2 step 4; the rule is this implementation's reading):
 * start from the ranks of confidence delta^2 and move each at least one
 * first-round spread (jL - jR, at least 1) beyond the first round's rank,
 * clipped to [0, s + 1].  A miss above a_R uses jR2, a miss below a_L uses jL2.
 */
int orc_widen_ranks(int64_t s, double pi, double delta, int64_t *jR2, int64_t *jL2)
{
    int64_t jR, jL, r2, l2;
    if (orc_binom_ranks(s, pi, delta, &jR, &jL) != 0) return -1;
    double d2 = delta * delta;
    if (d2 < 1e-300) d2 = 1e-300;
    if (orc_binom_ranks(s, pi, d2, &r2, &l2) != 0) return -1;
    int64_t spread = jL - jR;
    if (spread < 1) spread = 1;
    if (r2 > jR - spread) r2 = jR - spread;
    if (r2 < 0) r2 = 0;
    if (l2 < jL + spread) l2 = jL + spread;
    if (l2 > s + 1) l2 = s + 1;
    *jR2 = r2; *jL2 = l2;
    return 0;
}

/* Band membership [FL-2.2 step 2]: above r >= a_R; band a_L <= r < a_R; below r < a_L. */
void orc_counts(const float *r, int64_t n, float aL, float aR, int64_t *cL, int64_t *cB, int64_t *cR)
{
    int64_t L = 0, B = 0, R = 0;
#pragma omp parallel for schedule(static) reduction(+:L, B, R)
    for (int64_t i = 0; i < n; ++i) {
        float v = r[i];
        if (v >= aR) ++R;
        else if (v < aL) ++L;
        else if (v >= aL && v < aR) ++B;
    }
    *cL = L; *cB = B; *cR = R;
}

/*
 * Certification [FL-abs, FL-2.2 step 4]: the bracket holds iff
 * G(a_L) >= k > G(a_R) (G decreasing), both evaluated from the definition;
 * the verdict also requires the band to fit its buffer and the three
 * membership counts to cover every score (a non-finite score fails it).
 * Infinite ends: G(+inf) = 0, G(-inf) = n.
 */
int orc_certify(const float *r, int64_t n, double k, double t, float aL, float aR,
                int64_t band_cap, double *GaL, double *GaR,
                int64_t *cL, int64_t *cB, int64_t *cR)
{
    double gl, gr, sf;
    if (isinf(aL)) gl = (double)n; else orc_G(r, n, (double)aL, t, &gl, &sf);
    if (isinf(aR)) gr = 0.0;       else orc_G(r, n, (double)aR, t, &gr, &sf);
    orc_counts(r, n, aL, aR, cL, cB, cR);
    *GaL = gl; *GaR = gr;
    return (*cB <= band_cap) && (gl >= k) && (gr < k) && (*cL + *cB + *cR == n);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
