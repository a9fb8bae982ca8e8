/*
 * entmaxkv_oracle.c -- plain, slow, fp64 CPU oracle of the EntmaxKV decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link or call
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library: it reads the same raw input buffers (bf16 bit patterns, int32 page
 * tables) and writes its own plain arrays.
 *
 * Source of every definition: "EntmaxKV - Support-aware decoding for entmax
 * attention", technical summary at gist.science/es/paper/2605.21649 (and its
 * ja/ko/ar translations):
 *   section 2 "Methodology": alpha-entmax gives exact zeros; the selected set
 *     containing the support makes the sparse output equal the full one.
 *   section 2.A "Query-aware page scoring": per-page coordinate-wise k_min /
 *     k_max give an upper bound on the best score in the page; per-page key
 *     mean and variance give a Gaussian model of the page's token scores.
 *   section 2.B "Candidate selection": top-k pages by the bound, or an
 *     approximate normalisation equation solved for tau_hat and pages whose
 *     estimated max score exceeds tau_hat minus a margin Delta.
 *   section 2.C "Sparse entmax attention": entmax weights over the loaded set.
 *   section 4 "Efficiency": full-cache entmax and full-cache softmax decoding
 *     as the comparison points.
 * Where the pages are silent the readings are:
 *   p_i = [(alpha-1) s_i - tau]_+^{1/(alpha-1)},  s_i = q.k_i / sqrt(d);
 *   diagonal, population (divide by n) per-coordinate key variance;
 *   page score model N(mu_p, sigma_p^2), mu_p = q.mean/sqrt(d),
 *     sigma_p^2 = sum_j q_j^2 var_j / d;
 *   the approximate normalisation equation is sum_p n_p E[(X_p - tau)_+^r] = 1
 *     with X_p ~ N((alpha-1) mu_p, (alpha-1)^2 sigma_p^2), r = 1/(alpha-1);
 *   the "estimated max score" of a page is its bounding-box bound, compared on
 *     the z = (alpha-1) s scale: keep p if (alpha-1) u_p > tau_hat - Delta;
 *   a variant estimates it from the page's Gaussian model, capped by the
 *     bound: min(u_p, mu_p + z(n_p) sigma_p), z(n) = sqrt(2 ln n) (the usual
 *     estimate of the largest of n standard normal draws; z(1) = 0);
 *   top-k ties go to the lower page index; selections are listed ascending.
 *
 * Arithmetic rules (so that results are defined to the bit where stated):
 *   - every sum over coordinates or tokens runs in index order in fp64;
 *   - bf16 x bf16, bf16 x fp32 and bf16^2 x fp32 products are exact in fp64;
 *   - one final rounding to fp32 (round to nearest even).
 * Build with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

static double bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int n_pages_of(int seq_len, int P) { return (seq_len + P - 1) / P; }

static int tokens_in_page(int seq_len, int P, int p)
{
    int n = seq_len - p * P;
    return n > P ? P : (n < 0 ? 0 : n);
}

/* --------------------------------------------------------- page metadata */
/*
 * Section 2.A: per page and kv head, over the n valid tokens of the page and
 * for each coordinate j:
 *   kmin_j = min_t k_tj,  kmax_j = max_t k_tj   (the bf16 value itself; the
 *            first token holding the extreme wins on exact ties),
 *   mean_j = fp32( S1 / n ),
 *   var_j  = fp32( max(0, S2/n - (S1/n)^2) ),
 * with S1 = sum_t k_tj and S2 = sum_t k_tj^2 accumulated in fp64 in token order.
 * Output arrays are indexed by record = block * Hkv + kv_head, each of length d.
 */
void orc_build_meta(int B, int Hkv, int d, int P, int max_pages,
                    const uint16_t *K, const int32_t *page_table,
                    const int32_t *seq_lens,
                    uint16_t *kmin, uint16_t *kmax, float *mean, float *var)
{
    for (int b = 0; b < B; ++b) {
        int np = n_pages_of(seq_lens[b], P);
        for (int p = 0; p < np; ++p) {
            int blk = page_table[(size_t)b * max_pages + p];
            int n = tokens_in_page(seq_lens[b], P, p);
#pragma omp parallel for schedule(static)
            for (int kvh = 0; kvh < Hkv; ++kvh) {
                size_t rec = (size_t)blk * Hkv + kvh;
                const uint16_t *tile = K + rec * (size_t)P * d;
                for (int j = 0; j < d; ++j) {
                    uint16_t bmin = tile[j], bmax = tile[j];
                    double vmin = bf16_to_double(bmin), vmax = vmin;
                    double s1 = 0.0, s2 = 0.0;
                    for (int t = 0; t < n; ++t) {
                        uint16_t h = tile[(size_t)t * d + j];
                        double x = bf16_to_double(h);
                        if (x < vmin) { vmin = x; bmin = h; }
                        if (x > vmax) { vmax = x; bmax = h; }
                        s1 += x;
                        s2 += x * x;
                    }
                    double m = s1 / (double)n;
                    double v = s2 / (double)n - m * m;
                    if (v < 0.0) v = 0.0;
                    kmin[rec * d + j] = bmin;
                    kmax[rec * d + j] = bmax;
                    mean[rec * d + j] = (float)m;
                    var[rec * d + j] = (float)v;
                }
            }
        }
    }
}

/* ----------------------------------------------------------- page scores */
/*
 * Section 2.A, per (batch b, query head h, page p < ceil(seq_len/P)):
 *   bbox  u_p   = fp32( (sum_j max(q_j kmin_j, q_j kmax_j)) * (1/sqrt(d)) )
 *   mu_p        = fp32( (sum_j q_j mean_j) * (1/sqrt(d)) )
 *   sigma_p     = fp32( sqrt( (sum_j q_j^2 var_j) / d ) )
 * Outputs are [B][Hq][max_pages]; entries past the last page are not written.
 */
void orc_score_pages(int B, int Hq, int Hkv, int d, int P, int max_pages,
                     const uint16_t *q, const uint16_t *kmin,
                     const uint16_t *kmax, const float *mean, const float *var,
                     const int32_t *page_table, const int32_t *seq_lens,
                     float *bbox, float *mu, float *sigma)
{
    int G = Hq / Hkv;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int kvh = h / G;
            const uint16_t *qh = q + ((size_t)b * Hq + h) * d;
            int np = n_pages_of(seq_lens[b], P);
            for (int p = 0; p < np; ++p) {
                int blk = page_table[(size_t)b * max_pages + p];
                size_t rec = (size_t)blk * Hkv + kvh;
                double ab = 0.0, am = 0.0, av = 0.0;
                for (int j = 0; j < d; ++j) {
                    double qj = bf16_to_double(qh[j]);
                    double lo = qj * bf16_to_double(kmin[rec * d + j]);
                    double hi = qj * bf16_to_double(kmax[rec * d + j]);
                    ab += (lo > hi ? lo : hi);
                    am += qj * (double)mean[rec * d + j];
                    av += (qj * qj) * (double)var[rec * d + j];
                }
                size_t o = ((size_t)b * Hq + h) * max_pages + p;
                bbox[o] = (float)(ab * inv_sqrt_d);
                if (mu) mu[o] = (float)(am * inv_sqrt_d);
                if (sigma) sigma[o] = (float)sqrt(av / (double)d);
            }
        }
    }
}

/* ------------------------------------------- Gaussian partial moments J_r */
/*
 * For a standard normal Z and integer r >= 0:
 *   J_r(c) = E[(Z - c)_+^r] = sum_{i=0..r} C(r,i) (-c)^{r-i} M_i(c),
 *   M_i(c) = E[Z^i 1{Z > c}]:  M_0 = erfc(c/sqrt 2)/2,  M_1 = phi(c),
 *            M_i = c^{i-1} phi(c) + (i-1) M_{i-2}.
 * (integration by parts of z^{i-1} * z phi(z) over (c, inf)).
 */
double orc_gauss_J(int r, double c)
{
    double M[16];
    double phi = exp(-0.5 * c * c) / sqrt(2.0 * M_PI);
    M[0] = 0.5 * erfc(c / sqrt(2.0));
    if (r >= 1) M[1] = phi;
    for (int i = 2; i <= r; ++i) M[i] = pow(c, (double)(i - 1)) * phi + (double)(i - 1) * M[i - 2];
    double s = 0.0, binom = 1.0;
    for (int i = 0; i <= r; ++i) {
        /* binom = C(r, i) */
        s += binom * pow(-c, (double)(r - i)) * M[i];
        binom = binom * (double)(r - i) / (double)(i + 1);
    }
    return s < 0.0 ? 0.0 : s;
}

/* Expected mass n * E[(X - tau)_+^r], X ~ N(m, s^2); a point mass when s == 0. */
static double page_mass(int r, double m, double s, double n, double tau)
{
    if (s > 0.0) return n * pow(s, (double)r) * orc_gauss_J(r, (tau - m) / s);
    double x = m - tau;
    return x > 0.0 ? n * pow(x, (double)r) : 0.0;
}

/*
 * Section 2.B, Gaussian-aware selection, the approximate normalisation
 * equation:  F(tau) = sum_p n_p E[(X_p - tau)_+^r] = 1,
 * X_p ~ N((alpha-1) mu_p, (alpha-1)^2 sigma_p^2), r = 1/(alpha-1) integer.
 * Solved by bisection in fp64.  Lower end: max_p (alpha-1) mu_p - 1, where
 * F >= 1 by Jensen; upper end found by doubling steps until F < 1.
 * Returns NAN when r is not an integer in 1..8 or there are no pages.
 */
double orc_tau_hat(int n_pages, const float *mu, const float *sigma,
                   const int32_t *n_tok, double alpha)
{
    double rr = 1.0 / (alpha - 1.0);
    int r = (int)floor(rr + 0.5);
    if (fabs(rr - r) > 1e-9 || r < 1 || r > 8 || n_pages <= 0) return NAN;
    double a1 = alpha - 1.0;
    double mmax = -INFINITY;
    for (int p = 0; p < n_pages; ++p) {
        double m = a1 * (double)mu[p];
        if (m > mmax) mmax = m;
    }
    double lo = mmax - 1.0, hi = mmax, step = 1.0;
    for (int it = 0; it < 200; ++it) {
        double F = 0.0;
        for (int p = 0; p < n_pages; ++p)
            F += page_mass(r, a1 * (double)mu[p], a1 * (double)sigma[p], (double)n_tok[p], hi);
        if (F < 1.0) break;
        lo = hi;
        hi += step;
        step *= 2.0;
    }
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        double F = 0.0;
        for (int p = 0; p < n_pages; ++p)
            F += page_mass(r, a1 * (double)mu[p], a1 * (double)sigma[p], (double)n_tok[p], mid);
        if (F >= 1.0) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* ------------------------------------------------------------- selection */

typedef struct { float score; int idx; } scored_t;

static int cmp_desc_then_index(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_int(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/*
 * Section 2.B, policy 1: the k pages with the highest bounding-box bound
 * (k clipped to the page count, ties to the lower page index), listed in
 * ascending page order.  Returns the count.
 */
int orc_select_topk(int n_pages, const float *bbox, int k, int32_t *sel)
{
    if (k > n_pages) k = n_pages;
    if (k <= 0) return 0;
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)n_pages);
    for (int p = 0; p < n_pages; ++p) { v[p].score = bbox[p]; v[p].idx = p; }
    qsort(v, (size_t)n_pages, sizeof(scored_t), cmp_desc_then_index);
    for (int i = 0; i < k; ++i) sel[i] = v[i].idx;
    free(v);
    qsort(sel, (size_t)k, sizeof(int32_t), cmp_int);
    return k;
}

/*
 * Section 2.B, policy 2: every page whose bound, on the z scale, exceeds the
 * margin-adjusted threshold: (alpha-1) u_p > tau_hat - Delta.  Ascending order.
 */
int orc_select_gauss(int n_pages, const float *bbox, double alpha,
                     double tau_hat, double delta, int32_t *sel)
{
    int c = 0;
    double thr = tau_hat - delta;
    for (int p = 0; p < n_pages; ++p)
        if ((alpha - 1.0) * (double)bbox[p] > thr) sel[c++] = p;
    return c;
}

/*
 * Section 2.B, Gaussian rule with the estimated maximum taken from the page's
 * Gaussian model and capped by the bound (the bound is never below the true
 * maximum, the model's estimate may be):
 *   keep p if (alpha-1) min(u_p, mu_p + z(n_p) sigma_p) > tau_hat - Delta,
 *   z(n) = sqrt(2 ln n) for n >= 2, z(1) = 0.
 */
double orc_zmax_of(int n)
{
    return n >= 2 ? sqrt(2.0 * log((double)n)) : 0.0;
}

int orc_select_gauss_est(int n_pages, const float *bbox, const float *mu,
                         const float *sigma, const int32_t *n_tok, double alpha,
                         double tau_hat, double delta, int32_t *sel)
{
    int c = 0;
    double thr = tau_hat - delta;
    for (int p = 0; p < n_pages; ++p) {
        double est = (double)mu[p] + orc_zmax_of(n_tok[p]) * (double)sigma[p];
        if ((double)bbox[p] < est) est = (double)bbox[p];
        if ((alpha - 1.0) * est > thr) sel[c++] = p;
    }
    return c;
}

/* ------------------------------------------------------ entmax threshold */

static int cmp_double_desc(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/*
 * Sparsemax (alpha = 2) closed form: with z sorted descending,
 * k* = max{k : 1 + k z_(k) > sum_{i<=k} z_(i)},  tau = (sum_{i<=k*} z_(i) - 1)/k*.
 */
double orc_sparsemax_tau(const double *z, int n)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    memcpy(s, z, sizeof(double) * (size_t)n);
    qsort(s, (size_t)n, sizeof(double), cmp_double_desc);
    double cum = 0.0, cum_star = 0.0;
    int kstar = 1;
    for (int k = 1; k <= n; ++k) {
        cum += s[k - 1];
        if (1.0 + k * s[k - 1] > cum) { kstar = k; cum_star = cum; }
    }
    free(s);
    return (cum_star - 1.0) / kstar;
}

/*
 * Exact 1.5-entmax by sorting: with z sorted descending and the support taken
 * as the top k, sum_{i<=k} (z_i - tau)^2 = 1 gives
 *   tau_k = M_k - sqrt((1 - SS_k)/k),  M_k = mean of the top k,
 *   SS_k = sum_{i<=k} (z_i - M_k)^2;
 * the support size is the largest k with SS_k <= 1 and tau_k < z_(k).
 */
double orc_entmax15_tau(const double *z, int n)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    memcpy(s, z, sizeof(double) * (size_t)n);
    qsort(s, (size_t)n, sizeof(double), cmp_double_desc);
    double best = s[0] - 1.0;
    for (int k = 1; k <= n; ++k) {
        double m = 0.0;
        for (int i = 0; i < k; ++i) m += s[i];
        m /= k;
        double ss = 0.0;
        for (int i = 0; i < k; ++i) ss += (s[i] - m) * (s[i] - m);
        if (ss > 1.0) break;
        double tk = m - sqrt((1.0 - ss) / k);
        if (tk < s[k - 1]) best = tk;
    }
    free(s);
    return best;
}

static double mass_above(const double *z, int n, double tau, double r)
{
    double f = 0.0;
    for (int i = 0; i < n; ++i) {
        double x = z[i] - tau;
        if (x > 0.0) f += pow(x, r);
    }
    return f;
}

/*
 * General alpha > 1: tau solves sum_i [z_i - tau]_+^r = 1, r = 1/(alpha-1).
 * The root lies in [z_max - 1, z_max - n^(1-alpha)]: p_max <= 1 gives the lower
 * end and n equal shares give the upper.  Bisection in fp64 fixes the support,
 * then Newton on the support polishes tau to rounding level.
 */
double orc_entmax_tau(const double *z, int n, double alpha)
{
    double r = 1.0 / (alpha - 1.0);
    double zmax = -INFINITY;
    for (int i = 0; i < n; ++i) if (z[i] > zmax) zmax = z[i];
    double lo = zmax - 1.0, hi = zmax - pow((double)n, 1.0 - alpha);
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (mass_above(z, n, mid, r) >= 1.0) lo = mid; else hi = mid;
    }
    double tau = lo;
    for (int it = 0; it < 50; ++it) {
        double f = -1.0, fp = 0.0;
        for (int i = 0; i < n; ++i) {
            double x = z[i] - tau;
            if (x > 0.0) { f += pow(x, r); fp -= r * pow(x, r - 1.0); }
        }
        if (fp == 0.0) break;
        double nt = tau - f / fp;
        if (!(nt >= lo && nt <= hi)) break;
        if (nt == tau) break;
        tau = nt;
    }
    return tau;
}

/* --------------------------------------------------------------- decode */
/*
 * Section 2.C (sparse) and section 4 (full cache): for each (b, h) over the
 * token set T (the pages listed in sel[b][h][0..cnt) when sel != NULL, every
 * page of the sequence otherwise):
 *   s_t = (sum_j q_j k_tj) / sqrt(d)          (fp64, index order)
 *   alpha > 1:  z_t = (alpha-1) s_t, tau from orc_entmax_tau,
 *               p_t = [z_t - tau]_+^{1/(alpha-1)}
 *   alpha == 1: p_t = exp(s_t - max s) / sum exp(s - max s)   (softmax)
 *   o = sum_t p_t v_t                         (fp64)
 * Outputs: o [B][Hq][d], tau [B][Hq] (log sum exp(s) for softmax), and optionally
 * p_out [B][Hq][max_pages*P] in logical token order (only tokens of T written)
 * and z_out with the same layout (z for entmax, s for softmax).
 */
void orc_decode(int B, int Hq, int Hkv, int d, int P, int max_pages,
                const uint16_t *q, const uint16_t *K, const uint16_t *V,
                const int32_t *page_table, const int32_t *seq_lens,
                const int32_t *sel, const int32_t *cnt, int sel_stride,
                double alpha, double *o, double *tau_out,
                double *p_out, double *z_out)
{
    int G = Hq / Hkv;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            int kvh = h / G;
            size_t bh = (size_t)b * Hq + h;
            const uint16_t *qh = q + bh * d;
            int np = n_pages_of(seq_lens[b], P);
            int npl = sel ? cnt[bh] : np;
            size_t cap = (size_t)npl * P;
            double *zs = (double *)malloc(sizeof(double) * (cap ? cap : 1));
            size_t *src = (size_t *)malloc(sizeof(size_t) * (cap ? cap : 1));
            size_t *lpos = (size_t *)malloc(sizeof(size_t) * (cap ? cap : 1));
            int n = 0;
            for (int i = 0; i < npl; ++i) {
                int p = sel ? sel[bh * (size_t)sel_stride + i] : i;
                int blk = page_table[(size_t)b * max_pages + p];
                int nt = tokens_in_page(seq_lens[b], P, p);
                for (int t = 0; t < nt; ++t) {
                    size_t row = (((size_t)blk * Hkv + kvh) * P + t) * d;
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j)
                        acc += bf16_to_double(qh[j]) * bf16_to_double(K[row + j]);
                    double s = acc * inv_sqrt_d;
                    zs[n] = (alpha > 1.0) ? (alpha - 1.0) * s : s;
                    src[n] = row;
                    lpos[n] = (size_t)p * P + t;
                    ++n;
                }
            }
            double *oh = o + bh * d;
            for (int j = 0; j < d; ++j) oh[j] = 0.0;
            if (n == 0) { tau_out[bh] = NAN; free(zs); free(src); free(lpos); continue; }
            double tau;
            double *pw = (double *)malloc(sizeof(double) * (size_t)n);
            if (alpha > 1.0) {
                tau = orc_entmax_tau(zs, n, alpha);
                double r = 1.0 / (alpha - 1.0);
                for (int i = 0; i < n; ++i) {
                    double x = zs[i] - tau;
                    pw[i] = x > 0.0 ? pow(x, r) : 0.0;
                }
            } else {
                double m = -INFINITY, den = 0.0;
                for (int i = 0; i < n; ++i) if (zs[i] > m) m = zs[i];
                for (int i = 0; i < n; ++i) { pw[i] = exp(zs[i] - m); den += pw[i]; }
                for (int i = 0; i < n; ++i) pw[i] /= den;
                tau = m + log(den);  /* softmax: log-sum-exp of the scores */
            }
            for (int i = 0; i < n; ++i) {
                if (pw[i] == 0.0) continue;
                for (int j = 0; j < d; ++j) oh[j] += pw[i] * bf16_to_double(V[src[i] + j]);
            }
            tau_out[bh] = tau;
            size_t lstride = (size_t)max_pages * P;
            if (p_out) for (int i = 0; i < n; ++i) p_out[bh * lstride + lpos[i]] = pw[i];
            if (z_out) for (int i = 0; i < n; ++i) z_out[bh * lstride + lpos[i]] = zs[i];
            free(pw); free(zs); free(src); free(lpos);
        }
    }
}

/*
 * Scores and page selection for a whole batch (the middle of one decode step):
 * per (b, h) either top-k (policy 0), the Gaussian rule with the bound as the
 * estimated maximum (policy 1) or with the capped Gaussian estimate (policy 2).
 * sel is [B][Hq][max_pages], cnt and tau_hat are [B][Hq] (tau_hat NAN for top-k).
 */
void orc_select(int B, int Hq, int P, int max_pages, const int32_t *seq_lens,
                const float *bbox, const float *mu, const float *sigma,
                int policy, int k, double alpha, double delta,
                int32_t *sel, int32_t *cnt, double *tau_hat)
{
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            size_t bh = (size_t)b * Hq + h;
            int np = n_pages_of(seq_lens[b], P);
            const float *bb = bbox + bh * max_pages;
            int32_t *sl = sel + bh * max_pages;
            if (policy == 0) {
                cnt[bh] = orc_select_topk(np, bb, k, sl);
                tau_hat[bh] = NAN;
            } else {
                int32_t *nt = (int32_t *)malloc(sizeof(int32_t) * (size_t)(np ? np : 1));
                for (int p = 0; p < np; ++p) nt[p] = tokens_in_page(seq_lens[b], P, p);
                double th = orc_tau_hat(np, mu + bh * max_pages, sigma + bh * max_pages, nt, alpha);
                tau_hat[bh] = th;
                if (policy == 1)
                    cnt[bh] = orc_select_gauss(np, bb, alpha, th, delta, sl);
                else
                    cnt[bh] = orc_select_gauss_est(np, bb, mu + bh * max_pages, sigma + bh * max_pages, nt,
                                                   alpha, th, delta, sl);
                free(nt);
            }
        }
    }
}
