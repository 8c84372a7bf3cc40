/*
 * dct_oracle.c -- double-precision CPU oracle for per-token DCT mixing with
 * spectral-entropy routing.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
 * CPU-baseline leg of the benchmark are its only callers.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (Chiaroscuro Attention summary,
 * paper.rainbus.top/paper/2606.08327: "Prerequisites: DCT" and
 * "Prerequisites: spectral entropy" for the transform and H(x); "Method step
 * details" for DCTMix and the routing rule), for every token row x of length d:
 *
 *   X_k  = s_k * sum_n x_n cos(pi (2n+1) k / (2d)),  s_0 = sqrt(1/d),
 *          s_k = sqrt(2/d) for k > 0               (orthonormal Type-II DCT)
 *   p_k  = X_k^2 / sum_j X_j^2
 *   H(x) = -sum_k p_k ln p_k / ln d                (0 * ln 0 = 0; H = 0 for x = 0)
 *   route(x) = 1 if H(x) <= tau else 0             (1: the token takes the DCT branch)
 *   m_n  = sum_k s_k (w_k X_k) cos(pi (2n+1) k / (2d))   (orthonormal inverse)
 *   y    = LayerNorm_d(x + m; gamma, beta, eps)
 *
 * Readings of points the pages leave open:
 *   - the DCT is orthonormal: the pages call it an orthogonal transform, and
 *     only then is the power spectrum the energy per basis vector;
 *   - the entropy is normalised by ln d so that it lies in [0, 1] as stated;
 *   - the DCT and the filter act along the hidden dimension of each token,
 *     the same per-token spectrum the routing uses;
 *   - DCTMix's feed-forward network (a trained layer) is left out, so the
 *     mix is LayerNorm(x + iDCT(DCT(x) * w)); w is one filter of length d;
 *   - LayerNorm over d uses the biased variance with eps inside the root.
 *
 * Every sum is the plain O(d^2) definition; cos values come from a table of
 * cos(2 pi e / (4d)) with e = (2n+1)k reduced modulo 4d.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* stored element i of a row: dtype 0 = fp32, 1 = bf16 bit pattern */
static double dct_load(const void *p, size_t i, int dtype)
{
    if (dtype == 0) return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* cos(2 pi e / (4d)) for e in [0, 4d) */
static double *cos_table(long d)
{
    double *c = (double *)malloc((size_t)(4 * d) * sizeof(double));
    if (!c) return NULL;
    for (long e = 0; e < 4 * d; e++) c[e] = cos(2.0 * M_PI * (double)e / (double)(4 * d));
    return c;
}

static double dct_s(long k, long d) { return k == 0 ? sqrt(1.0 / (double)d) : sqrt(2.0 / (double)d); }

static void dct2_row(const double *x, double *X, long d, const double *ct)
{
    for (long k = 0; k < d; k++) {
        double acc = 0.0;
        for (long n = 0; n < d; n++) acc += x[n] * ct[((2 * n + 1) * k) % (4 * d)];
        X[k] = dct_s(k, d) * acc;
    }
}

static void dct3_row(const double *X, double *x, long d, const double *ct)
{
    for (long n = 0; n < d; n++) {
        double acc = 0.0;
        for (long k = 0; k < d; k++) acc += dct_s(k, d) * X[k] * ct[((2 * n + 1) * k) % (4 * d)];
        x[n] = acc;
    }
}

/* Orthonormal Type-II DCT of T rows of length d (fp64 in and out). */
int oracle_dct2(long T, long d, const double *x, double *X)
{
    if (T < 0 || d < 1 || !x || !X) return -1;
    double *ct = cos_table(d);
    if (!ct) return -2;
    for (long t = 0; t < T; t++) dct2_row(x + t * d, X + t * d, d, ct);
    free(ct);
    return 0;
}

/* Its inverse (the orthonormal Type-III DCT). */
int oracle_dct3(long T, long d, const double *X, double *x)
{
    if (T < 0 || d < 1 || !x || !X) return -1;
    double *ct = cos_table(d);
    if (!ct) return -2;
    for (long t = 0; t < T; t++) dct3_row(X + t * d, x + t * d, d, ct);
    free(ct);
    return 0;
}

/* Normalised spectral entropy of one row's coefficients. */
static double entropy_row(const double *X, long d)
{
    double e = 0.0;
    for (long k = 0; k < d; k++) e += X[k] * X[k];
    if (e == 0.0) return 0.0;
    double h = 0.0;
    for (long k = 0; k < d; k++) {
        double p = X[k] * X[k] / e;
        if (p > 0.0) h -= p * log(p);
    }
    return d > 1 ? h / log((double)d) : 0.0;
}

/*
 * The DCT mix of T token rows x[T][d] (stored fp32 or bf16, widened exactly):
 * mix[T][d] (before the residual), y[T][d], H[T] and route[T].  Any output
 * pointer may be NULL.  nthreads <= 0 uses the OpenMP default.
 */
int oracle_dct_mix(long T, long d, int dtype, const void *x, const float *w, const float *gamma,
                   const float *beta, double eps, double tau, double *mix, double *y, double *H,
                   unsigned char *route, int nthreads)
{
    if (T < 0 || d < 2 || !x || !w || !gamma || !beta || (dtype != 0 && dtype != 1)) return -1;
    double *ct = cos_table(d);
    if (!ct) return -2;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : bad)
#endif
    {
        double *buf = (double *)malloc((size_t)(4 * d) * sizeof(double));
        if (!buf) {
            bad = 1;
        } else {
            double *xr = buf, *X = buf + d, *m = buf + 2 * d, *z = buf + 3 * d;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
            for (long t = 0; t < T; t++) {
                const size_t base = (size_t)t * (size_t)d;
                for (long n = 0; n < d; n++) xr[n] = dct_load(x, base + (size_t)n, dtype);
                dct2_row(xr, X, d, ct);
                double h = entropy_row(X, d);
                if (H) H[t] = h;
                if (route) route[t] = (unsigned char)(h <= tau);
                for (long k = 0; k < d; k++) X[k] *= (double)w[k];
                dct3_row(X, m, d, ct);
                if (mix) memcpy(mix + base, m, (size_t)d * sizeof(double));
                double mean = 0.0;
                for (long n = 0; n < d; n++) {
                    z[n] = xr[n] + m[n];
                    mean += z[n];
                }
                mean /= (double)d;
                double var = 0.0;
                for (long n = 0; n < d; n++) var += (z[n] - mean) * (z[n] - mean);
                var /= (double)d;
                double rstd = 1.0 / sqrt(var + eps);
                if (y)
                    for (long n = 0; n < d; n++)
                        y[base + n] = (z[n] - mean) * rstd * (double)gamma[n] + (double)beta[n];
            }
            free(buf);
        }
    }
    free(ct);
    return bad ? -2 : 0;
}
