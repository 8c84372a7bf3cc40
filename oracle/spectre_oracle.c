/*
 * spectre_oracle.c -- double-precision CPU oracle for SPECTRE frequency-domain
 * token mixing.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference the CUDA path is
 * checked against.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  It shares no code, header, table or
 * helper with the CUDA library, and it must never be used to produce a result
 * for a user.
 *
 * What it computes (SPECTRE walk-through, hotelren.com/news/5925787, §2.2
 * pseudocode; §2.1 convolution theorem; §2.3 truncation):
 *
 *   for every batch row b and channel c = h*D + d (head h owns G[h, :]):
 *     Q = rfft(q[b,:,c]), K = rfft(k[b,:,c]), V = rfft(v[b,:,c])   (along L)
 *     O_f = Q_f * conj(K_f) * G[h,f] * V_f   for f <  F
 *     O_f = 0                                for F <= f <= L/2
 *     out[b,:,c] = irfft(O, n=L)
 *   y[b,t,:] = LayerNorm_C(out[b,t,:] + x[b,t,:]; gamma, beta, eps)
 *
 * Readings of points the pages leave open:
 *   - forward transform unscaled, inverse scaled by 1/L (the default norm of
 *     the fft/ifft calls in the §2.2 pseudocode);
 *   - real-input transforms (rfft/irfft): for real q,k,v and a real gate they
 *     equal fft followed by the real part of ifft;
 *   - "keep the first K bins" (§2.3) zeroes rfft bins f >= F, which keeps
 *     the output real;
 *   - the imaginary parts of the DC and Nyquist bins are ignored by the
 *     inverse, as irfft does;
 *   - the gate is a given real tensor G[H, L/2+1] multiplied in;
 *   - LayerNorm uses the biased variance with eps inside the square root.
 *
 * Precision: all arithmetic in double.  Inputs are read in their stored
 * format (fp32, or bf16 bit patterns) and widened exactly to double.
 *
 * The FFT is a plain recursive decimation-in-time transform over the prime
 * factors of n (2 and 3 on the lengths used here, any prime via a direct
 * DFT base step).  Twiddles exp(-2*pi*i*e/n) are taken from a table whose
 * exponents are reduced modulo n before the angle is formed.
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef double complex cplx;

/* ------------------------------------------------------------------------- */
/* twiddle table: w[e] = exp(sign * 2*pi*i * e / n), e in [0, n)              */
/* ------------------------------------------------------------------------- */
static cplx *make_twiddles(size_t n, int sign)
{
    cplx *w = (cplx *)malloc(n * sizeof(cplx));
    if (!w) return NULL;
    for (size_t e = 0; e < n; e++) {
        double ang = 2.0 * M_PI * (double)e / (double)n;
        w[e] = cos(ang) + (double)sign * sin(ang) * I;
    }
    return w;
}

static size_t smallest_factor(size_t n)
{
    if (n % 2 == 0) return 2;
    if (n % 3 == 0) return 3;
    for (size_t p = 5; p * p <= n; p += 2)
        if (n % p == 0) return p;
    return n;
}

/*
 * Recursive mixed-radix DIT FFT (Cooley-Tukey).  Length-n transform of
 * in[0], in[stride], ..., in[(n-1)*stride] into out[0..n-1].
 * N is the top-level length, w the length-N twiddle table; a sub-transform of
 * length n uses w[e * (N/n)].  tmp holds at least n values.
 *   X[k + m*s] = sum_{r<p} w_n^{r(k+m s)} * Y_r[k],   n = p*m,
 * where Y_r is the length-m transform of the samples with index = r mod p.
 */
static void fft_rec(const cplx *in, size_t stride, cplx *out, size_t n,
                    const cplx *w, size_t N, cplx *tmp)
{
    if (n == 1) {
        out[0] = in[0];
        return;
    }
    size_t p = smallest_factor(n);
    size_t m = n / p;
    for (size_t r = 0; r < p; r++)
        fft_rec(in + r * stride, stride * p, out + r * m, m, w, N, tmp);
    size_t step = N / n; /* w_n^e = w_N^{e*step} */
    for (size_t k = 0; k < m; k++) {
        for (size_t s = 0; s < p; s++) {
            cplx acc = 0.0;
            for (size_t r = 0; r < p; r++) {
                size_t e = (r * (k + m * s)) % n;
                acc += w[e * step] * out[r * m + k];
            }
            tmp[s] = acc;
        }
        for (size_t s = 0; s < p; s++) out[k + m * s] = tmp[s];
    }
}

/* Complex DFT of length n, sign -1 forward, +1 inverse (unscaled).
 * Returns 0 on success, -1 on allocation failure. */
int oracle_fft(long n, const double *in_re, const double *in_im,
               double *out_re, double *out_im, int sign)
{
    if (n <= 0) return -1;
    cplx *x = (cplx *)malloc((size_t)n * sizeof(cplx));
    cplx *y = (cplx *)malloc((size_t)n * sizeof(cplx));
    cplx *t = (cplx *)malloc((size_t)n * sizeof(cplx));
    cplx *w = make_twiddles((size_t)n, sign < 0 ? -1 : 1);
    if (!x || !y || !t || !w) {
        free(x); free(y); free(t); free(w);
        return -1;
    }
    for (long i = 0; i < n; i++) x[i] = in_re[i] + (in_im ? in_im[i] : 0.0) * I;
    fft_rec(x, 1, y, (size_t)n, w, (size_t)n, t);
    for (long i = 0; i < n; i++) {
        out_re[i] = creal(y[i]);
        out_im[i] = cimag(y[i]);
    }
    free(x); free(y); free(t); free(w);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* real transforms                                                            */
/* ------------------------------------------------------------------------- */
typedef struct {
    size_t L;
    cplx *wf, *wi;      /* forward / inverse twiddles, length L */
    cplx *a, *b, *tmp;  /* scratch, length L each */
} rt_ctx;

static int rt_init(rt_ctx *c, size_t L, const cplx *wf, const cplx *wi)
{
    c->L = L;
    c->wf = (cplx *)wf;
    c->wi = (cplx *)wi;
    c->a = (cplx *)malloc(L * sizeof(cplx));
    c->b = (cplx *)malloc(L * sizeof(cplx));
    c->tmp = (cplx *)malloc(L * sizeof(cplx));
    return (c->a && c->b && c->tmp) ? 0 : -1;
}

static void rt_free(rt_ctx *c)
{
    free(c->a); free(c->b); free(c->tmp);
}

/* rfft: bins 0..L/2 of the DFT of real x (forward, unscaled). */
static void rfft(rt_ctx *c, const double *x, cplx *X)
{
    for (size_t t = 0; t < c->L; t++) c->a[t] = x[t];
    fft_rec(c->a, 1, c->b, c->L, c->wf, c->L, c->tmp);
    for (size_t f = 0; f <= c->L / 2; f++) X[f] = c->b[f];
}

/* irfft: x[t] = (1/L) * Re sum_{f<L} Z_f e^{+2 pi i f t / L}, where Z is the
 * Hermitian extension of X[0..L/2] (Z_{L-f} = conj X_f) with the imaginary
 * parts of the DC and (even-L) Nyquist bins dropped. */
static void irfft(rt_ctx *c, const cplx *X, double *x)
{
    size_t L = c->L, h = L / 2;
    for (size_t f = 0; f <= h; f++) c->a[f] = X[f];
    c->a[0] = creal(X[0]);
    if (L % 2 == 0) c->a[h] = creal(X[h]);
    for (size_t f = 1; f < (L + 1) / 2; f++) c->a[L - f] = conj(X[f]);
    fft_rec(c->a, 1, c->b, L, c->wi, L, c->tmp);
    for (size_t t = 0; t < L; t++) x[t] = creal(c->b[t]) / (double)L;
}

/* ------------------------------------------------------------------------- */
/* input widening                                                             */
/* ------------------------------------------------------------------------- */
static double load_elem(const void *p, size_t i, int dtype)
{
    if (dtype == 0) return (double)((const float *)p)[i];
    /* bf16: the 16 stored bits are the top half of an IEEE fp32 */
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * out[b, :, c] for one channel (SPECTRE walk-through §2.2 pseudocode, with the
 * §2.3 truncation): gather the channel's column of q, k and v, take their
 * forward real FFTs, form the gated cross-spectrum times V's spectrum with
 * bins f >= F zeroed, and take the inverse real FFT into oc[0..L-1].
 */
typedef struct {
    rt_ctx ctx;
    double *col, *oc;
    cplx *Q, *K, *V;
    int ok;
} chan_ws;

static void chan_ws_init(chan_ws *w, long L, const cplx *wf, const cplx *wi)
{
    long nb = L / 2 + 1;
    w->col = (double *)malloc((size_t)L * sizeof(double));
    w->oc = (double *)malloc((size_t)L * sizeof(double));
    w->Q = (cplx *)malloc((size_t)nb * sizeof(cplx));
    w->K = (cplx *)malloc((size_t)nb * sizeof(cplx));
    w->V = (cplx *)malloc((size_t)nb * sizeof(cplx));
    w->ok = rt_init(&w->ctx, (size_t)L, wf, wi) == 0 && w->col && w->oc &&
            w->Q && w->K && w->V;
}

static void chan_ws_free(chan_ws *w)
{
    rt_free(&w->ctx);
    free(w->col); free(w->oc); free(w->Q); free(w->K); free(w->V);
}

static void mix_channel(chan_ws *w, long b, long c, long L, long C, int D,
                        int F, int dtype, const void *q, const void *k,
                        const void *v, const float *G, int cgate)
{
    long nb = L / 2 + 1;
    size_t base = (size_t)b * (size_t)L * (size_t)C + (size_t)c;
    for (long t = 0; t < L; t++) w->col[t] = load_elem(q, base + (size_t)t * C, dtype);
    rfft(&w->ctx, w->col, w->Q);
    for (long t = 0; t < L; t++) w->col[t] = load_elem(k, base + (size_t)t * C, dtype);
    rfft(&w->ctx, w->col, w->K);
    for (long t = 0; t < L; t++) w->col[t] = load_elem(v, base + (size_t)t * C, dtype);
    rfft(&w->ctx, w->col, w->V);
    /* real gate: G[h][f]; complex gate (a relative-position phase, §2.4):
     * G[h][f] = re + i im stored as pairs.  Bins f <= L/2 only: irfft
     * extends O Hermitian-symmetrically, so the complex gate acts as
     * conj(G[L - f]) above L/2 and the output stays real. */
    const float *Gh = G + (size_t)(c / D) * (size_t)nb * (cgate ? 2 : 1);
    for (long f = 0; f < nb; f++) {
        if (f < F) {
            cplx g = cgate ? (double)Gh[2 * f] + I * (double)Gh[2 * f + 1] : (double)Gh[f];
            w->Q[f] = w->Q[f] * conj(w->K[f]) * g * w->V[f];
        } else {
            w->Q[f] = 0.0;
        }
    }
    irfft(&w->ctx, w->Q, w->oc);
}

/*
 * oracle_spectre_out: the pre-LayerNorm mixer output for a channel range.
 *   q, k, v: [B, L, C] in dtype (0 = fp32, 1 = bf16 bits), row-major.
 *   G: [H, L/2+1] fp32, or with cgate [H, L/2+1, 2] (re, im); channel c
 *   uses row c / D.
 *   out: [B, L, c1 - c0] double (channel c written at column c - c0).
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_spectre_out(int B, long L, int H, int D, int F, int dtype,
                       const void *q, const void *k, const void *v,
                       const float *G, int c0, int c1, double *out,
                       int nthreads, int cgate)
{
    long C = (long)H * D;
    long nb = L / 2 + 1;
    if (B < 1 || L < 2 || H < 1 || D < 1 || F < 1 || F > nb || c0 < 0 ||
        c1 > C || c0 >= c1 || (dtype != 0 && dtype != 1))
        return -1;
    long W = c1 - c0;
    cplx *wf = make_twiddles((size_t)L, -1);
    cplx *wi = make_twiddles((size_t)L, +1);
    if (!wf || !wi) {
        free(wf); free(wi);
        return -1;
    }
    int failed = 0;
    long njobs = (long)B * W;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        chan_ws w;
        chan_ws_init(&w, L, wf, wi);
        if (!w.ok) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long job = 0; job < njobs; job++) {
            if (!w.ok) continue;
            long b = job / W, c = c0 + job % W;
            mix_channel(&w, b, c, L, C, D, F, dtype, q, k, v, G, cgate);
            for (long t = 0; t < L; t++)
                out[((size_t)b * (size_t)L + (size_t)t) * (size_t)W + (size_t)(c - c0)] = w.oc[t];
        }
        chan_ws_free(&w);
    }
    free(wf); free(wi);
    return failed ? -1 : 0;
}

/*
 * oracle_spectre_mix: y = LayerNorm_C(out + x) at selected tokens
 * (SPECTRE walk-through §2.2: layer_norm(out + x)), or one of the variants
 * the walk-through's §3.3 names (normalise before the residual; RMSNorm).
 *   tok: ntok token indices in [0, L) (NULL with ntok = L means every token).
 *   out_sel: [B, ntok, C] double or NULL; y_sel: [B, ntok, C] double.
 *   norm_mode: 0 y = LN(out + x); 1 y = LN(out) + x;
 *              2 y = RMS(out + x); 3 y = RMS(out) + x.
 * LN(z) = (z - mean) / sqrt(var + eps) * gamma + beta, mean and biased
 * variance over the C channels of one token; RMS(z) = z / sqrt(mean(z^2) +
 * eps) * gamma + beta.
 */
int oracle_spectre_mix(int B, long L, int H, int D, int F, int dtype,
                       double eps, const void *q, const void *k,
                       const void *v, const void *x, const float *G,
                       const float *gamma, const float *beta,
                       const long *tok, long ntok, double *out_sel,
                       double *y_sel, int nthreads, int norm_mode, int cgate)
{
    long C = (long)H * D;
    long nb = L / 2 + 1;
    if (B < 1 || L < 2 || H < 1 || D < 1 || F < 1 || F > nb || ntok < 1 ||
        (dtype != 0 && dtype != 1) || !y_sel || norm_mode < 0 || norm_mode > 3)
        return -1;
    if (!tok && ntok != L) return -1;
    for (long i = 0; tok && i < ntok; i++)
        if (tok[i] < 0 || tok[i] >= L) return -1;

    /* out at the selected tokens, channel by channel */
    double *o = out_sel ? out_sel
                        : (double *)malloc((size_t)B * (size_t)ntok * (size_t)C * sizeof(double));
    if (!o) return -1;
    cplx *wf = make_twiddles((size_t)L, -1);
    cplx *wi = make_twiddles((size_t)L, +1);
    if (!wf || !wi) {
        free(wf); free(wi);
        if (!out_sel) free(o);
        return -1;
    }
    int failed = 0;
    long njobs = (long)B * C;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        chan_ws w;
        chan_ws_init(&w, L, wf, wi);
        if (!w.ok) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long job = 0; job < njobs; job++) {
            if (!w.ok) continue;
            long b = job / C, c = job % C;
            mix_channel(&w, b, c, L, C, D, F, dtype, q, k, v, G, cgate);
            for (long i = 0; i < ntok; i++) {
                long t = tok ? tok[i] : i;
                o[((size_t)b * (size_t)ntok + (size_t)i) * (size_t)C + (size_t)c] = w.oc[t];
            }
        }
        chan_ws_free(&w);
    }
    free(wf); free(wi);
    if (failed) {
        if (!out_sel) free(o);
        return -1;
    }

    /* residual and normalisation over C, token by token */
    const int pre = norm_mode & 1, rms = norm_mode >> 1;
    for (long b = 0; b < B; b++) {
        for (long i = 0; i < ntok; i++) {
            long t = tok ? tok[i] : i;
            const double *orow = o + ((size_t)b * (size_t)ntok + (size_t)i) * (size_t)C;
            double *yrow = y_sel + ((size_t)b * (size_t)ntok + (size_t)i) * (size_t)C;
            size_t xbase = ((size_t)b * (size_t)L + (size_t)t) * (size_t)C;
            /* z: out + x, or out alone when x is added after the norm */
            for (long c = 0; c < C; c++)
                yrow[c] = orow[c] + (pre ? 0.0 : load_elem(x, xbase + (size_t)c, dtype));
            double mean = 0.0, var = 0.0;
            if (rms) {
                for (long c = 0; c < C; c++) var += yrow[c] * yrow[c];
                var /= (double)C;                       /* mean of squares */
            } else {
                for (long c = 0; c < C; c++) mean += yrow[c];
                mean /= (double)C;
                for (long c = 0; c < C; c++) var += (yrow[c] - mean) * (yrow[c] - mean);
                var /= (double)C;
            }
            double rstd = 1.0 / sqrt(var + eps);
            for (long c = 0; c < C; c++) {
                yrow[c] = (yrow[c] - mean) * rstd * (double)gamma[c] + (double)beta[c];
                if (pre) yrow[c] += load_elem(x, xbase + (size_t)c, dtype);
            }
        }
    }
    if (!out_sel) free(o);
    return 0;
}
