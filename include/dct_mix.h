/*
 * dct_mix.h -- C ABI of the per-token DCT mix with spectral-entropy routing
 * (part of libspectre_mix), on NVIDIA B200 (sm_100a).
 *
 * The operation (Chiaroscuro Attention summary,
 * paper.rainbus.top/paper/2606.08327: "Prerequisites: DCT", "Prerequisites:
 * spectral entropy", "Method step details"), for every token row x of x[T][d]:
 *
 *   X_k  = s_k * sum_n x_n cos(pi (2n+1) k / (2d))   orthonormal Type-II DCT,
 *          s_0 = sqrt(1/d), s_k = sqrt(2/d) for k > 0
 *   H    = -sum_k p_k ln p_k / ln d,  p_k = X_k^2 / sum_j X_j^2
 *          (normalised spectral entropy in [0, 1]; H = 0 for an all-zero row)
 *   route = 1 if H <= tau else 0      (1: the token takes the DCT branch)
 *   m    = iDCT(X * w)                orthonormal inverse, w[d] a spectral filter
 *   y    = LayerNorm over d of (x + m), with gamma, beta, eps
 *          (biased variance, eps inside the square root)
 *
 * The method's feed-forward layer inside DCTMix and its attention branch are
 * not part of this call: y is the DCT branch for every token and route says
 * which tokens take it.
 *
 * Supported shapes: d = 2^k with 64 <= d <= 1024; any T >= 0 (T = 0 does
 * nothing).  Numbers: x and y are fp32 (SPECTRE_F32) or bf16 (SPECTRE_BF16),
 * both of the plan's type; w, gamma, beta, H and the optional mix output are
 * fp32; route is one byte per token.  Arithmetic is fp32; a bf16 y is rounded
 * to nearest even.
 *
 * Layout: x, y, mix: [T][d] row-major; w, gamma, beta: [d]; H, route: [T].
 * Every tensor pointer must be 16-byte aligned (SPECTRE_ERR_ALIGN).
 *
 * Ownership: the caller owns every tensor.  The handle owns its twiddle
 * tables and, after the first dct_mix_run_host, a device staging buffer.
 *
 * Errors: the spectre_status codes of spectre_mix.h; no function throws or
 * exits.  Device faults of an asynchronous launch surface at the caller's
 * next synchronisation.
 */
#ifndef DCT_MIX_H
#define DCT_MIX_H

#include "spectre_mix.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dct_mix_s *dct_mix_t;

/*
 * Create a plan for rows of length d on the current CUDA device: validates d,
 * dtype and eps, computes the twiddle tables in double precision on the host
 * (stored as fp32) and uploads them.  Synchronous.
 *   out  : receives the handle (NULL on failure).
 *   d    : row length, 2^k in [64, 1024]  (SPECTRE_ERR_UNSUPPORTED_L otherwise).
 *   dtype: SPECTRE_F32 or SPECTRE_BF16; eps: LayerNorm epsilon, finite and > 0.
 * Returns SPECTRE_OK, SPECTRE_ERR_ARG, SPECTRE_ERR_UNSUPPORTED_L,
 * SPECTRE_ERR_DEVICE (no sm_100 device), SPECTRE_ERR_NOMEM or SPECTRE_ERR_CUDA.
 */
int dct_mix_create(dct_mix_t *out, int d, int dtype, float eps);

/*
 * Enqueue one DCT mix of T token rows on `stream` (a cudaStream_t, NULL for
 * the legacy default stream).  All pointers are device pointers:
 *   x     : [T][d] input rows (plan dtype).   w: [d] fp32 spectral filter.
 *   gamma, beta: [d] fp32 LayerNorm affine.   tau: routing threshold.
 *   y     : [T][d] output (plan dtype).       H: [T] fp32 entropies.
 *   route : [T] bytes, 1 where H <= tau (H as computed in fp32), else 0.
 * x and y may not overlap.  Returns SPECTRE_ERR_ARG for a NULL handle or
 * pointer (with T > 0) or T < 0, SPECTRE_ERR_ALIGN, SPECTRE_ERR_DEVICE when
 * the handle's device is not current, SPECTRE_ERR_CUDA for a failed launch.
 */
int dct_mix_run(dct_mix_t h, long long T, const void *x, const float *w, const float *gamma,
                const float *beta, float tau, void *y, float *H, unsigned char *route,
                void *stream);

/* dct_mix_run that also writes mix = iDCT(DCT(x) * w) (before the residual)
 * as fp32 [T][d] to `mix` (device, 16-byte aligned). */
int dct_mix_run_debug(dct_mix_t h, long long T, const void *x, const float *w,
                      const float *gamma, const float *beta, float tau, void *y, float *H,
                      unsigned char *route, float *mix, void *stream);

/* dct_mix_run on HOST buffers (pinned memory keeps the copies asynchronous):
 * enqueues the host-to-device copies of x, w, gamma, beta into a staging
 * buffer the handle owns (grown as T needs), the mix, and the device-to-host
 * copies of y, H and route, all on `stream`.  The results are in place once
 * `stream` has been synchronised. */
int dct_mix_run_host(dct_mix_t h, long long T, const void *x, const float *w,
                     const float *gamma, const float *beta, float tau, void *y, float *H,
                     unsigned char *route, void *stream);

/* Release the handle's device memory.  NULL-safe; returns SPECTRE_OK. */
int dct_mix_destroy(dct_mix_t h);

#ifdef __cplusplus
}
#endif

#endif /* DCT_MIX_H */
