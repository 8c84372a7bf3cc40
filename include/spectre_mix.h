/*
 * spectre_mix.h -- C ABI of libspectre_mix, SPECTRE frequency-domain token
 * mixing on NVIDIA B200 (sm_100a).
 *
 * The operation (SPECTRE walk-through, hotelren.com/news/5925787, §2.2
 * pseudocode, with the §2.3 low-frequency truncation):
 *
 *   q, k, v, x, y : [B, L, C] row-major, C = H * D contiguous,
 *                   channel c = h * D + d belongs to head h.
 *   for each (b, c):  Q = rfft(q[b,:,c]), K = rfft(k[b,:,c]), V = rfft(v[b,:,c])
 *                     O_f = Q_f * conj(K_f) * G[h, f] * V_f   for 0 <= f < F
 *                     O_f = 0                                 for F <= f <= L/2
 *                     out[b,:,c] = irfft(O, n = L)
 *   y[b,t,:] = LayerNorm over C of (out[b,t,:] + x[b,t,:]), with gamma, beta, eps
 *              (biased variance, eps inside the square root).
 *
 * The forward transform is unscaled and the inverse is scaled by 1/L.  The
 * imaginary parts of the DC and Nyquist bins are ignored by the inverse.  The
 * gate multiplies in as given (any sigmoid is applied by the caller).
 *
 * Supported shapes: L = 2^k (8 <= L <= 2^20) or L = 3 * 2^k (12 <= L <= 786432);
 * 1 <= B <= 65535; H, D >= 1; 1 <= F <= L/2 + 1; R * C * 4 bytes (R = 16, or 64
 * for L > 2^18) fits one block's shared memory.
 *
 * Numbers: q, k, v, x and y are fp32 (SPECTRE_F32) or bf16 (SPECTRE_BF16), all
 * of one type; G, gamma and beta are always fp32.  Arithmetic is fp32; y in
 * bf16 is rounded to nearest even.
 *
 * Ownership: the caller owns every tensor.  The handle owns its twiddle
 * tables, its workspace, one auxiliary CUDA stream and two events (created
 * by spectre_mix_create, released by spectre_mix_destroy).  spectre_mix_run
 * forks that stream from the caller's stream and joins it back before it
 * returns control of the work to `stream`, so stream ordering for the caller
 * is unchanged.
 *
 * Errors: every function returns a status code (SPECTRE_OK or a negative
 * SPECTRE_ERR_*), never throws and never exits.  Device faults of an
 * asynchronous launch surface at the caller's next synchronisation.
 */
#ifndef SPECTRE_MIX_H
#define SPECTRE_MIX_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct spectre_mix_s *spectre_mix_t;

enum spectre_dtype {
    SPECTRE_F32 = 0,  /* q, k, v, x, y stored as IEEE fp32 */
    SPECTRE_BF16 = 1  /* q, k, v, x, y stored as bfloat16 */
};

enum spectre_status {
    SPECTRE_OK = 0,
    SPECTRE_ERR_ARG = -1,           /* a null pointer, a bad size, F, dtype or eps */
    SPECTRE_ERR_UNSUPPORTED_L = -2, /* L is not 2^k or 3*2^k in the supported range */
    SPECTRE_ERR_ALIGN = -3,         /* a tensor pointer is not 16-byte aligned */
    SPECTRE_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed */
    SPECTRE_ERR_NOMEM = -5,         /* device or host allocation failed */
    SPECTRE_ERR_DEVICE = -6,        /* no usable sm_100 device, or wrong current device */
    SPECTRE_ERR_SCRATCH = -7,       /* problem too large for the no-allocation scratch */
    SPECTRE_ERR_TIMEOUT = -8        /* a bounded device-side wait gave up (see below) */
};

/* Size of the fixed device scratch behind spectre_mix_run_noalloc. */
#define SPECTRE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * Create a plan for one problem shape.  Validates the shape, picks the
 * decomposition L = R * M, allocates the twiddle tables and the workspace on
 * the current CUDA device and fills the tables there (double-precision
 * sines and cosines, stored as fp32).  Synchronous.
 *   out   : receives the handle (set to NULL on failure).
 *   B     : batch rows; L: sequence length; H: heads; D: channels per head.
 *   F     : number of low-frequency rfft bins kept (F = L/2 + 1 keeps all).
 *   dtype : SPECTRE_F32 or SPECTRE_BF16.
 *   eps   : LayerNorm epsilon, > 0.
 * Supported shapes: L = 2^k with 8 <= L <= 2^20, or L = 3 * 2^k with
 * 12 <= L <= 786432 (else SPECTRE_ERR_UNSUPPORTED_L); B in [1, 65535],
 * H, D >= 1 with C = H * D <= 2^20, 1 <= F <= L/2 + 1, and C narrow enough for
 * the inverse pass to hold R token rows of all channels in shared memory:
 * R * (C rounded up to a multiple of 32, plus 16) * 4 bytes <= 227 KiB, which
 * is C <= 3616 for R = 16 (L <= 2^18, or L = 3 * 2^k <= 196608) and C <= 864
 * for R = 64 (the longer L).  Other shapes give SPECTRE_ERR_ARG.
 */
int spectre_mix_create(spectre_mix_t *out, int B, int L, int H, int D, int F,
                       int dtype, float eps);

/*
 * Enqueue one mix on `stream` (a cudaStream_t; NULL = the legacy default
 * stream).  Asynchronous: returns after the launches are queued.
 *   q, k, v, x : device, [B, L, C] in the plan's dtype.
 *   G          : device, fp32 [H, L/2 + 1] (row h is head h's gate).
 *   gamma, beta: device, fp32 [C].
 *   y          : device, [B, L, C] in the plan's dtype; may not alias inputs.
 * Every pointer must be non-null and 16-byte aligned.  One handle must not run
 * on two streams at once: its workspace is shared by all its runs.  Calls on
 * one handle come from one host thread at a time (the handle keeps the
 * captured graph of its last pointer set, SPECTRE_OPT_GRAPH).
 */
int spectre_mix_run(spectre_mix_t h, const void *q, const void *k, const void *v,
                    const void *x, const float *G, const float *gamma,
                    const float *beta, void *y, void *stream);

/*
 * As spectre_mix_run, and also writes the pre-LayerNorm mixer output `out`
 * as fp32 [B, L, C] to `out_f32` (device, 16-byte aligned) when it is not
 * NULL.  For verification; the timed path is spectre_mix_run.
 */
int spectre_mix_run_debug(spectre_mix_t h, const void *q, const void *k,
                          const void *v, const void *x, const float *G,
                          const float *gamma, const float *beta, void *y,
                          float *out_f32, void *stream);

/*
 * End-to-end variant taking HOST buffers (same shapes and types as
 * spectre_mix_run).  Enqueues host-to-device copies of q, k, v, x, G, gamma
 * and beta into device staging buffers owned by the handle, the mix, and a
 * device-to-host copy of y, all on `stream`.  The staging buffers are
 * allocated on the first call (so that call is synchronous and must not be
 * made during stream capture).  With page-locked host memory the call is
 * asynchronous: synchronise `stream` before reading y or reusing the inputs.
 */
int spectre_mix_run_host(spectre_mix_t h, const void *q, const void *k,
                         const void *v, const void *x, const float *G,
                         const float *gamma, const float *beta, void *y,
                         void *stream);

/*
 * As spectre_mix_run, and also records CUDA events on `stream` around every
 * kernel launch of the path, for per-kernel timing.  The path is, for each
 * channel chunk, a row-pass launch then a slice-pass launch, and finally one
 * inverse-row-pass launch: n launches in all (see spectre_mix_plan_info).
 * spectre_mix_run overlaps one chunk's row pass with the previous chunk's
 * slice pass on a second stream the handle owns; the profiled run keeps all
 * launches on `stream`, one after another, so each event pair brackets one
 * kernel.  `events` points to nevents = n + 1 cudaEvent_t created by the caller;
 * events[i] is recorded before launch i and events[n] after the last.
 * Returns SPECTRE_ERR_ARG if nevents != n + 1 or an event is NULL.
 */
int spectre_mix_run_profiled(spectre_mix_t h, const void *q, const void *k,
                             const void *v, const void *x, const float *G,
                             const float *gamma, const float *beta, void *y,
                             void *const *events, int nevents, void *stream);

/*
 * One mix that allocates nothing.  The pages have no counterpart: this entry
 * point exists for callers that may not call cudaMalloc -- for instance code
 * running inside a framework whose caching allocator owns the device memory
 * and forbids side allocations, or a latency-critical loop that cannot accept
 * the device-wide synchronisation cudaMalloc and cudaFree can imply.
 *
 * Same operation, shapes, types and pointer rules as spectre_mix_run, with the
 * plan arguments of spectre_mix_create passed on every call (no handle).  The
 * caller still provides every input and output.  Instead of a workspace
 * allocated per plan, the call uses one fixed device array of
 * SPECTRE_NOALLOC_SCRATCH_BYTES (64 MiB) built into the library; every GPU
 * that loads the library holds that array until the process exits.  Twiddle
 * tables are rebuilt in the scratch by a small kernel on each call; the rest
 * of the scratch is fully overwritten before it is read, so nothing carries
 * over from the previous call.
 *
 *   Returns SPECTRE_ERR_SCRATCH when the tables plus the workspace of this
 *   shape (exactly what spectre_mix_workspace_bytes reports for the same
 *   shape's plan before any spectre_mix_run_host call adds staging) exceed
 *   the scratch; other errors as spectre_mix_create/spectre_mix_run.
 *   No error word is kept for this path: if a bounded tensor-core wait
 *   gives up, y comes out NaN (see spectre_mix_device_status).
 *
 * The first call on a device looks up the scratch's device address and loads
 * constant twiddles (synchronous); make that first call before any stream
 * capture.  All calls on a device share the one scratch array, so calls that
 * overlap on the GPU (other streams, other host threads) race: serialise them.
 * Asynchronous otherwise: returns after the launches are queued on `stream`.
 */
int spectre_mix_run_noalloc(int B, int L, int H, int D, int F, int dtype,
                            float eps, const void *q, const void *k,
                            const void *v, const void *x, const float *G,
                            const float *gamma, const float *beta, void *y,
                            void *stream);

enum spectre_option {
    /* 1 (default): plans with bf16 I/O, slice length M = 4096 (L = 65536) and
     * a truncation that leaves at most 16 live bins per slice row (F <= L/8
     * roughly) run the slice pass on the tensor cores: every 4096-point
     * transform as two DFT-64 passes of tcgen05 MMAs with fp16 operands
     * (power-of-two scaled per slice) and fp32 accumulation in tensor memory,
     * the truncation pruning the MMAs.  0: the CUDA-core slice pass (fp32
     * Stockham radix-16 butterflies) for every plan.  Plans outside the
     * tensor-core range always take the CUDA-core pass. */
    SPECTRE_OPT_TENSOR_CORES = 1,
    /* How the mixer output is normalised (enum spectre_norm; default
     * SPECTRE_NORM_POST_LN, the walk-through's §2.2 form).  The other values
     * are the §3.3 variants.  The no-allocation entry point always uses the
     * default. */
    SPECTRE_OPT_NORM = 2,
    /* 0 (default): G is real, [H][L/2+1] fp32.  1: G is complex, a gate with
     * a relative-position phase (walk-through §2.4): [H][L/2+1][2] fp32 as
     * (re, im) pairs, 16-byte aligned like every tensor.  Bins above L/2 use
     * conj(G[L - f]), so the output stays real; the imaginary parts at DC
     * and Nyquist are dropped, as an inverse real FFT does.  The
     * no-allocation entry point takes real gates only. */
    SPECTRE_OPT_COMPLEX_GATE = 3,
    /* 0 (default).  1: for tests of the failure path only.  In every
     * tensor-core slice launch, block 0 issues no MMA and waits only a few
     * 1 ms polls on its MMA barrier, so that wait gives up with nothing in
     * flight: the run's y is NaN and spectre_mix_device_status reports
     * SPECTRE_ERR_TIMEOUT.  No effect on plans that take the CUDA-core slice
     * pass. */
    SPECTRE_OPT_TEST_WAIT_TIMEOUT = 4,
    /* 0 (default): the row pass (the first stage of the forward transforms)
     * runs on the CUDA cores.  1: plans with bf16 I/O, R = 16 and a channel
     * count that is a multiple of 64 run it on the tensor cores: one TMA box
     * per 16 t2 x 64 channels, the 16-point DFT over t1 as bf16 MMAs with the
     * DFT matrix split into two bf16 terms (so the transform is accurate to
     * about 2^-17), fp32 accumulation in tensor memory.  Same results within
     * rounding; measured slower on B200 for the bf16 long workload (36 us
     * against 25 us per 128-channel launch), so it is off by default. */
    SPECTRE_OPT_ROW_TENSOR_CORES = 5,
    /* 1 (default): spectre_mix_run (and spectre_mix_run_host) replays the
     * step's launches as one CUDA graph,
     * captured at the first run with a given set of tensor pointers (and
     * again after a pointer or an option changes) on a stream the handle
     * owns, and launched on the caller's stream.  A capture costs about as
     * much as instantiating the graph; replays skip the per-launch host work.
     * A caller's stream that is itself being captured gets the plain
     * launches.  0: every run enqueues the launches directly.  Runs with
     * events (spectre_mix_run_profiled) or a debug output never use the
     * graph. */
    SPECTRE_OPT_GRAPH = 6
};

enum spectre_norm {
    SPECTRE_NORM_POST_LN = 0,   /* y = LayerNorm(out + x) */
    SPECTRE_NORM_PRE_LN = 1,    /* y = LayerNorm(out) + x */
    SPECTRE_NORM_POST_RMS = 2,  /* y = RMSNorm(out + x) */
    SPECTRE_NORM_PRE_RMS = 3    /* y = RMSNorm(out) + x */
    /* LayerNorm(z) = (z - mean) / sqrt(var + eps) * gamma + beta (biased
     * variance over C); RMSNorm(z) = z / sqrt(mean(z^2) + eps) * gamma + beta
     * (pass beta = 0 for the usual bias-free form). */
};

/* Set an option of the plan (see enum spectre_option).  Takes effect for
 * runs enqueued afterwards.  SPECTRE_ERR_ARG for a NULL handle, an unknown
 * option or a value out of range. */
int spectre_mix_set_option(spectre_mix_t h, int option, int value);

enum spectre_slice_pass {
    SPECTRE_SLICE_CUDA_CORES = 0,
    SPECTRE_SLICE_TENSOR_CORES = 1
};

/* Which slice pass runs of the plan launch under its current options
 * (enum spectre_slice_pass); SPECTRE_ERR_ARG for a NULL handle. */
int spectre_mix_slice_pass(spectre_mix_t h);

/*
 * Synchronise `stream` and report device-side failures of the handle's
 * earlier runs: SPECTRE_ERR_TIMEOUT if a bounded wait for a tensor-core MMA
 * gave up in any run since the last call, else SPECTRE_OK.  Clears the
 * recorded failure.  A block whose wait gives up (after about 4 s) stops,
 * releases its tensor memory and sets the scales of the slices it did not
 * finish to NaN, so every y of that run is NaN: the failure is visible in
 * the output as well (this is how spectre_mix_run_noalloc, which keeps no
 * error word, reports it).
 */
int spectre_mix_device_status(spectre_mix_t h, void *stream);

/* Free the handle, its tables, workspace and staging buffers.  NULL-safe.
 * Synchronises the device the handle lives on before freeing. */
int spectre_mix_destroy(spectre_mix_t h);

/* Static, human-readable text for a status code. */
const char *spectre_mix_error_string(int code);

/* Device bytes held by the handle (tables, workspace, staging), 0 for NULL. */
size_t spectre_mix_workspace_bytes(spectre_mix_t h);

/*
 * The decomposition the plan chose: L = R * M, with R-point transforms in the
 * row passes and M-point transforms per frequency slice (R/2 + 1 slices per
 * channel).  Channels are processed in waves of `channels_per_wave` so that
 * one wave's row-pass output stays in L2 until the slice pass reads it;
 * `launches` is the number of kernel launches of one run (2 per wave + 1).
 * Any out-pointer may be NULL.  Returns SPECTRE_ERR_ARG for a NULL handle.
 */
int spectre_mix_plan_info(spectre_mix_t h, int *R, int *M, int *slices_per_channel,
                          int *channels_per_wave, int *launches);

#ifdef __cplusplus
}
#endif

#endif /* SPECTRE_MIX_H */
