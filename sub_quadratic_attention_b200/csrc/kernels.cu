// kernels.cu -- the CUDA-core kernels of the SPECTRE spectral mixer on
// sm_100a (SPECTRE walk-through, hotelren.com/news/5925787: §2.2 pseudocode,
// §2.3 truncation, §3.1 real/imaginary parts carried as separate reals).
//
//   spectre_rows_fwd[_pipe]     : q, k, v rows -> R-point real transforms -> A
//   spectre_slices<M>           : per (b, c, f1) slice: three M-point FFTs, the
//                                 gated product, one inverse M-point FFT -> P
//   spectre_rows_inv_ln[_reg|_pipe] : P -> R-point inverse (real output) -> + x
//                                 -> LayerNorm over C -> y
//
// The _pipe variants are persistent and prefetch their next work item into
// shared memory with cp.async.  The tensor-core slice pass for M = 4096 is in
// slices_mma.cu.  The index algebra is in kernels.cuh.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>
#include <type_traits>

#include "fft_regs.cuh"
#include "kernels.cuh"
#include "tc_dft.cuh"

#ifndef SPECTRE_L2_HINTS
#define SPECTRE_L2_HINTS 1
#endif
// cap on the persistent row pass's blocks per multiprocessor
#ifndef SPECTRE_ROW_CTAS_PER_SM
#define SPECTRE_ROW_CTAS_PER_SM 4
#endif
// token columns per group of the prefetching inverse pass (1 or 2)
#ifndef SPECTRE_INV_COLS
#define SPECTRE_INV_COLS 2
#endif

namespace spectre {

// ---------------------------------------------------------------------------
// element I/O
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ __forceinline__ static float load(const float *p) { return __ldg(p); }
    __device__ __forceinline__ static float2 load2(const float *p) {
        return __ldg(reinterpret_cast<const float2 *>(p));
    }
    __device__ __forceinline__ static void store(float *p, float v) { *p = v; }
    __device__ __forceinline__ static void store2(float *p, float v0, float v1) {
        *reinterpret_cast<float2 *>(p) = make_float2(v0, v1);
    }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16 *p) {
        return __bfloat162float(__ldg(p));
    }
    __device__ __forceinline__ static float2 load2(const __nv_bfloat16 *p) {
        return __bfloat1622float2(__ldg(reinterpret_cast<const __nv_bfloat162 *>(p)));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
    __device__ __forceinline__ static void store2(__nv_bfloat16 *p, float v0, float v1) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v0, v1);
    }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One complex value of A: fp32 (float2), or with A16 a bf16 (re, im) pair.
// bf16 halves the intermediate's bytes; its 8-bit significand adds a
// relative error of at most 2^-9 per value, well inside the bf16-input bar.
template <bool A16> struct AElem;
template <> struct AElem<false> {
    using T = float2;
    __device__ __forceinline__ static void store(float2 *p, float2 v) { *p = v; }
    __device__ __forceinline__ static float2 load(const float2 *p) { return __ldg(p); }
};
template <> struct AElem<true> {
    using T = __nv_bfloat162;
    __device__ __forceinline__ static void store(__nv_bfloat162 *p, float2 v) {
        *p = __floats2bfloat162_rn(v.x, v.y);
    }
    __device__ __forceinline__ static float2 load(const __nv_bfloat162 *p) {
        return __bfloat1622float2(__ldg(p));
    }
};

// ---------------------------------------------------------------------------
// row pass: A[sig][b][c][f1][t2] = w_L^{f1 t2} sum_{t1} w_R^{f1 t1} sig[b][t1 M + t2][c]
// Block: 256 threads = 8 warps over 8 t2 values x 32 channel pairs; a warp
// covers 4 consecutive t2 x 8 consecutive channel pairs, lane = tl + 4 cpl.
// Each thread owns channels c0 = 2 cp, c0 + 1 at one t2, packed as one complex
// signal c0 + i c1.  Its 16-row loads are 32-byte segments per warp-row
// (8 channel pairs) and its stores are 32-byte segments (4 consecutive t2) of
// A, straight from registers.
// ---------------------------------------------------------------------------
template <int R, typename T, bool A16>
__global__ void __launch_bounds__(256, R <= 16 ? 4 : 1) spectre_rows_fwd(RowsFwdArgs a) {
    constexpr int NF = R / 2 + 1;
    using AT = typename AElem<A16>::T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t2 = blockIdx.x * 8 + (warp & 1) * 4 + (lane & 3);
    const int cp = blockIdx.y * 32 + (warp >> 1) * 8 + (lane >> 2);
    const int b = blockIdx.z;
    const int cl = 2 * cp;                 // channel within the wave
    const int c0 = a.c_lo + cl;
    const int cend = min(a.C, a.c_lo + a.Cw);
    const bool live = (t2 < a.M) && (c0 < cend);
    const bool has1 = live && (c0 + 1 < cend);
    const size_t rowstride = (size_t)a.M * a.C;
    const size_t plane = (size_t)a.B * a.Cw * NF * a.M;
    AT *dst0 = static_cast<AT *>(a.A) + ((size_t)b * a.Cw + cl) * NF * a.M + t2;
    AT *dst1 = dst0 + (size_t)NF * a.M;

#pragma unroll 1
    for (int sig = 0; sig < 3; sig++) {
        const T *src = static_cast<const T *>(sig == 0 ? a.q : (sig == 1 ? a.k : a.v));
        float2 z[R];
        if (live) {
            const T *p = src + ((size_t)b * a.L + t2) * a.C + c0;
            if (a.vec2) {
#pragma unroll
                for (int t1 = 0; t1 < R; t1++) z[t1] = Elem<T>::load2(p + t1 * rowstride);
            } else {
#pragma unroll
                for (int t1 = 0; t1 < R; t1++) {
                    z[t1].x = Elem<T>::load(p + t1 * rowstride);
                    z[t1].y = has1 ? Elem<T>::load(p + t1 * rowstride + 1) : 0.f;
                }
            }
        } else {
#pragma unroll
            for (int t1 = 0; t1 < R; t1++) z[t1] = make_float2(0.f, 0.f);
        }
        Dft<R>::run(z);
        // separate the two real channels, twiddle by w_L^{f1 t2}, store
        if (live) {
#pragma unroll
            for (int f1 = 0; f1 < NF; f1++) {
                float2 zf = z[f1], zc = cconj(z[(R - f1) % R]);
                float2 xa = cscale(cadd(zf, zc), 0.5f);
                float2 d = csub(zf, zc);
                float2 xb = make_float2(0.5f * d.y, -0.5f * d.x);
                if (f1 > 0) {
                    float2 w = __ldg(a.twL + f1 * t2);
                    xa = cmul(xa, w);
                    xb = cmul(xb, w);
                }
                AElem<A16>::store(dst0 + sig * plane + (size_t)f1 * a.M, xa);
                if (has1) AElem<A16>::store(dst1 + sig * plane + (size_t)f1 * a.M, xb);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// row pass, prefetching variant (R = 16, bf16 inputs, channel chunks that are
// multiples of 64).  Work items are (tile, signal) with tiles of 8 t2 x 64
// channels; a persistent block computes one item from a shared-memory stage
// while cp.async copies the next item's 16 x 8 row segments (64 bf16 each)
// into the other stage.  Rows are padded to 72 values so the warp's 8 t2 x 4
// channel-pair reads fall on 32 different banks.  Arithmetic and stores are
// those of spectre_rows_fwd.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :
                 : "r"((uint32_t)__cvta_generic_to_shared(smem_dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 16-byte copy of a streamed input row segment, marked first to leave L2 (so
// the row pass's reads do not push A, which the slice pass reads next, out of
// L2)
__device__ __forceinline__ void cp_async16_rows(void *smem_dst, const void *src, uint64_t pol) {
#if SPECTRE_L2_HINTS
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;"
                 :
                 : "r"((uint32_t)__cvta_generic_to_shared(smem_dst)), "l"(src), "l"(pol)
                 : "memory");
#else
    (void)pol;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :
                 : "r"((uint32_t)__cvta_generic_to_shared(smem_dst)), "l"(src)
                 : "memory");
#endif
}
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// one bf16 (re, im) pair of A, kept in L2 for the slice pass
__device__ __forceinline__ void store_a16_keep(__nv_bfloat162 *p, float2 v, uint64_t pol) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
#if SPECTRE_L2_HINTS
    asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;"
                 :
                 : "l"(p), "r"(*reinterpret_cast<const uint32_t *>(&h)), "l"(pol)
                 : "memory");
#else
    (void)pol;
    *p = h;
#endif
}

constexpr int kFwdPipeRow = 72;                          // bf16 per padded row (36 words)
constexpr int kFwdPipeStage = 16 * 8 * kFwdPipeRow / 2;  // 4-byte words per stage

template <bool A16>
__global__ void __launch_bounds__(256, 4) spectre_rows_fwd_pipe(RowsFwdArgs a) {
    constexpr int R = 16, NF = R / 2 + 1;
    using AT = typename AElem<A16>::T;
    extern __shared__ float4 smem_f4[];
    uint32_t *stage0 = reinterpret_cast<uint32_t *>(smem_f4);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // a warp covers 8 consecutive t2 x 4 channel pairs (lane = t2l + 8 (cpl % 4)),
    // so each of its stores to A is 8 consecutive t2 of one channel and slice
    // (a 32-byte sector for bf16 A); with 36-word rows the stage reads hit
    // bank 4 t2l + cpl mod 32, all different
    const int t2l = lane & 7;                              // 0..7
    const int cpl = warp * 4 + (lane >> 3);                // 0..31
    const int ntg = a.M / 8, ncg = a.Cw / 64;
    const int nitems = 3 * ntg * ncg * a.B;                // < 2^31 (checked by the launcher)
    const size_t rowstep = (size_t)a.M * a.C;
    const size_t plane = (size_t)a.B * a.Cw * NF * a.M;

    // item = ((b * ncg + cg) * ntg + tg) * 3 + sig, decoded with 32-bit
    // multiply-high division by the launch's fixed divisors
    auto decode = [&](int item, int &sig, int &tg, int &cg, int &b) {
        const uint32_t r1 = fdiv((uint32_t)item, a.fd3);
        sig = item - 3 * (int)r1;
        const uint32_t r2 = fdiv(r1, a.fd_ntg);
        tg = (int)r1 - ntg * (int)r2;
        const uint32_t r3 = fdiv(r2, a.fd_ncg);
        cg = (int)r2 - ncg * (int)r3;
        b = (int)r3;
    };
    const uint64_t pol_in = l2_evict_first(), pol_a = l2_evict_last();
    auto prefetch = [&](int item, int st) {
        int sig, tg, cg, b;
        decode(item, sig, tg, cg, b);
        uint32_t *dst = stage0 + st * kFwdPipeStage;
        const void *sp = sig == 0 ? a.q : (sig == 1 ? a.k : a.v);
        const __nv_bfloat16 *base = static_cast<const __nv_bfloat16 *>(sp) +
                                    ((size_t)b * a.L + (size_t)tg * 8) * a.C + a.c_lo + 64 * cg;
        for (int i = tid; i < 16 * 8 * 8; i += 256) {       // (t1, t2 row, 16-byte piece)
            const int piece = i & 7, rr = i >> 3, t1 = rr >> 3, tr = rr & 7;
            cp_async16_rows(dst + rr * (kFwdPipeRow / 2) + 4 * piece,
                            base + (size_t)t1 * rowstep + (size_t)tr * a.C + 8 * piece, pol_in);
        }
    };

    int it = blockIdx.x;
    if (it < nitems) prefetch(it, 0);
    cp_async_commit();
#pragma unroll 1
    for (int k = 0; it < nitems; k++, it += gridDim.x) {
        const int nxt = it + gridDim.x;
        if (nxt < nitems) prefetch(nxt, (k + 1) & 1);
        cp_async_commit();
        cp_async_wait1();
        __syncthreads();
        int sig, tg, cg, b;
        decode(it, sig, tg, cg, b);
        const uint32_t *stg = stage0 + (k & 1) * kFwdPipeStage;
        const int t2 = tg * 8 + t2l;
        const int cl = 64 * cg + 2 * cpl;                  // channel within the chunk
        // w_L^{t2}, loaded before the transform; w_L^{f1 t2} follow as its powers
        // (seven products in fp32 add far less than bf16's rounding)
        const float2 wt = __ldg(a.twL + t2);
        float2 z[R];
#pragma unroll
        for (int t1 = 0; t1 < R; t1++) {
            const uint32_t w = stg[(t1 * 8 + t2l) * (kFwdPipeRow / 2) + cpl];
            z[t1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
        }
        Dft<R>::run(z);
        AT *dst0 = static_cast<AT *>(a.A) + sig * plane + ((size_t)b * a.Cw + cl) * NF * a.M + t2;
        AT *dst1 = dst0 + (size_t)NF * a.M;
        // wh = w_L^{f1 t2} / 2 and wb = -i wh: channel a = (Z_f + conj Z_{R-f}) wh,
        // channel b = (Z_f - conj Z_{R-f}) wb
        float2 wh = make_float2(0.5f, 0.f);
#pragma unroll
        for (int f1 = 0; f1 < NF; f1++) {
            if (f1 > 0) wh = cmul(wh, wt);
            const float2 wb = make_float2(wh.y, -wh.x);
            const float2 zf = z[f1], zc = cconj(z[(R - f1) % R]);
            const float2 xa = cmul(cadd(zf, zc), wh);
            const float2 xb = cmul(csub(zf, zc), wb);
            if constexpr (A16) {
                store_a16_keep(dst0 + (size_t)f1 * a.M, xa, pol_a);
                store_a16_keep(dst1 + (size_t)f1 * a.M, xb, pol_a);
            } else {
                AElem<A16>::store(dst0 + (size_t)f1 * a.M, xa);
                AElem<A16>::store(dst1 + (size_t)f1 * a.M, xb);
            }
        }
        // every read of this stage is done before it is refilled
        __syncthreads();
    }
    cp_async_wait_all();
}

// ---------------------------------------------------------------------------
// slice pass
// ---------------------------------------------------------------------------
__device__ __forceinline__ int spad(int i) { return i + (i >> 4); }

// One in-place Stockham pass over shared memory:
//   butterfly bf < M/R reads buf[bf + r M/R], twiddles by w_{Ns R}^{(bf mod Ns) r}
//   (table entry tw[r Ns + bf mod Ns], so a warp's loads are contiguous),
//   and writes buf[(bf / Ns) Ns R + (bf mod Ns) + r Ns].
template <int R, int M, int NT, int NS>
__device__ __forceinline__ void smem_pass(float2 *buf, const float2 *__restrict__ tw, int j) {
    constexpr int NBF = M / R;
    constexpr int NB = (NBF + NT - 1) / NT;
    float2 v[NB][R];
#pragma unroll
    for (int i = 0; i < NB; i++) {
        int bf = j + i * NT;
        if (NBF % NT == 0 || bf < NBF) {
#pragma unroll
            for (int r = 0; r < R; r++) v[i][r] = buf[spad(bf + r * NBF)];
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NB; i++) {
        int bf = j + i * NT;
        if (NBF % NT == 0 || bf < NBF) {
            int kk = bf % NS;
            if (NS > 1) {
                const float2 *t = tw + kk;
#pragma unroll
                for (int r = 1; r < R; r++) v[i][r] = cmul(v[i][r], __ldg(t + r * NS));
            }
            Dft<R>::run(v[i]);
            int idxD = (bf / NS) * NS * R + kk;
#pragma unroll
            for (int r = 0; r < R; r++) buf[spad(idxD + r * NS)] = v[i][r];
        }
    }
    __syncthreads();
}

template <int M, int NT, int D, int P, int PEND> struct MidPasses {
    __device__ __forceinline__ static void run(float2 *buf, const SliceTables &tb, int j) {
        if constexpr (P < PEND) {
            constexpr int R = sched_radix(M, D, P);
            constexpr int NS = sched_stride(M, D, P);
            smem_pass<R, M, NT, NS>(buf, tb.tw[D][P], j);
            MidPasses<M, NT, D, P + 1, PEND>::run(buf, tb, j);
        }
    }
};

// Where the running product S = Q conj(K) G' / L lives between the three
// forward transforms of a slice.
enum SliceProduct { kProdSmem = 0, kProdRegs = 1, kProdGlobal = 2 };

constexpr int spb_warp_aligned(int nt) {
    int s = 256 / nt;
    while (s > 1 && (s * nt) % 32 != 0) s--;
    return s;
}

template <int M> struct SliceCfg {
    static constexpr RadList S = make_schedule(M);
    static constexpr int NP = S.n;
    static constexpr int RL = NP > 0 ? S.r[NP - 1] : 1;   // largest radix, last
    static constexpr int R0 = NP > 0 ? S.r[0] : 1;
    static constexpr int NT = M / RL;                      // threads per slice
    // slices per block: as many as fill 256 threads with a whole number of
    // warps (M = 768: 4 slices of 48 threads, not 5, whose 240 threads end in
    // half a warp; measured on B200 for the mixed-radix workload, the slice
    // pass went from 1.37 to 1.03 ms per step)
    static constexpr int SPB = NT >= 256 ? 1 : spb_warp_aligned(NT);
    static constexpr int THREADS = NT * SPB;
    static constexpr int BUF = NP >= 2 ? (M + M / 16) : 0; // float2 per slice (padded)
    static constexpr int PROD = (BUF + M) * SPB * 8 <= 72 * 1024 ? kProdSmem
                              : (NT <= 512 ? kProdRegs : kProdGlobal);
    static constexpr int SMEM = (BUF + (PROD == kProdSmem ? M : 0)) * SPB * 8;
    // blocks per SM the register budget must allow
    static constexpr int MINB0 = PROD == kProdSmem ? (SMEM > 0 ? (200 * 1024) / SMEM : 4) : 1;
    static constexpr int MINB = MINB0 > 4 ? 4 : MINB0;
    static constexpr int MINB_C = MINB < 1 ? 1 : (MINB * THREADS > 2048 ? 2048 / THREADS : MINB);
};

// Forward M-point transform of one slice of A.  On return thread j holds
// X[j + r NT], r < RL, in x[].  buf must not be in use by other threads'
// loads (callers separate uses with a barrier).
template <int M, bool A16>
__device__ __forceinline__ void slice_forward(const typename AElem<A16>::T *__restrict__ src, bool live,
                                              float2 *buf, const SliceTables &tb, int j,
                                              float2 (&x)[SliceCfg<M>::RL]) {
    using Cfg = SliceCfg<M>;
    using AE = AElem<A16>;
    constexpr int NP = Cfg::NP, NT = Cfg::NT;
    if constexpr (NP == 0) {
        x[0] = live ? AE::load(src) : make_float2(0.f, 0.f);
    } else if constexpr (NP == 1) {
        constexpr int R = Cfg::RL;
#pragma unroll
        for (int r = 0; r < R; r++) x[r] = live ? AE::load(src + j + r * NT) : make_float2(0.f, 0.f);
        Dft<R>::run(x);
    } else {
        // first pass: global -> registers -> smem (Ns = 1, no twiddle)
        constexpr int R = Cfg::R0;
        constexpr int NBF = M / R;
        constexpr int NB = (NBF + NT - 1) / NT;
#pragma unroll
        for (int i = 0; i < NB; i++) {
            int bf = j + i * NT;
            if (NBF % NT == 0 || bf < NBF) {
                float2 v[R];
#pragma unroll
                for (int r = 0; r < R; r++) v[r] = live ? AE::load(src + bf + r * NBF) : make_float2(0.f, 0.f);
                Dft<R>::run(v);
#pragma unroll
                for (int r = 0; r < R; r++) buf[spad(bf * R + r)] = v[r];
            }
        }
        __syncthreads();
        MidPasses<M, NT, 0, 1, NP - 1>::run(buf, tb, j);
        // last pass: smem -> registers, one butterfly per thread (Ns = NT)
        constexpr int RL = Cfg::RL;
#pragma unroll
        for (int r = 0; r < RL; r++) x[r] = buf[spad(j + r * NT)];
        const float2 *t = tb.tw[0][NP - 1] + j;
#pragma unroll
        for (int r = 1; r < RL; r++) x[r] = cmul(x[r], __ldg(t + r * NT));
        Dft<RL>::run(x);
    }
}

// Store of one slice of P.  With p16 the slice's values are scaled by a power
// of two s chosen from the slice's largest magnitude m (m s < 2^14) and stored
// as fp16 (round to nearest); pscale receives 1/s.  Otherwise fp32.  smax is
// this slice's shared max word, zeroed at kernel start.
struct PStore {
    void *dst;        // slice base (float2 *, or __half2 * at the channel's lane of its pair)
    float *pscale;    // this slice's scale slot
    int *smax;
    bool live, p16;
};

__device__ __forceinline__ float slice_scale(PStore &ps, float local_max) {
    if (!ps.p16) return 1.0f;
    atomicMax(ps.smax, __float_as_int(local_max));
    __syncthreads();
    const float m = __int_as_float(*ps.smax);
    int e = 0;
    if (m > 0.f) frexpf(m, &e);   // m < 2^e
    const int sexp = max(-126, min(126, 14 - e));
    return ldexpf(1.0f, sexp);
}

__device__ __forceinline__ void pstore(const PStore &ps, int t2, float2 v, float s) {
    if (!ps.live) return;
    if (ps.p16)
        static_cast<__half2 *>(ps.dst)[2 * t2] = __floats2half2_rn(v.x * s, v.y * s);
    else
        static_cast<float2 *>(ps.dst)[t2] = v;
}

// Inverse (unscaled) M-point transform of the values thread j holds at
// positions j + r NT, via conj -> forward passes in reversed radix order ->
// conj; writes P[t2] = w_L^{-f1 t2} * result[t2].
template <int M>
__device__ __forceinline__ void slice_inverse_store(float2 (&o)[SliceCfg<M>::RL], float2 *buf,
                                                    const SliceTables &tb, int j, PStore &ps,
                                                    const float2 *__restrict__ twL, int f1) {
    using Cfg = SliceCfg<M>;
    constexpr int NP = Cfg::NP, NT = Cfg::NT, RL = Cfg::RL;
#pragma unroll
    for (int r = 0; r < RL; r++) o[r] = cconj(o[r]);
    if constexpr (NP == 0) {
        float2 v = cconj(o[0]);  // f1 * 0 = 0: no twiddle
        float s = slice_scale(ps, fmaxf(fabsf(v.x), fabsf(v.y)));
        pstore(ps, 0, v, s);
    } else if constexpr (NP == 1) {
        Dft<RL>::run(o);
        // single butterfly (j = 0): output r at position r
        float mx = 0.f;
#pragma unroll
        for (int r = 0; r < RL; r++) {
            o[r] = cconj(cmul(o[r], __ldg(twL + f1 * r)));
            mx = fmaxf(mx, fmaxf(fabsf(o[r].x), fabsf(o[r].y)));
        }
        float s = slice_scale(ps, mx);
#pragma unroll
        for (int r = 0; r < RL; r++) pstore(ps, r, o[r], s);
    } else {
        // first inverse pass: radix RL, Ns = 1, registers -> smem
        Dft<RL>::run(o);
        __syncthreads();  // the forward's last-pass loads are done everywhere
#pragma unroll
        for (int r = 0; r < RL; r++) buf[spad(j * RL + r)] = o[r];
        __syncthreads();
        MidPasses<M, NT, 1, 1, NP - 1>::run(buf, tb, j);
        // last inverse pass: radix R0, Ns = M / R0
        constexpr int R = Cfg::R0;
        constexpr int NBF = M / R;
        constexpr int NB = (NBF + NT - 1) / NT;
        const float2 *tw = tb.tw[1][NP - 1];
        float2 v[NB][R];
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < NB; i++) {
            int bf = j + i * NT;
            if (NBF % NT == 0 || bf < NBF) {
#pragma unroll
                for (int r = 0; r < R; r++) v[i][r] = buf[spad(bf + r * NBF)];
#pragma unroll
                for (int r = 1; r < R; r++) v[i][r] = cmul(v[i][r], __ldg(tw + bf + r * NBF));
                Dft<R>::run(v[i]);
#pragma unroll
                for (int r = 0; r < R; r++) {
                    v[i][r] = cconj(cmul(v[i][r], __ldg(twL + f1 * (bf + r * NBF))));
                    mx = fmaxf(mx, fmaxf(fabsf(v[i][r].x), fabsf(v[i][r].y)));
                }
            }
        }
        float s = slice_scale(ps, mx);
#pragma unroll
        for (int i = 0; i < NB; i++) {
            int bf = j + i * NT;
            if (NBF % NT == 0 || bf < NBF) {
#pragma unroll
                for (int r = 0; r < R; r++) pstore(ps, bf + r * NBF, v[i][r], s);
            }
        }
    }
    if (ps.p16 && ps.live && j == 0) {
        int e = 0;
        const float m = __int_as_float(*ps.smax);
        if (m > 0.f) frexpf(m, &e);
        *ps.pscale = ldexpf(1.0f, -max(-126, min(126, 14 - e)));
    }
}

template <int M, bool A16>
__global__ void __launch_bounds__(SliceCfg<M>::THREADS, SliceCfg<M>::MINB_C) spectre_slices(SliceArgs a) {
    using Cfg = SliceCfg<M>;
    using AT = typename AElem<A16>::T;
    constexpr int NT = Cfg::NT, RL = Cfg::RL, PROD = Cfg::PROD;
    static_assert(!(A16 && PROD == kProdGlobal), "the product is parked in fp32 A");
    extern __shared__ float4 smem_f4[];
    const int sl = threadIdx.x / NT;
    const int j = threadIdx.x % NT;
    float2 *buf = reinterpret_cast<float2 *>(smem_f4) + sl * Cfg::BUF;
    float2 *sbuf = reinterpret_cast<float2 *>(smem_f4) + Cfg::SPB * Cfg::BUF + sl * M;
    __shared__ int smax[Cfg::SPB];
    if (j == 0) smax[sl] = 0;
    const long long sid = (long long)blockIdx.x * Cfg::SPB + sl;
    const bool live = sid < a.nslices;
    const int NF = a.R / 2 + 1;
    const long long sidc = live ? sid : 0;
    const int f1 = (int)(sidc % NF);
    const long long bcl = sidc / NF;            // b * Cw + (c - c_lo)
    const int b = (int)(bcl / a.Cw);
    const int c = a.c_lo + (int)(bcl % a.Cw);
    const int h = c / a.D;
    const size_t sig_stride = (size_t)a.B * a.Cw * NF * M;
    const AT *srcA = static_cast<const AT *>(a.A) + (size_t)bcl * NF * M + (size_t)f1 * M;
    PStore ps;
    if (a.p16) {
        const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
        ps.dst = static_cast<__half2 *>(a.P) + 2 * pslice * M + (c & 1);
        ps.pscale = a.pscale + 2 * pslice + (c & 1);
    } else {
        const size_t pslice = ((size_t)b * a.C + c) * NF + f1;
        ps.dst = static_cast<float2 *>(a.P) + pslice * M;
        ps.pscale = nullptr;
    }
    ps.smax = &smax[sl];
    ps.live = live;
    ps.p16 = a.p16 != 0;
    const float *Gh = a.G + (size_t)h * a.nbins * (a.cgate ? 2 : 1);
    __syncthreads();  // smax initialised

    float2 x[RL];
    float2 s[RL];
    // each thread owns bins f = f1 + R (j + r NT), r < RL, of the product;
    // with kProdGlobal S is parked in this slice's q row of A, which nothing
    // reads once the q transform has passed its first stage
    float2 *park = A16 ? nullptr : reinterpret_cast<float2 *>(const_cast<AT *>(srcA));
    auto put = [&](int r, float2 v) {
        if constexpr (PROD == kProdSmem) sbuf[j + r * NT] = v;
        else if constexpr (PROD == kProdRegs) s[r] = v;
        else { if (live) park[j + r * NT] = v; }
    };
    auto get = [&](int r) -> float2 {
        if constexpr (PROD == kProdSmem) return sbuf[j + r * NT];
        else if constexpr (PROD == kProdRegs) return s[r];
        else return live ? park[j + r * NT] : make_float2(0.f, 0.f);
    };

    // q: S = Q * G' / L
    slice_forward<M, A16>(srcA, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) {
        int f = f1 + a.R * (j + r * NT);
        int ff = min(f, a.L - f);
        if (a.cgate) {   // conj(G[L - f]) above L/2
            float2 gc = (live && ff < a.F) ? __ldg(reinterpret_cast<const float2 *>(Gh) + ff)
                                           : make_float2(0.f, 0.f);
            if (f > a.L - f) gc.y = -gc.y;
            put(r, cscale(cmul(x[r], gc), a.invL));
        } else {
            float g = (live && ff < a.F) ? __ldg(Gh + ff) * a.invL : 0.f;
            put(r, cscale(x[r], g));
        }
    }
    if constexpr (Cfg::NP >= 2) __syncthreads();
    // k: S *= conj(K)
    slice_forward<M, A16>(srcA + sig_stride, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) put(r, cmulc(get(r), x[r]));
    if constexpr (Cfg::NP >= 2) __syncthreads();
    // v: O = S * V
    slice_forward<M, A16>(srcA + 2 * sig_stride, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) x[r] = cmul(get(r), x[r]);
    slice_inverse_store<M>(x, buf, a.tabs, j, ps, a.twL, f1);
}

// ---------------------------------------------------------------------------
// inverse row pass + residual + LayerNorm
// ---------------------------------------------------------------------------
// NV: the plan uses a norm variant (residual after the norm, or RMSNorm);
// without it the default LayerNorm(out + x) code is compiled alone.
// The R = 64 inverse row transform of spectre_rows_inv_ln over two lanes per
// (column, channel pair).  Every lane of the block runs the same number of
// iterations (padded with idle items), so the exchange is a full-warp shuffle.
template <typename T, bool P16>
__device__ __forceinline__ void inv64_pairs(const RowsInvArgs &a, float *zbuf, int T2C, int ZS, int b, int t2base,
                                            int CP) {
    constexpr int R = 64, NF = R / 2 + 1;
    const int items = 2 * T2C * CP;
    const int h = threadIdx.x & 1;
    const int rounds = (items + blockDim.x - 1) / blockDim.x;
    for (int k = 0; k < rounds; k++) {
        const int it = threadIdx.x + k * blockDim.x;
        const int rest = it >> 1;
        const int tl = rest % T2C, cp = rest / T2C;
        const int t2 = t2base + tl;
        const bool ok = it < items && t2 < a.M;
        const int c0 = 2 * cp;
        const bool has1 = ok && c0 + 1 < a.C;
        const size_t sa = ok ? (P16 ? p16_pair_slice(b, c0, 0, a.C, NF) : ((size_t)b * a.C + c0) * NF) : 0;
        const size_t sb = sa + NF;
        auto ld2 = [&](int f1, float2 &pa, float2 &pb) {
            pa = pb = make_float2(0.f, 0.f);
            if (!ok) return;
            if constexpr (P16) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(a.P) + (sa + f1) * a.M + t2);
                const float2 sc = __ldg(reinterpret_cast<const float2 *>(a.pscale) + sa + f1);
                pa = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.x)), sc.x);
                if (has1) pb = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.y)), sc.y);
            } else {
                pa = __ldg(static_cast<const float2 *>(a.P) + (sa + f1) * a.M + t2);
                if (has1) pb = __ldg(static_cast<const float2 *>(a.P) + (sb + f1) * a.M + t2);
            }
        };
        // v[m] = Z[2 m + h], where Z[f1] = P_a + i P_b and Z[64 - f1] =
        // conj(P_a) + i conj(P_b) for 0 < f1 < 32, both stored conjugated, and
        // Z[0], Z[32] keep the real parts only.  Lane h reads P[f1] for f1 = 2 q
        // + h: Z[f1] is v[q], Z[64 - f1] is v[32 - q - h] (both of parity h).
        float2 v[32];
#pragma unroll
        for (int q = 0; q <= 16; q++) {
            if (q == 16 && h == 1) break;   // f1 = 33: none
            const int f1 = 2 * q + h;
            float2 pv, qv;
            ld2(f1, pv, qv);
            if (h == 0 && (q == 0 || q == 16)) {
                v[q] = make_float2(pv.x, -qv.x);
            } else {
                v[q] = make_float2(pv.x - qv.y, -(pv.y + qv.x));
                const float2 sec = make_float2(pv.x + qv.y, pv.y - qv.x);
                if (h == 0) {
                    if (q >= 1 && q <= 15) v[32 - q] = sec;
                } else {
                    v[31 - q] = sec;
                }
            }
        }
        Dft<32>::run(v);
        // odd lane: W[t] = w64^t O[t]; then lane 0 forms E + W (t < 32),
        // lane 1 E - W (t + 32)
#pragma unroll
        for (int t = 1; t < 32; t++)
            if (h == 1) v[t] = cmul(v[t], c_w64[t]);
        float *zr = zbuf + (size_t)tl * ZS + c0;
#pragma unroll
        for (int t = 0; t < 32; t++) {
            const float rx = __shfl_xor_sync(0xffffffffu, v[t].x, 1);
            const float ry = __shfl_xor_sync(0xffffffffu, v[t].y, 1);
            const float2 o = h == 0 ? make_float2(v[t].x + rx, v[t].y + ry) : make_float2(rx - v[t].x, ry - v[t].y);
            if (ok) {
                // inverse result = conj: real part -> channel c0, imaginary -> c0 + 1
                float *p = zr + (size_t)(t + 32 * h) * T2C * ZS;
                if (has1)
                    *reinterpret_cast<float2 *>(p) = make_float2(o.x, -o.y);
                else
                    p[0] = o.x;
            }
        }
    }
}

template <int R, typename T, bool DEBUG_OUT, bool NV>
__global__ void __launch_bounds__(512) spectre_rows_inv_ln(RowsInvArgs a) {
    constexpr int NF = R / 2 + 1;
    constexpr bool P16 = std::is_same<T, __nv_bfloat16>::value;  // bf16 I/O: fp16 P
    extern __shared__ float4 smem_f4[];
    float *zbuf = reinterpret_cast<float *>(smem_f4);  // [R * T2C][ZS]
    const int T2C = a.T2C, ZS = a.ZS;
    const int b = blockIdx.y;
    const int t2base = blockIdx.x * T2C;
    const int CP = (a.C + 1) / 2;
    if constexpr (R == 64) {
        // two lanes per (column, channel pair): lane h of an even/odd pair takes
        // the even (h = 0) or odd (h = 1) inputs Z[2m + h], a 32-point DFT each;
        // then DFT64[t] = E[t] + w64^t O[t] and DFT64[t + 32] = E[t] - w64^t O[t],
        // lane 0 forming t < 32 and lane 1 t >= 32 after one exchange
        inv64_pairs<T, P16>(a, zbuf, T2C, ZS, b, t2base, CP);
    } else {
    const int items = T2C * CP;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int tl = it % T2C, cp = it / T2C;
        const int t2 = t2base + tl;
        if (t2 >= a.M) continue;
        const int c0 = 2 * cp;
        const bool has1 = c0 + 1 < a.C;
        // fp32 P: slices (c0, f1) and (c0 + 1, f1); fp16 P: the pair's slice
        const size_t sa = P16 ? p16_pair_slice(b, c0, 0, a.C, NF) : ((size_t)b * a.C + c0) * NF;
        const size_t sb = sa + NF;
        auto ld2 = [&](int f1, float2 &pa, float2 &pb) {
            if constexpr (P16) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(a.P) + (sa + f1) * a.M + t2);
                const float2 sc = __ldg(reinterpret_cast<const float2 *>(a.pscale) + sa + f1);
                pa = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.x)), sc.x);
                pb = has1 ? cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.y)), sc.y)
                          : make_float2(0.f, 0.f);
            } else {
                pa = __ldg(static_cast<const float2 *>(a.P) + (sa + f1) * a.M + t2);
                pb = has1 ? __ldg(static_cast<const float2 *>(a.P) + (sb + f1) * a.M + t2)
                          : make_float2(0.f, 0.f);
            }
        };
        float2 Z[R];
        {
            float2 a0, aN, b0, bN;
            ld2(0, a0, b0);
            ld2(R / 2, aN, bN);
            // DC and Nyquist: imaginary parts dropped; conj() for the inverse
            Z[0] = make_float2(a0.x, -b0.x);
            Z[R / 2] = make_float2(aN.x, -bN.x);
        }
#pragma unroll
        for (int f1 = 1; f1 < R / 2; f1++) {
            float2 pv, qv;
            ld2(f1, pv, qv);
            // Z[f1] = P_a + i P_b ; Z[R - f1] = conj(P_a) + i conj(P_b); stored conjugated
            Z[f1] = make_float2(pv.x - qv.y, -(pv.y + qv.x));
            Z[R - f1] = make_float2(pv.x + qv.y, pv.y - qv.x);
        }
        Dft<R>::run(Z);
        // inverse result = conj(Z): real part -> channel c0, imaginary -> c0 + 1
        float *zr = zbuf + (size_t)tl * ZS + c0;
#pragma unroll
        for (int t1 = 0; t1 < R; t1++) {
            float *p = zr + (size_t)t1 * T2C * ZS;
            if (has1)
                *reinterpret_cast<float2 *>(p) = make_float2(Z[t1].x, -Z[t1].y);
            else
                p[0] = Z[t1].x;
        }
    }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y);
    const float invC = 1.0f / (float)a.C;
    const bool pre = NV && (a.norm & 1), rms = NV && ((a.norm >> 1) & 1);   // residual after the norm; RMSNorm
    for (int row = warp; row < R * T2C; row += nw) {
        const int t1 = row / T2C, tl = row % T2C;
        const int t2 = t2base + tl;
        if (t2 >= a.M) continue;
        const size_t tok = (size_t)b * a.L + (size_t)t1 * a.M + t2;
        const T *xr = x + tok * a.C;
        T *yr = y + tok * a.C;
        float *zr = zbuf + (size_t)row * ZS;
        if (a.vec2) {   // channel pairs: 2-wide loads and stores (ZS is even, C even)
            float2 *zr2 = reinterpret_cast<float2 *>(zr);
            const int C2 = a.C / 2;
            float s = 0.f;
            for (int c = lane; c < C2; c += 32) {
                const float2 o = zr2[c];
                if (DEBUG_OUT) *reinterpret_cast<float2 *>(a.out_f32 + tok * a.C + 2 * c) = o;
                float2 z = o;
                if (!pre) {
                    const float2 xv = Elem<T>::load2(xr + 2 * c);
                    z.x += xv.x;
                    z.y += xv.y;
                }
                zr2[c] = z;
                s = rms ? fmaf(z.x, z.x, fmaf(z.y, z.y, s)) : s + (z.x + z.y);
            }
            float mean = 0.f, rstd;
            if (rms) {
                rstd = rsqrtf(warp_sum(s) * invC + a.eps);
            } else {
                mean = warp_sum(s) * invC;
                float ss = 0.f;
                for (int c = lane; c < C2; c += 32) {
                    const float2 z = zr2[c];
                    const float d0 = z.x - mean, d1 = z.y - mean;
                    ss = fmaf(d0, d0, fmaf(d1, d1, ss));
                }
                rstd = rsqrtf(warp_sum(ss) * invC + a.eps);
            }
            for (int c = lane; c < C2; c += 32) {
                const float2 z = zr2[c];
                const float2 g = __ldg(reinterpret_cast<const float2 *>(a.gamma) + c);
                const float2 bb = __ldg(reinterpret_cast<const float2 *>(a.beta) + c);
                float y0 = fmaf((z.x - mean) * rstd, g.x, bb.x);
                float y1 = fmaf((z.y - mean) * rstd, g.y, bb.y);
                if (pre) {
                    const float2 xv = Elem<T>::load2(xr + 2 * c);
                    y0 += xv.x;
                    y1 += xv.y;
                }
                Elem<T>::store2(yr + 2 * c, y0, y1);
            }
            continue;
        }
        float s = 0.f;
        for (int c = lane; c < a.C; c += 32) {
            float o = zr[c];
            if (DEBUG_OUT) a.out_f32[tok * a.C + c] = o;
            float z = pre ? o : o + Elem<T>::load(xr + c);
            zr[c] = z;
            s = rms ? fmaf(z, z, s) : s + z;
        }
        float mean = 0.f, rstd;
        if (rms) {
            rstd = rsqrtf(warp_sum(s) * invC + a.eps);
        } else {
            mean = warp_sum(s) * invC;
            float ss = 0.f;
            for (int c = lane; c < a.C; c += 32) {
                float d = zr[c] - mean;
                ss = fmaf(d, d, ss);
            }
            rstd = rsqrtf(warp_sum(ss) * invC + a.eps);
        }
        for (int c = lane; c < a.C; c += 32) {
            float yv = fmaf((zr[c] - mean) * rstd, __ldg(a.gamma + c), __ldg(a.beta + c));
            if (pre) yv += Elem<T>::load(xr + c);
            Elem<T>::store(yr + c, yv);
        }
    }
}

// ---------------------------------------------------------------------------
// inverse row pass + residual + LayerNorm, register-resident variant.
// Block: T2C x CP threads (CP = ceil(C/2) channel pairs, T2C t2 values,
// thread = tl + T2C * cp).  Each thread inverts its channel pair's R-point
// spectrum at one t2 and keeps the R x 2 values of z = out + x in registers;
// the LayerNorm statistics of the R * T2C token rows are reduced with warp
// shuffles and one shared-memory stage, in two passes (mean, then the mean
// of squared deviations), in a fixed order.
// ---------------------------------------------------------------------------
// Sum N per-lane values over the lanes that differ in lane bits [BIT, BITEND),
// by recursive halving: at each bit a lane keeps half of its values and adds
// the partner's copy of that half, so N values cost about N shuffles in all
// rather than N per bit.  On return v[0 .. N >> (BITEND - BIT)) (at least one)
// hold the sums of rows row0 + i.
template <int N, int BIT, int BITEND> struct HalvingReduce {
    __device__ __forceinline__ static void run(float *v, int lane, int &row0) {
        if constexpr (BIT < BITEND && N > 1) {
            constexpr int H = N / 2;
            const bool up = (lane >> BIT) & 1;
#pragma unroll
            for (int i = 0; i < H; i++) {
                const float keep = up ? v[i + H] : v[i];
                const float send = up ? v[i] : v[i + H];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << BIT);
            }
            if (up) row0 += H;
            HalvingReduce<H, BIT + 1, BITEND>::run(v, lane, row0);
        } else if constexpr (BIT < BITEND) {
#pragma unroll
            for (int b = BIT; b < BITEND; b++) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1 << b);
        }
    }
};

constexpr int ilog2c(int v) { return v <= 1 ? 0 : 1 + ilog2c(v / 2); }

template <int R, int T2C, typename T, bool DEBUG_OUT, bool NV>
__global__ void __launch_bounds__(1024) spectre_rows_inv_ln_reg(RowsInvArgs a) {
    constexpr int NF = R / 2 + 1;
    constexpr bool P16 = std::is_same<T, __nv_bfloat16>::value;  // bf16 I/O: fp16 P
    extern __shared__ float4 smem_f4[];
    // per-warp partial sums as [T2C * R rows][nwarps + 1] (the pad keeps both
    // the per-warp writes and the per-row reads on distinct banks), then
    // stat[2][T2C][R]
    float *part = reinterpret_cast<float *>(smem_f4);
    const int nthr = blockDim.x;
    const int nwarps = nthr >> 5;
    const int PS = nwarps + 1;
    float *stat = part + T2C * R * PS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tl = tid & (T2C - 1), cp = tid / T2C;
    const int b = blockIdx.y;
    const int t2 = blockIdx.x * T2C + tl;
    const int c0 = 2 * cp;
    const bool live = (t2 < a.M) && (c0 < a.C);
    const bool has1 = live && (c0 + 1 < a.C);
    float z0[R], z1[R];
    {
        float2 Z[R];
        // fp32 P: slices (c0, f1) and (c0 + 1, f1); fp16 P: the pair's slice,
        // one 8-byte load for both channels
        const int cc = live ? c0 : 0, tt = live ? t2 : 0;
        const size_t sa = P16 ? p16_pair_slice(b, cc, 0, a.C, NF) : ((size_t)b * a.C + cc) * NF;
        const size_t pofs = sa * a.M + tt;
        const int fstride = a.M, cstride = NF * a.M;
        auto ld2 = [&](int f1, float2 &pa, float2 &pb) {
            pa = pb = make_float2(0.f, 0.f);
            if (!live) return;
            if constexpr (P16) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(a.P) + pofs + f1 * fstride);
                const float2 sc = __ldg(reinterpret_cast<const float2 *>(a.pscale) + sa + f1);
                pa = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.x)), sc.x);
                if (has1) pb = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.y)), sc.y);
            } else {
                const float2 *p = static_cast<const float2 *>(a.P) + pofs;
                pa = __ldg(p + f1 * fstride);
                if (has1) pb = __ldg(p + cstride + f1 * fstride);
            }
        };
        float2 a0, aN, b0, bN;
        ld2(0, a0, b0);
        ld2(R / 2, aN, bN);
        Z[0] = make_float2(a0.x, -b0.x);
        Z[R / 2] = make_float2(aN.x, -bN.x);
#pragma unroll
        for (int f1 = 1; f1 < R / 2; f1++) {
            float2 pv, qv;
            ld2(f1, pv, qv);
            Z[f1] = make_float2(pv.x - qv.y, -(pv.y + qv.x));
            Z[R - f1] = make_float2(pv.x + qv.y, pv.y - qv.x);
        }
        Dft<R>::run(Z);
#pragma unroll
        for (int t1 = 0; t1 < R; t1++) {
            z0[t1] = Z[t1].x;
            z1[t1] = -Z[t1].y;
        }
    }
    const T *x = static_cast<const T *>(a.x);
    const size_t tok0 = (size_t)b * a.L + (live ? t2 : 0);
    const int rowstep = a.M * a.C;                      // elements between t1 rows
    const T *xp = x + tok0 * a.C + (live ? c0 : 0);
    const bool pre = NV && (a.norm & 1), rms = NV && ((a.norm >> 1) & 1);   // residual after the norm; RMSNorm
    float s[R];
#pragma unroll
    for (int t1 = 0; t1 < R; t1++) {
        if (DEBUG_OUT && live) {
            float *op = a.out_f32 + tok0 * a.C + c0 + t1 * rowstep;
            if (has1 && a.vec2)
                *reinterpret_cast<float2 *>(op) = make_float2(z0[t1], z1[t1]);
            else {
                op[0] = z0[t1];
                if (has1) op[1] = z1[t1];
            }
        }
        if (pre) {
            z0[t1] = live ? z0[t1] : 0.f;
            z1[t1] = has1 ? z1[t1] : 0.f;
        } else if (has1 && a.vec2) {
            float2 xv = Elem<T>::load2(xp + t1 * rowstep);
            z0[t1] += xv.x;
            z1[t1] += xv.y;
        } else {
            z0[t1] = live ? z0[t1] + Elem<T>::load(xp + t1 * rowstep) : 0.f;
            z1[t1] = has1 ? z1[t1] + Elem<T>::load(xp + t1 * rowstep + 1) : 0.f;
        }
        s[t1] = rms ? fmaf(z0[t1], z0[t1], z1[t1] * z1[t1]) : z0[t1] + z1[t1];
    }
    const float invC = 1.0f / (float)a.C;
    // two reductions over the channels of each row: sum(z), then sum((z - mean)^2)
    // (RMSNorm: one, sum(z^2)); stat[0][.] holds the means (0 for RMSNorm),
    // stat[1][.] the reciprocal standard deviations
    const int npass = rms ? 1 : 2;
#pragma unroll 1
    for (int pass = 0; pass < npass; pass++) {
        if (pass == 1) {
#pragma unroll
            for (int t1 = 0; t1 < R; t1++) {
                const float mu = stat[tl * R + t1];
                float d0 = z0[t1] - mu, d1 = z1[t1] - mu;
                s[t1] = live ? fmaf(d0, d0, has1 ? d1 * d1 : 0.f) : 0.f;
            }
        }
        {
            // channel pairs of one t2 differ in lane bits [log2 T2C, 5)
            constexpr int B0 = ilog2c(T2C);
            constexpr int NOUT = (R >> (5 - B0)) > 0 ? (R >> (5 - B0)) : 1;
            float v[R];
#pragma unroll
            for (int t1 = 0; t1 < R; t1++) v[t1] = s[t1];
            int row0 = 0;
            HalvingReduce<R, B0, 5>::run(v, lane, row0);
#pragma unroll
            for (int i = 0; i < NOUT; i++) part[(tl * R + row0 + i) * PS + warp] = v[i];
        }
        __syncthreads();
        // a warp per row sums the row's per-warp partials (lane w: warp w's,
        // w < nwarps <= 32), in a fixed order
        for (int i = warp; i < T2C * R; i += nwarps) {
            float acc = lane < nwarps ? part[i * PS + lane] : 0.f;
            acc = warp_sum(acc) * invC;
            if (lane == 0) {
                if (rms) {
                    stat[i] = 0.f;
                    stat[T2C * R + i] = rsqrtf(acc + a.eps);
                } else {
                    stat[pass * T2C * R + i] = pass == 0 ? acc : rsqrtf(acc + a.eps);
                }
            }
        }
        __syncthreads();
    }
    T *y = static_cast<T *>(a.y);
    T *yp = y + tok0 * a.C + c0;
    const float g0 = live ? __ldg(a.gamma + c0) : 0.f, be0 = live ? __ldg(a.beta + c0) : 0.f;
    const float g1 = has1 ? __ldg(a.gamma + c0 + 1) : 0.f, be1 = has1 ? __ldg(a.beta + c0 + 1) : 0.f;
#pragma unroll
    for (int t1 = 0; t1 < R; t1++) {
        const float mu = stat[tl * R + t1];
        const float rstd = stat[T2C * R + tl * R + t1];
        float y0 = fmaf((z0[t1] - mu) * rstd, g0, be0);
        float y1 = fmaf((z1[t1] - mu) * rstd, g1, be1);
        if (pre) {
            if (has1 && a.vec2) {
                const float2 xv = Elem<T>::load2(xp + t1 * rowstep);
                y0 += xv.x;
                y1 += xv.y;
            } else {
                if (live) y0 += Elem<T>::load(xp + t1 * rowstep);
                if (has1) y1 += Elem<T>::load(xp + t1 * rowstep + 1);
            }
        }
        if (has1 && a.vec2) {
            Elem<T>::store2(yp + t1 * rowstep, y0, y1);
        } else if (live) {
            Elem<T>::store(yp + t1 * rowstep, y0);
            if (has1) Elem<T>::store(yp + t1 * rowstep + 1, y1);
        }
    }
}

// ---------------------------------------------------------------------------
// inverse row pass + residual + LayerNorm, prefetching variant (R = 16,
// bf16 I/O with fp16 P, C a multiple of 8, C <= 512).  A persistent block of
// 2 x CP threads (thread = tl + 2 cp: one of two token columns t2, one channel
// pair) walks pairs of columns; while it inverts and normalises one pair from
// a shared-memory stage, cp.async copies the next pair's P (per channel pair
// and f1, both columns' two fp16 complex values: 16 contiguous bytes) and its
// 2 x 16 rows of x into the other stage, so no register holds data in
// flight.  The x rows are padded by 32 values so the two columns' rows fall
// on different banks.  The arithmetic per column is that of
// spectre_rows_inv_ln_reg with T2C = 2.
// ---------------------------------------------------------------------------
constexpr int kInvPipeMaxC = 512;
constexpr uint32_t kInvWaitLimit = 1u << 12;   // polls of up to 1 ms each

// shared-memory words of one stage: P [NF][CP][T2C columns] as uint2 (the
// pair's two half2), then x [16 rows][T2C columns][C + 32] bf16
__host__ __device__ inline int inv_pipe_stage_words(int C, int T2C) {
    return 9 * (C / 2) * T2C * 2 + 16 * T2C * (C + 32) / 2;
}

// Before a 16-byte or 8-byte cp.async of P: T2C = 2 takes both columns of a
// pair slice in one 16-byte piece, T2C = 1 its one column's 8 bytes.
__device__ __forceinline__ void cp_async8(void *smem_dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;"
                 :
                 : "r"((uint32_t)__cvta_generic_to_shared(smem_dst)), "l"(src)
                 : "memory");
}

// T2C token columns per group: 2 (blocks of C threads, one per SM) or 1
// (blocks of C / 2 threads, two per SM, so one block's LayerNorm barriers
// overlap the other block's work)
template <bool DEBUG_OUT, bool NV, int T2C>
__global__ void __launch_bounds__(kInvPipeMaxC * T2C / 2, 2 / T2C) spectre_rows_inv_ln_pipe(RowsInvArgs a) {
    constexpr int R = 16, NF = R / 2 + 1;
    extern __shared__ float4 smem_f4[];
    const int C = a.C, CP = C / 2, XS = C + 32;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int stage_words = inv_pipe_stage_words(C, T2C);
    uint32_t *stage0 = reinterpret_cast<uint32_t *>(smem_f4);
    // per-warp partial sums as [T2C * R rows][nwarps + 1] (padded: distinct
    // banks for the writes and the per-row reads), then stat[2][T2C][R]
    const int PS = nwarps + 1;
    float *part = reinterpret_cast<float *>(stage0 + 2 * stage_words);
    float *stat = part + T2C * R * PS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tl = tid & (T2C - 1), cp = tid / T2C, c0 = 2 * cp;
    const bool live = cp < CP;
    const int npair_cols = a.M / T2C;
    const int ngroups = a.B * npair_cols;   // < 2^31 (checked by the launcher)
    const uint4 *P4 = static_cast<const uint4 *>(a.P);       // one uint4 = 2 columns of a pair
    const float2 *ps2 = reinterpret_cast<const float2 *>(a.pscale);
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(a.x);
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(a.y);
    const int rowstep = a.M * C;
    // one mbarrier per stage for its x rows (bulk copies)
    uint64_t *xbar = reinterpret_cast<uint64_t *>(stat + 2 * T2C * R);
    if (tid == 0) {
        tc::mbar_init(tc::smem_u32(xbar), 1);
        tc::mbar_init(tc::smem_u32(xbar + 1), 1);
    }
    __syncthreads();
    const uint32_t xrow_bytes = (uint32_t)C * 2;

    // P: 16-byte cp.async pieces (per channel pair and f1: both columns' two
    // fp16 complex values); x: the stage's 2 x 16 token rows, one bulk copy
    // of C bf16 per row, issued by the lanes of warp 0
    auto prefetch = [&](int grp, int st) {
        const int b = grp / npair_cols, t2 = (grp - b * npair_cols) * T2C;
        uint32_t *pst = stage0 + st * stage_words;
        uint32_t *xst = pst + NF * CP * 2 * T2C;
        for (int i = tid; i < NF * CP; i += nthr) {            // i = f1 * CP + pair
            const int f1 = (int)fdiv((uint32_t)i, a.fd_cp), pr = i - f1 * CP;
            const size_t slice = ((size_t)b * CP + pr) * NF + f1;
            if constexpr (T2C == 2)
                cp_async16(pst + 4 * i, P4 + (slice * a.M + t2) / 2);
            else
                cp_async8(pst + 2 * i, static_cast<const uint2 *>(a.P) + slice * a.M + t2);
        }
        if (warp == 0) {
            const uint32_t mb = tc::smem_u32(xbar + st);
            if (lane == 0) tc::mbar_arrive_expect_tx(mb, R * T2C * xrow_bytes);
            __syncwarp();
            if (lane < R * T2C) {
                const int t1 = lane / T2C, col = lane & (T2C - 1);   // lane = row t1 T2C + col
                const __nv_bfloat16 *src = x + ((size_t)b * a.L + t2 + col + (size_t)t1 * a.M) * C;
                tc::bulk_copy_g2s(tc::smem_u32(xst + lane * (XS / 2)), src, xrow_bytes, mb);
            }
        }
    };

    const float g0 = live ? __ldg(a.gamma + c0) : 0.f, be0 = live ? __ldg(a.beta + c0) : 0.f;
    const float g1 = live ? __ldg(a.gamma + c0 + 1) : 0.f, be1 = live ? __ldg(a.beta + c0 + 1) : 0.f;
    const float invC = 1.0f / (float)C;
    const bool pre = NV && (a.norm & 1), rms = NV && ((a.norm >> 1) & 1);   // residual after the norm; RMSNorm
    int grp = blockIdx.x;
    if (grp < ngroups) prefetch(grp, 0);
    cp_async_commit();
    bool late = false;      // a bounded wait for x rows gave up
    int done = grp;         // first group not finished
    int nissued = grp < ngroups ? 1 : 0;   // x fills issued / waited for (fill n: stage n & 1, phase (n >> 1) & 1)
    int nwaited = 0;
#pragma unroll 1
    for (int k = 0; grp < ngroups; k++, grp += gridDim.x) {
        const int nxt = grp + gridDim.x;
        if (nxt < ngroups) {
            prefetch(nxt, (k + 1) & 1);
            nissued++;
        }
        cp_async_commit();
        cp_async_wait1();
        if (tc::mbar_wait(tc::smem_u32(xbar + (k & 1)), (k >> 1) & 1, kInvWaitLimit)) nwaited++;
        else late = true;
        if (__syncthreads_or(late)) break;
        const uint32_t *pst = stage0 + (k & 1) * stage_words;
        const uint32_t *xst = pst + NF * CP * 2 * T2C;
        const int b = grp / npair_cols, t2 = (grp - b * npair_cols) * T2C + tl;
        float z0[R], z1[R], s[R];
        {
            float2 Z[R];
            const size_t sa = ((size_t)b * CP + (live ? cp : 0)) * NF;
            auto ld2 = [&](int f1, float2 &pa, float2 &pb) {
                pa = pb = make_float2(0.f, 0.f);
                if (!live) return;
                const uint2 u = reinterpret_cast<const uint2 *>(pst)[(f1 * CP + cp) * T2C + tl];
                const float2 sc = __ldg(ps2 + sa + f1);
                pa = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.x)), sc.x);
                pb = cscale(__half22float2(*reinterpret_cast<const __half2 *>(&u.y)), sc.y);
            };
            float2 a0, aN, b0, bN;
            ld2(0, a0, b0);
            ld2(R / 2, aN, bN);
            Z[0] = make_float2(a0.x, -b0.x);
            Z[R / 2] = make_float2(aN.x, -bN.x);
#pragma unroll
            for (int f1 = 1; f1 < R / 2; f1++) {
                float2 pv, qv;
                ld2(f1, pv, qv);
                Z[f1] = make_float2(pv.x - qv.y, -(pv.y + qv.x));
                Z[R - f1] = make_float2(pv.x + qv.y, pv.y - qv.x);
            }
            Dft<R>::run(Z);
            const size_t tok0 = (size_t)b * a.L + t2;
#pragma unroll
            for (int t1 = 0; t1 < R; t1++) {
                z0[t1] = Z[t1].x;
                z1[t1] = -Z[t1].y;
                if (DEBUG_OUT && live)
                    *reinterpret_cast<float2 *>(a.out_f32 + (tok0 + (size_t)t1 * a.M) * C + c0) =
                        make_float2(z0[t1], z1[t1]);
                const uint32_t xw = (live && !pre) ? xst[(t1 * T2C + tl) * (XS / 2) + cp] : 0u;
                const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xw));
                z0[t1] = live ? z0[t1] + xv.x : 0.f;
                z1[t1] = live ? z1[t1] + xv.y : 0.f;
                s[t1] = rms ? fmaf(z0[t1], z0[t1], z1[t1] * z1[t1]) : z0[t1] + z1[t1];
            }
        }
        // statistics of the 2 x R token rows: mean, then mean squared
        // deviation (RMSNorm: the mean square alone)
#pragma unroll 1
        for (int pass = 0; pass < (rms ? 1 : 2); pass++) {
            if (pass == 1) {
#pragma unroll
                for (int t1 = 0; t1 < R; t1++) {
                    const float mu = stat[tl * R + t1];
                    const float d0 = z0[t1] - mu, d1 = z1[t1] - mu;
                    s[t1] = live ? fmaf(d0, d0, d1 * d1) : 0.f;
                }
            }
            {
                // channel pairs of one column differ in lane bits [log2 T2C, 5)
                float v[R];
#pragma unroll
                for (int t1 = 0; t1 < R; t1++) v[t1] = s[t1];
                int row0 = 0;
                HalvingReduce<R, (T2C == 2 ? 1 : 0), 5>::run(v, lane, row0);
                part[(tl * R + row0) * PS + warp] = v[0];
            }
            __syncthreads();
            for (int i = warp; i < T2C * R; i += nwarps) {
                float acc = lane < nwarps ? part[i * PS + lane] : 0.f;
                acc = warp_sum(acc) * invC;
                if (lane == 0) {
                    if (rms) {
                        stat[i] = 0.f;
                        stat[T2C * R + i] = rsqrtf(acc + a.eps);
                    } else {
                        stat[pass * T2C * R + i] = pass == 0 ? acc : rsqrtf(acc + a.eps);
                    }
                }
            }
            __syncthreads();
        }
        if (live) {
            __nv_bfloat16 *yp = y + ((size_t)b * a.L + t2) * C + c0;
#pragma unroll
            for (int t1 = 0; t1 < R; t1++) {
                const float mu = stat[tl * R + t1], rstd = stat[T2C * R + tl * R + t1];
                float y0 = fmaf((z0[t1] - mu) * rstd, g0, be0);
                float y1 = fmaf((z1[t1] - mu) * rstd, g1, be1);
                if (pre) {   // the residual, still in this stage
                    const uint32_t xw = xst[(t1 * T2C + tl) * (XS / 2) + cp];
                    const float2 xv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&xw));
                    y0 += xv.x;
                    y1 += xv.y;
                }
                Elem<__nv_bfloat16>::store2(yp + t1 * rowstep, y0, y1);
            }
        }
        // every read of this stage and of stat is done before the stage is refilled
        __syncthreads();
        done = grp + gridDim.x;
    }
    cp_async_wait_all();
    if (__syncthreads_or(late)) {
        // a copy that never arrived: report it, let this block's own copies
        // land (bounded), and make y of the groups it did not finish NaN
        if (tid == 0) {
            if (a.err) atomicOr(a.err, 1);
            for (int n = nwaited; n < nissued; n++)
                tc::mbar_wait(tc::smem_u32(xbar + (n & 1)), (n >> 1) & 1, kInvWaitLimit);
        }
        for (int g = done; g < ngroups; g += gridDim.x) {
            const int b = g / npair_cols, t2 = (g - b * npair_cols) * T2C + tl;
            if (!live) continue;
            for (int t1 = 0; t1 < R; t1++)
                *reinterpret_cast<uint32_t *>(y + ((size_t)b * a.L + t2 + (size_t)t1 * a.M) * C + c0) = 0x7fc07fc0u;
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int R>
static cudaError_t rows_fwd_R(int dtype, const RowsFwdArgs &a0, cudaStream_t s) {
    if (R == 16 && dtype == 1 && a0.row_tc && rows_tc_applies(a0)) return launch_rows_fwd_tc(a0, s);
    const long long pipe_items = 3LL * (a0.M / 8) * (a0.Cw / 64) * a0.B;
    if (R == 16 && dtype == 1 && a0.vec2 && a0.C % 8 == 0 && a0.c_lo % 64 == 0 && a0.Cw % 64 == 0 &&
        a0.M % 8 == 0 && pipe_items < (1LL << 31)) {
        RowsFwdArgs a = a0;
        a.fd3 = make_fastdiv(3);
        a.fd_ntg = make_fastdiv((uint32_t)(a.M / 8));
        a.fd_ncg = make_fastdiv((uint32_t)(a.Cw / 64));
        const size_t smem = (size_t)2 * kFwdPipeStage * 4;
        auto k = a.a16 ? spectre_rows_fwd_pipe<true> : spectre_rows_fwd_pipe<false>;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        if (per_sm > SPECTRE_ROW_CTAS_PER_SM) per_sm = SPECTRE_ROW_CTAS_PER_SM;
        const long long cap = (long long)per_sm * (a.nsm > 0 ? a.nsm : 148);
        prefer_max_smem(k);
        k<<<(unsigned)(pipe_items < cap ? pipe_items : cap), 256, smem, s>>>(a);
        return cudaGetLastError();
    }
    dim3 grid((a0.M + 7) / 8, (a0.Cw + 63) / 64, a0.B);
    if (dtype == 0)
        a0.a16 ? spectre_rows_fwd<R, float, true><<<grid, 256, 0, s>>>(a0)
               : spectre_rows_fwd<R, float, false><<<grid, 256, 0, s>>>(a0);
    else
        a0.a16 ? spectre_rows_fwd<R, __nv_bfloat16, true><<<grid, 256, 0, s>>>(a0)
               : spectre_rows_fwd<R, __nv_bfloat16, false><<<grid, 256, 0, s>>>(a0);
    return cudaGetLastError();
}

cudaError_t launch_rows_fwd(int R, int dtype, const RowsFwdArgs &a, cudaStream_t s) {
    switch (R) {
    case 4: return rows_fwd_R<4>(dtype, a, s);
    case 8: return rows_fwd_R<8>(dtype, a, s);
    case 16: return rows_fwd_R<16>(dtype, a, s);
    case 64: return rows_fwd_R<64>(dtype, a, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int M>
static cudaError_t slices_M(const SliceArgs &a, cudaStream_t s) {
    using Cfg = SliceCfg<M>;
    size_t smem = (size_t)Cfg::SMEM;
    long long nblk = (a.nslices + Cfg::SPB - 1) / Cfg::SPB;
    auto k = spectre_slices<M, false>;
    if constexpr (Cfg::PROD != kProdGlobal) {
        if (a.a16) k = spectre_slices<M, true>;
    } else {
        if (a.a16) return cudaErrorInvalidValue;   // the product is parked in fp32 A
    }
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<(unsigned)nblk, Cfg::THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

template <int M> static void slice_geom_M(int *nt, int *spb, size_t *smem) {
    using Cfg = SliceCfg<M>;
    *nt = Cfg::NT;
    *spb = Cfg::SPB;
    *smem = (size_t)Cfg::SMEM;
}

#define SPECTRE_SLICE_LENGTHS(X)                                                              \
    X(1) X(2) X(4) X(8) X(16) X(32) X(64) X(128) X(256) X(512) X(1024) X(2048) X(4096)     \
    X(8192) X(16384) X(3) X(6) X(12) X(24) X(48) X(96) X(192) X(384) X(768) X(1536) X(3072) \
    X(6144) X(12288)

cudaError_t launch_slices(const SliceArgs &a, cudaStream_t s) {
    if (a.M == 4096 && a.use_mma) return launch_slices_mma4096(a, s);
    switch (a.M) {
#define X(m) case m: return slices_M<m>(a, s);
        SPECTRE_SLICE_LENGTHS(X)
#undef X
    default: return cudaErrorInvalidValue;
    }
}

template <int M> static bool parks_M() { return SliceCfg<M>::PROD == kProdGlobal; }

bool slice_parks_in_A(int M) {
    switch (M) {
#define X(m) case m: return parks_M<m>();
        SPECTRE_SLICE_LENGTHS(X)
#undef X
    default: return false;
    }
}

bool slice_length_supported(int M) {
    switch (M) {
#define X(m) case m: return true;
        SPECTRE_SLICE_LENGTHS(X)
#undef X
    default: return false;
    }
}

void slice_geometry(int M, int *nt, int *spb, size_t *smem) {
    *nt = 0;
    *spb = 0;
    *smem = 0;
    switch (M) {
#define X(m) case m: slice_geom_M<m>(nt, spb, smem); break;
        SPECTRE_SLICE_LENGTHS(X)
#undef X
    default: break;
    }
}

template <int R, typename T, bool NV>
static cudaError_t rows_inv_RTV(const RowsInvArgs &a, cudaStream_t s);

// NV selects the build of each inverse kernel that handles the norm variants
template <int R, typename T>
static cudaError_t rows_inv_RT(const RowsInvArgs &a, cudaStream_t s) {
    return a.norm != 0 ? rows_inv_RTV<R, T, true>(a, s) : rows_inv_RTV<R, T, false>(a, s);
}

template <int R, typename T, bool NV>
static cudaError_t rows_inv_RTV(const RowsInvArgs &a, cudaStream_t s) {
    if constexpr (R == 16 && std::is_same<T, __nv_bfloat16>::value) {
        constexpr int T2C = SPECTRE_INV_COLS;
        if (a.reg_variant && a.C % 8 == 0 && a.C <= kInvPipeMaxC && a.M % T2C == 0 &&
            (long long)a.B * (a.M / T2C) < (1LL << 31)) {
            const int threads = ((T2C * (a.C / 2) + 31) / 32) * 32;   // T2C columns x C / 2 pairs
            const size_t smem =
                ((size_t)2 * inv_pipe_stage_words(a.C, T2C) + (threads / 32 + 1) * 16 * T2C + 32 * T2C + 4) * 4;
            auto k = a.out_f32 ? spectre_rows_inv_ln_pipe<true, NV, T2C> : spectre_rows_inv_ln_pipe<false, NV, T2C>;
            cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            prefer_max_smem(k);
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, smem) != cudaSuccess ||
                per_sm < 1)
                per_sm = 1;
            const long long ngroups = (long long)a.B * (a.M / T2C);
            const long long cap = (long long)per_sm * (a.nsm > 0 ? a.nsm : 148);
            RowsInvArgs ap = a;
            ap.fd_cp = make_fastdiv((uint32_t)(a.C / 2));
            k<<<(unsigned)(ngroups < cap ? ngroups : cap), threads, smem, s>>>(ap);
            return cudaGetLastError();
        }
    }
    if constexpr (R <= 16) if (a.reg_variant) {
        dim3 grid((a.M + a.T2C - 1) / a.T2C, a.B);
        const int CP = (a.C + 1) / 2;
        const int threads = ((a.T2C * CP + 31) / 32) * 32;
        size_t smem = (size_t)((threads / 32 + 1) * a.T2C * R + 2 * a.T2C * R) * sizeof(float);
        switch (a.T2C) {
#define SPECTRE_INV_T2C(t2c)                                                              \
    case t2c:                                                                             \
        if (a.out_f32)                                                                    \
            spectre_rows_inv_ln_reg<R, t2c, T, true, NV><<<grid, threads, smem, s>>>(a);  \
        else                                                                              \
            spectre_rows_inv_ln_reg<R, t2c, T, false, NV><<<grid, threads, smem, s>>>(a); \
        break;
            SPECTRE_INV_T2C(1) SPECTRE_INV_T2C(2) SPECTRE_INV_T2C(4) SPECTRE_INV_T2C(8)
#undef SPECTRE_INV_T2C
        default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    dim3 grid((a.M + a.T2C - 1) / a.T2C, a.B);
    size_t smem = (size_t)R * a.T2C * a.ZS * sizeof(float);
    if (a.out_f32) {
        auto k = spectre_rows_inv_ln<R, T, true, NV>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 512, smem, s>>>(a);
    } else {
        auto k = spectre_rows_inv_ln<R, T, false, NV>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 512, smem, s>>>(a);
    }
    return cudaGetLastError();
}

template <int R>
static cudaError_t rows_inv_R(int dtype, const RowsInvArgs &a, cudaStream_t s) {
    return dtype == 0 ? rows_inv_RT<R, float>(a, s) : rows_inv_RT<R, __nv_bfloat16>(a, s);
}

cudaError_t launch_rows_inv_ln(int R, int dtype, const RowsInvArgs &a, cudaStream_t s) {
    switch (R) {
    case 4: return rows_inv_R<4>(dtype, a, s);
    case 8: return rows_inv_R<8>(dtype, a, s);
    case 16: return rows_inv_R<16>(dtype, a, s);
    case 64: return rows_inv_R<64>(dtype, a, s);
    default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------------------
// Fixed scratch for the entry point that allocates nothing.  The array lives
// in this module's global memory on every device that loads the library, from
// module load until process exit.  Host code reaches it only through the
// address cudaGetSymbolAddress returns for the current device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices];
}  // namespace

cudaError_t noalloc_scratch(void **ptr) {
    *ptr = nullptr;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        // once per device, with that device current: the scratch's device
        // address and the 64-point constant twiddles the R = 64 kernels use
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        float2 w64[64];
        for (int i = 0; i < 64; i++) {
            double ang = -2.0 * 3.14159265358979323846 * i / 64.0;
            w64[i] = make_float2((float)cos(ang), (float)sin(ang));
        }
        e = upload_w64(w64);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = addr;
    }
    *ptr = g_scratch_addr[dev];
    return cudaSuccess;
}

// Twiddle tables computed on the device (fp64 sincospi, stored fp32), in the
// layout spectre_mix_create builds on the host.
__global__ void spectre_make_tables(float2 *base, TableSegs segs) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    for (int sgi = 0; sgi < segs.n; sgi++) {
        const TableSeg &g = segs.seg[sgi];
        if (i < g.count) {
            if (g.ns == -1) {
                // slot i: bytes 8 i .. 8 i + 7 of the DFT-64 operand, four
                // K-consecutive fp16 values of one row
                const int byte = 8 * (int)i;
                const int n = (byte / 2048) * 8 + (byte % 128) / 16;
                const int k0 = ((byte % 2048) / 128) * 8 + (byte % 16) / 2;
                __half hv[4];
                for (int u = 0; u < 4; u++) {
                    long long e;
                    int part;
                    dft64_operand_angle(n, k0 + u, &e, &part);
                    double sn, cs;
                    sincospi(-2.0 * (double)e / 64.0, &sn, &cs);
                    const double val = (part == 0 || part == 3) ? cs : (part == 1 ? -sn : sn);
                    hv[u] = __float2half_rn((float)(val / 64.0));
                }
                float2 slot;
                memcpy(&slot, hv, sizeof(slot));
                base[g.offset + i] = slot;
                return;
            }
            long long e;
            if (g.ns == 0) {
                e = i;                                   // w_N^i
            } else {
                long long rr = i / g.ns, kk = i % g.ns;  // entry r * ns + k
                e = kk * rr;
            }
            double sn, cs;
            sincospi(-2.0 * (double)(e % g.N) / (double)g.N, &sn, &cs);
            base[g.offset + i] = make_float2((float)cs, (float)sn);
            return;
        }
        i -= g.count;
    }
}

cudaError_t launch_make_tables(float2 *base, const TableSegs &segs, cudaStream_t s) {
    long long total = 0;
    for (int i = 0; i < segs.n; i++) total += segs.seg[i].count;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    spectre_make_tables<<<(unsigned)((total + threads - 1) / threads), threads, 0, s>>>(base, segs);
    return cudaGetLastError();
}

cudaError_t upload_w64(const float2 *host64) {
    return cudaMemcpyToSymbol(c_w64, host64, 64 * sizeof(float2));
}

}  // namespace spectre
