// kernels.cu -- the three kernel families of the SPECTRE spectral mixer on
// sm_100a (SPECTRE walk-through, hotelren.com/news/5925787: §2.2 pseudocode,
// §2.3 truncation, §3.1 real/imaginary parts carried as separate reals).
//
//   spectre_rows_fwd    : q, k, v rows -> R-point real transforms -> A
//   spectre_slices<M>   : per (b, c, f1) slice: three M-point FFTs, the gated
//                         product, one inverse M-point FFT -> P
//   spectre_rows_inv_ln : P -> R-point inverse (real output) -> + x ->
//                         LayerNorm over C -> y
//
// The index algebra is in kernels.cuh.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>
#include <type_traits>

#include "fft_regs.cuh"
#include "kernels.cuh"

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

// ---------------------------------------------------------------------------
// row pass: A[sig][b][c][f1][t2] = w_L^{f1 t2} sum_{t1} w_R^{f1 t1} sig[b][t1 M + t2][c]
// Block: 256 threads = 8 warps over 8 t2 values x 32 channel pairs; a warp
// covers 4 consecutive t2 x 8 consecutive channel pairs, lane = tl + 4 cpl.
// Each thread owns channels c0 = 2 cp, c0 + 1 at one t2, packed as one complex
// signal c0 + i c1.  Its 16-row loads are 32-byte segments per warp-row
// (8 channel pairs) and its stores are 32-byte segments (4 consecutive t2) of
// A, straight from registers.
// ---------------------------------------------------------------------------
template <int R, typename T>
__global__ void __launch_bounds__(256, R <= 16 ? 4 : 1) spectre_rows_fwd(RowsFwdArgs a) {
    constexpr int NF = R / 2 + 1;
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
    float2 *dst0 = a.A + ((size_t)b * a.Cw + cl) * NF * a.M + t2;
    float2 *dst1 = dst0 + (size_t)NF * a.M;

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
                dst0[sig * plane + (size_t)f1 * a.M] = xa;
                if (has1) dst1[sig * plane + (size_t)f1 * a.M] = xb;
            }
        }
    }
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

template <int M> struct SliceCfg {
    static constexpr RadList S = make_schedule(M);
    static constexpr int NP = S.n;
    static constexpr int RL = NP > 0 ? S.r[NP - 1] : 1;   // largest radix, last
    static constexpr int R0 = NP > 0 ? S.r[0] : 1;
    static constexpr int NT = M / RL;                      // threads per slice
    static constexpr int SPB = NT >= 256 ? 1 : 256 / NT;   // slices per block
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
template <int M>
__device__ __forceinline__ void slice_forward(const float2 *__restrict__ src, bool live, float2 *buf,
                                              const SliceTables &tb, int j, float2 (&x)[SliceCfg<M>::RL]) {
    using Cfg = SliceCfg<M>;
    constexpr int NP = Cfg::NP, NT = Cfg::NT;
    if constexpr (NP == 0) {
        x[0] = live ? __ldg(src) : make_float2(0.f, 0.f);
    } else if constexpr (NP == 1) {
        constexpr int R = Cfg::RL;
#pragma unroll
        for (int r = 0; r < R; r++) x[r] = live ? __ldg(src + j + r * NT) : make_float2(0.f, 0.f);
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
                for (int r = 0; r < R; r++) v[r] = live ? __ldg(src + bf + r * NBF) : make_float2(0.f, 0.f);
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
    void *dst;        // slice base (float2 * or __half2 *)
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
        static_cast<__half2 *>(ps.dst)[t2] = __floats2half2_rn(v.x * s, v.y * s);
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

template <int M>
__global__ void __launch_bounds__(SliceCfg<M>::THREADS, SliceCfg<M>::MINB_C) spectre_slices(SliceArgs a) {
    using Cfg = SliceCfg<M>;
    constexpr int NT = Cfg::NT, RL = Cfg::RL, PROD = Cfg::PROD;
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
    const float2 *srcA = a.A + (size_t)bcl * NF * M + (size_t)f1 * M;
    const size_t pslice = ((size_t)b * a.C + c) * NF + f1;
    PStore ps;
    ps.dst = a.p16 ? static_cast<void *>(static_cast<__half2 *>(a.P) + pslice * M)
                   : static_cast<void *>(static_cast<float2 *>(a.P) + pslice * M);
    ps.pscale = a.pscale + pslice;
    ps.smax = &smax[sl];
    ps.live = live;
    ps.p16 = a.p16 != 0;
    const float *Gh = a.G + (size_t)h * a.nbins;
    __syncthreads();  // smax initialised

    float2 x[RL];
    float2 s[RL];
    // each thread owns bins f = f1 + R (j + r NT), r < RL, of the product;
    // with kProdGlobal S is parked in this slice's q row of A, which nothing
    // reads once the q transform has passed its first stage
    float2 *park = const_cast<float2 *>(srcA);
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
    slice_forward<M>(srcA, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) {
        int f = f1 + a.R * (j + r * NT);
        int ff = min(f, a.L - f);
        float g = (live && ff < a.F) ? __ldg(Gh + ff) * a.invL : 0.f;
        put(r, cscale(x[r], g));
    }
    if constexpr (Cfg::NP >= 2) __syncthreads();
    // k: S *= conj(K)
    slice_forward<M>(srcA + sig_stride, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) put(r, cmulc(get(r), x[r]));
    if constexpr (Cfg::NP >= 2) __syncthreads();
    // v: O = S * V
    slice_forward<M>(srcA + 2 * sig_stride, live, buf, a.tabs, j, x);
#pragma unroll
    for (int r = 0; r < RL; r++) x[r] = cmul(get(r), x[r]);
    slice_inverse_store<M>(x, buf, a.tabs, j, ps, a.twL, f1);
}

// ---------------------------------------------------------------------------
// inverse row pass + residual + LayerNorm
// ---------------------------------------------------------------------------
template <int R, typename T, bool DEBUG_OUT>
__global__ void __launch_bounds__(512) spectre_rows_inv_ln(RowsInvArgs a) {
    constexpr int NF = R / 2 + 1;
    constexpr bool P16 = std::is_same<T, __nv_bfloat16>::value;  // bf16 I/O: fp16 P
    extern __shared__ float4 smem_f4[];
    float *zbuf = reinterpret_cast<float *>(smem_f4);  // [R * T2C][ZS]
    const int T2C = a.T2C, ZS = a.ZS;
    const int b = blockIdx.y;
    const int t2base = blockIdx.x * T2C;
    const int CP = (a.C + 1) / 2;
    const int items = T2C * CP;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int tl = it % T2C, cp = it / T2C;
        const int t2 = t2base + tl;
        if (t2 >= a.M) continue;
        const int c0 = 2 * cp;
        const bool has1 = c0 + 1 < a.C;
        const size_t sa = ((size_t)b * a.C + c0) * NF;
        const size_t sb = sa + NF;
        auto ld = [&](size_t slice, bool ok) -> float2 {
            if (!ok) return make_float2(0.f, 0.f);
            if constexpr (P16) {
                float2 v = __half22float2(__ldg(static_cast<const __half2 *>(a.P) + slice * a.M + t2));
                return cscale(v, __ldg(a.pscale + slice));
            } else {
                return __ldg(static_cast<const float2 *>(a.P) + slice * a.M + t2);
            }
        };
        float2 Z[R];
        {
            float2 a0 = ld(sa, true), aN = ld(sa + R / 2, true);
            float2 b0 = ld(sb, has1);
            float2 bN = ld(sb + R / 2, has1);
            // DC and Nyquist: imaginary parts dropped; conj() for the inverse
            Z[0] = make_float2(a0.x, -b0.x);
            Z[R / 2] = make_float2(aN.x, -bN.x);
        }
#pragma unroll
        for (int f1 = 1; f1 < R / 2; f1++) {
            float2 pv = ld(sa + f1, true);
            float2 qv = ld(sb + f1, has1);
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
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y);
    const float invC = 1.0f / (float)a.C;
    for (int row = warp; row < R * T2C; row += nw) {
        const int t1 = row / T2C, tl = row % T2C;
        const int t2 = t2base + tl;
        if (t2 >= a.M) continue;
        const size_t tok = (size_t)b * a.L + (size_t)t1 * a.M + t2;
        const T *xr = x + tok * a.C;
        T *yr = y + tok * a.C;
        float *zr = zbuf + (size_t)row * ZS;
        float s = 0.f;
        for (int c = lane; c < a.C; c += 32) {
            float o = zr[c];
            if (DEBUG_OUT) a.out_f32[tok * a.C + c] = o;
            float z = o + Elem<T>::load(xr + c);
            zr[c] = z;
            s += z;
        }
        const float mean = warp_sum(s) * invC;
        float ss = 0.f;
        for (int c = lane; c < a.C; c += 32) {
            float d = zr[c] - mean;
            ss = fmaf(d, d, ss);
        }
        const float rstd = rsqrtf(warp_sum(ss) * invC + a.eps);
        for (int c = lane; c < a.C; c += 32)
            Elem<T>::store(yr + c, fmaf((zr[c] - mean) * rstd, __ldg(a.gamma + c), __ldg(a.beta + c)));
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

template <int R, int T2C, typename T, bool DEBUG_OUT>
__global__ void __launch_bounds__(1024) spectre_rows_inv_ln_reg(RowsInvArgs a) {
    constexpr int NF = R / 2 + 1;
    constexpr bool P16 = std::is_same<T, __nv_bfloat16>::value;  // bf16 I/O: fp16 P
    extern __shared__ float4 smem_f4[];
    float *part = reinterpret_cast<float *>(smem_f4);   // [nwarps][T2C][R], then stat[2][T2C][R]
    const int nthr = blockDim.x;
    const int nwarps = nthr >> 5;
    float *stat = part + nwarps * T2C * R;               // [T2C][R]
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
        const size_t sa = ((size_t)b * a.C + c0) * NF;       // slice index of (c0, f1 = 0)
        const size_t sb = sa + NF;
        auto ld = [&](size_t slice, bool ok) -> float2 {
            if (!ok) return make_float2(0.f, 0.f);
            if constexpr (P16) {
                float2 v = __half22float2(__ldg(static_cast<const __half2 *>(a.P) + slice * a.M + t2));
                return cscale(v, __ldg(a.pscale + slice));
            } else {
                return __ldg(static_cast<const float2 *>(a.P) + slice * a.M + t2);
            }
        };
        float2 a0 = ld(sa, live), aN = ld(sa + R / 2, live);
        float2 b0 = ld(sb, has1), bN = ld(sb + R / 2, has1);
        Z[0] = make_float2(a0.x, -b0.x);
        Z[R / 2] = make_float2(aN.x, -bN.x);
#pragma unroll
        for (int f1 = 1; f1 < R / 2; f1++) {
            float2 pv = ld(sa + f1, live);
            float2 qv = ld(sb + f1, has1);
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
    const size_t tok0 = (size_t)b * a.L + t2;
    const size_t rowstep = (size_t)a.M * a.C;
    const T *xp = x + tok0 * a.C + c0;
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
        if (has1 && a.vec2) {
            float2 xv = Elem<T>::load2(xp + t1 * rowstep);
            z0[t1] += xv.x;
            z1[t1] += xv.y;
        } else {
            z0[t1] = live ? z0[t1] + Elem<T>::load(xp + t1 * rowstep) : 0.f;
            z1[t1] = has1 ? z1[t1] + Elem<T>::load(xp + t1 * rowstep + 1) : 0.f;
        }
        s[t1] = z0[t1] + z1[t1];
    }
    const float invC = 1.0f / (float)a.C;
    // two reductions over the channels of each row: sum(z), then sum((z - mean)^2);
    // stat[0][.] holds the means, stat[1][.] the variances
#pragma unroll 1
    for (int pass = 0; pass < 2; pass++) {
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
            for (int i = 0; i < NOUT; i++) part[(warp * T2C + tl) * R + row0 + i] = v[i];
        }        __syncthreads();
        for (int i = tid; i < T2C * R; i += nthr) {
            float acc = 0.f;
            for (int w = 0; w < nwarps; w++) acc += part[w * T2C * R + i];
            stat[pass * T2C * R + i] = acc * invC;
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
        const float rstd = rsqrtf(stat[T2C * R + tl * R + t1] + a.eps);
        const float y0 = fmaf((z0[t1] - mu) * rstd, g0, be0);
        const float y1 = fmaf((z1[t1] - mu) * rstd, g1, be1);
        if (has1 && a.vec2) {
            Elem<T>::store2(yp + t1 * rowstep, y0, y1);
        } else if (live) {
            Elem<T>::store(yp + t1 * rowstep, y0);
            if (has1) Elem<T>::store(yp + t1 * rowstep + 1, y1);
        }
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int R>
static cudaError_t rows_fwd_R(int dtype, const RowsFwdArgs &a, cudaStream_t s) {
    dim3 grid((a.M + 7) / 8, (a.Cw + 63) / 64, a.B);
    if (dtype == 0)
        spectre_rows_fwd<R, float><<<grid, 256, 0, s>>>(a);
    else
        spectre_rows_fwd<R, __nv_bfloat16><<<grid, 256, 0, s>>>(a);
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
    auto k = spectre_slices<M>;
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

template <int R, typename T>
static cudaError_t rows_inv_RT(const RowsInvArgs &a, cudaStream_t s) {
    if constexpr (R <= 16) if (a.reg_variant) {
        dim3 grid((a.M + a.T2C - 1) / a.T2C, a.B);
        const int CP = (a.C + 1) / 2;
        const int threads = ((a.T2C * CP + 31) / 32) * 32;
        size_t smem = (size_t)((threads / 32) * a.T2C * R + 2 * a.T2C * R) * sizeof(float);
        switch (a.T2C) {
#define SPECTRE_INV_T2C(t2c)                                                          \
    case t2c:                                                                         \
        if (a.out_f32)                                                                \
            spectre_rows_inv_ln_reg<R, t2c, T, true><<<grid, threads, smem, s>>>(a);  \
        else                                                                          \
            spectre_rows_inv_ln_reg<R, t2c, T, false><<<grid, threads, smem, s>>>(a); \
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
        auto k = spectre_rows_inv_ln<R, T, true>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 512, smem, s>>>(a);
    } else {
        auto k = spectre_rows_inv_ln<R, T, false>;
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
