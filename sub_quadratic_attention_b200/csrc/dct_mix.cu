// dct_mix.cu -- per-token DCT mix with spectral-entropy routing (Chiaroscuro
// Attention summary, paper.rainbus.top/paper/2606.08327: "Prerequisites: DCT",
// "Prerequisites: spectral entropy", "Method step details"), and its C ABI.
//
// One warp transforms two token rows at once: row a in the real part and row b
// in the imaginary part of one d-point complex FFT.  The Type-II DCT of a row
// comes from the FFT of its even samples followed by its odd samples reversed
// (v[n] = x[2n], v[d-1-n] = x[2n+1]):  c_k = Re(exp(-i pi k / 2d) V_k), the
// unnormalised DCT, and X_k = s_k c_k.  The inverse runs the same steps back:
// V'_k = exp(i pi k / 2d) (g_k - i g_{d-k}) with g = c * w, an inverse FFT, and
// the even/odd interleave.  The FFT is a four-step split d = E * 32 held in
// registers: E-point DFTs down each lane's registers, a twiddle, and a 32-point
// DFT across the lanes as five radix-2 shuffle stages.  Every permutation (the
// even/odd reorder, the k <-> d-k pairing, the bit-reversed lane order) is a
// lane exchange, so the kernel uses no shared memory.  One pass over HBM: x
// read once (a second read for the residual hits L1/L2), y written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "dct_mix.h"
#include "fft_regs.cuh"

struct dct_mix_s {
    int d;
    int dtype;
    float eps;
    int device;
    int nsm;
    float2 *tables;   // twN[d] = exp(-2 pi i j / d), tq[d] = exp(-i pi k / (2d)), then the
                      // lane-major tables tl1[E][32], tl2[5][32], tl3[E][32] (E = d / 32)
    void *stage;      // dct_mix_run_host staging
    size_t stage_bytes;
};

namespace dctmix {

using spectre::cadd;
using spectre::cconj;
using spectre::cmul;
using spectre::csub;

struct Args {
    long long T;
    const void *x;
    const float *w, *gamma, *beta;
    float tau, eps;
    void *y;
    float *H;
    unsigned char *route;
    float *mix;
    const float2 *twN;
    const float2 *tq;
    // lane-major copies, so that a warp's table load is one contiguous 256-byte
    // access: tl1[k][l] = w_N^{l k}; tl2[s][l] = the lane-stage twiddle
    // w_{2h}^{l mod h} of stage h = 16 >> s; tl3[k][l] = tq[k + E brev5(l)]
    const float2 *tl1, *tl2, *tl3;
};

template <typename T> struct Row;
template <> struct Row<float> {
    __device__ __forceinline__ static float2 load2(const float *p) {
        return __ldg(reinterpret_cast<const float2 *>(p));
    }
    __device__ __forceinline__ static void store2(float *p, float a, float b) {
        *reinterpret_cast<float2 *>(p) = make_float2(a, b);
    }
};
template <> struct Row<__nv_bfloat16> {
    __device__ __forceinline__ static float2 load2(const __nv_bfloat16 *p) {
        const unsigned int u = __ldg(reinterpret_cast<const unsigned int *>(p));
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
    }
    __device__ __forceinline__ static void store2(__nv_bfloat16 *p, float a, float b) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
    }
};

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float2 shfl_xor2(float2 v, int m) {
    return make_float2(__shfl_xor_sync(kFull, v.x, m), __shfl_xor_sync(kFull, v.y, m));
}
__device__ __forceinline__ float2 shfl2(float2 v, int src) {
    return make_float2(__shfl_sync(kFull, v.x, src), __shfl_sync(kFull, v.y, src));
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Unscaled forward DFT of length E down one lane's registers, natural order.
template <int E> struct RegDft {
    __device__ __forceinline__ static void run(float2 (&v)[E], const float2 *) {
        spectre::Dft<E>::run(v);
    }
};
// E = 32: one radix-2 decimation-in-frequency step, a[i] = v[i] + v[i+16]
// and b[i] = (v[i] - v[i+16]) w_32^i, then 16-point DFTs of a (the even
// outputs) and b (the odd ones).  w_32^i = twN[32 i] of the d = 1024 table.
template <> struct RegDft<32> {
    __device__ __forceinline__ static void run(float2 (&v)[32], const float2 *twN) {
        float2 a[16], b[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            a[i] = cadd(v[i], v[i + 16]);
            const float2 t = csub(v[i], v[i + 16]);
            b[i] = i == 0 ? t : cmul(t, __ldg(twN + 32 * i));
        }
        spectre::Dft<16>::run(a);
        spectre::Dft<16>::run(b);
#pragma unroll
        for (int m = 0; m < 16; m++) {
            v[2 * m] = a[m];
            v[2 * m + 1] = b[m];
        }
    }
};

// Forward N-point FFT of the warp's N values.  On entry lane l, register r
// holds z[l + 32 r]; on exit it holds Z[r + E * brev5(l)].
template <int N>
__device__ __forceinline__ void fft_forward(float2 (&v)[N / 32], int lane, const Args &a) {
    constexpr int E = N / 32;
    RegDft<E>::run(v, a.twN);
#pragma unroll
    for (int k = 1; k < E; k++) v[k] = cmul(v[k], __ldg(a.tl1 + 32 * k + lane));
    // 32-point DFT across lanes, radix-2 decimation in frequency: at stage h
    // the lanes l and l ^ h form a butterfly with twiddle w_{2h}^{l mod h}.
#pragma unroll
    for (int h = 16, st = 0; h >= 1; h >>= 1, st++) {
        const bool up = (lane & h) != 0;
        const float2 t = __ldg(a.tl2 + 32 * st + lane);
#pragma unroll
        for (int k = 0; k < E; k++) {
            const float2 p = shfl_xor2(v[k], h);
            v[k] = up ? cmul(csub(p, v[k]), t) : cadd(v[k], p);
        }
    }
}

// The adjoint of fft_forward (N times the inverse FFT): the lane stages in
// reverse order with conjugate twiddles, the conjugate twiddle, then the
// E-point DFT's adjoint conj(DFT(conj(.))).  Layouts swap: in, register r of
// lane l holds Y[r + E * brev5(l)]; out, it holds N * y[l + 32 r].
template <int N>
__device__ __forceinline__ void fft_adjoint(float2 (&v)[N / 32], int lane, const Args &a) {
    constexpr int E = N / 32;
#pragma unroll
    for (int h = 1, st = 4; h <= 16; h <<= 1, st--) {
        const bool up = (lane & h) != 0;
        const float2 t = cconj(__ldg(a.tl2 + 32 * st + lane));
#pragma unroll
        for (int k = 0; k < E; k++) {
            const float2 p = shfl_xor2(v[k], h);
            v[k] = up ? csub(p, cmul(t, v[k])) : cadd(v[k], cmul(t, p));
        }
    }
#pragma unroll
    for (int k = 1; k < E; k++) v[k] = cmul(v[k], cconj(__ldg(a.tl1 + 32 * k + lane)));
#pragma unroll
    for (int k = 0; k < E; k++) v[k] = cconj(v[k]);
    RegDft<E>::run(v, a.twN);
#pragma unroll
    for (int k = 0; k < E; k++) v[k] = cconj(v[k]);
}

struct Entropy {
    float s1a = 0.f, s2a = 0.f, s1b = 0.f, s2b = 0.f;  // sum P, sum P ln P per row
    __device__ __forceinline__ void add(float ca, float cb, float s2) {
        const float pa = s2 * ca * ca, pb = s2 * cb * cb;
        s1a += pa;
        s1b += pb;
        // terms below 1e-30 add less than 1e-28 to the sum: skipped, which
        // also keeps the fast logarithm away from denormals
        if (pa > 1e-30f) s2a += pa * __logf(pa);
        if (pb > 1e-30f) s2b += pb * __logf(pb);
    }
};

// Frequency f of the pair (rows a, b) with Zf = Z[f], Zp = Z[N - f] (Z[0]
// for f = 0): the DCT coefficients c[f] (entropy), then the filtered and
// re-twiddled spectrum Y[f] = V'_a[f] + i V'_b[f] of the inverse.
// ws: the filter w in shared memory, entry i at i + i / 32 (one pad word per
// 32: the bit-reversed frequencies of a warp's lanes fall on distinct banks)
template <int N>
__device__ __forceinline__ float2 spectrum(float2 Zf, float2 Zp, int k, int lane, const Args &a,
                                           const float *ws, Entropy &en) {
    constexpr int E = N / 32;
    const int f = k + E * (int)(__brev((unsigned)lane) >> 27);
    // the two real rows' FFTs: V_a = (Zf + conj Zp) / 2, V_b = (Zf - conj Zp) / 2i
    const float2 Va = make_float2(0.5f * (Zf.x + Zp.x), 0.5f * (Zf.y - Zp.y));
    const float2 Vb = make_float2(0.5f * (Zf.y + Zp.y), 0.5f * (Zp.x - Zf.x));
    const float2 q = __ldg(a.tl3 + 32 * k + lane);     // (cos, -sin)(pi f / 2N)
    const float cf = q.x, sf = -q.y;
    // c[f] = Re(e^{-i pi f/2N} V[f]); c[N-f] = Re(e^{-i pi (N-f)/2N} conj V[f])
    const float caf = cf * Va.x + sf * Va.y, cap = sf * Va.x - cf * Va.y;
    const float cbf = cf * Vb.x + sf * Vb.y, cbp = sf * Vb.x - cf * Vb.y;
    en.add(caf, cbf, (f == 0 ? 1.0f : 2.0f) / (float)N);
    const float wf = ws[f + (f >> 5)];
    const float wp = f == 0 ? 0.0f : ws[(N - f) + ((N - f) >> 5)];   // c[N] = 0 for f = 0
    const float gaf = caf * wf, gap = cap * wp, gbf = cbf * wf, gbp = cbp * wp;
    // V'[f] = e^{i pi f/2N} (g[f] - i g[N-f])
    const float2 Pa = make_float2(cf * gaf + sf * gap, sf * gaf - cf * gap);
    const float2 Pb = make_float2(cf * gbf + sf * gbp, sf * gbf - cf * gbp);
    return make_float2(Pa.x - Pb.y, Pa.y + Pb.x);
}

// Blocks of 256 threads, 2 per SM for d >= 512 (128 registers a thread) and 3
// below (80): the register caps cost a few spilled bytes and double or triple
// the warps each SM has to hide load and shuffle latency.
template <int N> constexpr int dct_blocks_per_sm() { return N >= 512 ? 2 : 3; }

template <int N, typename T, bool DEBUG>
__global__ void __launch_bounds__(256, dct_blocks_per_sm<N>()) dct_mix_kernel(Args a) {
    constexpr int E = N / 32;   // complex values per lane
    constexpr int H2 = E / 2;   // (even, odd) sample pairs per lane and row
    const int lane = threadIdx.x & 31;
    const int mrev = (int)(__brev((unsigned)lane) >> 27);
    const int src0 = (int)(__brev((unsigned)((32 - mrev) & 31)) >> 27);   // holds Z[N - E*mrev]
    const long long npairs = (a.T + 1) >> 1;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const T *X = static_cast<const T *>(a.x);
    T *Y = static_cast<T *>(a.y);
    __shared__ float ws[N + N / 32];
    for (int i = threadIdx.x; i < N; i += blockDim.x) ws[i + (i >> 5)] = __ldg(a.w + i);
    __syncthreads();

    for (long long pr = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; pr < npairs;
         pr += nwarps) {
        const long long ta = 2 * pr;
        const bool hasb = ta + 1 < a.T;
        const T *xa = X + ta * N;
        const T *xb = xa + N;

        // z[n] = x_a[j] + i x_b[j] with j = 2n (n < N/2) or j = 2(N-1-n)+1;
        // lane l loads the pairs x[2n], x[2n+1] at n = l + 32 q
        float2 v[E];
        float2 od[H2];
#pragma unroll
        for (int q = 0; q < H2; q++) {
            const int n = lane + 32 * q;
            const float2 pa = Row<T>::load2(xa + 2 * n);
            const float2 pb = hasb ? Row<T>::load2(xb + 2 * n) : make_float2(0.f, 0.f);
            v[q] = make_float2(pa.x, pb.x);
            od[q] = make_float2(pa.y, pb.y);
        }
        // z[l + 32 r] for r >= E/2 is the odd sample that lane 31-l loaded at q = E-1-r
#pragma unroll
        for (int r = H2; r < E; r++) v[r] = shfl_xor2(od[E - 1 - r], 31);

        fft_forward<N>(v, lane, a);

        // register k of lane l holds Z[f], f = k + E * mrev; Z[N - f] sits in
        // register E-k of lane l^31 (k > 0) or register 0 of lane src0 (k = 0)
        Entropy en;
        {
            const float2 zp = shfl2(v[0], src0);
            v[0] = spectrum<N>(v[0], zp, 0, lane, a, ws, en);
        }
#pragma unroll
        for (int k = 1; k <= E / 2; k++) {
            if (k < E - k) {
                const float2 pk = shfl_xor2(v[E - k], 31);
                const float2 pj = shfl_xor2(v[k], 31);
                const float2 yk = spectrum<N>(v[k], pk, k, lane, a, ws, en);
                const float2 yj = spectrum<N>(v[E - k], pj, E - k, lane, a, ws, en);
                v[k] = yk;
                v[E - k] = yj;
            } else {   // k = E/2 pairs with itself across lanes
                const float2 pk = shfl_xor2(v[k], 31);
                v[k] = spectrum<N>(v[k], pk, k, lane, a, ws, en);
            }
        }

        // entropy per row: H = (ln S1 - S2 / S1) / ln N
        const float s1a = warp_sum(en.s1a), s2a = warp_sum(en.s2a);
        const float s1b = warp_sum(en.s1b), s2b = warp_sum(en.s2b);
        const float inv_ln = 1.0f / logf((float)N);
        const float Ha = s1a > 0.f ? (logf(s1a) - s2a / s1a) * inv_ln : 0.f;
        const float Hb = s1b > 0.f ? (logf(s1b) - s2b / s1b) * inv_ln : 0.f;
        if (lane == 0) {
            a.H[ta] = Ha;
            a.route[ta] = Ha <= a.tau ? 1 : 0;
        } else if (lane == 1 && hasb) {
            a.H[ta + 1] = Hb;
            a.route[ta + 1] = Hb <= a.tau ? 1 : 0;
        }

        fft_adjoint<N>(v, lane, a);

        // m[2n] = u[n], m[2n+1] = u[N-1-n] with u = adjoint / N; lane l owns
        // n = l + 32 q, and u[N-1-n] is register E-1-q of lane 31-l
        float2 uo[H2];
#pragma unroll
        for (int q = 0; q < H2; q++) uo[q] = shfl_xor2(v[E - 1 - q], 31);
        const float invN = 1.0f / (float)N;
        float2 ze[H2], zo[H2];   // residual sums (row a, row b) at j = 2n and 2n+1
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int q = 0; q < H2; q++) {
            const int n = lane + 32 * q;
            const float2 me = make_float2(v[q].x * invN, v[q].y * invN);
            const float2 mo = make_float2(uo[q].x * invN, uo[q].y * invN);
            if (DEBUG) {
                *reinterpret_cast<float2 *>(a.mix + ta * N + 2 * n) = make_float2(me.x, mo.x);
                if (hasb) *reinterpret_cast<float2 *>(a.mix + (ta + 1) * N + 2 * n) = make_float2(me.y, mo.y);
            }
            const float2 pa = Row<T>::load2(xa + 2 * n);
            const float2 pb = hasb ? Row<T>::load2(xb + 2 * n) : make_float2(0.f, 0.f);
            ze[q] = make_float2(pa.x + me.x, pb.x + me.y);
            zo[q] = make_float2(pa.y + mo.x, pb.y + mo.y);
            sa += ze[q].x + zo[q].x;
            sb += ze[q].y + zo[q].y;
        }
        const float mean_a = warp_sum(sa) * invN, mean_b = warp_sum(sb) * invN;
        float va = 0.f, vb = 0.f;
#pragma unroll
        for (int q = 0; q < H2; q++) {
            float t;
            t = ze[q].x - mean_a; va += t * t;
            t = zo[q].x - mean_a; va += t * t;
            t = ze[q].y - mean_b; vb += t * t;
            t = zo[q].y - mean_b; vb += t * t;
        }
        const float rs_a = rsqrtf(warp_sum(va) * invN + a.eps);
        const float rs_b = rsqrtf(warp_sum(vb) * invN + a.eps);
#pragma unroll
        for (int q = 0; q < H2; q++) {
            const int j = 2 * (lane + 32 * q);
            const float2 g = __ldg(reinterpret_cast<const float2 *>(a.gamma + j));
            const float2 b = __ldg(reinterpret_cast<const float2 *>(a.beta + j));
            Row<T>::store2(Y + ta * N + j, (ze[q].x - mean_a) * rs_a * g.x + b.x,
                           (zo[q].x - mean_a) * rs_a * g.y + b.y);
            if (hasb)
                Row<T>::store2(Y + (ta + 1) * N + j, (ze[q].y - mean_b) * rs_b * g.x + b.x,
                               (zo[q].y - mean_b) * rs_b * g.y + b.y);
        }
    }
}

template <int N, typename T>
cudaError_t launch_NT(const Args &a, bool debug, int nsm, cudaStream_t s) {
    const long long npairs = (a.T + 1) / 2;
    const long long want = (npairs + 7) / 8;                  // 8 warps per block
    const long long cap = (long long)nsm * dct_blocks_per_sm<N>();   // one resident wave
    const int grid = (int)(want < cap ? want : cap);
    if (debug)
        dct_mix_kernel<N, T, true><<<grid, 256, 0, s>>>(a);
    else
        dct_mix_kernel<N, T, false><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_T(int d, const Args &a, bool debug, int nsm, cudaStream_t s) {
    switch (d) {
    case 64: return launch_NT<64, T>(a, debug, nsm, s);
    case 128: return launch_NT<128, T>(a, debug, nsm, s);
    case 256: return launch_NT<256, T>(a, debug, nsm, s);
    case 512: return launch_NT<512, T>(a, debug, nsm, s);
    case 1024: return launch_NT<1024, T>(a, debug, nsm, s);
    default: return cudaErrorInvalidValue;
    }
}

int status_of(cudaError_t e) {
    if (e == cudaSuccess) return SPECTRE_OK;
    if (e == cudaErrorMemoryAllocation) return SPECTRE_ERR_NOMEM;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorInvalidDevice)
        return SPECTRE_ERR_DEVICE;
    return SPECTRE_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool current_device_is(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return cur == dev;
}

int run(dct_mix_s *h, long long T, const void *x, const float *w, const float *gamma,
        const float *beta, float tau, void *y, float *H, unsigned char *route, float *mix,
        bool debug, void *stream) {
    if (!h || T < 0) return SPECTRE_ERR_ARG;
    if (T == 0) return SPECTRE_OK;
    if (!x || !w || !gamma || !beta || !y || !H || !route || (debug && !mix)) return SPECTRE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y) ||
        !aligned16(H) || !aligned16(route) || (debug && !aligned16(mix)))
        return SPECTRE_ERR_ALIGN;
    if (!current_device_is(h->device)) return SPECTRE_ERR_DEVICE;
    Args a;
    a.T = T;
    a.x = x;
    a.w = w;
    a.gamma = gamma;
    a.beta = beta;
    a.tau = tau;
    a.eps = h->eps;
    a.y = y;
    a.H = H;
    a.route = route;
    a.mix = mix;
    a.twN = h->tables;
    a.tq = h->tables + h->d;
    a.tl1 = h->tables + 2 * h->d;
    a.tl2 = a.tl1 + h->d;          // E x 32 = d entries
    a.tl3 = a.tl2 + 5 * 32;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = h->dtype == SPECTRE_F32
                              ? launch_T<float>(h->d, a, debug, h->nsm, s)
                              : launch_T<__nv_bfloat16>(h->d, a, debug, h->nsm, s);
    return status_of(e);
}

size_t align_up(size_t v, size_t al) { return (v + al - 1) / al * al; }

}  // namespace dctmix

extern "C" {

int dct_mix_create(dct_mix_t *out, int d, int dtype, float eps) {
    if (!out) return SPECTRE_ERR_ARG;
    *out = nullptr;
    if (dtype != SPECTRE_F32 && dtype != SPECTRE_BF16) return SPECTRE_ERR_ARG;
    if (!(eps > 0.0f) || !std::isfinite(eps)) return SPECTRE_ERR_ARG;
    if (d < 64 || d > 1024 || (d & (d - 1)) != 0) return SPECTRE_ERR_UNSUPPORTED_L;
    int dev = -1, major = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    if (major != 10) return SPECTRE_ERR_DEVICE;
    // twN, tq, then the lane-major tl1 [E][32], tl2 [5][32], tl3 [E][32]
    const int E = d / 32;
    std::vector<float2> tab(4 * (size_t)d + 5 * 32);
    for (int j = 0; j < d; j++) {
        const double ang = 2.0 * M_PI * (double)j / (double)d;
        tab[j] = make_float2((float)std::cos(ang), (float)-std::sin(ang));
        const double half = M_PI * (double)j / (2.0 * (double)d);
        tab[d + j] = make_float2((float)std::cos(half), (float)-std::sin(half));
    }
    float2 *tl1 = tab.data() + 2 * d, *tl2 = tl1 + d, *tl3 = tl2 + 5 * 32;
    for (int k = 0; k < E; k++)
        for (int l = 0; l < 32; l++) {
            tl1[32 * k + l] = tab[(size_t)((l * k) % d)];
            int rev = 0;
            for (int bit = 0; bit < 5; bit++) rev |= ((l >> bit) & 1) << (4 - bit);
            tl3[32 * k + l] = tab[d + k + E * rev];
        }
    for (int st = 0; st < 5; st++) {
        const int hh = 16 >> st;
        for (int l = 0; l < 32; l++) tl2[32 * st + l] = tab[(size_t)((l & (hh - 1)) * (16 / hh) * E)];
    }
    dct_mix_s *h = new (std::nothrow) dct_mix_s();
    if (!h) return SPECTRE_ERR_NOMEM;
    h->d = d;
    h->dtype = dtype;
    h->eps = eps;
    h->device = dev;
    h->nsm = nsm;
    cudaError_t e = cudaMalloc(&h->tables, tab.size() * sizeof(float2));
    if (e == cudaSuccess)
        e = cudaMemcpy(h->tables, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (h->tables) cudaFree(h->tables);
        delete h;
        return dctmix::status_of(e);
    }
    *out = h;
    return SPECTRE_OK;
}

int dct_mix_run(dct_mix_t h, long long T, const void *x, const float *w, const float *gamma,
                const float *beta, float tau, void *y, float *H, unsigned char *route,
                void *stream) {
    return dctmix::run(h, T, x, w, gamma, beta, tau, y, H, route, nullptr, false, stream);
}

int dct_mix_run_debug(dct_mix_t h, long long T, const void *x, const float *w,
                      const float *gamma, const float *beta, float tau, void *y, float *H,
                      unsigned char *route, float *mix, void *stream) {
    return dctmix::run(h, T, x, w, gamma, beta, tau, y, H, route, mix, true, stream);
}

int dct_mix_run_host(dct_mix_t h, long long T, const void *x, const float *w,
                     const float *gamma, const float *beta, float tau, void *y, float *H,
                     unsigned char *route, void *stream) {
    using dctmix::align_up;
    if (!h || T < 0) return SPECTRE_ERR_ARG;
    if (T == 0) return SPECTRE_OK;
    if (!x || !w || !gamma || !beta || !y || !H || !route) return SPECTRE_ERR_ARG;
    if (!dctmix::current_device_is(h->device)) return SPECTRE_ERR_DEVICE;
    const size_t es = h->dtype == SPECTRE_F32 ? 4 : 2;
    const size_t nx = (size_t)T * (size_t)h->d * es, nv = (size_t)h->d * sizeof(float);
    const size_t nh = (size_t)T * sizeof(float), nr = (size_t)T;
    const size_t o_x = align_up(nx, 256), o_v = align_up(nv, 256);
    const size_t o_h = align_up(nh, 256), o_r = align_up(nr, 256);
    const size_t need = 2 * o_x + 3 * o_v + o_h + o_r;
    if (h->stage && h->stage_bytes < need) {
        cudaFree(h->stage);
        h->stage = nullptr;
        h->stage_bytes = 0;
    }
    if (!h->stage) {
        cudaError_t e = cudaMalloc(&h->stage, need);
        if (e != cudaSuccess) {
            cudaGetLastError();
            h->stage = nullptr;
            return dctmix::status_of(e);
        }
        h->stage_bytes = need;
    }
    char *base = static_cast<char *>(h->stage);
    void *dx = base, *dy = base + o_x;
    float *dw = reinterpret_cast<float *>(base + 2 * o_x);
    float *dg = reinterpret_cast<float *>(base + 2 * o_x + o_v);
    float *db = reinterpret_cast<float *>(base + 2 * o_x + 2 * o_v);
    float *dH = reinterpret_cast<float *>(base + 2 * o_x + 3 * o_v);
    unsigned char *dr = reinterpret_cast<unsigned char *>(base + 2 * o_x + 3 * o_v + o_h);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(dx, x, nx, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dw, w, nv, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dg, gamma, nv, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(db, beta, nv, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return dctmix::status_of(e);
    }
    int st = dctmix::run(h, T, dx, dw, dg, db, tau, dy, dH, dr, nullptr, false, stream);
    if (st != SPECTRE_OK) return st;
    e = cudaMemcpyAsync(y, dy, nx, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(H, dH, nh, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(route, dr, nr, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return dctmix::status_of(e);
    }
    return SPECTRE_OK;
}

int dct_mix_destroy(dct_mix_t h) {
    if (!h) return SPECTRE_OK;
    if (h->tables) cudaFree(h->tables);
    if (h->stage) cudaFree(h->stage);
    delete h;
    return SPECTRE_OK;
}

}  // extern "C"
