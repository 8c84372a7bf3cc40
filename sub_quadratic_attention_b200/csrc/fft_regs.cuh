// fft_regs.cuh -- complex helpers and in-register DFTs for the SPECTRE mixer.
//
// All transforms here are forward (exp(-2*pi*i*n*k/N)), unscaled, with inputs
// and outputs in natural order; inverses are taken as conj(DFT(conj(x))).
// Array indices are compile-time constants after unrolling, so the arrays
// live in registers.
#pragma once

#include <cuda_runtime.h>

namespace spectre {

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
// a * b
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
// -i * a
__device__ __forceinline__ float2 cmul_mi(float2 a) { return make_float2(a.y, -a.x); }
// +i * a
__device__ __forceinline__ float2 cmul_pi(float2 a) { return make_float2(-a.y, a.x); }

// cos/sin of multiples of pi/8, as fp32 constants
constexpr float kC8 = 0.70710678118654752f;  // cos(pi/4)
constexpr float kC16 = 0.92387953251128674f; // cos(pi/8)
constexpr float kS16 = 0.38268343236508977f; // sin(pi/8)
constexpr float kS3 = 0.86602540378443865f;  // sin(pi/3)

// exp(-2*pi*i*e/16) for compile-time e in [0, 16)
__device__ __forceinline__ float2 w16_mul(float2 a, int e) {
    switch (e & 15) {
    case 0: return a;
    case 1: return cmul(a, make_float2(kC16, -kS16));
    case 2: return make_float2((a.x + a.y) * kC8, (a.y - a.x) * kC8);
    case 3: return cmul(a, make_float2(kS16, -kC16));
    case 4: return cmul_mi(a);
    case 5: return cmul(a, make_float2(-kS16, -kC16));
    case 6: return make_float2((a.y - a.x) * kC8, -(a.x + a.y) * kC8);
    case 7: return cmul(a, make_float2(-kC16, -kS16));
    case 8: return make_float2(-a.x, -a.y);
    case 9: return cmul(a, make_float2(-kC16, kS16));
    case 10: return make_float2(-(a.x + a.y) * kC8, (a.x - a.y) * kC8);
    case 11: return cmul(a, make_float2(-kS16, kC16));
    case 12: return cmul_pi(a);
    case 13: return cmul(a, make_float2(kS16, kC16));
    case 14: return make_float2((a.x - a.y) * kC8, (a.x + a.y) * kC8);
    default: return cmul(a, make_float2(kC16, kS16));
    }
}

__device__ __forceinline__ void dft2(float2 &a, float2 &b) {
    float2 t = a;
    a = cadd(t, b);
    b = csub(t, b);
}

// length-4 DFT of (a0, a1, a2, a3) in place
__device__ __forceinline__ void dft4(float2 &a0, float2 &a1, float2 &a2, float2 &a3) {
    float2 s02 = cadd(a0, a2), d02 = csub(a0, a2);
    float2 s13 = cadd(a1, a3), d13 = cmul_mi(csub(a1, a3));
    a0 = cadd(s02, s13);
    a2 = csub(s02, s13);
    a1 = cadd(d02, d13);
    a3 = csub(d02, d13);
}

__device__ __forceinline__ void dft3(float2 &a, float2 &b, float2 &c) {
    float2 t1 = cadd(b, c);
    float2 t2 = make_float2(fmaf(-0.5f, t1.x, a.x), fmaf(-0.5f, t1.y, a.y));
    float2 t3 = cscale(csub(b, c), kS3);  // sin(pi/3) * (b - c)
    a = cadd(a, t1);
    // y1 = t2 - i*t3, y2 = t2 + i*t3
    b = make_float2(t2.x + t3.y, t2.y - t3.x);
    c = make_float2(t2.x - t3.y, t2.y + t3.x);
}

template <int R> struct Dft;

template <> struct Dft<1> {
    __device__ __forceinline__ static void run(float2 *) {}
};
template <> struct Dft<2> {
    __device__ __forceinline__ static void run(float2 *v) { dft2(v[0], v[1]); }
};
template <> struct Dft<3> {
    __device__ __forceinline__ static void run(float2 *v) { dft3(v[0], v[1], v[2]); }
};
template <> struct Dft<4> {
    __device__ __forceinline__ static void run(float2 *v) { dft4(v[0], v[1], v[2], v[3]); }
};
template <> struct Dft<8> {
    // radix-2 split into two length-4 DFTs over even and odd samples
    __device__ __forceinline__ static void run(float2 *v) {
        float2 e0 = v[0], e1 = v[2], e2 = v[4], e3 = v[6];
        float2 o0 = v[1], o1 = v[3], o2 = v[5], o3 = v[7];
        dft4(e0, e1, e2, e3);
        dft4(o0, o1, o2, o3);
        o1 = w16_mul(o1, 2);
        o2 = cmul_mi(o2);
        o3 = w16_mul(o3, 6);
        v[0] = cadd(e0, o0); v[4] = csub(e0, o0);
        v[1] = cadd(e1, o1); v[5] = csub(e1, o1);
        v[2] = cadd(e2, o2); v[6] = csub(e2, o2);
        v[3] = cadd(e3, o3); v[7] = csub(e3, o3);
    }
};
template <> struct Dft<16> {
    // 4 x 4: length-4 DFTs over samples r, r+4, r+8, r+12, twiddle by
    // w16^{r*k}, then length-4 DFTs across r; output k + 4*s.
    __device__ __forceinline__ static void run(float2 *v) {
#pragma unroll
        for (int r = 0; r < 4; r++) dft4(v[r], v[r + 4], v[r + 8], v[r + 12]);
        // v[r + 4k] now holds Y_r[k]
#pragma unroll
        for (int r = 1; r < 4; r++)
#pragma unroll
            for (int k = 1; k < 4; k++) v[r + 4 * k] = w16_mul(v[r + 4 * k], r * k);
#pragma unroll
        for (int k = 0; k < 4; k++) dft4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        // v[4k + s] holds X[k + 4s]; transpose to natural order
        float2 t[16];
#pragma unroll
        for (int k = 0; k < 4; k++)
#pragma unroll
            for (int s = 0; s < 4; s++) t[k + 4 * s] = v[4 * k + s];
#pragma unroll
        for (int i = 0; i < 16; i++) v[i] = t[i];
    }
};

// exp(-2*pi*i*e/64), filled from the host at plan creation by kernels.cu.
// Each translation unit that includes this header gets its own copy, and only
// kernels.cu's is filled: other units (dct_mix.cu) use Dft<R> for R <= 16 only,
// never Dft<32> or Dft<64>.
static __constant__ float2 c_w64[64];

// Composite R = R1 * R2 (R2 <= 16): length-R1 DFTs over samples r, r+R2, ...
// for each r < R2, twiddle Y_r[k] by w_R^{r k}, length-R2 DFTs across r.
template <int R1, int R2> struct DftComposite {
    __device__ __forceinline__ static void run(float2 *v) {
        constexpr int R = R1 * R2;
        float2 y[R];
#pragma unroll
        for (int r = 0; r < R2; r++) {
            float2 s[R1];
#pragma unroll
            for (int m = 0; m < R1; m++) s[m] = v[r + R2 * m];
            Dft<R1>::run(s);
#pragma unroll
            for (int k = 0; k < R1; k++)
                y[r + R2 * k] = (r * k == 0) ? s[k] : cmul(s[k], c_w64[((r * k) % R) * (64 / R)]);
        }
#pragma unroll
        for (int k = 0; k < R1; k++) {
            float2 s[R2];
#pragma unroll
            for (int r = 0; r < R2; r++) s[r] = y[r + R2 * k];
            Dft<R2>::run(s);
#pragma unroll
            for (int r = 0; r < R2; r++) v[k + R1 * r] = s[r];
        }
    }
};
template <> struct Dft<32> {
    __device__ __forceinline__ static void run(float2 *v) { DftComposite<16, 2>::run(v); }
};
template <> struct Dft<64> {
    __device__ __forceinline__ static void run(float2 *v) { DftComposite<16, 4>::run(v); }
};

}  // namespace spectre
