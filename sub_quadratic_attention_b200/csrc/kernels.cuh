// kernels.cuh -- launch interface between the plan (api.cu) and the kernels
// of the SPECTRE mixer (kernels.cu: row passes, CUDA-core slice pass, inverse
// passes; slices_mma.cu: tensor-core slice pass).
//
// Decomposition (four-step Cooley-Tukey along L, split L = R * M, token
// t = t1 * M + t2, rfft bin f = f1 + R * f2):
//   row pass      A[f1][t2] = w_L^{f1 t2} * sum_{t1<R} w_R^{f1 t1} x[t1 M + t2]
//                 (f1 in [0, R/2]: the real-input half; pairs of channels
//                 share one complex R-point transform)
//   slice pass    X[f1 + R f2] = DFT_M(A[f1][.])[f2] for q, k, v; the gated
//                 product O = Q conj(K) G' V / L on those bins (G' mirrors G
//                 to f > L/2 and is 0 where min(f, L-f) >= F); then
//                 P[f1][t2] = w_L^{-f1 t2} * IDFT_M(O[f1 + R .])[t2]
//   inverse rows  out[t1 M + t2] = sum_{f1<R} w_R^{-f1 t1} P~[f1][t2], with P~
//                 the Hermitian extension P~[R - f1] = conj(P[f1]); then
//                 residual + LayerNorm over C on whole token rows.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace spectre {

constexpr int kMaxPasses = 6;

// Division by a divisor fixed for a launch, for numerators n < 2^31:
// q = (umulhi(n, m) + n) >> s with s = ceil(log2 d) and
// m = floor(2^32 (2^s - d) / d) + 1 (exact on that range; the sum stays
// below 2^32).  Work-item decoding uses it instead of 64-bit division.
struct FastDiv {
    uint32_t d, m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    f.s = 0;
    while ((1ull << f.s) < d) f.s++;
    f.m = (uint32_t)((((1ull << 32) * ((1ull << f.s) - d)) / d) + 1);
    return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
    return (__umulhi(n, f.m) + n) >> f.s;
}

// Per-pass twiddle tables of the M-point slice transforms.  Pass p of
// direction d (0 = forward radix order, 1 = reversed) with radix R_p and
// stride Ns_p (product of the earlier radices) uses
//   tw[d][p][r * Ns_p + k] = exp(-2 pi i k r / (Ns_p R_p)),  k < Ns_p, r < R_p.
struct SliceTables {
    const float2 *tw[2][kMaxPasses];
};

struct RowsFwdArgs {
    const void *q, *k, *v;
    void *A;              // [3][B][Cw][R/2+1][M]: channels c_lo .. c_lo + Cw - 1;
                          // float2, or __nv_bfloat162 (re, im) with a16
    int a16;
    const float2 *twL;    // exp(-2 pi i e / L), e in [0, L/2]
    int B, L, M, C;
    int c_lo, Cw;         // channel wave (c_lo even)
    int vec2;             // C even: load channel pairs as one vector
    int nsm;              // multiprocessors (grid of the persistent variant)
    FastDiv fd3, fd_ntg, fd_ncg;   // set by the launcher of the persistent variant
    int *err;             // device error word (tensor-core variant: bit 0 = a bounded wait gave up)
    int row_tc;           // take the tensor-core variant where it applies
};

// fp16 P (bf16 I/O) interleaves the two channels c = 2 cp, 2 cp + 1 of a pair:
// the half2 of (b, c, f1, t2) is number 2 (pslice M + t2) + (c & 1), and its
// scale pscale[2 pslice + (c & 1)], with pslice = (b CP + cp) NF + f1,
// CP = ceil(C / 2), NF = R / 2 + 1.  fp32 P (fp32 I/O) is [B][C][NF][M].
__host__ __device__ inline size_t p16_pair_slice(int b, int c, int f1, int C, int NF) {
    return ((size_t)b * ((C + 1) / 2) + c / 2) * NF + f1;
}

struct SliceArgs {
    const void *A;        // [3][B][Cw][R/2+1][M]: the chunk's channels, float2 or (a16) bf16 pairs
    int a16;
    void *P;              // float2 [B][C][NF][M], or __half2 pair-interleaved (p16_pair_slice)
    float *pscale;        // p16: P = stored * pscale, pair-interleaved like P
    const float2 *twL;
    const float *G;       // [H][L/2+1], or with cgate [H][L/2+1][2] (re, im)
    int cgate;            // complex gate: conj(G[L - f]) above L/2
    SliceTables tabs;
    int B, L, R, M, C, D, F, nbins;
    int c_lo, Cw;         // channel wave
    int p16;              // store P as fp16 with a power-of-two scale per slice
    int use_mma;          // M = 4096 as two DFT-64 passes on the tensor cores
    int nsm;              // multiprocessors of the device (grid of the MMA slice pass)
    const float2 *twMM;   // [64][64]: entry k1 * 64 + n2 = w_4096^{n2 k1}
    const void *w64op;    // DFT-64 / 64 as a 128 x 128 fp16 operand (canonical layout)
    int *err;             // device error word: bit 0 = a tensor-core wait timed out,
                          // bit 1 = a slice exceeded the tensor-memory product budget
    int test_stall;       // wait-timeout test: block 0 of the tensor-core pass issues no MMA
    long long nslices;    // B * Cw * (R/2+1)
    float invL;
};

struct RowsInvArgs {
    const void *P;        // float2 [B][C][NF][M] (fp32 I/O) or pair-interleaved __half2 with pscale
    const float *pscale;
    const void *x;
    const float *gamma, *beta;
    void *y;
    float *out_f32;       // nullable
    int B, L, M, C;
    int T2C, ZS;          // t2 values per block, padded row stride of the z buffer
    int reg_variant;      // 1: register-resident LayerNorm (R <= 16, C <= 2048)
    int vec2;             // C even: channel pairs as one vector
    int nsm;              // multiprocessors (grid of the persistent variant)
    int norm;             // bit 0: residual after the norm; bit 1: RMSNorm (no mean)
    float eps;
    FastDiv fd_cp;        // set by the launcher of the prefetching variant: C / 2
    int *err;             // device error word (prefetching variant: bit 0 = a bounded wait gave up)
};

// Returns cudaSuccess or the launch error.  dtype: 0 fp32, 1 bf16.
cudaError_t launch_rows_fwd(int R, int dtype, const RowsFwdArgs &a, cudaStream_t s);
// the tensor-core row pass (bf16 in, bf16 A, R = 16; rows_tc.cu) and whether
// it covers a launch
bool rows_tc_applies(const RowsFwdArgs &a);
cudaError_t launch_rows_fwd_tc(const RowsFwdArgs &a, cudaStream_t s);
cudaError_t launch_slices(const SliceArgs &a, cudaStream_t s);
cudaError_t launch_slices_mma4096(const SliceArgs &a, cudaStream_t s);
cudaError_t launch_rows_inv_ln(int R, int dtype, const RowsInvArgs &a, cudaStream_t s);

// Slice-transform schedule for length M (radices ascending, largest last).
// Shared-memory carveout of the row, slice and inverse kernels.  With
// SPECTRE_CARVEOUT_MAX every one of them asks for the largest shared-memory
// share of the L1/shared array, so consecutive kernels of a step need no
// reconfiguration of it between them.
#ifndef SPECTRE_CARVEOUT_MAX
#define SPECTRE_CARVEOUT_MAX 0
#endif
template <class K> inline void prefer_max_smem(K k) {
#if SPECTRE_CARVEOUT_MAX
    cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
#else
    (void)k;
#endif
}

struct RadList {
    int n;
    int r[kMaxPasses];
};

constexpr RadList make_schedule(int M) {
    RadList s{0, {0, 0, 0, 0, 0, 0}};
    int m = M;
    bool three = false;
    if (m % 3 == 0) {
        three = true;
        m /= 3;
    }
    int k = 0;
    while ((1 << k) < m) k++;
    int n16 = k / 4, rem = 1 << (k % 4);
    if (rem > 1) s.r[s.n++] = rem;
    if (three) s.r[s.n++] = 3;
    for (int i = 0; i < n16; i++) s.r[s.n++] = 16;
    for (int i = 0; i < s.n; i++)
        for (int j = 0; j + 1 < s.n - i; j++)
            if (s.r[j] > s.r[j + 1]) {
                int t = s.r[j];
                s.r[j] = s.r[j + 1];
                s.r[j + 1] = t;
            }
    return s;
}

// Radix and stride of pass p in direction d (0 forward order, 1 reversed).
constexpr int sched_radix(int M, int d, int p) {
    RadList s = make_schedule(M);
    return d == 0 ? s.r[p] : s.r[s.n - 1 - p];
}
constexpr int sched_stride(int M, int d, int p) {
    int ns = 1;
    for (int i = 0; i < p; i++) ns *= sched_radix(M, d, i);
    return ns;
}

// The tensor-core slice pass (M = 4096) keeps the product of at most this
// many k2 groups (8 bins of a slice row each) in tensor memory.
constexpr int kMmaMaxGroups = 2;

// Whether k2 group g (f2 = k1 + 64 k2, k2 in [8 g, 8 g + 8), k1 < 64) of
// slice f1 holds a bin f = f1 + R f2 with min(f, L - f) < F.
__host__ __device__ inline bool mma_group_live(int g, int f1, int R, int L, int F) {
    const long long flo = f1 + (long long)R * (64 * 8 * g);
    const long long fhi = f1 + (long long)R * (63 + 64 * (8 * g + 7));
    return flo < F || fhi > (long long)L - F;
}

// Element (n, k) of the real 128 x 128 form of the DFT-64 matrix / 64:
// n = 2 o + (0 re | 1 im) indexes outputs, k = 2 i + (0 re | 1 im) inputs,
// so that out = sum_k B[n][k] in[k] gives (re, im) of sum_i w64^{o i} in_i / 64.
__host__ __device__ inline void dft64_operand_angle(int n, int k, long long *e, int *part) {
    *e = (long long)((n >> 1) * (k >> 1)) & 63;      // w64^e
    *part = ((n & 1) << 1) | (k & 1);                 // 0: Fr, 1: -Fi, 2: Fi, 3: Fr
}
// byte offset of (n, k) in the canonical K-major no-swizzle layout with
// LBO 128 and SBO 2048 (K = 128 fp16 values per row)
__host__ __device__ inline int dft64_operand_offset(int n, int k) {
    return (n >> 3) * 2048 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

// whether M is a supported slice length (2^k <= 16384 or 3*2^k <= 12288)
bool slice_length_supported(int M);
// whether the CUDA-core slice pass for M parks its running product in A (fp32
// A required)
bool slice_parks_in_A(int M);
// threads per slice and slices per block the slice kernel uses for M
void slice_geometry(int M, int *threads_per_slice, int *slices_per_block, size_t *smem_bytes);

// Upload exp(-2 pi i e / 64), e < 64, to the constant bank of the current device.
cudaError_t upload_w64(const float2 *host64);

// Fixed scratch of the no-allocation entry point (kernels.cu).
constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;
// Device address of the scratch on the current device.  The first call on a
// device looks it up (and loads the constant twiddles); later calls reuse it.
cudaError_t noalloc_scratch(void **ptr);

// One segment of twiddle table: count entries at base + offset.  ns == 0:
// entry i = w_N^i.  ns > 0: entry r * ns + k = w_N^{k r} (a slice-pass table).
// ns == -1: the fp16 DFT-64 operand (count = 4096 eight-byte slots).
struct TableSeg {
    long long offset;
    long long count;
    long long ns;
    long long N;
};
struct TableSegs {
    int n;
    TableSeg seg[3 + 2 * kMaxPasses];
};
cudaError_t launch_make_tables(float2 *base, const TableSegs &segs, cudaStream_t s);

}  // namespace spectre
