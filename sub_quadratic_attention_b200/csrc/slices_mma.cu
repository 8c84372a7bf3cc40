// slices_mma.cu -- the slice pass for M = 4096 on the tensor cores.
//
// What is computed is what spectre_slices<4096> computes (SPECTRE walk-through,
// hotelren.com/news/5925787, §2.2 pseudocode and §2.3 truncation): for each
// (b, c, f1) slice, the three 4096-point transforms of A's q, k, v rows, the
// gated product O = Q conj(K) G' V / L on the slice's bins f = f1 + R f2, and
// P[t2] = w_L^{-f1 t2} IDFT_4096(O)[t2], stored as fp16 with a per-slice
// power-of-two scale.  Only the arithmetic is arranged differently.
//
// Each 4096-point transform runs as two 64-point DFT passes (t = 64 n1 + n2,
// k = k1 + 64 k2):
//   pass 1   Y[n2][k1] = sum_{n1} w64^{n1 k1} a[64 n1 + n2]      (row n2)
//   twiddle  Y[n2][k1] *= w4096^{n2 k1}
//   pass 2   X[k1 + 64 k2] = sum_{n2} w64^{n2 k2} Y[n2][k1]      (row k1)
// Each pass is one tcgen05 MMA chain: the operand tile holds one length-64
// complex input per row in fp16 (K = 128 reals, re/im interleaved), the
// constant operand is the real 128 x 128 form of the DFT-64 matrix / 64, and
// the fp32 result lands in tensor memory, one row per TMEM lane.  A block of
// 256 threads carries two slices (channels c, c + 1 at the same f1): tile
// row = TMEM lane, and the two warps of a lane quarter split each row's 64
// columns into halves.  Between the passes each thread twiddles its half row
// and writes it transposed into the tile (a padded layout keeps those 4-byte
// writes free of bank conflicts).
//
// Truncation prunes the tensor work: the gate is zero outside min(f, L-f) < F,
// so pass 2 of the forward transforms computes only the k2 groups (8 k2
// values = one 16-column MMA) that hold a live bin, and pass 1 of the inverse
// runs only the K steps of those groups.  The product S lives in tensor
// memory between the transforms.
//
// Scaling: every pass-1 input is scaled by a power of two s with
// max |component| * s in [2^13, 2^14); the DFT matrix carries 1/64, so no
// intermediate exceeds sqrt(2) * 2^14 in magnitude (fp16-safe), and the
// power-of-two factors are gathered into the slice's P scale.
//
// All waits on the MMA mbarrier are bounded; a timeout sets bit 0 of the
// device error word and the block stops after releasing its tensor memory
// (results of that run are invalid).
#include <cuda_fp16.h>

#include "fft_regs.cuh"
#include "kernels.cuh"
#include "tc_dft.cuh"

namespace spectre {
namespace {

constexpr int kM = 4096;
constexpr int kThreads = 256;
constexpr int kBlocksPerSM = 2;                  // register budget: 128 per thread
constexpr uint32_t kTileLBO = 144;              // K-adjacent core matrices (padded)
constexpr uint32_t kTileSBO = 16 * kTileLBO;    // 8-row groups
constexpr uint32_t kTileBytes = 16 * kTileSBO;  // 128 rows
constexpr uint32_t kOpBytes = 128 * 128 * 2;    // DFT-64 operand, LBO 128, SBO 2048
constexpr uint32_t kDCols = 128;                // pass results
constexpr uint32_t kSCols = 16 * kMmaMaxGroups; // the running product S
constexpr uint32_t kWaitLimit = 1u << 12;       // polls of up to 1 ms each
constexpr size_t kSmemBytes = kTileBytes + kOpBytes + 64;

__device__ __forceinline__ uint32_t tile_off(uint32_t row, uint32_t k) {
    return (row >> 3) * kTileSBO + (k >> 3) * kTileLBO + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint32_t h2_bits(float x, float y) {
    __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// exponent a with m * 2^a in [2^13, 2^14) (0 for m == 0), clamped to fp32 range
__device__ __forceinline__ int scale_shift(float m) {
    if (!(m > 0.f)) return 0;
    int e = 0;
    frexpf(m, &e);   // m < 2^e
    return max(-126, min(126, 14 - e));
}

struct Mma {
    uint32_t tile, op, mbar, dcol, phase;
    bool late;   // this thread's last wait gave up

    // One elected thread issues the chain after a block barrier; every thread
    // then waits for the commit's mbarrier phase itself (bounded), so no second
    // barrier is needed.  A wait that gave up anywhere is seen by the whole
    // block at the next issue barrier (run returns false, uniformly) or in
    // any_late().  full_n: all 128 result
    // columns, over the K steps (16 reals each) whose bit is set in ksteps.
    // Otherwise all 8 K steps, and for each group g in gmask the 16 result
    // columns of DFT-matrix rows 16 g .. 16 g + 15 (outputs 8 g .. 8 g + 7),
    // packed side by side from column 0.
    __device__ __forceinline__ bool run(uint32_t ksteps, uint32_t gmask, bool full_n) {
        tc::fence_proxy_async();
        tc::fence_before();
        if (__syncthreads_or(late)) return false;
        if (threadIdx.x == 0) {
            tc::fence_after();
            if (full_n) {
                uint32_t acc = 0;
                for (uint32_t km = ksteps; km; km &= km - 1) {
                    const int ks = __ffs(km) - 1;
                    tc::mma_f16(dcol, tc::make_desc(tile + ks * 2 * kTileLBO, kTileLBO, kTileSBO),
                                tc::make_desc(op + ks * 2 * 128, 128, 2048), tc::idesc_f16(128), acc);
                    acc = 1;
                }
            } else {
                uint32_t gi = 0;
                for (uint32_t gm = gmask; gm; gm &= gm - 1) {
                    const int g = __ffs(gm) - 1;
                    for (int ks = 0; ks < 8; ks++)
                        tc::mma_f16(dcol + 16 * gi,
                                    tc::make_desc(tile + ks * 2 * kTileLBO, kTileLBO, kTileSBO),
                                    tc::make_desc(op + 2 * g * 2048 + ks * 2 * 128, 128, 2048),
                                    tc::idesc_f16(16), ks > 0);
                    gi++;
                }
            }
            tc::commit(mbar);
        }
        late = !tc::mbar_wait(mbar, phase, kWaitLimit);
        phase ^= 1u;
        tc::fence_after();
        return true;
    }

    // whether any thread's last wait gave up (a block-wide barrier)
    __device__ __forceinline__ bool any_late() { return __syncthreads_or(late); }
};

// Pass-1 epilogue shared by all four transforms: read this thread's half row
// of the pass result (32 complex, columns k1 = 32 half .. 32 half + 31),
// twiddle by w4096^{row k1}, and write it transposed into the tile: row
// (slice base + k1), K = 2 row.  The twiddles run as recurrences
// t <- t w4096^{row} from w4096^{16 q row}, which itself steps by
// w4096^{16 row} (at most 18 steps in all; the fp32 rounding they add is far
// below fp16's).
__device__ __forceinline__ void twiddle_transpose(uint32_t tl, const float2 *__restrict__ twMM,
                                                  unsigned char *tile, int sbase, int row, int half) {
    const float2 w1 = __ldg(twMM + 64 + row), w16 = __ldg(twMM + 16 * 64 + row);
    float2 tq = half ? cmul(w16, w16) : make_float2(1.f, 0.f);
    // column K = 2 row of tile row sbase + 16 q + i sits at colbase + (2q + i/8) SBO + (i%8) 16
    unsigned char *colbase = tile + tile_off(sbase, 2 * row);
#pragma unroll 1
    for (int q = 2 * half; q < 2 * half + 2; q++) {
        float d[32];
        tc::tmem_ld32(tl + 32 * q, d);
        float2 t = tq;
        tq = cmul(tq, w16);
        unsigned char *qb = colbase + 2 * q * kTileSBO;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float2 y = cmul(make_float2(d[2 * i], d[2 * i + 1]), t);
            *reinterpret_cast<uint32_t *>(qb + (i >> 3) * kTileSBO + (i & 7) * 16) = h2_bits(y.x, y.y);
            t = cmul(t, w1);
        }
    }
}

// Bring a 32 KB slice row into L2 ahead of its use (one bulk prefetch).
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" : : "l"(p), "r"(32768u) : "memory");
}

// largest value of v over the four warps that carry slice sl
__device__ __forceinline__ float slice_max(float v, float *red, int warp, int lane, int sl) {
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    return fmaxf(fmaxf(red[2 * sl], red[2 * sl + 1]), fmaxf(red[2 * sl + 4], red[2 * sl + 5]));
}

}  // namespace

__global__ void __launch_bounds__(kThreads, kBlocksPerSM) spectre_slices_mma4096(SliceArgs a) {
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *tile = smem;
    unsigned char *op = smem + kTileBytes;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(op + kOpBytes);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 1);   // [0] D, [1] S
    float *red = reinterpret_cast<float *>(tslot + 2);           // per-warp maxima

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int trow = 32 * quarter + lane;                        // tile row = TMEM lane
    const int sl = trow >> 6, row = trow & 63, sbase = 64 * sl;

    if (warp == 0) {
        tc::tmem_alloc_keep(&tslot[0], kDCols);
        tc::tmem_alloc_keep(&tslot[1], kSCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) tc::mbar_init(tc::smem_u32(mbar), 1);
    {
        const uint4 *src = static_cast<const uint4 *>(a.w64op);
        uint4 *dst = reinterpret_cast<uint4 *>(op);
#pragma unroll 4
        for (int i = tid; i < (int)(kOpBytes / 16); i += kThreads) dst[i] = __ldg(src + i);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    Mma mma;
    mma.tile = tc::smem_u32(tile);
    mma.op = tc::smem_u32(op);
    mma.mbar = tc::smem_u32(mbar);
    mma.dcol = tslot[0];
    mma.phase = 0;
    mma.late = false;
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const uint32_t tlD = tslot[0] + lane_base;
    const uint32_t tlS = tslot[1] + lane_base;

    const int NF = a.R / 2 + 1;
    const int npair = (a.Cw + 1) / 2;
    const long long nitems = (long long)a.B * npair * NF;
    const size_t sig_stride = (size_t)a.B * a.Cw * NF * kM;
    const bool lead = row == 0 && half == 0;   // one thread per slice
    // first row of item `it` in signal sig (channel of this thread's slice)
    auto item_row = [&](long long item, int sig, bool *ok) -> const float2 * {
        const int ff1 = (int)(item % NF);
        const long long r = item / NF;
        const int ccl = 2 * (int)(r % npair) + sl;
        const int bb = (int)(r / npair);
        *ok = ccl < a.Cw && a.c_lo + ccl < a.C;
        return a.A + sig * sig_stride + ((size_t)(bb * a.Cw + (*ok ? ccl : 0)) * NF + ff1) * kM;
    };
    bool abort = false;
    if (lead && blockIdx.x < nitems) {   // the first item's q rows
        bool ok;
        const float2 *p = item_row(blockIdx.x, 0, &ok);
        if (ok) prefetch_l2(p);
    }

#pragma unroll 1
    for (long long it = blockIdx.x; it < nitems && !abort; it += gridDim.x) {
        const int f1 = (int)(it % NF);
        const long long rest = it / NF;
        const int cl = 2 * (int)(rest % npair) + sl;
        const int b = (int)(rest / npair);
        const int c = a.c_lo + cl;
        const bool live = cl < a.Cw && c < a.C;
        const float *Gh = a.G + (size_t)(live ? c / a.D : 0) * a.nbins * (a.cgate ? 2 : 1);
        const float2 *srcA = a.A + ((size_t)(b * a.Cw + (live ? cl : 0)) * NF + f1) * kM;

        // k2 groups (8 k2 values) that hold a bin with a nonzero gate
        uint32_t gmask = 0;
#pragma unroll
        for (int g = 0; g < 8; g++)
            if (mma_group_live(g, f1, a.R, a.L, a.F)) gmask |= 1u << g;
        if (__popc(gmask) > kMmaMaxGroups) {   // excluded by the plan; never reached
            if (tid == 0 && a.err) atomicOr(a.err, 2);
            break;
        }
        if (gmask == 0) {   // every gate of the slice is zero: P = 0
            if (live) {
                const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
                uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (c & 1);
                for (int m2 = 32 * half; m2 < 32 * half + 32; m2++) dst[2 * (row + 64 * m2)] = 0u;
                if (lead) a.pscale[2 * pslice + (c & 1)] = 1.0f;
            }
            continue;
        }

        int shift_sum = 0;   // sum of the applied input shifts of the four transforms
        float omax = 0.f;
#pragma unroll 1
        for (int sig = 0; sig < 3 && !abort; sig++) {
            // the next signal's rows (after v: the next item's q rows) into L2
            if (lead) {
                bool ok = live;
                const float2 *p = nullptr;
                if (sig < 2)
                    p = srcA + (sig + 1) * sig_stride;
                else if (it + gridDim.x < nitems)
                    p = item_row(it + gridDim.x, 0, &ok);
                if (p && ok) prefetch_l2(p);
            }
            // pass-1 input: row n2 = row holds a[64 n1 + row]; this thread
            // the n1 of its half
            {
                const float2 *src = srcA + sig * sig_stride + row + 64 * 32 * half;
                float2 v[32];
#pragma unroll
                for (int n = 0; n < 32; n++)
                    v[n] = live ? __ldcs(src + 64 * n) : make_float2(0.f, 0.f);
                float mx = 0.f;
#pragma unroll
                for (int n = 0; n < 32; n += 4) {
                    const float m01 = fmaxf(fmaxf(fabsf(v[n].x), fabsf(v[n].y)),
                                            fmaxf(fabsf(v[n + 1].x), fabsf(v[n + 1].y)));
                    const float m23 = fmaxf(fmaxf(fabsf(v[n + 2].x), fabsf(v[n + 2].y)),
                                            fmaxf(fabsf(v[n + 3].x), fabsf(v[n + 3].y)));
                    mx = fmaxf(mx, fmaxf(m01, m23));
                }
                const int sh = scale_shift(slice_max(mx, red, warp, lane, sl));
                shift_sum += sh;
                const float s = ldexpf(1.0f, sh);
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    uint4 u;
                    u.x = h2_bits(v[4 * j].x * s, v[4 * j].y * s);
                    u.y = h2_bits(v[4 * j + 1].x * s, v[4 * j + 1].y * s);
                    u.z = h2_bits(v[4 * j + 2].x * s, v[4 * j + 2].y * s);
                    u.w = h2_bits(v[4 * j + 3].x * s, v[4 * j + 3].y * s);
                    *reinterpret_cast<uint4 *>(tile + tile_off(trow, 64 * half + 8 * j)) = u;
                }
            }
            if (!mma.run(0xFFu, 0, true)) { abort = true; break; }
            twiddle_transpose(tlD, a.twMM, tile, sbase, row, half);
            if (!mma.run(0xFFu, gmask, false)) { abort = true; break; }
            // pass-2 result: X[row + 64 k2] for the k2 of each live group;
            // the two halves take alternate groups
            uint32_t gi = 0;
#pragma unroll 1
            for (uint32_t gm = gmask; gm; gm &= gm - 1, gi++) {
                const int g = __ffs(gm) - 1;
                if ((gi & 1u) == (uint32_t)half) {
                    float d[16], sv[16];
                    tc::tmem_ld16(tlD + 16 * gi, d);
                    if (sig > 0) tc::tmem_ld16(tlS + 16 * gi, sv);
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const float2 X = make_float2(d[2 * j], d[2 * j + 1]);
                        float2 S;
                        if (sig == 0) {
                            const int f = f1 + a.R * (row + 64 * (8 * g + j));
                            const int ff = min(f, a.L - f);
                            if (a.cgate) {   // conj(G[L - f]) above L/2
                                float2 gc = (live && ff < a.F)
                                                ? __ldg(reinterpret_cast<const float2 *>(Gh) + ff)
                                                : make_float2(0.f, 0.f);
                                if (f > a.L - f) gc.y = -gc.y;
                                S = cscale(cmul(X, gc), a.invL);
                            } else {
                                const float gate = (live && ff < a.F) ? __ldg(Gh + ff) * a.invL : 0.f;
                                S = cscale(X, gate);
                            }
                        } else if (sig == 1) {
                            S = cmulc(make_float2(sv[2 * j], sv[2 * j + 1]), X);
                        } else {
                            S = cmul(make_float2(sv[2 * j], sv[2 * j + 1]), X);
                            omax = fmaxf(omax, fmaxf(fabsf(S.x), fabsf(S.y)));
                        }
                        sv[2 * j] = S.x;
                        sv[2 * j + 1] = S.y;
                    }
                    tc::tmem_st16(tlS + 16 * gi, sv);
                }
            }
        }
        if (abort) break;

        // inverse: conj(O) scaled into the tile rows (K steps of the live groups)
        {
            const int sh = scale_shift(slice_max(omax, red, warp, lane, sl));
            shift_sum += sh;
            const float s = ldexpf(1.0f, sh);
            uint32_t gi = 0;
#pragma unroll 1
            for (uint32_t gm = gmask; gm; gm &= gm - 1, gi++) {
                const int g = __ffs(gm) - 1;
                if ((gi & 1u) == (uint32_t)half) {
                    float sv[16];
                    tc::tmem_ld16(tlS + 16 * gi, sv);
#pragma unroll
                    for (int hh = 0; hh < 2; hh++) {
                        uint4 u;
                        u.x = h2_bits(sv[8 * hh + 0] * s, -sv[8 * hh + 1] * s);
                        u.y = h2_bits(sv[8 * hh + 2] * s, -sv[8 * hh + 3] * s);
                        u.z = h2_bits(sv[8 * hh + 4] * s, -sv[8 * hh + 5] * s);
                        u.w = h2_bits(sv[8 * hh + 6] * s, -sv[8 * hh + 7] * s);
                        *reinterpret_cast<uint4 *>(tile + tile_off(trow, 16 * g + 8 * hh)) = u;
                    }
                }
            }
        }
        if (!mma.run(gmask, 0, true)) { abort = true; break; }
        twiddle_transpose(tlD, a.twMM, tile, sbase, row, half);
        if (!mma.run(0xFFu, 0, true)) { abort = true; break; }

        // P[t2] = conj(U[t2] w_L^{f1 t2}) at t2 = row + 64 m2; the scale
        // gathers 4096 / s of each transform: 2^(48 - sum of shifts)
        {
            const int cc = live ? c : 0;
            const size_t pslice = p16_pair_slice(b, cc, f1, a.C, NF);
            uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (cc & 1);
            // w_L^{f1 t2} by recurrences in m2 (step w_L^{64 f1}) from
            // w_L^{f1 (row + 1024 q)}
            const float2 step = __ldg(a.twL + 64 * f1);
#pragma unroll 1
            for (int q = 2 * half; q < 2 * half + 2; q++) {
                float2 t = __ldg(a.twL + f1 * (row + 1024 * q));
                float d[32];
                tc::tmem_ld32(tlD + 32 * q, d);
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const float2 u = cmul(make_float2(d[2 * i], d[2 * i + 1]), t);
                    if (live) dst[2 * (row + 64 * (16 * q + i))] = h2_bits(u.x, -u.y);
                    t = cmul(t, step);
                }
            }
            if (live && lead)
                a.pscale[2 * pslice + (cc & 1)] = ldexpf(1.0f, min(127, 48 - shift_sum));
        }
    }
    if (mma.any_late()) abort = true;   // also a timeout in the last wait
    if (abort && tid == 0 && a.err) atomicOr(a.err, 1);
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tslot[1], kSCols);
        tc::tmem_dealloc(tslot[0], kDCols);
    }
}

cudaError_t launch_slices_mma4096(const SliceArgs &a, cudaStream_t s) {
    const int NF = a.R / 2 + 1;
    const long long nitems = (long long)a.B * ((a.Cw + 1) / 2) * NF;
    if (nitems <= 0) return cudaSuccess;
    const long long cap = (long long)kBlocksPerSM * (a.nsm > 0 ? a.nsm : 148);
    const unsigned grid = (unsigned)(nitems < cap ? nitems : cap);
    cudaFuncSetAttribute(spectre_slices_mma4096, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kSmemBytes);
    spectre_slices_mma4096<<<grid, kThreads, kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace spectre
