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
// A is bf16 (re, im) pairs.  One thread stages the next signal's two slice
// rows (16 KB each) into shared memory with bulk asynchronous copies while
// the block works on the current one, so the transform's input is read from
// shared memory rather than waited for from L2 or DRAM.
//
// All waits (MMA and staging mbarriers) are bounded; a timeout sets bit 0 of
// the device error word, and the block waits (bounded) for its own copy in
// flight, sets the scales of its unfinished slices to NaN, releases its
// tensor memory and stops (results of that run are invalid).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "fft_regs.cuh"
#include "kernels.cuh"
#include "tc_dft.cuh"

#ifndef SPECTRE_SLICE_TWO_TILES
#define SPECTRE_SLICE_TWO_TILES 0
#endif
// drop each line of A from L2 once the slice pass has read it, so the dirty
// intermediate is never written back to DRAM
#ifndef SPECTRE_A_DISCARD
#define SPECTRE_A_DISCARD 0
#endif

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
constexpr uint32_t kTestWaitLimit = 4;          // the wait-timeout test's block
constexpr uint32_t kRowBytes = kM * 4;           // one bf16 slice row of A
constexpr uint32_t kStageBytes = 2 * kRowBytes;  // the two slices of an item
constexpr size_t kSmemBytes = kTileBytes + kOpBytes + kStageBytes + 64;

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
    uint32_t limit;   // polls per wait
    bool late;        // this thread's last wait gave up
    bool no_issue;    // the wait-timeout test: wait without issuing any MMA

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
        if (threadIdx.x == 0 && !no_issue) {
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
        late = !tc::mbar_wait(mbar, phase, limit);
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
// t <- t w1 (w1 = w4096^{row}) from tq = w4096^{32 half row}, which steps by
// w16 = w4096^{16 row} (at most 18 steps in all; the fp32 rounding they add is
// far below fp16's).
__device__ __forceinline__ void twiddle_transpose(uint32_t tl, float2 w1, float2 w16, float2 tq,
                                                  unsigned char *tile, int sbase, int row, int half) {
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

// a bf16 (re, im) pair widened exactly to fp32
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// largest value of v over the four warps that carry slice sl; also a block
// barrier, which returns whether any thread passed `bad`
__device__ __forceinline__ float slice_max(float v, float *red, int warp, int lane, int sl, bool bad,
                                           bool *any_bad) {
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    *any_bad = __syncthreads_or(bad) != 0;
    return fmaxf(fmaxf(red[2 * sl], red[2 * sl + 1]), fmaxf(red[2 * sl + 4], red[2 * sl + 5]));
}

}  // namespace

// CG: complex gate (SPECTRE_OPT_COMPLEX_GATE), else real
template <bool CG>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM) spectre_slices_mma4096(SliceArgs a) {
    using GateT = typename std::conditional<CG, float2, float>::type;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *tile = smem;
    unsigned char *op = smem + kTileBytes;
    const uint32_t *stage = reinterpret_cast<const uint32_t *>(op + kOpBytes);   // [2][4096] bf16 pairs
    uint64_t *mbar = reinterpret_cast<uint64_t *>(op + kOpBytes + kStageBytes);  // [0] MMA, [1] stage
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 2);    // [0] D, [1] S
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
    if (tid == 0) {
        tc::mbar_init(tc::smem_u32(mbar), 1);
        tc::mbar_init(tc::smem_u32(mbar + 1), 1);
    }
    {
        const uint4 *src = static_cast<const uint4 *>(a.w64op);
        uint4 *dst = reinterpret_cast<uint4 *>(op);
#pragma unroll 4
        for (int i = tid; i < (int)(kOpBytes / 16); i += kThreads) dst[i] = __ldg(src + i);
    }
    // per-row twiddle constants of the pass-1 epilogue: w4096^{row},
    // w4096^{16 row} and the start w4096^{32 half row}
    const float2 w1 = __ldg(a.twMM + 64 + row), w16 = __ldg(a.twMM + 16 * 64 + row);
    const float2 tq0 = half ? cmul(w16, w16) : make_float2(1.f, 0.f);
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
    // the wait-timeout test: block 0 issues nothing, so its first wait runs
    // out after a few polls with no MMA in flight
    mma.no_issue = a.test_stall != 0 && blockIdx.x == 0;
    mma.limit = mma.no_issue ? kTestWaitLimit : kWaitLimit;
    const uint32_t smbar = tc::smem_u32(mbar + 1);
    const uint32_t sdst = tc::smem_u32(stage);
    // staging fills issued (thread 0) and consumed (every thread); fill n
    // completes phase n & 1 of the staging mbarrier, and at most one fill is
    // outstanding: the next is issued only after every thread consumed this one
    uint32_t nfill = 0, nused = 0;
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const uint32_t tlD = tslot[0] + lane_base;
    const uint32_t tlS = tslot[1] + lane_base;

    const int NF = a.R / 2 + 1;
    const int npair = (a.Cw + 1) / 2;
    const int nitems = a.B * npair * NF;   // < 2^31 (checked by the launcher)
    const uint32_t *Abase = static_cast<const uint32_t *>(a.A);
    const size_t sig_stride = (size_t)a.B * a.Cw * NF * kM;
    auto live_groups = [&](int f1) -> uint32_t {
        uint32_t m = 0;
#pragma unroll
        for (int g = 0; g < 8; g++)
            if (mma_group_live(g, f1, a.R, a.L, a.F)) m |= 1u << g;
        return m;
    };
    // thread 0: stage signal sig of item j (both slices' rows) into shared
    // memory, completing on the staging mbarrier
    auto stage_copy = [&](int j, int sig) {
        const int r = j / NF;
        const int ff1 = j - r * NF;
        const int rb = r / npair;
        const int ccl = 2 * (r - rb * npair);
        const bool ok1 = ccl + 1 < a.Cw && a.c_lo + ccl + 1 < a.C;
        const uint32_t *src = Abase + sig * sig_stride + ((size_t)(rb * a.Cw + ccl) * NF + ff1) * kM;
        tc::mbar_arrive_expect_tx(smbar, ok1 ? 2 * kRowBytes : kRowBytes);
        tc::bulk_copy_g2s(sdst, src, kRowBytes, smbar);
        if (ok1) tc::bulk_copy_g2s(sdst + kRowBytes, src + (size_t)NF * kM, kRowBytes, smbar);
        nfill++;
    };
    // thread 0: stage the q rows of item j if it is one that reads A
    auto stage_item = [&](int j) {
        if (j < nitems && live_groups(j % NF) != 0) stage_copy(j, 0);
    };
    bool abort = false;
    int cur = -1;   // the item in progress
    if (tid == 0) stage_item(blockIdx.x);

#pragma unroll 1
    for (int it = blockIdx.x; it < nitems && !abort; it += gridDim.x) {
        cur = it;
        const int rest = it / NF;
        const int f1 = it - rest * NF;
        const int b = rest / npair;
        const int cl = 2 * (rest - b * npair) + sl;
        const int c = a.c_lo + cl;
        const bool live = cl < a.Cw && c < a.C;
        const float *Gh = a.G + (size_t)(live ? c / a.D : 0) * a.nbins * (CG ? 2 : 1);

        // k2 groups (8 k2 values) that hold a bin with a nonzero gate
        const uint32_t gmask = live_groups(f1);
        if (__popc(gmask) > kMmaMaxGroups) {   // excluded by the plan; never reached
            if (tid == 0 && a.err) atomicOr(a.err, 2);
            abort = true;
            break;
        }
        if (gmask == 0) {   // every gate of the slice is zero: P = 0
            if (live) {
                const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
                uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (c & 1);
                for (int m2 = 32 * half; m2 < 32 * half + 32; m2++) dst[2 * (row + 64 * m2)] = 0u;
                if (row == 0 && half == 0) a.pscale[2 * pslice + (c & 1)] = 1.0f;
            }
            if (tid == 0) stage_item(it + gridDim.x);
            continue;
        }
        // this thread's k2 group in the pass-2 epilogues (ordinal `half`
        // among the live groups), or -1
        int gmine = -1;
        {
            uint32_t gm = gmask;
            if (half) gm &= gm - 1;
            if (gm) gmine = __ffs(gm) - 1;
        }

        int shift_sum = 0;   // sum of the applied input shifts of the four transforms
        float omax = 0.f;
        GateT gate[8];       // the gates of this thread's pass-2 bins / L (loaded early)
#pragma unroll 1
        for (int sig = 0; sig < 3 && !abort; sig++) {
            // pass-1 input: row n2 = row holds a[64 n1 + row]; this thread
            // the n1 of its half, read from the staged rows
            {
                const bool ok = tc::mbar_wait(smbar, nused & 1u, mma.limit);
                if (ok) nused++;
                const uint32_t *src = stage + sl * kM + row + 64 * 32 * half;
                float2 v[32];
#pragma unroll
                for (int n = 0; n < 32; n++) v[n] = live ? bf2_to_f2(src[64 * n]) : make_float2(0.f, 0.f);
                float mx = 0.f;
#pragma unroll
                for (int n = 0; n < 32; n += 4) {
                    const float m01 = fmaxf(fmaxf(fabsf(v[n].x), fabsf(v[n].y)),
                                            fmaxf(fabsf(v[n + 1].x), fabsf(v[n + 1].y)));
                    const float m23 = fmaxf(fmaxf(fabsf(v[n + 2].x), fabsf(v[n + 2].y)),
                                            fmaxf(fabsf(v[n + 3].x), fabsf(v[n + 3].y)));
                    mx = fmaxf(mx, fmaxf(m01, m23));
                }
                bool bad;
                const int sh = scale_shift(slice_max(mx, red, warp, lane, sl, !ok, &bad));
                if (bad) {
                    abort = true;
                    break;
                }
#if SPECTRE_A_DISCARD
                {   // the staged rows are in shared memory: drop their lines from L2
                    const int ccl0 = cl - sl;   // the pair's first channel
                    const bool ok1 = ccl0 + 1 < a.Cw && a.c_lo + ccl0 + 1 < a.C;
                    const int s2 = tid >> 7;    // 128 threads per row, one 128-byte line each
                    if (s2 == 0 || ok1) {
                        const uint32_t *rowp = Abase + sig * sig_stride +
                                               ((size_t)(b * a.Cw + ccl0 + s2) * NF + f1) * kM;
                        asm volatile("discard.global.L2 [%0], 128;" : : "l"(rowp + 32 * (tid & 127)) : "memory");
                    }
                }
#endif
                if (tid == 0) {
                    // every read of the staged rows is done: stage the next
                    // signal, or the next item's q rows
                    if (sig < 2)
                        stage_copy(it, sig + 1);
                    else
                        stage_item(it + gridDim.x);
                }
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
            if (sig == 0) {   // this thread's gates, loaded while the MMAs run
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int f = f1 + a.R * (row + 64 * (8 * (gmine < 0 ? 0 : gmine) + j));
                    const int ff = min(f, a.L - f);
                    const bool on = live && gmine >= 0 && ff < a.F;
                    if constexpr (CG) {   // conj(G[L - f]) above L/2
                        float2 gc = on ? __ldg(reinterpret_cast<const float2 *>(Gh) + ff)
                                       : make_float2(0.f, 0.f);
                        if (f > a.L - f) gc.y = -gc.y;
                        gate[j] = cscale(gc, a.invL);
                    } else {
                        gate[j] = on ? __ldg(Gh + ff) * a.invL : 0.f;
                    }
                }
            }
            if (!mma.run(0xFFu, 0, true)) { abort = true; break; }
            twiddle_transpose(tlD, w1, w16, tq0, tile, sbase, row, half);
            if (!mma.run(0xFFu, gmask, false)) { abort = true; break; }
            // pass-2 result: X[row + 64 k2] for the k2 of this thread's group
            if (gmine >= 0) {
                const int gi = half;
                float d[16], sv[16];
                tc::tmem_ld16(tlD + 16 * gi, d);
                if (sig > 0) tc::tmem_ld16(tlS + 16 * gi, sv);
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const float2 X = make_float2(d[2 * j], d[2 * j + 1]);
                    float2 S;
                    if (sig == 0) {
                        if constexpr (CG) S = cmul(X, gate[j]);
                        else S = cscale(X, gate[j]);
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
        if (abort) break;

        // the final epilogue's twiddles w_L^{f1 (row + 1024 q)} and the step
        // w_L^{64 f1}, loaded while the inverse MMAs run
        const float2 step = __ldg(a.twL + 64 * f1);
        const float2 tstart0 = __ldg(a.twL + f1 * (row + 1024 * (2 * half)));
        const float2 tstart1 = __ldg(a.twL + f1 * (row + 1024 * (2 * half + 1)));
        // inverse: conj(O) scaled into the tile rows (K steps of the live groups)
        {
            bool bad;
            const int sh = scale_shift(slice_max(omax, red, warp, lane, sl, false, &bad));
            shift_sum += sh;
            const float s = ldexpf(1.0f, sh);
            if (gmine >= 0) {
                float sv[16];
                tc::tmem_ld16(tlS + 16 * half, sv);
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    uint4 u;
                    u.x = h2_bits(sv[8 * hh + 0] * s, -sv[8 * hh + 1] * s);
                    u.y = h2_bits(sv[8 * hh + 2] * s, -sv[8 * hh + 3] * s);
                    u.z = h2_bits(sv[8 * hh + 4] * s, -sv[8 * hh + 5] * s);
                    u.w = h2_bits(sv[8 * hh + 6] * s, -sv[8 * hh + 7] * s);
                    *reinterpret_cast<uint4 *>(tile + tile_off(trow, 16 * gmine + 8 * hh)) = u;
                }
            }
        }
        if (!mma.run(gmask, 0, true)) { abort = true; break; }
        twiddle_transpose(tlD, w1, w16, tq0, tile, sbase, row, half);
        if (!mma.run(0xFFu, 0, true)) { abort = true; break; }

        // P[t2] = conj(U[t2] w_L^{f1 t2}) at t2 = row + 64 m2; the scale
        // gathers 4096 / s of each transform: 2^(48 - sum of shifts)
        {
            const int cc = live ? c : 0;
            const size_t pslice = p16_pair_slice(b, cc, f1, a.C, NF);
            uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (cc & 1);
            // w_L^{f1 t2} by recurrences in m2 (step w_L^{64 f1}) from
            // w_L^{f1 (row + 1024 q)}
#pragma unroll 1
            for (int qq = 0; qq < 2; qq++) {
                const int q = 2 * half + qq;
                float2 t = qq ? tstart1 : tstart0;
                float d[32];
                tc::tmem_ld32(tlD + 32 * q, d);
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const float2 u = cmul(make_float2(d[2 * i], d[2 * i + 1]), t);
                    if (live) dst[2 * (row + 64 * (16 * q + i))] = h2_bits(u.x, -u.y);
                    t = cmul(t, step);
                }
            }
            if (live && row == 0 && half == 0)
                a.pscale[2 * pslice + (cc & 1)] = ldexpf(1.0f, min(127, 48 - shift_sum));
        }
    }
    if (mma.any_late()) abort = true;   // also a timeout in the last wait
    if (abort && tid == 0) {
        if (a.err) atomicOr(a.err, 1);
        // a staging copy still in flight lands before the block leaves
        if (nfill > nused) tc::mbar_wait(smbar, (nfill - 1) & 1u, kWaitLimit);
        // this block's slices from the one in progress on were not (fully)
        // computed: a NaN scale makes every y of the run NaN (the LayerNorm
        // mixes all channels), so the failure shows in the output too
        for (int j = cur; j >= 0 && j < nitems; j += gridDim.x) {
            const int rest = j / NF;
            const int f1 = j - rest * NF;
            const int b = rest / npair, cp = rest - b * npair;
            const int c = a.c_lo + 2 * cp;
            if (c < a.C) {
                const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
                a.pscale[2 * pslice] = __int_as_float(0x7fc00000);
                a.pscale[2 * pslice + 1] = __int_as_float(0x7fc00000);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tslot[1], kSCols);
        tc::tmem_dealloc(tslot[0], kDCols);
    }
}

// ---------------------------------------------------------------------------
// Two-tile variant.  Pass-1 inputs go to one tile (tin) and pass-2 inputs to
// another (tmid), so pass 2 of one signal and pass 1 of the next are issued
// as one MMA chain: six waits per item instead of eight (q; q2 + k; k2 + v;
// v2; inverse 1; inverse 2).  The next signal's bf16 A words are loaded into
// registers just before each wait, so their latency overlaps the MMAs and the
// epilogues.  Same arithmetic, scaling and outputs as the kernel above.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kSmem2Bytes = 2 * kTileBytes + kOpBytes + 64;

struct Chain {
    uint32_t mbar, phase, limit;
    bool late, no_issue;

    // block barrier, then one thread issues `issue` and commits; every thread
    // waits (bounded) for the commit.  false: a wait gave up somewhere.
    template <class F>
    __device__ __forceinline__ bool run(F &&issue) {
        tc::fence_proxy_async();
        tc::fence_before();
        if (__syncthreads_or(late)) return false;
        if (threadIdx.x == 0 && !no_issue) {
            tc::fence_after();
            issue();
            tc::commit(mbar);
        }
        late = !tc::mbar_wait(mbar, phase, limit);
        phase ^= 1u;
        tc::fence_after();
        return true;
    }
};

// full 128-column pass over the K steps set in ksteps
__device__ __forceinline__ void issue_full(uint32_t tile, uint32_t op, uint32_t d, uint32_t ksteps) {
    uint32_t acc = 0;
    for (uint32_t km = ksteps; km; km &= km - 1) {
        const int ks = __ffs(km) - 1;
        tc::mma_f16(d, tc::make_desc(tile + ks * 2 * kTileLBO, kTileLBO, kTileSBO),
                    tc::make_desc(op + ks * 2 * 128, 128, 2048), tc::idesc_f16(128), acc);
        acc = 1;
    }
}
// the live k2 groups' 16 columns each, packed from column 0
__device__ __forceinline__ void issue_groups(uint32_t tile, uint32_t op, uint32_t d, uint32_t gmask) {
    uint32_t gi = 0;
    for (uint32_t gm = gmask; gm; gm &= gm - 1) {
        const int g = __ffs(gm) - 1;
        for (int ks = 0; ks < 8; ks++)
            tc::mma_f16(d + 16 * gi, tc::make_desc(tile + ks * 2 * kTileLBO, kTileLBO, kTileSBO),
                        tc::make_desc(op + 2 * g * 2048 + ks * 2 * 128, 128, 2048), tc::idesc_f16(16),
                        ks > 0);
        gi++;
    }
}

}  // namespace

template <bool CG>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM) spectre_slices_mma4096_2t(SliceArgs a) {
    using GateT = typename std::conditional<CG, float2, float>::type;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *tin = smem;
    unsigned char *tmid = smem + kTileBytes;
    unsigned char *op = smem + 2 * kTileBytes;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(op + kOpBytes);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 1);   // [0] D1, [1] D2, [2] S
    float *red = reinterpret_cast<float *>(tslot + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int trow = 32 * quarter + lane;
    const int sl = trow >> 6, row = trow & 63, sbase = 64 * sl;

    if (warp == 0) {
        tc::tmem_alloc_keep(&tslot[0], kDCols);
        tc::tmem_alloc_keep(&tslot[1], 16 * kMmaMaxGroups);
        tc::tmem_alloc_keep(&tslot[2], kSCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) tc::mbar_init(tc::smem_u32(mbar), 1);
    {
        const uint4 *src = static_cast<const uint4 *>(a.w64op);
        uint4 *dst = reinterpret_cast<uint4 *>(op);
#pragma unroll 4
        for (int i = tid; i < (int)(kOpBytes / 16); i += kThreads) dst[i] = __ldg(src + i);
    }
    const float2 w1 = __ldg(a.twMM + 64 + row), w16 = __ldg(a.twMM + 16 * 64 + row);
    const float2 tq0 = half ? cmul(w16, w16) : make_float2(1.f, 0.f);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    Chain ch;
    ch.mbar = tc::smem_u32(mbar);
    ch.phase = 0;
    ch.late = false;
    ch.no_issue = a.test_stall != 0 && blockIdx.x == 0;
    ch.limit = ch.no_issue ? kTestWaitLimit : kWaitLimit;
    const uint32_t utin = tc::smem_u32(tin), utmid = tc::smem_u32(tmid), uop = tc::smem_u32(op);
    const uint32_t dD1 = tslot[0], dD2 = tslot[1], dS = tslot[2];
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const uint32_t tlD1 = dD1 + lane_base, tlD2 = dD2 + lane_base, tlS = dS + lane_base;

    const int NF = a.R / 2 + 1;
    const int npair = (a.Cw + 1) / 2;
    const int nitems = a.B * npair * NF;
    const uint32_t *Abase = static_cast<const uint32_t *>(a.A);
    const size_t sig_stride = (size_t)a.B * a.Cw * NF * kM;
    auto live_groups = [&](int f1) -> uint32_t {
        uint32_t m = 0;
#pragma unroll
        for (int g = 0; g < 8; g++)
            if (mma_group_live(g, f1, a.R, a.L, a.F)) m |= 1u << g;
        return m;
    };
    // this thread's 32 A words (bf16 pairs) of signal sig of item j: row
    // n2 = row, n1 = 32 half .. 32 half + 31
    uint32_t araw[32];
    auto load_a = [&](int j, int sig) {
        const int r = j / NF;
        const int ff1 = j - r * NF;
        const int rb = r / npair;
        const int ccl = 2 * (r - rb * npair) + sl;
        const bool ok = ccl < a.Cw && a.c_lo + ccl < a.C;
        const uint32_t *src = Abase + sig * sig_stride + ((size_t)(rb * a.Cw + (ok ? ccl : 0)) * NF + ff1) * kM +
                              row + 64 * 32 * half;
#pragma unroll
        for (int n = 0; n < 32; n++) araw[n] = ok ? __ldcs(src + 64 * n) : 0u;
    };
    // after araw of signal sig of item j is consumed: lane l drops the
    // 128-byte line its warp read with load n = l
    auto discard_a = [&](int j, int sig) {
#if SPECTRE_A_DISCARD
        const int r = j / NF;
        const int ff1 = j - r * NF;
        const int rb = r / npair;
        const int ccl = 2 * (r - rb * npair) + sl;
        if (ccl < a.Cw && a.c_lo + ccl < a.C) {
            const uint32_t *src = Abase + sig * sig_stride + ((size_t)(rb * a.Cw + ccl) * NF + ff1) * kM +
                                  (row & ~31) + 64 * 32 * half + 64 * lane;
            asm volatile("discard.global.L2 [%0], 128;" : : "l"(src) : "memory");
        }
#else
        (void)j;
        (void)sig;
#endif
    };
    // pass-1 input tile from araw: the slice maximum (a block barrier), a
    // power-of-two scale, fp16 into tin.  Returns the applied shift.
    auto prologue = [&]() -> int {
        float mx = 0.f;
#pragma unroll
        for (int n = 0; n < 32; n++) {
            const float2 v = bf2_to_f2(araw[n]);
            mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
        }
        bool bad;
        const int sh = scale_shift(slice_max(mx, red, warp, lane, sl, false, &bad));
        const float s = ldexpf(1.0f, sh);
#pragma unroll
        for (int j = 0; j < 8; j++) {
            float2 v0 = bf2_to_f2(araw[4 * j]), v1 = bf2_to_f2(araw[4 * j + 1]);
            float2 v2 = bf2_to_f2(araw[4 * j + 2]), v3 = bf2_to_f2(araw[4 * j + 3]);
            uint4 u;
            u.x = h2_bits(v0.x * s, v0.y * s);
            u.y = h2_bits(v1.x * s, v1.y * s);
            u.z = h2_bits(v2.x * s, v2.y * s);
            u.w = h2_bits(v3.x * s, v3.y * s);
            *reinterpret_cast<uint4 *>(tin + tile_off(trow, 64 * half + 8 * j)) = u;
        }
        return sh;
    };

    bool abort = false;
    int cur = -1;
    // the first item's q words
    int it = blockIdx.x;
    while (it < nitems && live_groups(it % NF) == 0) {   // all-zero slices: P = 0, no A read
        const int rest = it / NF, f1 = it - rest * NF, b = rest / npair;
        const int c = a.c_lo + 2 * (rest - b * npair) + sl;
        if (2 * (rest - b * npair) + sl < a.Cw && c < a.C) {
            const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
            uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (c & 1);
            for (int m2 = 32 * half; m2 < 32 * half + 32; m2++) dst[2 * (row + 64 * m2)] = 0u;
            if (row == 0 && half == 0) a.pscale[2 * pslice + (c & 1)] = 1.0f;
        }
        it += gridDim.x;
    }
    if (it < nitems) load_a(it, 0);

#pragma unroll 1
    while (it < nitems && !abort) {
        cur = it;
        const int rest = it / NF;
        const int f1 = it - rest * NF;
        const int b = rest / npair;
        const int cl = 2 * (rest - b * npair) + sl;
        const int c = a.c_lo + cl;
        const bool live = cl < a.Cw && c < a.C;
        const float *Gh = a.G + (size_t)(live ? c / a.D : 0) * a.nbins * (CG ? 2 : 1);
        const uint32_t gmask = live_groups(f1);
        if (__popc(gmask) > kMmaMaxGroups) {   // excluded by the plan; never reached
            if (tid == 0 && a.err) atomicOr(a.err, 2);
            abort = true;
            break;
        }
        int gmine = -1;
        {
            uint32_t gm = gmask;
            if (half) gm &= gm - 1;
            if (gm) gmine = __ffs(gm) - 1;
        }
        // the next item that reads A (all-zero slices in between are written here)
        int nxt = it + gridDim.x;
        while (nxt < nitems && live_groups(nxt % NF) == 0) {
            const int r2 = nxt / NF, ff1 = nxt - r2 * NF, bb = r2 / npair;
            const int cc = a.c_lo + 2 * (r2 - bb * npair) + sl;
            if (2 * (r2 - bb * npair) + sl < a.Cw && cc < a.C) {
                const size_t pslice = p16_pair_slice(bb, cc, ff1, a.C, NF);
                uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (cc & 1);
                for (int m2 = 32 * half; m2 < 32 * half + 32; m2++) dst[2 * (row + 64 * m2)] = 0u;
                if (row == 0 && half == 0) a.pscale[2 * pslice + (cc & 1)] = 1.0f;
            }
            nxt += gridDim.x;
        }

        int shift_sum = prologue();   // q into tin (its words were loaded earlier)
        discard_a(it, 0);
        GateT gate[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int f = f1 + a.R * (row + 64 * (8 * (gmine < 0 ? 0 : gmine) + j));
            const int ff = min(f, a.L - f);
            const bool on = live && gmine >= 0 && ff < a.F;
            if constexpr (CG) {
                float2 gc = on ? __ldg(reinterpret_cast<const float2 *>(Gh) + ff) : make_float2(0.f, 0.f);
                if (f > a.L - f) gc.y = -gc.y;
                gate[j] = cscale(gc, a.invL);
            } else {
                gate[j] = on ? __ldg(Gh + ff) * a.invL : 0.f;
            }
        }
        load_a(it, 1);   // k words, in flight during the q pass
        if (!ch.run([&] { issue_full(utin, uop, dD1, 0xFFu); })) { abort = true; break; }
        twiddle_transpose(tlD1, w1, w16, tq0, tmid, sbase, row, half);
        shift_sum += prologue();   // k into tin
        discard_a(it, 1);
        load_a(it, 2);   // v words
        if (!ch.run([&] {
                issue_groups(utmid, uop, dD2, gmask);
                issue_full(utin, uop, dD1, 0xFFu);
            })) { abort = true; break; }
        float omax = 0.f;
        // q's pass-2 result times the gate / L -> S
        if (gmine >= 0) {
            float d[16], sv[16];
            tc::tmem_ld16(tlD2 + 16 * half, d);
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float2 X = make_float2(d[2 * j], d[2 * j + 1]);
                float2 S;
                if constexpr (CG) S = cmul(X, gate[j]);
                else S = cscale(X, gate[j]);
                sv[2 * j] = S.x;
                sv[2 * j + 1] = S.y;
            }
            tc::tmem_st16(tlS + 16 * half, sv);
        }
        twiddle_transpose(tlD1, w1, w16, tq0, tmid, sbase, row, half);
        shift_sum += prologue();   // v into tin
        discard_a(it, 2);
        if (nxt < nitems) load_a(nxt, 0);   // the next item's q words
        if (!ch.run([&] {
                issue_groups(utmid, uop, dD2, gmask);
                issue_full(utin, uop, dD1, 0xFFu);
            })) { abort = true; break; }
        if (gmine >= 0) {   // S *= conj(K)
            float d[16], sv[16];
            tc::tmem_ld16(tlD2 + 16 * half, d);
            tc::tmem_ld16(tlS + 16 * half, sv);
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float2 S = cmulc(make_float2(sv[2 * j], sv[2 * j + 1]), make_float2(d[2 * j], d[2 * j + 1]));
                sv[2 * j] = S.x;
                sv[2 * j + 1] = S.y;
            }
            tc::tmem_st16(tlS + 16 * half, sv);
        }
        twiddle_transpose(tlD1, w1, w16, tq0, tmid, sbase, row, half);
        if (!ch.run([&] { issue_groups(utmid, uop, dD2, gmask); })) { abort = true; break; }
        float sv[16];
        if (gmine >= 0) {   // O = S V
            float d[16];
            tc::tmem_ld16(tlD2 + 16 * half, d);
            tc::tmem_ld16(tlS + 16 * half, sv);
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float2 S = cmul(make_float2(sv[2 * j], sv[2 * j + 1]), make_float2(d[2 * j], d[2 * j + 1]));
                omax = fmaxf(omax, fmaxf(fabsf(S.x), fabsf(S.y)));
                sv[2 * j] = S.x;
                sv[2 * j + 1] = S.y;
            }
        }
        const float2 step = __ldg(a.twL + 64 * f1);
        const float2 tstart0 = __ldg(a.twL + f1 * (row + 1024 * (2 * half)));
        const float2 tstart1 = __ldg(a.twL + f1 * (row + 1024 * (2 * half + 1)));
        {   // inverse input: conj(O) scaled into tin (K steps of the live groups)
            bool bad;
            const int sh = scale_shift(slice_max(omax, red, warp, lane, sl, false, &bad));
            shift_sum += sh;
            const float s = ldexpf(1.0f, sh);
            if (gmine >= 0) {
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    uint4 u;
                    u.x = h2_bits(sv[8 * hh + 0] * s, -sv[8 * hh + 1] * s);
                    u.y = h2_bits(sv[8 * hh + 2] * s, -sv[8 * hh + 3] * s);
                    u.z = h2_bits(sv[8 * hh + 4] * s, -sv[8 * hh + 5] * s);
                    u.w = h2_bits(sv[8 * hh + 6] * s, -sv[8 * hh + 7] * s);
                    *reinterpret_cast<uint4 *>(tin + tile_off(trow, 16 * gmine + 8 * hh)) = u;
                }
            }
        }
        if (!ch.run([&] { issue_full(utin, uop, dD1, gmask); })) { abort = true; break; }
        twiddle_transpose(tlD1, w1, w16, tq0, tmid, sbase, row, half);
        if (!ch.run([&] { issue_full(utmid, uop, dD1, 0xFFu); })) { abort = true; break; }
        {
            const int cc = live ? c : 0;
            const size_t pslice = p16_pair_slice(b, cc, f1, a.C, NF);
            uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (cc & 1);
#pragma unroll 1
            for (int qq = 0; qq < 2; qq++) {
                const int q = 2 * half + qq;
                float2 t = qq ? tstart1 : tstart0;
                float d[32];
                tc::tmem_ld32(tlD1 + 32 * q, d);
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const float2 u = cmul(make_float2(d[2 * i], d[2 * i + 1]), t);
                    if (live) dst[2 * (row + 64 * (16 * q + i))] = h2_bits(u.x, -u.y);
                    t = cmul(t, step);
                }
            }
            if (live && row == 0 && half == 0)
                a.pscale[2 * pslice + (cc & 1)] = ldexpf(1.0f, min(127, 48 - shift_sum));
        }
        it = nxt;
    }
    if (__syncthreads_or(ch.late)) abort = true;   // also a timeout in the last wait
    if (abort && tid == 0) {
        if (a.err) atomicOr(a.err, 1);
        for (int j = cur; j >= 0 && j < nitems; j += gridDim.x) {
            const int rest = j / NF;
            const int f1 = j - rest * NF;
            const int b = rest / npair, cp = rest - b * npair;
            const int c = a.c_lo + 2 * cp;
            if (c < a.C) {
                const size_t pslice = p16_pair_slice(b, c, f1, a.C, NF);
                a.pscale[2 * pslice] = __int_as_float(0x7fc00000);
                a.pscale[2 * pslice + 1] = __int_as_float(0x7fc00000);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tslot[2], kSCols);
        tc::tmem_dealloc(tslot[1], 16 * kMmaMaxGroups);
        tc::tmem_dealloc(tslot[0], kDCols);
    }
}

cudaError_t launch_slices_mma4096(const SliceArgs &a, cudaStream_t s) {
    const int NF = a.R / 2 + 1;
    const long long nitems = (long long)a.B * ((a.Cw + 1) / 2) * NF;
    if (nitems <= 0) return cudaSuccess;
    if (nitems >= (1LL << 31)) return cudaErrorInvalidValue;
    const long long cap = (long long)kBlocksPerSM * (a.nsm > 0 ? a.nsm : 148);
    const unsigned grid = (unsigned)(nitems < cap ? nitems : cap);
    if (!a.a16) return cudaErrorInvalidValue;   // the pass reads bf16 A
#if SPECTRE_SLICE_TWO_TILES
    auto k = a.cgate ? spectre_slices_mma4096_2t<true> : spectre_slices_mma4096_2t<false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem2Bytes);
    k<<<grid, kThreads, kSmem2Bytes, s>>>(a);
#else
    auto k = a.cgate ? spectre_slices_mma4096<true> : spectre_slices_mma4096<false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    k<<<grid, kThreads, kSmemBytes, s>>>(a);
#endif
    return cudaGetLastError();
}

}  // namespace spectre
