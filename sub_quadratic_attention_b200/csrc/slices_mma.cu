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
// values = 16 result columns) that hold a live bin, as one chain of 8 MMAs
// over those groups' DFT-operand rows gathered side by side, and pass 1 of
// the inverse runs only the K steps of those groups.  The product S lives in tensor
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

// drop each line of A from L2 once the slice pass has read it, so the dirty
// intermediate is never written back to DRAM
#ifndef SPECTRE_A_DISCARD
#define SPECTRE_A_DISCARD 1
#endif
// warps per TMEM lane quarter in the tensor-core slice pass (2: 256 threads,
// 4: 512 threads per block; measured on B200 for the bf16 long workload, 4 was
// slower, 221 us against 189 us per step)
#ifndef SPECTRE_SLICE_PARTS
#define SPECTRE_SLICE_PARTS 2
#endif
// persistent blocks per multiprocessor of the tensor-core slice pass (at most
// 2: shared memory and tensor memory fit two)
#ifndef SPECTRE_SLICE_CTAS_PER_SM
#define SPECTRE_SLICE_CTAS_PER_SM 2
#endif

namespace spectre {
namespace {

constexpr int kM = 4096;
constexpr int kBlocksPerSM = 2;                  // register budget: 128 per thread
constexpr uint32_t kTileLBO = 144;              // K-adjacent core matrices (padded)
constexpr uint32_t kTileSBO = 16 * kTileLBO;    // 8-row groups
constexpr uint32_t kTileBytes = 16 * kTileSBO;  // 128 rows
constexpr uint32_t kOpBytes = 128 * 128 * 2;    // DFT-64 operand, LBO 128, SBO 2048
constexpr uint32_t kGroupOpBytes = 2 * 2048;     // one k2 group's 16 operand rows (two 8-row groups)
// the operand rows of the item's live k2 groups, side by side, so that pass 2
// of a forward transform is one 8-MMA chain of N = 16 x (live groups)
constexpr uint32_t kOp2Bytes = kMmaMaxGroups * kGroupOpBytes;
constexpr uint32_t kDCols = 128;                // pass results
constexpr uint32_t kSCols = 16 * kMmaMaxGroups; // the running product S
constexpr uint32_t kWaitLimit = 1u << 12;       // polls of up to 1 ms each
constexpr uint32_t kTestWaitLimit = 4;          // the wait-timeout test's block
constexpr uint32_t kRowBytes = kM * 4;           // one bf16 slice row of A
constexpr uint32_t kStageBytes = 2 * kRowBytes;  // the two slices of an item
constexpr size_t kSmemBytes = kTileBytes + kOpBytes + kOp2Bytes + kStageBytes + 64;

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
    uint32_t tile, op, op2, mbar, dcol, phase;
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
    // packed side by side from column 0: one MMA per K step over the gathered
    // rows in op2, which hold gmask's groups in ascending order.
    __device__ __forceinline__ bool run(uint32_t ksteps, uint32_t gmask, bool full_n) {
        return run(ksteps, gmask, full_n, [] {});
    }
    // as above; thread 0 first calls pre() once every thread has passed the
    // barrier (and so is done with what it read before the call)
    template <class Pre>
    __device__ __forceinline__ bool run(uint32_t ksteps, uint32_t gmask, bool full_n, Pre &&pre) {
        tc::fence_proxy_async();
        tc::fence_before();
        if (__syncthreads_or(late)) return false;
        if (threadIdx.x == 0) pre();
        if (threadIdx.x == 0 && !no_issue) {
            tc::fence_after();
            if (full_n) {
                const uint64_t da = tc::make_desc(tile, kTileLBO, kTileSBO);
                const uint64_t db = tc::make_desc(op, 128, 2048);
                if (ksteps == 0xFFu) {
#pragma unroll
                    for (int ks = 0; ks < 8; ks++)
                        tc::mma_f16(dcol, da + ks * (2 * kTileLBO / 16), db + ks * (2 * 128 / 16),
                                    tc::idesc_f16(128), ks > 0);
                } else {
                    uint32_t acc = 0;
                    for (uint32_t km = ksteps; km; km &= km - 1) {
                        const int ks = __ffs(km) - 1;
                        tc::mma_f16(dcol, da + ks * (2 * kTileLBO / 16), db + ks * (2 * 128 / 16),
                                    tc::idesc_f16(128), acc);
                        acc = 1;
                    }
                }
            } else {
                const uint32_t idesc = tc::idesc_f16(16 * __popc(gmask));
                const uint64_t da = tc::make_desc(tile, kTileLBO, kTileSBO);
                const uint64_t db = tc::make_desc(op2, 128, 2048);
#pragma unroll
                for (int ks = 0; ks < 8; ks++)   // the start address sits in the low bits (16-byte units)
                    tc::mma_f16(dcol, da + ks * (2 * kTileLBO / 16), db + ks * (2 * 128 / 16), idesc, ks > 0);
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

// Pass-1 epilogue shared by all four transforms: read this thread's part of
// the row's pass result (NQ blocks of 32 columns = 16 complex each, from block
// q0), twiddle by w4096^{row k1}, and write it transposed into the tile: row
// (slice base + k1), K = 2 row.  The twiddles run as recurrences
// t <- t w1 (w1 = w4096^{row}) from tq = w4096^{16 q0 row}, which steps by
// w16 = w4096^{16 row} per block (at most 18 steps in all; the fp32 rounding
// they add is far below fp16's).
template <int NQ>
__device__ __forceinline__ void twiddle_transpose(uint32_t tl, float2 w1, float2 w16, float2 tq,
                                                  unsigned char *tile, int sbase, int row, int q0) {
    // column K = 2 row of tile row sbase + 16 q + i sits at colbase + (2q + i/8) SBO + (i%8) 16
    unsigned char *colbase = tile + tile_off(sbase, 2 * row);
#pragma unroll 1
    for (int qq = 0; qq < NQ; qq++) {
        const int q = q0 + qq;
        float2 t = tq;
        tq = cmul(tq, w16);
        unsigned char *qb = colbase + 2 * q * kTileSBO;
        if constexpr (NQ == 2) {
            // 256-thread blocks: the second 16-column chunk's TMEM load is in
            // flight while the first is processed
            uint32_t ra[16], rb[16];
            tc::tmem_ld16_issue(tl + 32 * q, ra);
            tc::tmem_wait_ld16(ra);
            tc::tmem_ld16_issue(tl + 32 * q + 16, rb);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 y = cmul(make_float2(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1])), t);
                *reinterpret_cast<uint32_t *>(qb + i * 16) = h2_bits(y.x, y.y);
                t = cmul(t, w1);
            }
            tc::tmem_wait_ld16(rb);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 y = cmul(make_float2(__uint_as_float(rb[2 * i]), __uint_as_float(rb[2 * i + 1])), t);
                *reinterpret_cast<uint32_t *>(qb + kTileSBO + i * 16) = h2_bits(y.x, y.y);
                t = cmul(t, w1);
            }
        } else {
            // 512-thread blocks (64 registers): one 16-column chunk at a time
#pragma unroll 1
            for (int hh = 0; hh < 2; hh++) {
                float r[16];
                tc::tmem_ld16(tl + 32 * q + 16 * hh, r);
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const float2 y = cmul(make_float2(r[2 * i], r[2 * i + 1]), t);
                    *reinterpret_cast<uint32_t *>(qb + hh * kTileSBO + i * 16) = h2_bits(y.x, y.y);
                    t = cmul(t, w1);
                }
            }
        }
    }
}

// a bf16 (re, im) pair widened exactly to fp32
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// largest value of v over the warps that carry slice sl (lane quarters 2 sl
// and 2 sl + 1 of each of the NP parts; warp = quarter + 4 part); also a block
// barrier, which returns whether any thread passed `bad`
template <int NP = 2>
__device__ __forceinline__ float slice_max(float v, float *red, int warp, int lane, int sl, bool bad,
                                           bool *any_bad) {
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    *any_bad = __syncthreads_or(bad) != 0;
    float m = 0.f;
#pragma unroll
    for (int p = 0; p < NP; p++) m = fmaxf(m, fmaxf(red[2 * sl + 4 * p], red[2 * sl + 1 + 4 * p]));
    return m;
}

}  // namespace

// CG: complex gate (SPECTRE_OPT_COMPLEX_GATE), else real.  NP: warps per TMEM
// lane quarter (the block has 128 NP threads; each row's 64 complex columns
// are split into NP parts of 64 / NP).
template <bool CG, int NP>
__global__ void __launch_bounds__(128 * NP, kBlocksPerSM) spectre_slices_mma4096(SliceArgs a) {
    using GateT = typename std::conditional<CG, float2, float>::type;
    constexpr int NT = 128 * NP;       // threads
    constexpr int NV = 64 / NP;        // complex values of a row per thread
    constexpr int NQ = NV / 16;        // 32-column TMEM blocks per thread (1 or 2)
    constexpr int GPP = NP / 2;        // parts per live k2 group in the pass-2 epilogues
    constexpr int GJ = 8 / GPP;        // complex values of a group per thread there
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *tile = smem;
    unsigned char *op = smem + kTileBytes;
    unsigned char *op2 = op + kOpBytes;
    const uint32_t *stage = reinterpret_cast<const uint32_t *>(op2 + kOp2Bytes);   // [2][4096] bf16 pairs
    uint64_t *mbar = reinterpret_cast<uint64_t *>(op2 + kOp2Bytes + kStageBytes);  // [0] MMA, [1] stage
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 2);    // [0] D, [1] S
    float *red = reinterpret_cast<float *>(tslot + 2);           // per-warp maxima

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, part = warp >> 2;
    const int trow = 32 * quarter + lane;                        // tile row = TMEM lane
    const int sl = trow >> 6, row = trow & 63, sbase = 64 * sl;
    const int gi = part / GPP, jsub = (part % GPP) * GJ;         // pass-2 group ordinal, first value

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
        for (int i = tid; i < (int)(kOpBytes / 16); i += NT) dst[i] = __ldg(src + i);
    }
    // per-row twiddle constants of the pass-1 epilogue: w4096^{row},
    // w4096^{16 row} and the start w4096^{NV part row}
    const float2 w1 = __ldg(a.twMM + 64 + row), w16 = __ldg(a.twMM + 16 * 64 + row);
    const float2 tq0 = part == 0 ? make_float2(1.f, 0.f) : __ldg(a.twMM + (NV * part) * 64 + row);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();

    Mma mma;
    mma.tile = tc::smem_u32(tile);
    mma.op = tc::smem_u32(op);
    mma.op2 = tc::smem_u32(op2);
    uint32_t op2_mask = 0;   // the groups whose operand rows op2 holds
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
                for (int m2 = NV * part; m2 < NV * part + NV; m2++) dst[2 * (row + 64 * m2)] = 0u;
                if (row == 0 && part == 0) a.pscale[2 * pslice + (c & 1)] = 1.0f;
            }
            if (tid == 0) stage_item(it + gridDim.x);
            continue;
        }
        // this thread's live k2 group in the pass-2 epilogues (ordinal gi among
        // the live groups), or -1
        int gmine = -1;
        {
            uint32_t gm = gmask;
            for (int i = 0; i < gi && gm; i++) gm &= gm - 1;
            if (gm) gmine = __ffs(gm) - 1;
        }
        // gather the live groups' operand rows for pass 2 (the previous
        // item's MMAs, the last readers, have completed; the first MMA
        // chain's proxy fence and barrier publish the copy)
        if (gmask != op2_mask) {
            for (int i = tid; i < __popc(gmask) * (int)(kGroupOpBytes / 16); i += NT) {
                const int gk = i / (int)(kGroupOpBytes / 16);
                uint32_t gm = gmask;
                for (int j = 0; j < gk; j++) gm &= gm - 1;
                const int g = __ffs(gm) - 1;
                reinterpret_cast<uint4 *>(op2)[i] = reinterpret_cast<const uint4 *>(
                    op + g * kGroupOpBytes)[i - gk * (int)(kGroupOpBytes / 16)];
            }
            op2_mask = gmask;
        }
        // this thread's gates, issued now and first used in the first pass-2
        // epilogue, so the loads are in flight through the q transform
        GateT graw[GJ];
#pragma unroll
        for (int j = 0; j < GJ; j++) {
            const int f = f1 + a.R * (row + 64 * (8 * (gmine < 0 ? 0 : gmine) + jsub + j));
            const int ff = min(f, a.L - f);
            const bool on = live && gmine >= 0 && ff < a.F;
            if constexpr (CG) graw[j] = on ? __ldg(reinterpret_cast<const float2 *>(Gh) + ff) : make_float2(0.f, 0.f);
            else graw[j] = on ? __ldg(Gh + ff) : 0.f;
        }

        int shift_sum = 0;   // sum of the applied input shifts of the four transforms
        float omax = 0.f;
#pragma unroll 1
        for (int sig = 0; sig < 3 && !abort; sig++) {
            // pass-1 input: row n2 = row holds a[64 n1 + row]; this thread
            // the n1 of its part, read from the staged rows
            {
                const bool ok = tc::mbar_wait(smbar, nused & 1u, mma.limit);
                if (ok) nused++;
                const uint32_t *src = stage + sl * kM + row + 64 * NV * part;
                // two passes over the staged values: the largest magnitude,
                // then (after the slice maximum) scale, round and store
                float mx = 0.f;
#pragma unroll
                for (int n = 0; n < NV; n++) {
                    const float2 v = bf2_to_f2(src[64 * n]);
                    mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
                }
                if (!live) mx = 0.f;
                bool bad;
                const int sh = scale_shift(slice_max<NP>(mx, red, warp, lane, sl, !ok, &bad));
                if (bad) {
                    abort = true;
                    break;
                }
#if SPECTRE_A_DISCARD
                if (tid < 256) {   // the staged rows are in shared memory: drop their lines from L2
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
                shift_sum += sh;
                const float s = live ? ldexpf(1.0f, sh) : 0.f;
#pragma unroll
                for (int j = 0; j < NV / 4; j++) {
                    const float2 v0 = bf2_to_f2(src[64 * (4 * j)]), v1 = bf2_to_f2(src[64 * (4 * j + 1)]);
                    const float2 v2 = bf2_to_f2(src[64 * (4 * j + 2)]), v3 = bf2_to_f2(src[64 * (4 * j + 3)]);
                    uint4 u;
                    u.x = h2_bits(v0.x * s, v0.y * s);
                    u.y = h2_bits(v1.x * s, v1.y * s);
                    u.z = h2_bits(v2.x * s, v2.y * s);
                    u.w = h2_bits(v3.x * s, v3.y * s);
                    *reinterpret_cast<uint4 *>(tile + tile_off(trow, 2 * NV * part + 8 * j)) = u;
                }
            }
            // after the chain's barrier every thread is done with the staged
            // rows: thread 0 stages the next signal, or the next item's q rows
            if (!mma.run(0xFFu, 0, true, [&] {
                    if (sig < 2)
                        stage_copy(it, sig + 1);
                    else
                        stage_item(it + gridDim.x);
                })) { abort = true; break; }
            twiddle_transpose<NQ>(tlD, w1, w16, tq0, tile, sbase, row, NQ * part);
            if (!mma.run(0xFFu, gmask, false)) { abort = true; break; }
            // pass-2 result: X[row + 64 k2] for this thread's values of its group
            if (gmine >= 0) {
                float d[2 * GJ], sv[2 * GJ];
                if constexpr (GJ == 8) {
                    tc::tmem_ld16(tlD + 16 * gi, d);
                    if (sig > 0) tc::tmem_ld16(tlS + 16 * gi, sv);
                } else {
                    tc::tmem_ld8(tlD + 16 * gi + 2 * jsub, d);
                    if (sig > 0) tc::tmem_ld8(tlS + 16 * gi + 2 * jsub, sv);
                }
#pragma unroll
                for (int j = 0; j < GJ; j++) {
                    const float2 X = make_float2(d[2 * j], d[2 * j + 1]);
                    float2 S;
                    if (sig == 0) {
                        if constexpr (CG) {   // conj(G[L - f]) above L/2
                            const int f = f1 + a.R * (row + 64 * (8 * gmine + jsub + j));
                            float2 gc = graw[j];
                            if (f > a.L - f) gc.y = -gc.y;
                            S = cmul(X, cscale(gc, a.invL));
                        } else {
                            S = cscale(X, graw[j] * a.invL);
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
                if constexpr (GJ == 8) tc::tmem_st16(tlS + 16 * gi, sv);
                else tc::tmem_st8(tlS + 16 * gi + 2 * jsub, sv);
            }
        }
        if (abort) break;

        // the final epilogue's twiddles w_L^{f1 (row + 1024 q)} and the step
        // w_L^{64 f1}, loaded while the inverse MMAs run
        const float2 step = __ldg(a.twL + 64 * f1);
        float2 tstart[NQ];
#pragma unroll
        for (int qq = 0; qq < NQ; qq++) tstart[qq] = __ldg(a.twL + f1 * (row + 1024 * (NQ * part + qq)));
        // inverse: conj(O) scaled into the tile rows (K steps of the live groups)
        {
            bool bad;
            const int sh = scale_shift(slice_max<NP>(omax, red, warp, lane, sl, false, &bad));
            shift_sum += sh;
            const float s = ldexpf(1.0f, sh);
            if (gmine >= 0) {
                float sv[2 * GJ];
                if constexpr (GJ == 8) tc::tmem_ld16(tlS + 16 * gi, sv);
                else tc::tmem_ld8(tlS + 16 * gi + 2 * jsub, sv);
#pragma unroll
                for (int hh = 0; hh < GJ / 4; hh++) {
                    uint4 u;
                    u.x = h2_bits(sv[8 * hh + 0] * s, -sv[8 * hh + 1] * s);
                    u.y = h2_bits(sv[8 * hh + 2] * s, -sv[8 * hh + 3] * s);
                    u.z = h2_bits(sv[8 * hh + 4] * s, -sv[8 * hh + 5] * s);
                    u.w = h2_bits(sv[8 * hh + 6] * s, -sv[8 * hh + 7] * s);
                    *reinterpret_cast<uint4 *>(tile + tile_off(trow, 16 * gmine + 2 * jsub + 8 * hh)) = u;
                }
            }
        }
        if (!mma.run(gmask, 0, true)) { abort = true; break; }
        twiddle_transpose<NQ>(tlD, w1, w16, tq0, tile, sbase, row, NQ * part);
        if (!mma.run(0xFFu, 0, true)) { abort = true; break; }

        // P[t2] = conj(U[t2] w_L^{f1 t2}) at t2 = row + 64 m2; the scale
        // gathers 4096 / s of each transform: 2^(48 - sum of shifts)
        {
            const int cc = live ? c : 0;
            const size_t pslice = p16_pair_slice(b, cc, f1, a.C, NF);
            uint32_t *dst = static_cast<uint32_t *>(a.P) + 2 * pslice * kM + (cc & 1);
            // w_L^{f1 t2} by recurrences in m2 (step w_L^{64 f1}) from
            // w_L^{f1 (row + 1024 q)}; within each 32-column block the second
            // 16-column TMEM load is in flight while the first is stored
#pragma unroll 1
            for (int qq = 0; qq < NQ; qq++) {
                const int q = NQ * part + qq;
                float2 t = tstart[qq];
                if constexpr (NQ == 2) {
                    uint32_t ra[16], rb[16];
                    tc::tmem_ld16_issue(tlD + 32 * q, ra);
                    tc::tmem_wait_ld16(ra);
                    tc::tmem_ld16_issue(tlD + 32 * q + 16, rb);
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const float2 u = cmul(make_float2(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1])), t);
                        if (live) dst[2 * (row + 64 * (16 * q + i))] = h2_bits(u.x, -u.y);
                        t = cmul(t, step);
                    }
                    tc::tmem_wait_ld16(rb);
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const float2 u = cmul(make_float2(__uint_as_float(rb[2 * i]), __uint_as_float(rb[2 * i + 1])), t);
                        if (live) dst[2 * (row + 64 * (16 * q + 8 + i))] = h2_bits(u.x, -u.y);
                        t = cmul(t, step);
                    }
                } else {
#pragma unroll 1
                    for (int hh = 0; hh < 2; hh++) {
                        float r[16];
                        tc::tmem_ld16(tlD + 32 * q + 16 * hh, r);
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            const float2 u = cmul(make_float2(r[2 * i], r[2 * i + 1]), t);
                            if (live) dst[2 * (row + 64 * (16 * q + 8 * hh + i))] = h2_bits(u.x, -u.y);
                            t = cmul(t, step);
                        }
                    }
                }
            }
            if (live && row == 0 && part == 0)
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

cudaError_t launch_slices_mma4096(const SliceArgs &a, cudaStream_t s) {
    const int NF = a.R / 2 + 1;
    const long long nitems = (long long)a.B * ((a.Cw + 1) / 2) * NF;
    if (nitems <= 0) return cudaSuccess;
    if (nitems >= (1LL << 31)) return cudaErrorInvalidValue;
    const long long cap = (long long)SPECTRE_SLICE_CTAS_PER_SM * (a.nsm > 0 ? a.nsm : 148);
    const unsigned grid = (unsigned)(nitems < cap ? nitems : cap);
    if (!a.a16) return cudaErrorInvalidValue;   // the pass reads bf16 A
    constexpr int NP = SPECTRE_SLICE_PARTS;
    auto k = a.cgate ? spectre_slices_mma4096<true, NP> : spectre_slices_mma4096<false, NP>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    prefer_max_smem(k);
    k<<<grid, 128 * NP, kSmemBytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace spectre
