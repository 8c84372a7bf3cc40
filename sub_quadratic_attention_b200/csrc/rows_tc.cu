// rows_tc.cu -- the row pass for bf16 inputs with R = 16 on the tensor cores.
//
// What is computed is what spectre_rows_fwd_pipe computes (SPECTRE walk-through,
// hotelren.com/news/5925787, §2.2: the forward real FFT along L, here its first
// four-step stage):
//   A[f1][t2] = w_L^{f1 t2} sum_{t1 < 16} w16^{f1 t1} x[t1 M + t2],  f1 = 0..8,
// for every channel of the chunk, stored as bf16 (re, im) pairs.
//
// The 16-point DFT over t1 of real inputs is a real 16 x 16 matrix product: for
// each column (t2, c), D[n] = sum_t1 W[t1][n] x[t1] with n = 0: Re X0, 1: Re X8,
// 2f: Re Xf, 2f + 1: Im Xf (f = 1..7); the imaginary parts of X0 and X8 are 0.
// One work item is 16 t2 x 64 channels of one signal.  A 4-D TMA box
// {64 channels, 16 t1, 16 t2, 1 batch row} with 128-byte swizzling lands in
// shared memory exactly in the tensor cores' MN-major layout (the 64 channels
// of one t2 as one 128-byte row per t1; the next t2 2 KB further on), so the
// MMA reads the inputs as loaded: 8 MMAs of M = 128 (64 channels at t2 = j
// and j + 8), N = 16, K = 16, each issued twice, with W rounded to bf16 (hi)
// and the remainder W - hi (lo) accumulated into the same fp32 result, so the
// transform's coefficients are exact to about 2^-17.  The epilogue reads
// each thread's TMEM lane (one channel at 8 consecutive t2), multiplies by the
// twiddles w_L^{f1 t2} (a per-item table in shared memory), rounds to bf16
// pairs and stages them so that every store to A is 16 contiguous bytes.
//
// Waits on the TMA and MMA mbarriers are bounded; a block whose wait gives up
// sets bit 0 of the device error word, fills A of its unfinished items with NaN
// (so y of the run is NaN), waits (bounded) for its own copies and MMAs in
// flight, releases its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "fft_regs.cuh"
#include "kernels.cuh"
#include "tc_dft.cuh"

namespace spectre {
namespace {

constexpr int kRT2 = 16;                          // t2 per item
constexpr int kRCB = 64;                          // channels per item
constexpr int kRThreads = 128;
constexpr uint32_t kRInBytes = kRCB * 16 * kRT2 * 2;   // 32 KB per input buffer
constexpr uint32_t kRWBytes = 512;                     // one 16 x 16 bf16 operand
constexpr uint32_t kRTwBytes = 8 * kRT2 * 8;           // w_L^{f1 t2}, f1 = 1..8, one item's t2
constexpr size_t kRSmemBytes = 1024 + 2 * kRInBytes + 2 * kRWBytes + 2 * kRTwBytes + 64;
constexpr uint32_t kRWaitLimit = 1u << 12;

struct RowsTcMaps {
    CUtensorMap m[3];   // q, k, v
};

// shared-memory descriptor of a 128-byte-swizzled operand (layout type 2)
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return tc::make_desc(saddr, lbo, sbo) | ((uint64_t)2 << 61);
}

// kind::f16 with bf16 A (MN-major) and bf16 B (K-major), fp32 D, M = 128, N = 16
constexpr uint32_t kRIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((16u >> 3) << 17) |
                             ((128u >> 4) << 24);

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            int c3, uint32_t mbar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar),
          "l"(pol)
        : "memory");
}

__device__ __forceinline__ uint32_t bf2_bits(float x, float y) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}

}  // namespace

__global__ void __launch_bounds__(kRThreads, 2) spectre_rows_fwd_tc(const __grid_constant__ RowsTcMaps maps,
                                                                    RowsFwdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    const uint32_t raw = tc::smem_u32(smem_raw);
    unsigned char *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    unsigned char *in0 = base;                               // [2][t2 16][t1 16][64 c] bf16, swizzled
    unsigned char *whi = base + 2 * kRInBytes;
    unsigned char *wlo = whi + kRWBytes;
    float2 *tw = reinterpret_cast<float2 *>(wlo + kRWBytes);   // [2 items][8 f1 - 1][16 t2]
    uint64_t *mbar = reinterpret_cast<uint64_t *>(reinterpret_cast<unsigned char *>(tw) + 2 * kRTwBytes);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mbar + 3);   // mbar: [0], [1] input buffers, [2] MMA

    const int tid = threadIdx.x, warp = tid >> 5;
    const int ntile = a.M / kRT2, ncb = a.Cw / kRCB;
    const int per_sig = a.B * ntile * ncb;
    const int nitems = 3 * per_sig;   // < 2^31 (checked by the launcher)
    constexpr int NF = 9;

    if (warp == 0) {
        tc::tmem_alloc_keep(&tslot[0], 128);
        tc::tmem_relinquish();
    }
    if (tid == 0)
        for (int i = 0; i < 3; i++) tc::mbar_init(tc::smem_u32(mbar + i), 1);
    // W[t1][n] as the B operand (n rows, K = t1), K-major, core matrices of
    // 8 rows x 16 bytes: (n, k) at (n / 8) 256 + (k / 8) 128 + (n % 8) 16 + (k % 8) 2
    for (int e = tid; e < 256; e += kRThreads) {
        const int n = e >> 4, k = e & 15;
        double w;
        if (n == 0) w = 1.0;
        else if (n == 1) w = (k & 1) ? -1.0 : 1.0;
        else {
            const int f = n >> 1;
            double sn, cs;
            sincospi((double)((f * k) & 15) / 8.0, &sn, &cs);
            w = (n & 1) ? -sn : cs;
        }
        const __nv_bfloat16 hi = __double2bfloat16(w);
        const __nv_bfloat16 lo = __double2bfloat16(w - (double)__bfloat162float(hi));
        const int off = (n >> 3) * 256 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
        *reinterpret_cast<__nv_bfloat16 *>(whi + off) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(wlo + off) = lo;
    }
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t dcol = tslot[0];
    const uint32_t uin = tc::smem_u32(in0), uwhi = tc::smem_u32(whi), uwlo = tc::smem_u32(wlo);
    const uint64_t pol_in = [] {
        uint64_t p;
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
        return p;
    }();
    const uint64_t pol_a = [] {
        uint64_t p;
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
        return p;
    }();

    // item = ((sig B + b) ntile + tile) ncb + cb
    auto decode = [&](int item, int &sig, int &b, int &tile, int &cb) {
        sig = item / per_sig;
        int r = item - sig * per_sig;
        cb = r % ncb;
        r /= ncb;
        tile = r % ntile;
        b = r / ntile;
    };
    auto issue_tma = [&](int item, int buf) {
        int sig, b, tile, cb;
        decode(item, sig, b, tile, cb);
        const uint32_t mb = tc::smem_u32(mbar + buf);
        tc::mbar_arrive_expect_tx(mb, kRInBytes);
        tma_load_4d(uin + buf * kRInBytes, &maps.m[sig], a.c_lo + cb * kRCB, 0, tile * kRT2, b, mb, pol_in);
    };
    auto issue_mma = [&](int buf) {
        tc::fence_after();
        const uint32_t ab = uin + buf * kRInBytes;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const uint64_t ad = desc_sw128(ab + 2048 * j, 16384, 1024);
            tc::mma_f16(dcol + 16 * j, ad, tc::make_desc(uwhi, 128, 256), kRIdesc, 0);
            tc::mma_f16(dcol + 16 * j, ad, tc::make_desc(uwlo, 128, 256), kRIdesc, 1);
        }
        tc::commit(tc::smem_u32(mbar + 2));
    };

    bool late = false;
    // (thread 0) copies issued into / waited for on each input buffer, MMA
    // chains committed; (every thread) MMA chains waited for
    uint32_t nissue[2] = {0, 0}, nfull[2] = {0, 0}, ncommit = 0, nmma = 0;
    int it = blockIdx.x;
    if (tid == 0) {
        if (it < nitems) { issue_tma(it, 0); nissue[0]++; }
        if (it + (int)gridDim.x < nitems) { issue_tma(it + gridDim.x, 1); nissue[1]++; }
        if (it < nitems) {
            late = !tc::mbar_wait(tc::smem_u32(mbar), 0, kRWaitLimit);
            if (!late) { nfull[0]++; issue_mma(0); ncommit++; }
        }
    }
    const int c = tid & 63, h = tid >> 6;   // this thread's channel and t2 half
    const uint32_t tl = dcol + ((uint32_t)(32 * warp) << 16);
    // this thread's entry of an item's twiddle table: w_L^{f1 t2}, f1 = 1 + tid / 16
    const int twf1 = 1 + (tid >> 4), twt = tid & 15;
    auto tw_entry = [&](int item) -> float2 {
        int sig, b, tile, cb;
        decode(item, sig, b, tile, cb);
        return __ldg(a.twL + twf1 * (tile * kRT2 + twt));
    };
    if (it < nitems) tw[tid] = tw_entry(it);
    __syncthreads();
    int k = 0;
    int done = it;   // first item this block has not finished
#pragma unroll 1
    for (; it < nitems; it += gridDim.x, k++) {
        int sig, b, tile, cb;
        decode(it, sig, b, tile, cb);
        const int t20 = tile * kRT2;
        const int nit = it + gridDim.x;
        // the next item's twiddle entry, in flight while this item is processed
        const float2 twn = nit < nitems ? tw_entry(nit) : make_float2(0.f, 0.f);
        if (tc::mbar_wait(tc::smem_u32(mbar + 2), nmma & 1, kRWaitLimit)) nmma++;
        else late = true;
        tc::fence_after();
        // the MMA has read buffer k & 1: refill it two items ahead
        if (tid == 0 && !late && it + 2 * (int)gridDim.x < nitems) {
            issue_tma(it + 2 * gridDim.x, k & 1);
            nissue[k & 1]++;
        }
        // a wait that gave up is acted on uniformly at the end of the item (the
        // item is then not counted done, so the abort path fills it with NaN)
        const float2 *twk = tw + (k & 1) * (8 * kRT2);
        // this thread's channel c at t2 = t20 + 8 h + j: 16 TMEM columns per j,
        // loaded four j at a time with one wait
        uint32_t outv[9][8];
#pragma unroll
        for (int jb = 0; jb < 8; jb += 4) {
            uint32_t r[4][16];
#pragma unroll
            for (int jj = 0; jj < 4; jj++) tc::tmem_ld16_issue(tl + 16 * (jb + jj), r[jj]);
#pragma unroll
            for (int jj = 0; jj < 4; jj++) tc::tmem_wait_ld16(r[jj]);
#pragma unroll
            for (int jj = 0; jj < 4; jj++) {
                const int j = jb + jj, tt = 8 * h + j;
                const float *d = reinterpret_cast<const float *>(r[jj]);
                outv[0][j] = bf2_bits(d[0], 0.f);
#pragma unroll
                for (int f = 1; f < 8; f++) {
                    const float2 y = cmul(make_float2(d[2 * f], d[2 * f + 1]), twk[(f - 1) * kRT2 + tt]);
                    outv[f][j] = bf2_bits(y.x, y.y);
                }
                const float2 w8 = twk[7 * kRT2 + tt];
                outv[8][j] = bf2_bits(d[1] * w8.x, d[1] * w8.y);
            }
        }
        // A[sig][b][c_chunk][f1][t2]: this thread's 8 consecutive t2 of each
        // slice are one 32-byte sector
        uint32_t *A = static_cast<uint32_t *>(a.A);
        const size_t crow = ((size_t)(sig * a.B + b) * a.Cw + (size_t)cb * kRCB + c) * NF;
#pragma unroll
        for (int f = 0; f < NF; f++) {
            uint32_t *dst = A + (crow + f) * a.M + t20 + 8 * h;
            asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;"
                         :
                         : "l"(dst), "r"(outv[f][0]), "r"(outv[f][1]), "r"(outv[f][2]), "r"(outv[f][3]), "l"(pol_a)
                         : "memory");
            asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;"
                         :
                         : "l"(dst + 4), "r"(outv[f][4]), "r"(outv[f][5]), "r"(outv[f][6]), "r"(outv[f][7]),
                           "l"(pol_a)
                         : "memory");
        }
        tw[((k + 1) & 1) * (8 * kRT2) + tid] = twn;
        tc::fence_before();
        // every TMEM read of this item done, the next twiddle table written
        if (__syncthreads_or(late)) break;
        done = nit;
        if (tid == 0 && nit < nitems) {
            const int nb = (k + 1) & 1;
            if (tc::mbar_wait(tc::smem_u32(mbar + nb), nfull[nb] & 1, kRWaitLimit)) {
                nfull[nb]++;
                issue_mma(nb);
                ncommit++;
            } else {
                late = true;
            }
        }
    }
    if (__syncthreads_or(late)) {
        if (tid == 0) {
            if (a.err) atomicOr(a.err, 1);
            // copies and MMAs this block still has in flight (at most one each)
            for (int bb = 0; bb < 2; bb++)
                if (nissue[bb] > nfull[bb]) tc::mbar_wait(tc::smem_u32(mbar + bb), nfull[bb] & 1, kRWaitLimit);
            if (ncommit > nmma) tc::mbar_wait(tc::smem_u32(mbar + 2), nmma & 1, kRWaitLimit);
        }
        // this block's unfinished items: A = NaN, so the run's y is NaN
        uint32_t *A = static_cast<uint32_t *>(a.A);
        for (int j = done; j < nitems; j += gridDim.x) {
            int sig, b, tile, cb;
            decode(j, sig, b, tile, cb);
            const size_t cbase = ((size_t)(sig * a.B + b) * a.Cw + (size_t)cb * kRCB) * NF;
            for (int e = tid; e < kRCB * NF * kRT2; e += kRThreads) {
                const int tt = e & 15, rowi = e >> 4;
                A[(cbase + rowi) * a.M + tile * kRT2 + tt] = 0x7fc07fc0u;
            }
        }
        __syncthreads();
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tslot[0], 128);
    }
}

namespace {
std::mutex g_encode_mutex;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encode(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
    std::lock_guard<std::mutex> lock(g_encode_mutex);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode;
    return cudaSuccess;
}
}  // namespace

bool rows_tc_applies(const RowsFwdArgs &a) {
    return a.a16 && a.vec2 && a.C % 64 == 0 && a.c_lo % 64 == 0 && a.Cw % 64 == 0 && a.M % kRT2 == 0 &&
           3LL * a.B * (a.M / kRT2) * (a.Cw / kRCB) < (1LL << 31);
}

cudaError_t launch_rows_fwd_tc(const RowsFwdArgs &a, cudaStream_t s) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    cudaError_t e = get_encode(&encode);
    if (e != cudaSuccess) return e;
    RowsTcMaps maps;
    const void *src[3] = {a.q, a.k, a.v};
    // dims (channel, t1, t2, batch row); strides in bytes of dims 1..3
    const cuuint64_t dims[4] = {(cuuint64_t)a.C, 16, (cuuint64_t)a.M, (cuuint64_t)a.B};
    const cuuint64_t strides[3] = {(cuuint64_t)a.M * a.C * 2, (cuuint64_t)a.C * 2, (cuuint64_t)a.L * a.C * 2};
    const cuuint32_t box[4] = {kRCB, 16, kRT2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    for (int i = 0; i < 3; i++) {
        CUresult r = encode(&maps.m[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(src[i]), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const long long nitems = 3LL * a.B * (a.M / kRT2) * (a.Cw / kRCB);
    if (nitems <= 0) return cudaSuccess;
    cudaFuncSetAttribute(spectre_rows_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRSmemBytes);
    const long long cap = 2LL * (a.nsm > 0 ? a.nsm : 148);
    spectre_rows_fwd_tc<<<(unsigned)(nitems < cap ? nitems : cap), kRThreads, kRSmemBytes, s>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace spectre
