// tc_dft.cuh -- a 16-point DFT on the 5th-generation tensor cores (tcgen05).
//
// Each of up to 128 rows of an fp16 operand tile A holds one length-16 complex
// input vector, K = 32 values interleaved as (re, im) of inputs 0..15.  The
// constant operand B is the DFT matrix w16^{sr} / 16 written as a real
// 32 x 32 matrix, so D = A B^T gives, per row, (re, im) of the 16 outputs in
// fp32 in tensor memory:
//   B[2s][2r] = Fr, B[2s][2r+1] = -Fi, B[2s+1][2r] = Fi, B[2s+1][2r+1] = Fr,
//   F = w16^{s r} / 16 (the 1/16 keeps every stage within fp16 range).
// Both tiles use the K-major, no-swizzle canonical layout: 8-row x 16-byte
// core matrices of 128 contiguous bytes, consecutive K chunks LBO = 128 bytes
// apart, consecutive 8-row groups SBO = 512 bytes apart.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spectre {
namespace tc {

constexpr uint32_t kLBO = 128;   // bytes between the 8-element K chunks
constexpr uint32_t kSBO = 512;   // bytes between 8-row groups (4 K chunks)
constexpr uint32_t kRowTile = 128 * 64;  // bytes of one 128-row, K = 32 tile

// byte offset of element (row, k) in a K = 32 canonical tile
__device__ __forceinline__ uint32_t tile_offset(uint32_t row, uint32_t k) {
    return (row >> 3) * kSBO + (k >> 3) * kLBO + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// shared-memory matrix descriptor: K-major, no swizzle, version 1
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((kLBO >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((kSBO >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;           // descriptor version for sm_100
    return d;                          // base offset 0, layout SWIZZLE_NONE
}

// instruction descriptor: kind::f16, A = B = fp16, D = fp32, both K-major,
// N = 32, M = 128
constexpr uint32_t kIdesc = (1u << 4)            // D format f32
                          | (0u << 7)            // A format f16
                          | (0u << 10)           // B format f16
                          | ((32u >> 3) << 17)   // N >> 3
                          | ((128u >> 4) << 24); // M >> 4

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :
                 : "r"(mbar)
                 : "memory");
}

__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" : : "r"(mbar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Wait for the mbarrier phase with parity `phase`; each poll may suspend the
// thread for up to kSuspendNs until the phase completes.  Gives up after
// `limit` polls and returns false (the caller records the timeout).
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t phase, uint32_t limit) {
    for (uint32_t i = 0; i < limit; i++) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(phase), "r"(kSuspendNs)
            : "memory");
        if (done) return true;
    }
    return false;
}

// one warp allocates ncols columns of tensor memory; the base lands in *slot
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :
                 : "r"(smem_u32(slot)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" : : "r"(base), "r"(ncols)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// Fill the 32 x 32 fp16 DFT16/16 operand (2 KB) in canonical layout; all
// threads of the block participate.  w16^e = cos(pi e / 8) - i sin(pi e / 8)
// comes from cos(pi m / 8), m = 0..4, by symmetry.
__device__ __forceinline__ float cos_pi8(int m) {  // cos(pi m / 8), m in [0, 16)
    const float c[5] = {1.0f, 0.92387953251128674f, 0.70710678118654752f,
                        0.38268343236508977f, 0.0f};
    m &= 15;
    if (m > 8) m = 16 - m;             // cos is even about pi
    return m <= 4 ? c[m] : -c[8 - m];  // cos(pi - x) = -cos(x)
}
__device__ __forceinline__ void fill_dft16_operand(unsigned char *b_tile) {
    for (int i = threadIdx.x; i < 32 * 32; i += blockDim.x) {
        const int n = i >> 5, k = i & 31;
        const int e = ((n >> 1) * (k >> 1)) & 15;
        const float cs = cos_pi8(e), sn = cos_pi8(e - 4);   // sin x = cos(x - pi/2)
        const float fr = cs * 0.0625f, fi = -sn * 0.0625f;
        float val;
        if ((n & 1) == 0)
            val = (k & 1) == 0 ? fr : -fi;
        else
            val = (k & 1) == 0 ? fi : fr;
        *reinterpret_cast<__half *>(b_tile + tile_offset(n, k)) = __float2half_rn(val);
    }
}

// Store this thread's 16 complex values (times s when SCALED) as row `row`
// of an A tile.
template <bool SCALED>
__device__ __forceinline__ void put_row(unsigned char *a_tile, uint32_t row, const float2 (&v)[16],
                                        float s) {
    auto h = [&](float2 x) {
        return SCALED ? __floats2half2_rn(x.x * s, x.y * s) : __floats2half2_rn(x.x, x.y);
    };
#pragma unroll
    for (int c = 0; c < 4; c++) {
        __half2 h0 = h(v[4 * c]);
        __half2 h1 = h(v[4 * c + 1]);
        __half2 h2 = h(v[4 * c + 2]);
        __half2 h3 = h(v[4 * c + 3]);
        uint4 u;
        u.x = *reinterpret_cast<uint32_t *>(&h0);
        u.y = *reinterpret_cast<uint32_t *>(&h1);
        u.z = *reinterpret_cast<uint32_t *>(&h2);
        u.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(a_tile + tile_offset(row, 8 * c)) = u;
    }
}

}  // namespace tc
}  // namespace spectre
