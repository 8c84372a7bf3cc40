// api.cu -- the C ABI of libspectre_mix (declared in include/spectre_mix.h):
// argument validation, the plan (decomposition, twiddle tables, workspace)
// and the launch sequence.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/spectre_mix.h"
#include "kernels.cuh"

using namespace spectre;

// Shape, decomposition and launch geometry of one problem.
struct PathGeom {
    int B, L, H, D, C, F, dtype;
    float eps;
    int R, M, NF;
    int W;               // channels per wave (A of one wave kept in L2)
    int p16;             // P stored as fp16 with per-slice scales (bf16 I/O)
    int T2C, ZS;         // inverse row pass
    int inv_reg;         // register-resident LayerNorm variant
    int tc_mode;         // option: slice pass on the tensor cores where mma_ok (1) or CUDA cores (0)
    int norm_mode;       // option: enum spectre_norm
    int cgate;           // option: complex gate
    int mma_ok;          // the DFT-64 MMA slice pass applies (M = 4096, fp16 P, few live groups)
    int nsm;             // multiprocessors of the device
    int chunk;           // channels per pipeline chunk (multiple of 64, or C)
    size_t a_bytes, p_bytes, s_bytes;
};

// Device buffers the launch sequence works in.
struct PathBuffers {
    const float2 *twL;
    SliceTables tabs;
    const float2 *twMM;  // M = 4096: w_4096^{n2 k1} as [k1][n2]
    const void *w64op;   // M = 4096: the fp16 DFT-64 operand
    float2 *A;           // [3][B][W][NF][M]
    void *P;             // [B][C][NF][M] float2 or __half2
    float *pscale;       // [B][C][NF]
    int *err;            // device error word (bit 0: a tensor-core wait timed out)
};

struct spectre_mix_s {
    int device;
    PathGeom g;
    // second stream and fork/join events: the row pass of one channel chunk
    // overlaps the slice pass of the previous chunk
    cudaStream_t aux;
    cudaEvent_t ev_fork, ev_join;
    // device memory owned by the handle
    void *tables;       // twL followed by the slice tables
    void *ws;           // A, P, pscale
    PathBuffers bufs;
    size_t table_bytes, ws_bytes;
    // staging for spectre_mix_run_host, allocated on first use
    void *stage;
    size_t stage_bytes;
};

namespace {

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SPECTRE_OK;
    if (e == cudaErrorMemoryAllocation) return SPECTRE_ERR_NOMEM;
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver || e == cudaErrorInvalidDevice)
        return SPECTRE_ERR_DEVICE;
    return SPECTRE_ERR_CUDA;
}

bool fault_requested(const char *what) {
    const char *f = std::getenv("SPECTRE_MIX_FAULT");
    return f && std::strcmp(f, what) == 0;
}

bool is_pow2(long v) { return v > 0 && (v & (v - 1)) == 0; }

// L = R * M: R-point row transforms, M-point slice transforms.
bool choose_split(int L, int *R, int *M) {
    bool three = (L % 3 == 0);
    long p = three ? L / 3 : L;
    if (!is_pow2(p)) return false;
    if (!three && (L < 8 || L > (1 << 20))) return false;
    if (three && (L < 12 || L > 786432)) return false;
    int r;
    if (!three && L <= 16)
        r = L;
    else if (three && L == 12)
        r = 4;
    else if (three && L == 24)
        r = 8;
    else
        r = (L / 16 <= (three ? 12288 : 16384)) ? 16 : 64;
    *R = r;
    *M = L / r;
    return slice_length_supported(*M);
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device(int *dev_out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    if (major != 10) return SPECTRE_ERR_DEVICE;  // the library holds sm_100a code only
    *dev_out = dev;
    return SPECTRE_OK;
}

void free_handle(spectre_mix_s *h) {
    if (!h) return;
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->aux) cudaStreamDestroy(h->aux);
    if (h->tables) cudaFree(h->tables);
    if (h->ws) cudaFree(h->ws);
    if (h->stage) cudaFree(h->stage);
    delete h;
}

// Validate a shape and derive its geometry.  l2_bytes sizes the channel
// waves: one wave's A (3 signals x B x W channels x (R/2+1) x M complex fp32)
// is kept within half of L2 so the slice pass reads it back from L2.
int make_geom(int B, int L, int H, int D, int F, int dtype, float eps, size_t l2_bytes, PathGeom *g) {
    if (B < 1 || B > 65535 || H < 1 || D < 1 || L < 1) return SPECTRE_ERR_ARG;
    if (dtype != SPECTRE_F32 && dtype != SPECTRE_BF16) return SPECTRE_ERR_ARG;
    if (!(eps > 0.0f) || !std::isfinite(eps)) return SPECTRE_ERR_ARG;
    if ((long long)H * D > (1 << 20)) return SPECTRE_ERR_ARG;
    int R = 0, M = 0;
    if (!choose_split(L, &R, &M)) return SPECTRE_ERR_UNSUPPORTED_L;
    if (F < 1 || F > L / 2 + 1) return SPECTRE_ERR_ARG;
    const int C = H * D;
    const int NF = R / 2 + 1;
    // inverse row pass: R rows x T2C x padded C floats must fit one block's smem
    const int ZS = (int)align_up((size_t)C, 32) + 16;
    if ((size_t)R * ZS * sizeof(float) > 227 * 1024) return SPECTRE_ERR_ARG;
    g->B = B; g->L = L; g->H = H; g->D = D; g->C = C; g->F = F; g->dtype = dtype; g->eps = eps;
    g->R = R; g->M = M; g->NF = NF;
    g->ZS = ZS;
    g->p16 = dtype == SPECTRE_BF16 ? 1 : 0;
    // channel waves: with kWaveL2Fraction > 0, one wave's A is sized to that
    // fraction of L2 so the slice pass could read it back from L2.  Measured on
    // B200 for the bf16 long workload, waves were slower (each wave's grid
    // fills the SMs only ~1.2 times and L2 still wrote most of A back to
    // DRAM), so the plan uses a single wave.
    constexpr double kWaveL2Fraction = 0.0;
    const size_t per_ch = (size_t)3 * B * NF * M * sizeof(float2);
    const size_t budget = (size_t)(kWaveL2Fraction * (double)l2_bytes);
    int W = C;
    if (budget > 0 && per_ch * (size_t)C > budget) {
        size_t w = budget / per_ch;
        w -= w % 64;
        if (w >= 64) W = (int)w;
    }
    g->W = W;
    // inverse row pass: register-resident LayerNorm when a block of
    // T2C x ceil(C/2) <= 1024 threads covers the channels; else the
    // shared-memory variant (R rows x T2C x padded C floats per block)
    const int CP = (C + 1) / 2;
    g->inv_reg = (R <= 16 && CP <= 1024) ? 1 : 0;
    int T2C;
    if (g->inv_reg) {
        T2C = 1;
        while (T2C < 8 && T2C * 2 * CP <= (CP > 512 ? 1024 : 512) && T2C * 2 <= M) T2C *= 2;
    } else {
        T2C = 8;
        while (T2C > 1 && (size_t)R * T2C * ZS * sizeof(float) > 160 * 1024) T2C /= 2;
    }
    g->T2C = T2C;
    // tensor-core slice pass: M = 4096 as two DFT-64 MMA passes, for fp16 P,
    // when no slice has more than kMmaMaxGroups live k2 groups
    g->mma_ok = 0;
    if (M == 4096 && g->p16) {
        int worst = 0;
        for (int f1 = 0; f1 < NF; f1++) {
            int n = 0;
            for (int grp = 0; grp < 8; grp++) n += mma_group_live(grp, f1, R, L, F) ? 1 : 0;
            worst = n > worst ? n : worst;
        }
        g->mma_ok = worst <= kMmaMaxGroups ? 1 : 0;
    }
    g->tc_mode = 1;
    g->norm_mode = SPECTRE_NORM_POST_LN;
    g->cgate = 0;
    g->nsm = 148;
    // pipeline chunks: four channel chunks when each still fills the GPU
    g->chunk = C;
    if (W == C && C >= 256) g->chunk = (int)align_up((size_t)(C + 3) / 4, 64);
    const size_t slices = (size_t)B * C * NF;
    g->a_bytes = align_up((size_t)3 * B * W * NF * M * sizeof(float2), 256);
    // fp16 P interleaves channel pairs: 2 ceil(C / 2) channel lanes
    const size_t pslices = g->p16 ? (size_t)B * 2 * ((C + 1) / 2) * NF : slices;
    g->p_bytes = align_up(pslices * M * (g->p16 ? 4 : 8), 256);
    g->s_bytes = align_up(pslices * sizeof(float), 256) + 256;   // scales, then the error word
    return SPECTRE_OK;
}

// Whether the slice pass runs on the tensor cores (option on and the plan in
// the tensor-core kernel's range).
bool uses_mma(const PathGeom &g) { return g.tc_mode == 1 && g.mma_ok; }

// Channels per pipeline chunk.  Measured on B200 for the bf16 long workload:
// four chunks suit the CUDA-core slice pass (0.573 ms per mix against 0.60 ms
// unchunked); the tensor-core slice pass, whose blocks each carry a long
// chain of dependent phases, does best with two (0.454 ms against 0.460 with
// four and 0.464 unchunked), which keep more blocks per launch.
int chunk_channels(const PathGeom &g) {
    if (!uses_mma(g) || g.chunk >= g.W) return g.chunk;
    return (int)align_up((size_t)(g.C + 1) / 2, 64);
}

// The launch sequence of one mix.  Per channel chunk (within each wave) the
// row pass then the slice pass, then the inverse row pass with residual +
// LayerNorm.  Each chunk has its own region of A, so with an auxiliary stream
// the chunks alternate between `s` and `aux` and the row pass of chunk k + 1
// runs while the slice pass of chunk k does; `aux` forks from and joins back
// into `s`.  events (nullable, one per launch + 1) are recorded before every
// launch and after the last; with events the schedule is single-stream.
int launch_path(const PathGeom &g, const PathBuffers &bf, const void *q, const void *k, const void *v,
                const void *x, const float *G, const float *gamma, const float *beta, void *y,
                float *out_f32, void *const *events, cudaStream_t s, cudaStream_t aux,
                cudaEvent_t ev_fork, cudaEvent_t ev_join) {
    int ev = 0;
    auto mark = [&](cudaStream_t st) -> cudaError_t {
        return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), st) : cudaSuccess;
    };
    const int chunk = chunk_channels(g);
    const bool two = aux && !events && chunk < g.W;
    cudaError_t e = cudaSuccess;
    if (two) {
        e = cudaEventRecord(ev_fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(aux, ev_fork, 0);
        if (e != cudaSuccess) return cuda_status(e);
    }
    int idx = 0;
    for (int w_lo = 0; w_lo < g.C; w_lo += g.W) {
        const int w_hi = g.C - w_lo < g.W ? g.C : w_lo + g.W;
        for (int c_lo = w_lo; c_lo < w_hi; c_lo += chunk, idx++) {
            const int Cw = w_hi - c_lo < chunk ? w_hi - c_lo : chunk;
            cudaStream_t st = (two && (idx & 1)) ? aux : s;
            // this chunk's region of A: [3][B][Cw][NF][M] at its offset in the wave
            float2 *A = bf.A + (size_t)3 * g.B * (c_lo - w_lo) * g.NF * g.M;
            RowsFwdArgs fa;
            fa.q = q; fa.k = k; fa.v = v;
            fa.A = A;
            fa.twL = bf.twL;
            fa.B = g.B; fa.L = g.L; fa.M = g.M; fa.C = g.C;
            fa.c_lo = c_lo; fa.Cw = Cw;
            fa.vec2 = (g.C % 2 == 0) ? 1 : 0;
            fa.nsm = g.nsm;
            e = mark(st);
            if (e == cudaSuccess) e = launch_rows_fwd(g.R, g.dtype, fa, st);
            if (e != cudaSuccess) return cuda_status(e);

            SliceArgs sa;
            sa.A = A; sa.P = bf.P; sa.pscale = bf.pscale; sa.twL = bf.twL; sa.G = G; sa.tabs = bf.tabs;
            sa.B = g.B; sa.L = g.L; sa.R = g.R; sa.M = g.M; sa.C = g.C; sa.D = g.D; sa.F = g.F;
            sa.c_lo = c_lo; sa.Cw = Cw;
            sa.p16 = g.p16;
            sa.use_mma = uses_mma(g) ? 1 : 0;
            sa.nsm = g.nsm;
            sa.twMM = bf.twMM;
            sa.w64op = bf.w64op;
            sa.err = bf.err;
            sa.nbins = g.L / 2 + 1;
            sa.cgate = g.cgate;
            sa.nslices = (long long)g.B * Cw * g.NF;
            sa.invL = 1.0f / (float)g.L;
            e = mark(st);
            if (e == cudaSuccess) e = launch_slices(sa, st);
            if (e != cudaSuccess) return cuda_status(e);
        }
    }
    if (two) {
        e = cudaEventRecord(ev_join, aux);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_join, 0);
        if (e != cudaSuccess) return cuda_status(e);
    }
    RowsInvArgs ia;
    ia.P = bf.P; ia.pscale = bf.pscale;
    ia.x = x; ia.gamma = gamma; ia.beta = beta; ia.y = y; ia.out_f32 = out_f32;
    ia.B = g.B; ia.L = g.L; ia.M = g.M; ia.C = g.C;
    ia.T2C = g.T2C; ia.ZS = g.ZS; ia.eps = g.eps;
    ia.reg_variant = g.inv_reg;
    ia.vec2 = (g.C % 2 == 0) ? 1 : 0;
    ia.nsm = g.nsm;
    ia.norm = g.norm_mode;
    e = mark(s);
    if (e == cudaSuccess) e = launch_rows_inv_ln(g.R, g.dtype, ia, s);
    if (e == cudaSuccess) e = mark(s);
    if (e != cudaSuccess) return cuda_status(e);
    return SPECTRE_OK;
}

int launch_count(const PathGeom &g) {
    int n = 0;
    for (int w_lo = 0; w_lo < g.C; w_lo += g.W) {
        const int w_hi = g.C - w_lo < g.W ? g.C : w_lo + g.W;
        n += 2 * ((w_hi - w_lo + chunk_channels(g) - 1) / chunk_channels(g));
    }
    return n + 1;
}

size_t l2_size(int dev) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess || v <= 0) {
        cudaGetLastError();
        return (size_t)32 << 20;
    }
    return (size_t)v;
}

}  // namespace

extern "C" {

const char *spectre_mix_error_string(int code) {
    switch (code) {
    case SPECTRE_OK: return "ok";
    case SPECTRE_ERR_ARG: return "invalid argument (null pointer, size, F, dtype or eps)";
    case SPECTRE_ERR_UNSUPPORTED_L: return "unsupported L (need 2^k in [8, 2^20] or 3*2^k in [12, 786432])";
    case SPECTRE_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case SPECTRE_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
    case SPECTRE_ERR_NOMEM: return "out of memory";
    case SPECTRE_ERR_DEVICE: return "no usable sm_100 device, or the handle's device is not current";
    case SPECTRE_ERR_SCRATCH: return "problem needs more than the 64 MiB no-allocation scratch holds";
    case SPECTRE_ERR_TIMEOUT: return "a bounded wait on the tensor cores timed out; results of the run are invalid";
    default: return "unknown status";
    }
}

int spectre_mix_create(spectre_mix_t *out, int B, int L, int H, int D, int F, int dtype, float eps) {
    if (!out) return SPECTRE_ERR_ARG;
    *out = nullptr;
    PathGeom g;
    // validate with a provisional L2 size; the waves are re-derived below
    int st = make_geom(B, L, H, D, F, dtype, eps, (size_t)32 << 20, &g);
    if (st != SPECTRE_OK) return st;
    if (fault_requested("alloc")) return SPECTRE_ERR_NOMEM;

    int dev = -1;
    st = check_device(&dev);
    if (st != SPECTRE_OK) return st;
    make_geom(B, L, H, D, F, dtype, eps, l2_size(dev), &g);

    spectre_mix_s *h = new (std::nothrow) spectre_mix_s();
    if (!h) return SPECTRE_ERR_NOMEM;
    h->device = dev;
    h->g = g;
    const int M = g.M;

    // ---- twiddle tables (double on the host, stored fp32)
    const RadList sch = make_schedule(M);
    std::vector<float2> host;
    const size_t nL = (size_t)L / 2 + 1;
    host.resize(nL);
    for (size_t e = 0; e < nL; e++) {
        double ang = -2.0 * M_PI * (double)e / (double)L;
        host[e] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
    size_t offs[2][kMaxPasses] = {};
    for (int d = 0; d < 2; d++) {
        int ns = 1;
        for (int p = 0; p < sch.n; p++) {
            int r = d == 0 ? sch.r[p] : sch.r[sch.n - 1 - p];
            if (p > 0) {
                size_t base = align_up(host.size(), 2);
                host.resize(base);
                offs[d][p] = base;
                for (int rr = 0; rr < r; rr++)
                    for (int kk = 0; kk < ns; kk++) {
                        long long e = (long long)kk * rr;
                        double ang = -2.0 * M_PI * (double)e / (double)(ns * r);
                        host.push_back(make_float2((float)std::cos(ang), (float)std::sin(ang)));
                    }
            }
            ns *= r;
        }
    }
    // M = 4096: the twiddles between the two DFT-64 passes and the fp16
    // DFT-64 operand of the tensor-core slice pass
    size_t off_mm = 0, off_op = 0;
    if (M == 4096) {
        off_mm = align_up(host.size(), 2);
        host.resize(off_mm);
        for (int k1 = 0; k1 < 64; k1++)
            for (int n2 = 0; n2 < 64; n2++) {
                double ang = -2.0 * M_PI * (double)(n2 * k1) / 4096.0;
                host.push_back(make_float2((float)std::cos(ang), (float)std::sin(ang)));
            }
        off_op = align_up(host.size(), 2);
        host.resize(off_op + 4096);
        unsigned char *bytes = reinterpret_cast<unsigned char *>(host.data() + off_op);
        for (int n = 0; n < 128; n++)
            for (int kk = 0; kk < 128; kk++) {
                long long ee;
                int part;
                dft64_operand_angle(n, kk, &ee, &part);
                const double ang = -2.0 * M_PI * (double)ee / 64.0;
                const double val = (part == 0 || part == 3) ? std::cos(ang)
                                 : (part == 1 ? -std::sin(ang) : std::sin(ang));
                const __half hv = __float2half_rn((float)(val / 64.0));
                std::memcpy(bytes + dft64_operand_offset(n, kk), &hv, sizeof(hv));
            }
    }
    float2 w64[64];
    for (int e = 0; e < 64; e++) {
        double ang = -2.0 * M_PI * e / 64.0;
        w64[e] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }

    cudaError_t e;
    h->table_bytes = host.size() * sizeof(float2);
    e = cudaMalloc(&h->tables, h->table_bytes);
    if (e == cudaSuccess) e = cudaMemcpy(h->tables, host.data(), h->table_bytes, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = upload_w64(w64);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    h->bufs.twL = static_cast<float2 *>(h->tables);
    h->bufs.twMM = M == 4096 ? h->bufs.twL + off_mm : nullptr;
    h->bufs.w64op = M == 4096 ? static_cast<const void *>(h->bufs.twL + off_op) : nullptr;
    {
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
            h->g.nsm = nsm;
        cudaGetLastError();
    }
    for (int d = 0; d < 2; d++)
        for (int p = 0; p < kMaxPasses; p++)
            h->bufs.tabs.tw[d][p] = (p > 0 && p < sch.n) ? h->bufs.twL + offs[d][p] : nullptr;

    // ---- workspace: A of one wave, P, P scales
    h->ws_bytes = g.a_bytes + g.p_bytes + g.s_bytes;
    e = cudaMalloc(&h->ws, h->ws_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    char *base = static_cast<char *>(h->ws);
    h->bufs.A = reinterpret_cast<float2 *>(base);
    h->bufs.P = base + g.a_bytes;
    h->bufs.pscale = reinterpret_cast<float *>(base + g.a_bytes + g.p_bytes);
    h->bufs.err = reinterpret_cast<int *>(base + g.a_bytes + g.p_bytes + g.s_bytes - 256);
    e = cudaMemset(h->bufs.err, 0, sizeof(int));
    if (e == cudaSuccess && g.chunk < g.W) {
        e = cudaStreamCreateWithFlags(&h->aux, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    *out = h;
    return SPECTRE_OK;
}

static int run_impl(spectre_mix_t h, const void *q, const void *k, const void *v, const void *x,
                    const float *G, const float *gamma, const float *beta, void *y, float *out_f32,
                    void *const *events, void *stream) {
    if (!h) return SPECTRE_ERR_ARG;
    if (!q || !k || !v || !x || !G || !gamma || !beta || !y) return SPECTRE_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(x) || !aligned16(G) ||
        !aligned16(gamma) || !aligned16(beta) || !aligned16(y) || (out_f32 && !aligned16(out_f32)))
        return SPECTRE_ERR_ALIGN;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    if (fault_requested("launch")) return SPECTRE_ERR_CUDA;
    return launch_path(h->g, h->bufs, q, k, v, x, G, gamma, beta, y, out_f32, events,
                       static_cast<cudaStream_t>(stream), h->aux, h->ev_fork, h->ev_join);
}

int spectre_mix_run(spectre_mix_t h, const void *q, const void *k, const void *v, const void *x,
                    const float *G, const float *gamma, const float *beta, void *y, void *stream) {
    return run_impl(h, q, k, v, x, G, gamma, beta, y, nullptr, nullptr, stream);
}

int spectre_mix_run_debug(spectre_mix_t h, const void *q, const void *k, const void *v, const void *x,
                          const float *G, const float *gamma, const float *beta, void *y,
                          float *out_f32, void *stream) {
    return run_impl(h, q, k, v, x, G, gamma, beta, y, out_f32, nullptr, stream);
}

int spectre_mix_run_profiled(spectre_mix_t h, const void *q, const void *k, const void *v,
                             const void *x, const float *G, const float *gamma, const float *beta,
                             void *y, void *const *events, int nevents, void *stream) {
    if (!h || !events) return SPECTRE_ERR_ARG;
    const int need = launch_count(h->g) + 1;
    if (nevents != need) return SPECTRE_ERR_ARG;
    for (int i = 0; i < need; i++)
        if (!events[i]) return SPECTRE_ERR_ARG;
    return run_impl(h, q, k, v, x, G, gamma, beta, y, nullptr, events, stream);
}

int spectre_mix_run_host(spectre_mix_t h, const void *q, const void *k, const void *v, const void *x,
                         const float *G, const float *gamma, const float *beta, void *y, void *stream) {
    if (!h) return SPECTRE_ERR_ARG;
    if (!q || !k || !v || !x || !G || !gamma || !beta || !y) return SPECTRE_ERR_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    const PathGeom &g = h->g;
    const size_t es = g.dtype == SPECTRE_F32 ? 4 : 2;
    const size_t nt = (size_t)g.B * g.L * g.C * es;
    const size_t ng = (size_t)g.H * (g.L / 2 + 1) * sizeof(float) * (g.cgate ? 2 : 1);
    const size_t nc = (size_t)g.C * sizeof(float);
    const size_t o_t = align_up(nt, 256), o_g = align_up(ng, 256), o_c = align_up(nc, 256);
    const size_t need = 5 * o_t + o_g + 2 * o_c;
    if (h->stage && h->stage_bytes < need) {   // the gate grew (complex-gate option)
        cudaFree(h->stage);
        h->stage = nullptr;
        h->stage_bytes = 0;
    }
    if (!h->stage) {
        cudaError_t e = cudaMalloc(&h->stage, need);
        if (e != cudaSuccess) {
            cudaGetLastError();
            h->stage = nullptr;
            return cuda_status(e);
        }
        h->stage_bytes = need;
    }
    char *base = static_cast<char *>(h->stage);
    void *dq = base, *dk = base + o_t, *dv = base + 2 * o_t, *dx = base + 3 * o_t, *dy = base + 4 * o_t;
    float *dG = reinterpret_cast<float *>(base + 5 * o_t);
    float *dgam = reinterpret_cast<float *>(base + 5 * o_t + o_g);
    float *dbet = reinterpret_cast<float *>(base + 5 * o_t + o_g + o_c);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(dq, q, nt, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dk, k, nt, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dv, v, nt, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dx, x, nt, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dG, G, ng, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dgam, gamma, nc, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dbet, beta, nc, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    int st = run_impl(h, dq, dk, dv, dx, dG, dgam, dbet, dy, nullptr, nullptr, stream);
    if (st != SPECTRE_OK) return st;
    e = cudaMemcpyAsync(y, dy, nt, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    return SPECTRE_OK;
}

int spectre_mix_run_noalloc(int B, int L, int H, int D, int F, int dtype, float eps, const void *q,
                            const void *k, const void *v, const void *x, const float *G,
                            const float *gamma, const float *beta, void *y, void *stream) {
    // the same validation as spectre_mix_create and spectre_mix_run
    PathGeom g;
    int st = make_geom(B, L, H, D, F, dtype, eps, (size_t)32 << 20, &g);
    if (st != SPECTRE_OK) return st;
    if (!q || !k || !v || !x || !G || !gamma || !beta || !y) return SPECTRE_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(x) || !aligned16(G) ||
        !aligned16(gamma) || !aligned16(beta) || !aligned16(y))
        return SPECTRE_ERR_ALIGN;
    int dev = -1;
    st = check_device(&dev);
    if (st != SPECTRE_OK) return st;
    make_geom(B, L, H, D, F, dtype, eps, l2_size(dev), &g);

    // scratch layout: twiddle tables (as spectre_mix_create lays them out),
    // then A of one wave, P and the P scales
    const RadList sch = make_schedule(g.M);
    TableSegs segs;
    segs.n = 0;
    size_t n_tab = (size_t)L / 2 + 1;
    segs.seg[segs.n++] = TableSeg{0, (long long)n_tab, 0, (long long)L};
    for (int d = 0; d < 2; d++) {
        int ns = 1;
        for (int p = 0; p < sch.n; p++) {
            int r = d == 0 ? sch.r[p] : sch.r[sch.n - 1 - p];
            if (p > 0) {
                size_t base = align_up(n_tab, 2);
                segs.seg[segs.n++] = TableSeg{(long long)base, (long long)ns * r, (long long)ns,
                                              (long long)ns * r};
                n_tab = base + (size_t)ns * r;
            }
            ns *= r;
        }
    }
    long long seg_mm = -1, seg_op = -1;
    if (g.M == 4096) {
        size_t base = align_up(n_tab, 2);
        seg_mm = segs.n;
        segs.seg[segs.n++] = TableSeg{(long long)base, 4096, 64, 4096};
        base = align_up(base + 4096, 2);
        seg_op = segs.n;
        segs.seg[segs.n++] = TableSeg{(long long)base, 4096, -1, 64};
        n_tab = base + 4096;
    }
    const size_t tab_bytes = align_up(n_tab * sizeof(float2), 256);
    const size_t need = tab_bytes + g.a_bytes + g.p_bytes + g.s_bytes;
    if (need > kNoAllocScratchBytes) return SPECTRE_ERR_SCRATCH;
    if (fault_requested("launch")) return SPECTRE_ERR_CUDA;
    void *scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(scratch);
    PathBuffers bf;
    float2 *tw = reinterpret_cast<float2 *>(base);
    bf.twL = tw;
    bf.A = reinterpret_cast<float2 *>(base + tab_bytes);
    bf.P = base + tab_bytes + g.a_bytes;
    bf.pscale = reinterpret_cast<float *>(base + tab_bytes + g.a_bytes + g.p_bytes);
    bf.err = nullptr;   // no error word: the no-allocation path reports launch errors only
    bf.twMM = seg_mm >= 0 ? tw + segs.seg[seg_mm].offset : nullptr;
    bf.w64op = seg_op >= 0 ? static_cast<const void *>(tw + segs.seg[seg_op].offset) : nullptr;
    {
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
            g.nsm = nsm;
        cudaGetLastError();
    }
    {
        int si = 1;
        for (int d = 0; d < 2; d++)
            for (int p = 0; p < kMaxPasses; p++)
                bf.tabs.tw[d][p] = (p > 0 && p < sch.n) ? tw + segs.seg[si++].offset : nullptr;
    }
    e = launch_make_tables(tw, segs, s);
    if (e != cudaSuccess) return cuda_status(e);
    // single stream: this path creates no streams or events
    return launch_path(g, bf, q, k, v, x, G, gamma, beta, y, nullptr, nullptr, s, nullptr, nullptr,
                       nullptr);
}

int spectre_mix_set_option(spectre_mix_t h, int option, int value) {
    if (!h) return SPECTRE_ERR_ARG;
    switch (option) {
    case SPECTRE_OPT_TENSOR_CORES:
        if (value != 0 && value != 1) return SPECTRE_ERR_ARG;
        h->g.tc_mode = value;
        return SPECTRE_OK;
    case SPECTRE_OPT_COMPLEX_GATE:
        if (value != 0 && value != 1) return SPECTRE_ERR_ARG;
        h->g.cgate = value;
        return SPECTRE_OK;
    case SPECTRE_OPT_NORM:
        if (value < SPECTRE_NORM_POST_LN || value > SPECTRE_NORM_PRE_RMS) return SPECTRE_ERR_ARG;
        h->g.norm_mode = value;
        return SPECTRE_OK;
    default: return SPECTRE_ERR_ARG;
    }
}

int spectre_mix_slice_pass(spectre_mix_t h) {
    if (!h) return SPECTRE_ERR_ARG;
    return uses_mma(h->g) ? SPECTRE_SLICE_TENSOR_CORES : SPECTRE_SLICE_CUDA_CORES;
}

int spectre_mix_device_status(spectre_mix_t h, void *stream) {
    if (!h) return SPECTRE_ERR_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) {
        cudaGetLastError();
        return SPECTRE_ERR_DEVICE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, h->bufs.err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(h->bufs.err, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    return word ? SPECTRE_ERR_TIMEOUT : SPECTRE_OK;
}

int spectre_mix_destroy(spectre_mix_t h) {
    if (!h) return SPECTRE_OK;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(h->device);
    cudaError_t e = cudaDeviceSynchronize();
    free_handle(h);
    if (prev >= 0) cudaSetDevice(prev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    return SPECTRE_OK;
}

size_t spectre_mix_workspace_bytes(spectre_mix_t h) {
    if (!h) return 0;
    return h->table_bytes + h->ws_bytes + h->stage_bytes;
}

int spectre_mix_plan_info(spectre_mix_t h, int *R, int *M, int *slices_per_channel,
                          int *channels_per_wave, int *launches) {
    if (!h) return SPECTRE_ERR_ARG;
    if (R) *R = h->g.R;
    if (M) *M = h->g.M;
    if (slices_per_channel) *slices_per_channel = h->g.NF;
    if (channels_per_wave) *channels_per_wave = h->g.W;
    if (launches) *launches = launch_count(h->g);
    return SPECTRE_OK;
}

}  // extern "C"
