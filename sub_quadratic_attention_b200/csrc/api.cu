// api.cu -- the C ABI of libspectre_mix (declared in include/spectre_mix.h):
// argument validation, the plan (decomposition, twiddle tables, workspace)
// and the launch sequence.
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

struct spectre_mix_s {
    int device;
    int B, L, H, D, C, F, dtype;
    float eps;
    int R, M, NF;
    // device memory owned by the handle
    void *tables;       // twL followed by the slice tables
    float2 *twL;
    SliceTables tabs;
    float2 *A, *P;
    size_t table_bytes, ws_bytes;
    // geometry
    int T2C, ZS;         // inverse row pass
    int inv_reg;         // register-resident LayerNorm variant
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
    if (h->tables) cudaFree(h->tables);
    if (h->A) cudaFree(h->A);
    if (h->P) cudaFree(h->P);
    if (h->stage) cudaFree(h->stage);
    delete h;
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
    default: return "unknown status";
    }
}

int spectre_mix_create(spectre_mix_t *out, int B, int L, int H, int D, int F, int dtype, float eps) {
    if (!out) return SPECTRE_ERR_ARG;
    *out = nullptr;
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
    const size_t smem_max = 227 * 1024;
    if ((size_t)R * ZS * sizeof(float) > smem_max) return SPECTRE_ERR_ARG;
    if (fault_requested("alloc")) return SPECTRE_ERR_NOMEM;

    int dev = -1;
    int st = check_device(&dev);
    if (st != SPECTRE_OK) return st;

    spectre_mix_s *h = new (std::nothrow) spectre_mix_s();
    if (!h) return SPECTRE_ERR_NOMEM;
    h->device = dev;
    h->B = B; h->L = L; h->H = H; h->D = D; h->C = C; h->F = F; h->dtype = dtype; h->eps = eps;
    h->R = R; h->M = M; h->NF = NF;

    // ---- geometry
    // inverse row pass: register-resident LayerNorm when a block of
    // T2C x ceil(C/2) <= 1024 threads covers the channels; else the
    // shared-memory variant (R rows x T2C x padded C floats per block)
    const int CP = (C + 1) / 2;
    h->inv_reg = (R <= 16 && CP <= 1024) ? 1 : 0;
    int T2C;
    if (h->inv_reg) {
        T2C = 1;
        while (T2C < 8 && T2C * 2 * CP <= (CP > 512 ? 1024 : 512) && T2C * 2 <= M) T2C *= 2;
    } else {
        T2C = 8;
        while (T2C > 1 && (size_t)R * T2C * ZS * sizeof(float) > 160 * 1024) T2C /= 2;
    }
    h->T2C = T2C;
    h->ZS = ZS;

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
    h->twL = static_cast<float2 *>(h->tables);
    for (int d = 0; d < 2; d++)
        for (int p = 0; p < kMaxPasses; p++)
            h->tabs.tw[d][p] = (p > 0 && p < sch.n) ? h->twL + offs[d][p] : nullptr;

    // ---- workspace
    const size_t slice_elems = (size_t)B * C * NF * M;
    e = cudaMalloc(reinterpret_cast<void **>(&h->A), 3 * slice_elems * sizeof(float2));
    if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void **>(&h->P), slice_elems * sizeof(float2));
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    h->ws_bytes = 4 * slice_elems * sizeof(float2);
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto mark = [&](int i) -> cudaError_t {
        return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s) : cudaSuccess;
    };

    RowsFwdArgs fa;
    fa.q = q; fa.k = k; fa.v = v;
    fa.A = h->A;
    fa.twL = h->twL;
    fa.B = h->B; fa.L = h->L; fa.M = h->M; fa.C = h->C;
    fa.vec2 = (h->C % 2 == 0) ? 1 : 0;
    cudaError_t e = mark(0);
    if (e == cudaSuccess) e = launch_rows_fwd(h->R, h->dtype, fa, s);
    if (e != cudaSuccess) return cuda_status(e);

    SliceArgs sa;
    sa.A = h->A; sa.P = h->P; sa.twL = h->twL; sa.G = G; sa.tabs = h->tabs;
    sa.B = h->B; sa.L = h->L; sa.R = h->R; sa.M = h->M; sa.C = h->C; sa.D = h->D; sa.F = h->F;
    sa.nbins = h->L / 2 + 1;
    sa.nslices = (long long)h->B * h->C * h->NF;
    sa.invL = 1.0f / (float)h->L;
    e = mark(1);
    if (e == cudaSuccess) e = launch_slices(sa, s);
    if (e != cudaSuccess) return cuda_status(e);

    RowsInvArgs ia;
    ia.P = h->P; ia.x = x; ia.gamma = gamma; ia.beta = beta; ia.y = y; ia.out_f32 = out_f32;
    ia.B = h->B; ia.L = h->L; ia.M = h->M; ia.C = h->C;
    ia.T2C = h->T2C; ia.ZS = h->ZS; ia.eps = h->eps;
    ia.reg_variant = h->inv_reg;
    ia.vec2 = (h->C % 2 == 0) ? 1 : 0;
    e = mark(2);
    if (e == cudaSuccess) e = launch_rows_inv_ln(h->R, h->dtype, ia, s);
    if (e == cudaSuccess) e = mark(3);
    if (e != cudaSuccess) return cuda_status(e);
    return SPECTRE_OK;
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
                             void *y, void *const *events, void *stream) {
    if (!events || !events[0] || !events[1] || !events[2] || !events[3]) return SPECTRE_ERR_ARG;
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
    const size_t es = h->dtype == SPECTRE_F32 ? 4 : 2;
    const size_t nt = (size_t)h->B * h->L * h->C * es;
    const size_t ng = (size_t)h->H * (h->L / 2 + 1) * sizeof(float);
    const size_t nc = (size_t)h->C * sizeof(float);
    const size_t o_t = align_up(nt, 256), o_g = align_up(ng, 256), o_c = align_up(nc, 256);
    const size_t need = 5 * o_t + o_g + 2 * o_c;
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
    if (B < 1 || B > 65535 || H < 1 || D < 1 || L < 1) return SPECTRE_ERR_ARG;
    if (dtype != SPECTRE_F32 && dtype != SPECTRE_BF16) return SPECTRE_ERR_ARG;
    if (!(eps > 0.0f) || !std::isfinite(eps)) return SPECTRE_ERR_ARG;
    if ((long long)H * D > (1 << 20)) return SPECTRE_ERR_ARG;
    int R = 0, M = 0;
    if (!choose_split(L, &R, &M)) return SPECTRE_ERR_UNSUPPORTED_L;
    if (F < 1 || F > L / 2 + 1) return SPECTRE_ERR_ARG;
    const int C = H * D;
    const int NF = R / 2 + 1;
    const int ZS = (int)align_up((size_t)C, 32) + 16;
    if ((size_t)R * ZS * sizeof(float) > 227 * 1024) return SPECTRE_ERR_ARG;
    if (!q || !k || !v || !x || !G || !gamma || !beta || !y) return SPECTRE_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(x) || !aligned16(G) ||
        !aligned16(gamma) || !aligned16(beta) || !aligned16(y))
        return SPECTRE_ERR_ALIGN;

    // scratch layout: twiddle tables (as spectre_mix_create lays them out),
    // then A [3][B][C][NF][M] and P [B][C][NF][M], all fp32 complex
    const RadList sch = make_schedule(M);
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
    const size_t tab_bytes = align_up(n_tab * sizeof(float2), 256);
    const size_t slice_elems = (size_t)B * C * NF * M;
    const size_t need = tab_bytes + 4 * slice_elems * sizeof(float2);
    if (need > kNoAllocScratchBytes) return SPECTRE_ERR_SCRATCH;

    int dev = -1;
    int st = check_device(&dev);
    if (st != SPECTRE_OK) return st;
    if (fault_requested("launch")) return SPECTRE_ERR_CUDA;
    void *scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_status(e);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float2 *tw = static_cast<float2 *>(scratch);
    float2 *A = reinterpret_cast<float2 *>(static_cast<char *>(scratch) + tab_bytes);
    float2 *P = A + 3 * slice_elems;
    e = launch_make_tables(tw, segs, s);
    if (e != cudaSuccess) return cuda_status(e);

    SliceTables tabs;
    {
        int si = 1;
        for (int d = 0; d < 2; d++)
            for (int p = 0; p < kMaxPasses; p++)
                tabs.tw[d][p] = (p > 0 && p < sch.n) ? tw + segs.seg[si++].offset : nullptr;
    }
    const int CP = (C + 1) / 2;
    const int inv_reg = (R <= 16 && CP <= 1024) ? 1 : 0;
    int T2C;
    if (inv_reg) {
        T2C = 1;
        while (T2C < 8 && T2C * 2 * CP <= (CP > 512 ? 1024 : 512) && T2C * 2 <= M) T2C *= 2;
    } else {
        T2C = 8;
        while (T2C > 1 && (size_t)R * T2C * ZS * sizeof(float) > 160 * 1024) T2C /= 2;
    }

    RowsFwdArgs fa;
    fa.q = q; fa.k = k; fa.v = v; fa.A = A; fa.twL = tw;
    fa.B = B; fa.L = L; fa.M = M; fa.C = C;
    fa.vec2 = (C % 2 == 0) ? 1 : 0;
    e = launch_rows_fwd(R, dtype, fa, s);
    if (e != cudaSuccess) return cuda_status(e);

    SliceArgs sa;
    sa.A = A; sa.P = P; sa.twL = tw; sa.G = G; sa.tabs = tabs;
    sa.B = B; sa.L = L; sa.R = R; sa.M = M; sa.C = C; sa.D = D; sa.F = F;
    sa.nbins = L / 2 + 1;
    sa.nslices = (long long)B * C * NF;
    sa.invL = 1.0f / (float)L;
    e = launch_slices(sa, s);
    if (e != cudaSuccess) return cuda_status(e);

    RowsInvArgs ia;
    ia.P = P; ia.x = x; ia.gamma = gamma; ia.beta = beta; ia.y = y; ia.out_f32 = nullptr;
    ia.B = B; ia.L = L; ia.M = M; ia.C = C;
    ia.T2C = T2C; ia.ZS = ZS; ia.eps = eps;
    ia.reg_variant = inv_reg;
    ia.vec2 = (C % 2 == 0) ? 1 : 0;
    e = launch_rows_inv_ln(R, dtype, ia, s);
    if (e != cudaSuccess) return cuda_status(e);
    return SPECTRE_OK;
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

int spectre_mix_plan_info(spectre_mix_t h, int *R, int *M, int *slices_per_channel) {
    if (!h) return SPECTRE_ERR_ARG;
    if (R) *R = h->R;
    if (M) *M = h->M;
    if (slices_per_channel) *slices_per_channel = h->NF;
    return SPECTRE_OK;
}

}  // extern "C"
