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
    int a16;             // A stored as bf16 (re, im) pairs (bf16 I/O, slice pass does not park in A)
    int regions;         // A regions: 1 (chunks run one after another and reuse it) or 2 (alternating streams)
    int p16;             // P stored as fp16 with per-slice scales (bf16 I/O)
    int T2C, ZS;         // inverse row pass
    int inv_reg;         // register-resident LayerNorm variant
    int tc_mode;         // option: slice pass on the tensor cores where mma_ok (1) or CUDA cores (0)
    int norm_mode;       // option: enum spectre_norm
    int cgate;           // option: complex gate
    int test_stall;      // option: the wait-timeout test (tensor-core slice pass)
    int row_tc;          // option: the row pass on the tensor cores where it applies
    int mma_ok;          // the DFT-64 MMA slice pass applies (M = 4096, fp16 P, few live groups)
    int nsm;             // multiprocessors of the device
    int chunk;           // channels per chunk (a multiple of 64, or C)
    size_t a_bytes, p_bytes, s_bytes;
};

// Device buffers the launch sequence works in.
struct PathBuffers {
    const float2 *twL;
    SliceTables tabs;
    const float2 *twMM;  // M = 4096: w_4096^{n2 k1} as [k1][n2]
    const void *w64op;   // M = 4096: the fp16 DFT-64 operand
    void *A;             // regions x [3][B][chunk][NF][M], float2 or bf16 pairs (a16)
    void *P;             // [B][C][NF][M] float2 or __half2
    float *pscale;       // [B][C][NF]
    int *err;            // device error word (bit 0: a tensor-core wait timed out)
};

// Streams of the chunk pipeline: chunk i runs on stream i % n (0: the
// caller's stream, k > 0: aux[k - 1]), so a region's next chunk follows its
// previous one in stream order.  ev_fork orders the aux streams after the
// caller's earlier work; ev_join[k] orders the caller's stream after aux[k].
constexpr int kMaxRegions = 4;
struct ChunkStreams {
    int n = 1;
    cudaStream_t aux[kMaxRegions - 1] = {};
    cudaEvent_t ev_fork = nullptr;
    cudaEvent_t ev_join[kMaxRegions - 1] = {};
};

struct spectre_mix_s {
    int device;
    PathGeom g;
    // one stream per A region beyond the first, with fork/join events: the
    // chunks of different regions overlap
    ChunkStreams cs;
    // device memory owned by the handle
    void *tables;       // twL followed by the slice tables
    void *ws;           // A, P, pscale
    PathBuffers bufs;
    size_t table_bytes, ws_bytes;
    // staging for spectre_mix_run_host, allocated on first use
    void *stage;
    size_t stage_bytes;
    // the step as a CUDA graph (SPECTRE_OPT_GRAPH): captured on `cap` for the
    // pointer set gkey, replayed on the caller's stream
    int use_graph;
    cudaStream_t cap;
    cudaGraphExec_t gexec;
    const void *gkey[8];
    int gvalid;
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

// Fraction of L2 that all regions' A together may fill.  Measured on B200:
// data written by one kernel and read back by the next comes entirely from
// L2 up to about 64 MB (of 126 MB) when nothing else streams through; in the
// mix the region being read is the one written one chunk earlier, and with
// 0.9 (two regions of 128 channels, 113 MB, for the bf16 long workload) the
// slice passes still read only 5 MB of DRAM per step.  0.9 against 0.45 (two
// regions of 64 channels): 0.3256 against 0.3297 ms per mix for the bf16 long
// workload, 1.420 against 1.435 ms for the mixed-radix one, the same time for
// the others.
#ifndef SPECTRE_L2_FRACTION
#define SPECTRE_L2_FRACTION 0.9
#endif
// Two regions let one chunk's row pass run beside the previous chunk's slice
// pass (measured on B200 for the bf16 long workload: 0.340 ms per mix with
// two regions of 64 channels against 0.366 ms with one of 128).
#ifndef SPECTRE_A_REGIONS
#define SPECTRE_A_REGIONS 2
#endif
// whether a handle replays its launches as a CUDA graph by default
// (SPECTRE_OPT_GRAPH; measured on B200: the same time for the bf16 long
// workload, 2-3 % less for the 65-launch mixed-radix step and fp32 mid)
#ifndef SPECTRE_GRAPH_DEFAULT
#define SPECTRE_GRAPH_DEFAULT 1
#endif
constexpr double kL2Fraction = SPECTRE_L2_FRACTION;
constexpr int kARegions = SPECTRE_A_REGIONS;
static_assert(kARegions >= 1 && kARegions <= 4, "one to four A regions");

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
    if (h->gexec) cudaGraphExecDestroy(h->gexec);
    if (h->cap) cudaStreamDestroy(h->cap);
    if (h->cs.ev_fork) cudaEventDestroy(h->cs.ev_fork);
    for (int i = 0; i < kMaxRegions - 1; i++) {
        if (h->cs.ev_join[i]) cudaEventDestroy(h->cs.ev_join[i]);
        if (h->cs.aux[i]) cudaStreamDestroy(h->cs.aux[i]);
    }
    if (h->tables) cudaFree(h->tables);
    if (h->ws) cudaFree(h->ws);
    if (h->stage) cudaFree(h->stage);
    delete h;
}

// Validate a shape and derive its geometry.  l2_bytes sizes the channel
// chunks: one chunk's A (3 signals x B x chunk channels x (R/2+1) x M complex
// values) is kept within a fraction of L2, so the slice pass reads A back
// from L2 and the next chunk's row pass overwrites those lines in L2 rather
// than DRAM receiving them.
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
    // A in bf16 pairs where the slice pass reads it (it parks its running
    // product in fp32 A only for the longest slices)
    g->a16 = (g->p16 && !slice_parks_in_A(M)) ? 1 : 0;
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
    if (M == 4096 && g->p16 && g->a16) {
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
    g->test_stall = 0;
    g->row_tc = 0;
    g->nsm = 148;
    // channel chunks: the largest multiple of 64 channels whose A fits the L2
    // budget (at least 64), all of C when that fits
    const size_t per_ch = (size_t)3 * B * NF * M * (g->a16 ? 4 : 8);
    const int regions = kARegions;
    const size_t budget = (size_t)(kL2Fraction * (double)l2_bytes) / (size_t)regions;
    int chunk = C;
    if (per_ch * (size_t)C > budget && C > 64) {
        size_t w = budget / per_ch;
        w -= w % 64;
        chunk = (int)(w < 64 ? 64 : w);
        if (chunk > C) chunk = C;
    }
    g->chunk = chunk;
    g->regions = chunk < C ? regions : 1;
    const size_t slices = (size_t)B * C * NF;
    g->a_bytes = align_up((size_t)g->regions * per_ch * (size_t)chunk, 256);
    // fp16 P interleaves channel pairs: 2 ceil(C / 2) channel lanes
    const size_t pslices = g->p16 ? (size_t)B * 2 * ((C + 1) / 2) * NF : slices;
    g->p_bytes = align_up(pslices * M * (g->p16 ? 4 : 8), 256);
    g->s_bytes = align_up(pslices * sizeof(float), 256) + 256;   // scales, then the error word
    return SPECTRE_OK;
}

// Layout of the plan's twiddle tables in one device buffer, as segments the
// table kernel fills (fp64 sincospi, stored fp32): the L-point table w_L^e
// (e <= L/2), the slice-pass tables of each pass and direction, and for
// M = 4096 the twiddles w_4096^{n2 k1} ([k1][n2]) and the fp16 DFT-64 operand.
// The handle and the no-allocation entry point use this one layout and the
// one kernel, so both compute bit-identical tables.
struct TableLayout {
    TableSegs segs;
    size_t bytes;        // rounded up to 256
    long long off_slice[2][kMaxPasses];
    long long off_mm, off_op;   // -1 when absent
};

TableLayout table_layout(const PathGeom &g) {
    TableLayout t;
    t.segs.n = 0;
    t.off_mm = t.off_op = -1;
    for (int d = 0; d < 2; d++)
        for (int p = 0; p < kMaxPasses; p++) t.off_slice[d][p] = -1;
    const RadList sch = make_schedule(g.M);
    size_t n = (size_t)g.L / 2 + 1;
    t.segs.seg[t.segs.n++] = TableSeg{0, (long long)n, 0, (long long)g.L};
    for (int d = 0; d < 2; d++) {
        int ns = 1;
        for (int p = 0; p < sch.n; p++) {
            const int r = d == 0 ? sch.r[p] : sch.r[sch.n - 1 - p];
            if (p > 0) {
                const size_t base = align_up(n, 2);
                t.off_slice[d][p] = (long long)base;
                t.segs.seg[t.segs.n++] = TableSeg{(long long)base, (long long)ns * r, (long long)ns,
                                                  (long long)ns * r};
                n = base + (size_t)ns * r;
            }
            ns *= r;
        }
    }
    if (g.M == 4096) {
        size_t base = align_up(n, 2);
        t.off_mm = (long long)base;
        t.segs.seg[t.segs.n++] = TableSeg{(long long)base, 4096, 64, 4096};
        base = align_up(base + 4096, 2);
        t.off_op = (long long)base;
        t.segs.seg[t.segs.n++] = TableSeg{(long long)base, 4096, -1, 64};
        n = base + 4096;
    }
    t.bytes = align_up(n * sizeof(float2), 256);
    return t;
}

// Table pointers of a plan whose tables start at tw.
void bind_tables(const TableLayout &t, float2 *tw, PathBuffers *bf) {
    bf->twL = tw;
    for (int d = 0; d < 2; d++)
        for (int p = 0; p < kMaxPasses; p++)
            bf->tabs.tw[d][p] = t.off_slice[d][p] >= 0 ? tw + t.off_slice[d][p] : nullptr;
    bf->twMM = t.off_mm >= 0 ? tw + t.off_mm : nullptr;
    bf->w64op = t.off_op >= 0 ? static_cast<const void *>(tw + t.off_op) : nullptr;
}

// exp(-2 pi i e / 64), e < 64, for the constant bank of the R = 64 kernels
void host_w64(float2 (&w64)[64]) {
    for (int e = 0; e < 64; e++) {
        double ang = -2.0 * M_PI * e / 64.0;
        w64[e] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
}

// Whether the slice pass runs on the tensor cores (option on and the plan in
// the tensor-core kernel's range).
bool uses_mma(const PathGeom &g) { return g.tc_mode == 1 && g.mma_ok; }

// The launch sequence of one mix: per channel chunk the row pass then the
// slice pass, then the inverse row pass with residual + LayerNorm.  With one
// A region the chunks run one after another on `s` and each overwrites the
// previous chunk's A (still in L2).  With n regions (and cs with n streams)
// chunk i uses region i % n on stream i % n, so the row passes of up to n - 1
// later chunks can run while a chunk's slice pass does, and a region is
// rewritten only after its previous chunk's slice pass (stream order).  The
// aux streams fork from and join back into `s`.  events (nullable, one per
// launch + 1) are recorded before every launch and after the last; with
// events the schedule is single-stream.
int launch_path(const PathGeom &g, const PathBuffers &bf, const void *q, const void *k, const void *v,
                const void *x, const float *G, const float *gamma, const float *beta, void *y,
                float *out_f32, void *const *events, cudaStream_t s, const ChunkStreams *cs) {
    int ev = 0;
    auto mark = [&](cudaStream_t st) -> cudaError_t {
        return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), st) : cudaSuccess;
    };
    const int chunk = g.chunk;
    const int nst = (cs && !events && cs->n == g.regions) ? g.regions : 1;
    const size_t region_elems = (size_t)3 * g.B * chunk * g.NF * g.M;
    const size_t elem = g.a16 ? 4 : 8;
    cudaError_t e = cudaSuccess;
    if (nst > 1) {
        e = cudaEventRecord(cs->ev_fork, s);
        for (int i = 0; i < nst - 1 && e == cudaSuccess; i++) e = cudaStreamWaitEvent(cs->aux[i], cs->ev_fork, 0);
        if (e != cudaSuccess) return cuda_status(e);
    }
    int idx = 0;
    for (int c_lo = 0; c_lo < g.C; c_lo += chunk, idx++) {
        const int Cw = g.C - c_lo < chunk ? g.C - c_lo : chunk;
        const int si = nst > 1 ? idx % nst : 0;
        cudaStream_t st = si == 0 ? s : cs->aux[si - 1];
        // this chunk's region of A: [3][B][Cw][NF][M]
        void *A = static_cast<char *>(bf.A) + (size_t)(idx % g.regions) * region_elems * elem;
        RowsFwdArgs fa;
        fa.q = q; fa.k = k; fa.v = v;
        fa.A = A;
        fa.a16 = g.a16;
        fa.twL = bf.twL;
        fa.B = g.B; fa.L = g.L; fa.M = g.M; fa.C = g.C;
        fa.c_lo = c_lo; fa.Cw = Cw;
        fa.vec2 = (g.C % 2 == 0) ? 1 : 0;
        fa.nsm = g.nsm;
        fa.err = bf.err;
        fa.row_tc = g.row_tc;
        e = mark(st);
        if (e == cudaSuccess) e = launch_rows_fwd(g.R, g.dtype, fa, st);
        if (e != cudaSuccess) return cuda_status(e);

        SliceArgs sa;
        sa.A = A; sa.a16 = g.a16;
        sa.P = bf.P; sa.pscale = bf.pscale; sa.twL = bf.twL; sa.G = G; sa.tabs = bf.tabs;
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
        sa.test_stall = g.test_stall;
        sa.nslices = (long long)g.B * Cw * g.NF;
        sa.invL = 1.0f / (float)g.L;
        e = mark(st);
        if (e == cudaSuccess) e = launch_slices(sa, st);
        if (e != cudaSuccess) return cuda_status(e);
    }
    for (int i = 0; i < nst - 1; i++) {
        e = cudaEventRecord(cs->ev_join[i], cs->aux[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, cs->ev_join[i], 0);
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
    ia.err = bf.err;
    e = mark(s);
    if (e == cudaSuccess) e = launch_rows_inv_ln(g.R, g.dtype, ia, s);
    if (e == cudaSuccess) e = mark(s);
    if (e != cudaSuccess) return cuda_status(e);
    return SPECTRE_OK;
}

int launch_count(const PathGeom &g) { return 2 * ((g.C + g.chunk - 1) / g.chunk) + 1; }

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
    case SPECTRE_ERR_TIMEOUT: return "a bounded wait on the tensor cores timed out; results of the run are invalid (y is NaN)";
    default: return "unknown status";
    }
}

int spectre_mix_create(spectre_mix_t *out, int B, int L, int H, int D, int F, int dtype, float eps) {
    if (!out) return SPECTRE_ERR_ARG;
    *out = nullptr;
    PathGeom g;
    // validate with a provisional L2 size; the chunks are re-derived below
    int st = make_geom(B, L, H, D, F, dtype, eps, (size_t)32 << 20, &g);
    if (st != SPECTRE_OK) return st;
    if (fault_requested("alloc")) return SPECTRE_ERR_NOMEM;

    int dev = -1;
    st = check_device(&dev);
    if (st != SPECTRE_OK) return st;
    make_geom(B, L, H, D, F, dtype, eps, l2_size(dev), &g);

    spectre_mix_s *h = new (std::nothrow) spectre_mix_s();
    if (!h) return SPECTRE_ERR_NOMEM;
    h->use_graph = SPECTRE_GRAPH_DEFAULT;
    h->device = dev;
    h->g = g;

    // ---- twiddle tables: fp64 on the device (the table kernel), stored fp32
    const TableLayout tl = table_layout(g);
    float2 w64[64];
    host_w64(w64);
    cudaError_t e;
    h->table_bytes = tl.bytes;
    e = cudaMalloc(&h->tables, h->table_bytes);
    if (e == cudaSuccess) e = launch_make_tables(static_cast<float2 *>(h->tables), tl.segs, 0);
    if (e == cudaSuccess) e = cudaStreamSynchronize(0);
    if (e == cudaSuccess) e = upload_w64(w64);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    bind_tables(tl, static_cast<float2 *>(h->tables), &h->bufs);
    {
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
            h->g.nsm = nsm;
        cudaGetLastError();
    }

    // ---- workspace: A (one or two chunk regions), P, P scales
    h->ws_bytes = g.a_bytes + g.p_bytes + g.s_bytes;
    e = cudaMalloc(&h->ws, h->ws_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    char *base = static_cast<char *>(h->ws);
    h->bufs.A = base;
    h->bufs.P = base + g.a_bytes;
    h->bufs.pscale = reinterpret_cast<float *>(base + g.a_bytes + g.p_bytes);
    h->bufs.err = reinterpret_cast<int *>(base + g.a_bytes + g.p_bytes + g.s_bytes - 256);
    e = cudaMemset(h->bufs.err, 0, sizeof(int));
    if (e == cudaSuccess && g.regions > 1) {
        e = cudaEventCreateWithFlags(&h->cs.ev_fork, cudaEventDisableTiming);
        for (int i = 0; i < g.regions - 1 && e == cudaSuccess; i++) {
            e = cudaStreamCreateWithFlags(&h->cs.aux[i], cudaStreamNonBlocking);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->cs.ev_join[i], cudaEventDisableTiming);
        }
        if (e == cudaSuccess) h->cs.n = g.regions;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_handle(h);
        return cuda_status(e);
    }
    *out = h;
    return SPECTRE_OK;
}

// One run as the handle's CUDA graph: captured (on the handle's own stream,
// so that the caller's stream may be the legacy default stream) when the
// pointer set or the plan changed since the last capture, then launched on
// the caller's stream.  A re-capture updates the executable graph in place
// where the topology allows, else re-instantiates it.
static int run_graph(spectre_mix_t h, const void *q, const void *k, const void *v, const void *x,
                     const float *G, const float *gamma, const float *beta, void *y, cudaStream_t s) {
    const void *key[8] = {q, k, v, x, G, gamma, beta, y};
    bool same = h->gvalid != 0;
    for (int i = 0; i < 8 && same; i++) same = key[i] == h->gkey[i];
    cudaError_t e = cudaSuccess;
    if (!same) {
        h->gvalid = 0;
        if (!h->cap) {
            e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking);
            if (e != cudaSuccess) {
                cudaGetLastError();
                h->cap = nullptr;
                return cuda_status(e);
            }
        }
        e = cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_status(e);
        }
        const int rc = launch_path(h->g, h->bufs, q, k, v, x, G, gamma, beta, y, nullptr, nullptr, h->cap,
                                   &h->cs);
        cudaGraph_t graph = nullptr;
        e = cudaStreamEndCapture(h->cap, &graph);
        if (rc != SPECTRE_OK || e != cudaSuccess) {
            if (graph) cudaGraphDestroy(graph);
            cudaGetLastError();
            return rc != SPECTRE_OK ? rc : cuda_status(e);
        }
        if (h->gexec) {
            cudaGraphExecUpdateResultInfo info;
            if (cudaGraphExecUpdate(h->gexec, graph, &info) != cudaSuccess) {
                cudaGetLastError();
                cudaGraphExecDestroy(h->gexec);
                h->gexec = nullptr;
            }
        }
        if (!h->gexec) e = cudaGraphInstantiate(&h->gexec, graph, 0);
        cudaGraphDestroy(graph);
        if (e != cudaSuccess) {
            cudaGetLastError();
            h->gexec = nullptr;
            return cuda_status(e);
        }
        for (int i = 0; i < 8; i++) h->gkey[i] = key[i];
        h->gvalid = 1;
    }
    e = cudaGraphLaunch(h->gexec, s);
    return cuda_status(e);
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
    if (h->use_graph && !events && !out_f32) {
        // a caller that is capturing its own graph gets the launches themselves
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess) {
            cudaGetLastError();
            cs = cudaStreamCaptureStatusActive;
        }
        if (cs == cudaStreamCaptureStatusNone)
            return run_graph(h, q, k, v, x, G, gamma, beta, y, static_cast<cudaStream_t>(stream));
    }
    return launch_path(h->g, h->bufs, q, k, v, x, G, gamma, beta, y, out_f32, events,
                       static_cast<cudaStream_t>(stream), &h->cs);
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

    // scratch layout: twiddle tables (the layout spectre_mix_create uses),
    // then A, P and the P scales
    const TableLayout tl = table_layout(g);
    const size_t need = tl.bytes + g.a_bytes + g.p_bytes + g.s_bytes;
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
    bind_tables(tl, tw, &bf);
    bf.A = base + tl.bytes;
    bf.P = base + tl.bytes + g.a_bytes;
    bf.pscale = reinterpret_cast<float *>(base + tl.bytes + g.a_bytes + g.p_bytes);
    bf.err = nullptr;   // no error word: a tensor-core wait that gives up poisons y with NaN
    {
        int nsm = 0;
        if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && nsm > 0)
            g.nsm = nsm;
        cudaGetLastError();
    }
    e = launch_make_tables(tw, tl.segs, s);
    if (e != cudaSuccess) return cuda_status(e);
    // single stream: this path creates no streams or events
    return launch_path(g, bf, q, k, v, x, G, gamma, beta, y, nullptr, nullptr, s, nullptr);
}

int spectre_mix_set_option(spectre_mix_t h, int option, int value) {
    if (!h) return SPECTRE_ERR_ARG;
    h->gvalid = 0;   // the plan may change: the next run captures again
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
    case SPECTRE_OPT_TEST_WAIT_TIMEOUT:
        if (value != 0 && value != 1) return SPECTRE_ERR_ARG;
        h->g.test_stall = value;
        return SPECTRE_OK;
    case SPECTRE_OPT_ROW_TENSOR_CORES:
        if (value != 0 && value != 1) return SPECTRE_ERR_ARG;
        h->g.row_tc = value;
        return SPECTRE_OK;
    case SPECTRE_OPT_GRAPH:
        if (value != 0 && value != 1) return SPECTRE_ERR_ARG;
        h->use_graph = value;
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
    if (channels_per_wave) *channels_per_wave = h->g.chunk;
    if (launches) *launches = launch_count(h->g);
    return SPECTRE_OK;
}

}  // extern "C"
