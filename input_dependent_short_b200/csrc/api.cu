// C entry points of libdsc.so: argument checks, then dispatch to the kernels.
// The contract of every function is in include/dsc.h.
#include <atomic>
#include <mutex>

#include "edges.cuh"

namespace dsc {

static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsc_status validate(const dsc_problem *p, bool lowrank) {
    if (!p) return DSC_ERR_INVALID_ARG;
    if (p->B < 1 || p->T < 1 || p->D < 1 || p->W < 1 || p->W > 8 || p->H < 1) return DSC_ERR_INVALID_ARG;
    if (p->D % p->H) return DSC_ERR_INVALID_ARG;
    if (p->dtype != DSC_F32 && p->dtype != DSC_BF16) return DSC_ERR_INVALID_ARG;
    if (p->T > (int64_t)1 << 30 || p->B > (int64_t)1 << 30) return DSC_ERR_UNSUPPORTED;
    if (lowrank && (p->R < 1 || p->R > 256)) return DSC_ERR_INVALID_ARG;
    return DSC_OK;
}

static dsc_status check_ptrs(std::initializer_list<const void *> ptrs) {
    for (const void *q : ptrs)
        if (!q) return DSC_ERR_INVALID_ARG;
    for (const void *q : ptrs)
        if (!aligned16(q)) return DSC_ERR_MISALIGNED;
    return DSC_OK;
}

static int sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;
    }
    std::lock_guard<std::mutex> g(mu);
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

static Ctx ctx(void *stream) { return Ctx{static_cast<cudaStream_t>(stream), sm_count()}; }

static dsc_status done(cudaError_t e) { return e == cudaSuccess ? DSC_OK : DSC_ERR_CUDA; }

static GenArgs gen_args(const dsc_problem &p, int wmode) {
    GenArgs a{};
    a.B = p.B; a.T = p.T; a.D = p.D; a.H = p.H; a.G = p.D / p.H;
    a.W = (int)p.W;
    a.residual = p.residual ? 1 : 0;
    a.wmode = wmode;
    return a;
}

static dsc_problem static_view(const dsc_problem &p) {
    dsc_problem q = p;
    q.H = 1;  // one filter per channel
    return q;
}

static size_t lr_generic_fwd_bytes(const dsc_problem &p) {
    return (size_t)(p.B * p.T) * (size_t)((p.D / p.H) * p.W) * sizeof(float);
}

// decode.cu: one decode step (mode 0 head-wise filters [B,G,W] in the input
// dtype, 1 low-rank filters as fp32 [B,G,W], 2 static [D,W]), the state taken
// from the last W-1 tokens of a prompt [B,T,D], and the low-rank step with the
// token's filters formed on chip (tensor cores, or CUDA cores for shapes with
// D a multiple of the vector width and H dividing or divided by it).
cudaError_t launch_decode(const Ctx &c, const dsc_problem &p, int mode, const void *x, const void *w, void *state,
                          void *y);
cudaError_t launch_decode_state(const Ctx &c, const dsc_problem &p, const void *x, void *state);
bool decode_lowrank_fused_ok(const dsc_problem &p);
cudaError_t launch_decode_lowrank_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z,
                                        const void *U, void *state, void *y);
// lowrank_tc_dec.cu: the tensor-core decode's plan and the status word of its bounded waits
bool decode_lowrank_tc_ok(const dsc_problem &p);
int take_tc_dec_status(cudaStream_t stream);

}  // namespace dsc

using namespace dsc;

extern "C" {

int dsc_version(void) { return 100; }

uint64_t dsc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *dsc_status_string(dsc_status s) {
    switch (s) {
    case DSC_OK: return "ok";
    case DSC_ERR_INVALID_ARG: return "invalid argument";
    case DSC_ERR_UNSUPPORTED: return "unsupported problem";
    case DSC_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case DSC_ERR_CUDA: return "CUDA error";
    case DSC_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

dsc_status dsc_fwd_headwise(const dsc_problem *p, const void *x, const void *w, void *y, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_ptrs({x, w, y});
    if (s != DSC_OK) return s;
    const Ctx c = ctx(stream);
    HwArgs a{};
    if (stream_plan(*p, a.m)) {
        a.x = x; a.w = w; a.y = y;
        return done(launch_hw_fwd(c, *p, a));
    }
    GenArgs g = gen_args(*p, WMODE_HEADWISE);
    g.x = x; g.w = w; g.y = y;
    return done(launch_gen_fwd(c, *p, g, false));
}

dsc_status dsc_bwd_headwise(const dsc_problem *p, const void *x, const void *w, const void *dy, void *dx, void *dw,
                            void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_ptrs({x, w, dy, dx, dw});
    if (s != DSC_OK) return s;
    const Ctx c = ctx(stream);
    HwArgs a{};
    if (stream_plan(*p, a.m)) {
        a.x = x; a.w = w; a.dy = dy; a.dx = dx; a.dw = dw;
        return done(launch_hw_bwd(c, *p, a));
    }
    GenArgs g = gen_args(*p, WMODE_HEADWISE);
    g.x = x; g.w = w; g.dy = dy; g.dx = dx; g.dw = dw;
    cudaError_t e = launch_gen_dx(c, *p, g, false);
    if (e == cudaSuccess) e = launch_gen_dw(c, *p, g, false);
    return done(e);
}

dsc_status dsc_fwd_static(const dsc_problem *p, const void *x, const void *ws, void *y, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_ptrs({x, ws, y});
    if (s != DSC_OK) return s;
    const dsc_problem q = static_view(*p);
    const Ctx c = ctx(stream);
    HwArgs a{};
    if (stream_plan(q, a.m)) {
        a.x = x; a.w = ws; a.y = y;
        return done(launch_st_fwd(c, q, a));
    }
    GenArgs g = gen_args(q, WMODE_STATIC);
    g.x = x; g.w = ws; g.y = y;
    return done(launch_gen_fwd(c, q, g, false));
}

size_t dsc_bwd_static_workspace_bytes(const dsc_problem *p) {
    if (validate(p, false) != DSC_OK) return 0;
    const dsc_problem q = static_view(*p);
    StreamMap m;
    size_t parts;
    if (stream_plan(q, m)) parts = st_partial_count(ctx(nullptr), q);
    else parts = (size_t)(q.B * ((q.T + 63) / 64));
    return parts * (size_t)(q.D * q.W) * sizeof(float);
}

dsc_status dsc_bwd_static(const dsc_problem *p, const void *x, const void *ws, const void *dy, void *dx, float *dws,
                          void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_ptrs({x, ws, dy, dx, dws, workspace});
    if (s != DSC_OK) return s;
    if (workspace_bytes < dsc_bwd_static_workspace_bytes(p)) return DSC_ERR_INVALID_ARG;
    const dsc_problem q = static_view(*p);
    const Ctx c = ctx(stream);
    HwArgs a{};
    if (stream_plan(q, a.m)) {
        a.x = x; a.w = ws; a.dy = dy; a.dx = dx;
        a.partial = static_cast<float *>(workspace);
        return done(launch_st_bwd(c, q, a, dws));
    }
    GenArgs g = gen_args(q, WMODE_STATIC);
    g.x = x; g.w = ws; g.dy = dy; g.dx = dx;
    cudaError_t e = launch_gen_dx(c, q, g, false);
    if (e == cudaSuccess) e = launch_gen_dws(c, q, g, dws, static_cast<float *>(workspace), 0);
    return done(e);
}

int dsc_lowrank_kernels(const dsc_problem *p, int backward) {
    if (validate(p, true) != DSC_OK) return -1;
    if (backward == 2) {  // decode step
        if (p->T != 1) return -1;
        if (decode_lowrank_tc_ok(*p)) return DSC_LR_TENSOR_CORE;
        return decode_lowrank_fused_ok(*p) ? DSC_LR_FUSED : DSC_LR_UNFUSED;
    }
    if (backward ? lowrank_tc_bwd_ok(*p, sm_count()) : lowrank_tc_ok(*p)) return DSC_LR_TENSOR_CORE;
    if (lowrank_fused_ok(*p)) return DSC_LR_FUSED;
    return DSC_LR_UNFUSED;
}

size_t dsc_fwd_lowrank_workspace_bytes(const dsc_problem *p) {
    if (validate(p, true) != DSC_OK) return 0;
    if (lowrank_tc_ok(*p)) return lr_tc_fwd_ws_bytes(*p);
    if (lowrank_fused_ok(*p)) return 0;
    return lr_generic_fwd_bytes(*p);
}

size_t dsc_bwd_lowrank_workspace_bytes(const dsc_problem *p) {
    if (validate(p, true) != DSC_OK) return 0;
    if (lowrank_tc_bwd_ok(*p, sm_count())) return lr_tc_bwd_ws_bytes(*p, sm_count());
    if (lowrank_fused_ok(*p)) return lr_bwd_fused_ws_bytes(ctx(nullptr), *p);
    return 2 * lr_generic_fwd_bytes(*p);
}

dsc_status dsc_fwd_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, void *y,
                           void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_ptrs({x, z, U, y});
    if (s != DSC_OK) return s;
    const Ctx c = ctx(stream);
    if (lowrank_tc_ok(*p)) {
        const size_t need = lr_tc_fwd_ws_bytes(*p);
        if (need && (!workspace || workspace_bytes < need)) return DSC_ERR_INVALID_ARG;
        if (need && !aligned16(workspace)) return DSC_ERR_MISALIGNED;
        return done(launch_lr_fwd_tc(c, *p, x, z, U, y, workspace, workspace_bytes));
    }
    if (lowrank_fused_ok(*p)) return done(launch_lr_fwd_fused(c, *p, x, z, U, y));
    // Unfused fallback: filters w = zU in the workspace, then the per-channel kernel.
    if (!workspace) return DSC_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return DSC_ERR_MISALIGNED;
    if (workspace_bytes < lr_generic_fwd_bytes(*p)) return DSC_ERR_INVALID_ARG;
    float *wf = static_cast<float *>(workspace);
    cudaError_t e = launch_lr_filters(c, *p, z, U, wf);
    GenArgs g = gen_args(*p, WMODE_HEADWISE);
    g.x = x; g.w = wf; g.y = y;
    if (e == cudaSuccess) e = launch_gen_fwd(c, *p, g, true);
    return done(e);
}

dsc_status dsc_bwd_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, const void *dy,
                           void *dx, void *dz, float *dU, void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_ptrs({x, z, U, dy, dx, dz, dU});
    if (s != DSC_OK) return s;
    const size_t need = dsc_bwd_lowrank_workspace_bytes(p);
    if (need && (!workspace || workspace_bytes < need)) return DSC_ERR_INVALID_ARG;
    if (need && !aligned16(workspace)) return DSC_ERR_MISALIGNED;
    const Ctx c = ctx(stream);
    if (lowrank_tc_bwd_ok(*p, c.sms))
        return done(launch_lr_bwd_tc(c, *p, x, z, U, dy, dx, dz, dU, workspace, workspace_bytes));
    if (lowrank_fused_ok(*p)) return done(launch_lr_bwd_fused(c, *p, x, z, U, dy, dx, dz, dU, workspace, workspace_bytes));
    // Unfused fallback: w = zU and dw in the workspace; dz = dw U^T; dU = z^T dw.
    const int64_t N = p->B * p->T, GW = (p->D / p->H) * p->W;
    float *wf = static_cast<float *>(workspace);
    float *dwf = wf + N * GW;
    const bool bf = p->dtype == DSC_BF16;
    cudaError_t e = launch_lr_filters(c, *p, z, U, wf);
    GenArgs g = gen_args(*p, WMODE_HEADWISE);
    g.x = x; g.w = wf; g.dy = dy; g.dx = dx; g.dw = dwf;
    if (e == cudaSuccess) e = launch_gen_dx(c, *p, g, true);
    if (e == cudaSuccess) e = launch_gen_dw(c, *p, g, true);
    if (e == cudaSuccess)  // dz[n][r] = sum_j dw[n][j] U[r][j]
        e = launch_gemm(c, (int)N, (int)p->R, (int)GW, dwf, true, GW, 1, U, !bf, GW, 1, dz, !bf, p->R, bf);
    if (e == cudaSuccess)  // dU[r][j] = sum_n z[n][r] dw[n][j]
        e = launch_gemm(c, (int)p->R, (int)GW, (int)N, z, !bf, 1, p->R, dwf, true, 1, GW, dU, true, GW, bf);
    return done(e);
}

// ------------------------------------------------------------------ decode ---

static dsc_status validate_decode(const dsc_problem *p, bool lowrank) {
    dsc_status s = validate(p, lowrank);
    if (s == DSC_OK && p->T != 1) s = DSC_ERR_INVALID_ARG;
    return s;
}

static dsc_status check_state(const dsc_problem *p, const void *state) {
    return p->W > 1 ? check_ptrs({state}) : DSC_OK;
}

dsc_status dsc_decode_headwise(const dsc_problem *p, const void *x, const void *w, void *state, void *y,
                               void *stream) {
    dsc_status s = validate_decode(p, false);
    if (s == DSC_OK) s = check_ptrs({x, w, y});
    if (s == DSC_OK) s = check_state(p, state);
    if (s != DSC_OK) return s;
    return done(launch_decode(ctx(stream), *p, 0, x, w, state, y));
}

dsc_status dsc_decode_static(const dsc_problem *p, const void *x, const void *ws, void *state, void *y,
                             void *stream) {
    dsc_status s = validate_decode(p, false);
    if (s == DSC_OK) s = check_ptrs({x, ws, y});
    if (s == DSC_OK) s = check_state(p, state);
    if (s != DSC_OK) return s;
    return done(launch_decode(ctx(stream), *p, 2, x, ws, state, y));
}

size_t dsc_decode_lowrank_workspace_bytes(const dsc_problem *p) {
    if (validate_decode(p, true) != DSC_OK || decode_lowrank_fused_ok(*p)) return 0;
    return (size_t)p->B * (size_t)(p->D / p->H) * (size_t)p->W * sizeof(float);
}

dsc_status dsc_decode_lowrank(const dsc_problem *p, const void *x, const void *z, const void *U, void *state, void *y,
                              void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate_decode(p, true);
    if (s == DSC_OK) s = check_ptrs({x, z, U, y});
    if (s == DSC_OK) s = check_state(p, state);
    if (s != DSC_OK) return s;
    const Ctx c = ctx(stream);
    if (decode_lowrank_fused_ok(*p)) return done(launch_decode_lowrank_fused(c, *p, x, z, U, state, y));
    // other shapes: the token's filters through a scratch
    s = check_ptrs({workspace});
    if (s != DSC_OK) return s;
    if (workspace_bytes < dsc_decode_lowrank_workspace_bytes(p)) return DSC_ERR_INVALID_ARG;
    float *wf = static_cast<float *>(workspace);
    cudaError_t e = launch_lr_filters(c, *p, z, U, wf);  // w[b, g*W+k] = z_b . U[:, g*W+k]
    if (e == cudaSuccess) e = launch_decode(c, *p, 1, x, wf, state, y);
    return done(e);
}

dsc_status dsc_decode_state(const dsc_problem *p, const void *x, void *state, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_ptrs({x});
    if (s == DSC_OK) s = check_state(p, state);
    if (s != DSC_OK) return s;
    return done(launch_decode_state(ctx(stream), *p, x, state));
}

// ------------------------------------------- packed documents and chunks ---

static size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

static dsc_status check_varlen(const dsc_problem *p, const int32_t *cu, int64_t n_docs) {
    if (p->B != 1 || n_docs < 1 || !cu) return DSC_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(cu) & 3u) return DSC_ERR_MISALIGNED;
    // the fix-up grids have one block per (edge row, 256 channels)
    if (n_docs * (p->W - 1) * ((p->D + 255) / 256) >= ((int64_t)1 << 31)) return DSC_ERR_UNSUPPORTED;
    return DSC_OK;
}

static dsc_status check_chunk(const dsc_problem *p) {
    if (p->B * (p->W - 1) * ((p->D + 255) / 256) >= ((int64_t)1 << 31)) return DSC_ERR_UNSUPPORTED;
    return DSC_OK;
}

// Halo pointers of a chunk: present ones must be 16-byte aligned; the filters
// of the next tokens must come with their dy.
static dsc_status check_halos(const dsc_problem *p, const void *x_prev, const void *dy_next, const void *f_next,
                              bool needs_f) {
    if (p->W < 2) return DSC_OK;
    for (const void *q : {x_prev, dy_next, f_next})
        if (q && !aligned16(q)) return DSC_ERR_MISALIGNED;
    if (dy_next && needs_f && !f_next) return DSC_ERR_INVALID_ARG;
    return DSC_OK;
}

static EdgeArgs varlen_edges(const dsc_problem &p, int kind, const int32_t *cu, int64_t n_docs) {
    EdgeArgs a{};
    edge_args(p, kind, a);
    a.cu = cu;
    a.nseg = n_docs;
    a.early = 1;  // every packed-document call runs the row pass first
    return a;
}

static EdgeArgs chunk_edges(const dsc_problem &p, int kind, const void *x_prev, const void *dy_next,
                            const void *f_next, int edges_only) {
    EdgeArgs a{};
    edge_args(p, kind, a);
    a.early = !edges_only;
    a.cu = nullptr;
    a.nseg = p.B;
    if (p.W > 1) {
        a.x_prev = x_prev;
        a.dy_next = dy_next;
        a.f_next = f_next;
    }
    return a;
}

static dsc_status edges_fwd(void *stream, const dsc_problem *p, EdgeArgs a) {
    if (a.nseg < 1 || p->W < 2) return DSC_OK;
    if (!a.cu && !a.x_prev) return DSC_OK;  // a sequence's first chunk: the plain call is the whole result
    return done(launch_edges_fwd(ctx(stream), *p, a));
}

static dsc_status edges_bwd(void *stream, const dsc_problem *p, EdgeArgs a) {
    if (a.nseg < 1 || p->W < 2) return DSC_OK;
    if (!a.cu && !a.x_prev && !a.dy_next) return DSC_OK;
    return done(launch_edges_bwd(ctx(stream), *p, a));
}

dsc_status dsc_fwd_headwise_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                   const void *w, void *y, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = dsc_fwd_headwise(p, x, w, y, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = varlen_edges(*p, EDGE_HEADWISE, cu_seqlens, n_docs);
    a.x = x; a.w = w; a.y = y;
    return edges_fwd(stream, p, a);
}

dsc_status dsc_bwd_headwise_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                   const void *w, const void *dy, void *dx, void *dw, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = dsc_bwd_headwise(p, x, w, dy, dx, dw, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = varlen_edges(*p, EDGE_HEADWISE, cu_seqlens, n_docs);
    a.x = x; a.w = w; a.dy = dy; a.dx = dx; a.dw = dw;
    return edges_bwd(stream, p, a);
}

dsc_status dsc_fwd_lowrank_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                  const void *z, const void *U, void *y, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = dsc_fwd_lowrank(p, x, z, U, y, workspace, workspace_bytes, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = varlen_edges(*p, EDGE_LOWRANK, cu_seqlens, n_docs);
    a.x = x; a.z = z; a.U = U; a.y = y;
    return edges_fwd(stream, p, a);
}

size_t dsc_bwd_lowrank_varlen_workspace_bytes(const dsc_problem *p, int64_t n_docs) {
    if (validate(p, true) != DSC_OK || n_docs < 1) return 0;
    return up256(dsc_bwd_lowrank_workspace_bytes(p)) + edge_scratch_bytes(*p, EDGE_LOWRANK, n_docs);
}

// Low-rank backward with fix-ups: the plain call's workspace first, then the
// fix-up scratch (dw rows of the fixed tokens and their cross-edge part).
static dsc_status lowrank_bwd_edges(const dsc_problem *p, EdgeArgs a, const void *x, const void *z, const void *U,
                                    const void *dy, void *dx, void *dz, float *dU, void *workspace,
                                    size_t workspace_bytes, size_t main_bytes, bool run_main, void *stream) {
    const size_t edge = edge_scratch_bytes(*p, EDGE_LOWRANK, a.nseg);
    const size_t off = run_main ? up256(main_bytes) : 0;
    if ((off + edge) && (!workspace || workspace_bytes < off + edge)) return DSC_ERR_INVALID_ARG;
    if ((off + edge) && !aligned16(workspace)) return DSC_ERR_MISALIGNED;
    if (run_main) {
        const dsc_status s = dsc_bwd_lowrank(p, x, z, U, dy, dx, dz, dU, main_bytes ? workspace : nullptr, main_bytes,
                                             stream);
        if (s != DSC_OK) return s;
    }
    a.x = x; a.z = z; a.U = U; a.dy = dy; a.dx = dx; a.dz = dz; a.dU = dU;
    if (edge) {
        a.dwfull = reinterpret_cast<float *>(static_cast<char *>(workspace) + off);
        a.dwdelta = a.dwfull + edge / (2 * sizeof(float));
    }
    return edges_bwd(stream, p, a);
}

dsc_status dsc_bwd_lowrank_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                  const void *z, const void *U, const void *dy, void *dx, void *dz, float *dU,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = check_ptrs({x, z, U, dy, dx, dz, dU});
    if (s != DSC_OK) return s;
    return lowrank_bwd_edges(p, varlen_edges(*p, EDGE_LOWRANK, cu_seqlens, n_docs), x, z, U, dy, dx, dz, dU,
                             workspace, workspace_bytes, dsc_bwd_lowrank_workspace_bytes(p), true, stream);
}

dsc_status dsc_fwd_static_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                 const void *ws, void *y, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = dsc_fwd_static(p, x, ws, y, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = varlen_edges(*p, EDGE_STATIC, cu_seqlens, n_docs);
    a.x = x; a.w = ws; a.y = y;
    return edges_fwd(stream, p, a);
}

dsc_status dsc_bwd_static_varlen(const dsc_problem *p, const int32_t *cu_seqlens, int64_t n_docs, const void *x,
                                 const void *ws, const void *dy, void *dx, float *dws, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_varlen(p, cu_seqlens, n_docs);
    if (s == DSC_OK) s = dsc_bwd_static(p, x, ws, dy, dx, dws, workspace, workspace_bytes, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = varlen_edges(*p, EDGE_STATIC, cu_seqlens, n_docs);
    a.x = x; a.w = ws; a.dy = dy; a.dx = dx; a.dws = dws;
    return edges_bwd(stream, p, a);
}

dsc_status dsc_fwd_headwise_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *w, void *y,
                                  int edges_only, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, w, y});
    if (s == DSC_OK) s = check_halos(p, x_prev, nullptr, nullptr, false);
    if (s == DSC_OK && !edges_only) s = dsc_fwd_headwise(p, x, w, y, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = chunk_edges(*p, EDGE_HEADWISE, x_prev, nullptr, nullptr, edges_only);
    a.x = x; a.w = w; a.y = y;
    return edges_fwd(stream, p, a);
}

dsc_status dsc_bwd_headwise_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next, const void *w_next,
                                  const void *x, const void *w, const void *dy, void *dx, void *dw, int edges_only,
                                  void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, w, dy, dx, dw});
    if (s == DSC_OK) s = check_halos(p, x_prev, dy_next, w_next, true);
    if (s == DSC_OK && !edges_only) s = dsc_bwd_headwise(p, x, w, dy, dx, dw, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = chunk_edges(*p, EDGE_HEADWISE, x_prev, dy_next, w_next, edges_only);
    a.x = x; a.w = w; a.dy = dy; a.dx = dx; a.dw = dw;
    return edges_bwd(stream, p, a);
}

dsc_status dsc_fwd_lowrank_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *z, const void *U,
                                 void *y, void *workspace, size_t workspace_bytes, int edges_only, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, z, U, y});
    if (s == DSC_OK) s = check_halos(p, x_prev, nullptr, nullptr, false);
    if (s == DSC_OK && !edges_only) s = dsc_fwd_lowrank(p, x, z, U, y, workspace, workspace_bytes, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = chunk_edges(*p, EDGE_LOWRANK, x_prev, nullptr, nullptr, edges_only);
    a.x = x; a.z = z; a.U = U; a.y = y;
    return edges_fwd(stream, p, a);
}

size_t dsc_bwd_lowrank_chunk_workspace_bytes(const dsc_problem *p) {
    if (validate(p, true) != DSC_OK) return 0;
    return up256(dsc_bwd_lowrank_workspace_bytes(p)) + edge_scratch_bytes(*p, EDGE_LOWRANK, p->B);
}

dsc_status dsc_bwd_lowrank_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next, const void *z_next,
                                 const void *x, const void *z, const void *U, const void *dy, void *dx, void *dz,
                                 float *dU, void *workspace, size_t workspace_bytes, int edges_only, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, z, U, dy, dx, dz, dU});
    if (s == DSC_OK) s = check_halos(p, x_prev, dy_next, z_next, true);
    if (s != DSC_OK) return s;
    return lowrank_bwd_edges(p, chunk_edges(*p, EDGE_LOWRANK, x_prev, dy_next, z_next, edges_only), x, z, U, dy, dx, dz, dU,
                             workspace, workspace_bytes, dsc_bwd_lowrank_workspace_bytes(p), !edges_only, stream);
}

dsc_status dsc_fwd_static_chunk(const dsc_problem *p, const void *x_prev, const void *x, const void *ws, void *y,
                                int edges_only, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, ws, y});
    if (s == DSC_OK) s = check_halos(p, x_prev, nullptr, nullptr, false);
    if (s == DSC_OK && !edges_only) s = dsc_fwd_static(p, x, ws, y, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = chunk_edges(*p, EDGE_STATIC, x_prev, nullptr, nullptr, edges_only);
    a.x = x; a.w = ws; a.y = y;
    return edges_fwd(stream, p, a);
}

dsc_status dsc_bwd_static_chunk(const dsc_problem *p, const void *x_prev, const void *dy_next, const void *x,
                                const void *ws, const void *dy, void *dx, float *dws, void *workspace,
                                size_t workspace_bytes, int edges_only, void *stream) {
    dsc_status s = validate(p, false);
    if (s == DSC_OK) s = check_chunk(p);
    if (s == DSC_OK) s = check_ptrs({x, ws, dy, dx, dws});
    if (s == DSC_OK) s = check_halos(p, x_prev, dy_next, nullptr, false);
    if (s == DSC_OK && !edges_only) s = dsc_bwd_static(p, x, ws, dy, dx, dws, workspace, workspace_bytes, stream);
    if (s != DSC_OK) return s;
    EdgeArgs a = chunk_edges(*p, EDGE_STATIC, x_prev, dy_next, nullptr, edges_only);
    a.x = x; a.w = ws; a.dy = dy; a.dx = dx; a.dws = dws;
    return edges_bwd(stream, p, a);
}

// ------------------------------------------------ first projection z = hV ---

static dsc_status check_dmodel(int64_t d_model) {
    return (d_model < 1 || d_model > ((int64_t)1 << 30)) ? DSC_ERR_INVALID_ARG : DSC_OK;
}

size_t dsc_fwd_lowrank_proj_workspace_bytes(const dsc_problem *p, int64_t d_model) {
    if (validate(p, true) != DSC_OK || check_dmodel(d_model) != DSC_OK) return 0;
    return dsc_fwd_lowrank_workspace_bytes(p);
}

dsc_status dsc_fwd_lowrank_proj(const dsc_problem *p, int64_t d_model, const void *x, const void *h, const void *V,
                                const void *U, void *z, void *y, void *workspace, size_t workspace_bytes,
                                void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_dmodel(d_model);
    if (s == DSC_OK) s = check_ptrs({x, h, V, U, z, y});
    if (s != DSC_OK) return s;
    s = done(launch_proj_z(ctx(stream), *p, d_model, h, V, z));
    if (s != DSC_OK) return s;
    return dsc_fwd_lowrank(p, x, z, U, y, workspace, workspace_bytes, stream);
}

// Workspace of the backward with the projection: dz [B,T,R] (input dtype),
// then the low-rank backward's workspace, then the dV partials.
static size_t proj_dz_bytes(const dsc_problem &p) {
    return up256((size_t)(p.B * p.T) * (size_t)p.R * (p.dtype == DSC_BF16 ? 2 : 4));
}

size_t dsc_bwd_lowrank_proj_workspace_bytes(const dsc_problem *p, int64_t d_model) {
    if (validate(p, true) != DSC_OK || check_dmodel(d_model) != DSC_OK) return 0;
    return proj_dz_bytes(*p) + up256(dsc_bwd_lowrank_workspace_bytes(p)) + proj_dV_part_bytes(*p, d_model, sm_count());
}

dsc_status dsc_bwd_lowrank_proj(const dsc_problem *p, int64_t d_model, const void *x, const void *h, const void *V,
                                const void *z, const void *U, const void *dy, void *dx, void *dh, float *dV,
                                float *dU, void *workspace, size_t workspace_bytes, void *stream) {
    dsc_status s = validate(p, true);
    if (s == DSC_OK) s = check_dmodel(d_model);
    if (s == DSC_OK) s = check_ptrs({x, h, V, z, U, dy, dx, dh, dV, dU, workspace});
    if (s != DSC_OK) return s;
    if (workspace_bytes < dsc_bwd_lowrank_proj_workspace_bytes(p, d_model)) return DSC_ERR_INVALID_ARG;
    char *w = static_cast<char *>(workspace);
    void *dz = w;
    const size_t main_bytes = dsc_bwd_lowrank_workspace_bytes(p);
    void *wmain = w + proj_dz_bytes(*p);
    float *part = reinterpret_cast<float *>(w + proj_dz_bytes(*p) + up256(main_bytes));
    s = dsc_bwd_lowrank(p, x, z, U, dy, dx, dz, dU, main_bytes ? wmain : nullptr, main_bytes, stream);
    if (s != DSC_OK) return s;
    return done(launch_proj_bwd(ctx(stream), *p, d_model, h, V, dz, dh, dV, part));
}

dsc_status dsc_selftest_timeout(void *stream) {
    return launch_wait_selftest(static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSC_OK : DSC_ERR_CUDA;
}

dsc_status dsc_check(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSC_ERR_CUDA;
    const int st = take_device_status(static_cast<cudaStream_t>(stream));
    const int st_tc = take_tc_status(static_cast<cudaStream_t>(stream));
    const int st_dec = take_tc_dec_status(static_cast<cudaStream_t>(stream));
    const int st_pj = take_proj_status(static_cast<cudaStream_t>(stream));
    if (st < 0 || st_tc < 0 || st_dec < 0 || st_pj < 0) return DSC_ERR_CUDA;
    return static_cast<dsc_status>(st ? st : (st_tc ? st_tc : (st_dec ? st_dec : st_pj)));
}

}  // extern "C"
