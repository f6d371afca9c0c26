// Sequence edges inside a call: packed documents (variable-length batches)
// and time chunks of longer sequences (context parallelism).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Mechanism": y_t = sum_k w(t)_k (.) x_{t-k}, causal, so a token
// depends only on the W-1 tokens before it, and (backward) on the W-1 after
// it.  Two uses need other values than zero at a sequence edge:
//  - packed documents (one row holding several documents, cu_seqlens
//    offsets): every document start is a sequence start, so taps that reach
//    across it read zero, and dx of a document's last tokens takes nothing
//    from the next document;
//  - a time chunk of longer sequences: taps before the chunk read the W-1
//    inputs of the previous chunk (x_prev), and dx of the chunk's last tokens
//    takes dy and the filters of the next chunk's first W-1 tokens.
//
// Design.  The streaming and tensor-core kernels stay as they are: each call
// first runs them on the row (or chunk) as one zero-padded sequence, which is
// already right for every output more than W-1 tokens from an edge.  The
// kernels here then recompute, from the definition, only the outputs that
// differ: y and dw/dz of the first W-1 tokens after a left edge, dx of the
// last W-1 tokens before a right edge; the token reductions dU and dws get
// the difference of the cross-edge terms added.  That costs O(edges * W * D)
// work (plus one R x (G*W) contraction per fixed token for low-rank), and
// the roofline kernels keep their inner loops free of per-token edge tests.
// The fix-up kernels read only the call's inputs before their first store, so
// when the row pass runs in the same call they load and compute while it
// finishes (programmatic dependent launch) and wait for it only to store: the
// row pass itself waited for the stream's earlier kernels before it let them
// start, so the inputs are complete.  A call that runs the fix-ups alone has
// no such pass before them, and its first fix-up kernel waits before it reads.
#include "edges.cuh"

namespace dsc {

namespace {

constexpr int ED_THREADS = 256;

template <typename T> __device__ __forceinline__ float ldf(const void *p, int64_t i) {
    return to_f<T>(static_cast<const T *>(p)[i]);
}

// Segment i of the call: row b, tokens [s, e).  Packed documents: row 0,
// offsets clamped into [0, T] so that malformed offsets stay in bounds.
// Chunks: segment b is row b, all T tokens.
__device__ __forceinline__ void segment(const EdgeArgs &a, int64_t i, int64_t &b, int64_t &s, int64_t &e) {
    if (a.cu) {
        b = 0;
        s = min(max((int64_t)a.cu[i], (int64_t)0), a.T);
        e = min(max((int64_t)a.cu[i + 1], s), a.T);
    } else {
        b = i;
        s = 0;
        e = a.T;
    }
}
// The zero-padded pass was wrong at the segment's left / right edge.
__device__ __forceinline__ bool left_edge(const EdgeArgs &a, int64_t i) { return a.cu ? i > 0 : a.x_prev != nullptr; }
__device__ __forceinline__ bool right_edge(const EdgeArgs &a, int64_t i) {
    return a.cu ? i + 1 < a.nseg : a.dy_next != nullptr;
}

// Tap k of channel c's filter at local token t of row b.
template <typename T>
__device__ __forceinline__ float tap(const EdgeArgs &a, int64_t b, int64_t t, int64_t c, int k) {
    if (a.kind == EDGE_STATIC) return ldf<T>(a.w, c * a.W + k);
    const int64_t g = c / a.H;
    if (a.kind == EDGE_HEADWISE) return ldf<T>(a.w, ((b * a.T + t) * a.G + g) * a.W + k);
    float s = 0.f;
    for (int r = 0; r < a.R; ++r) s = fmaf(ldf<T>(a.z, (b * a.T + t) * a.R + r), ldf<T>(a.U, r * a.GW + g * a.W + k), s);
    return s;
}

// Tap k of channel c's filter at token j of the next chunk (row b).
template <typename T>
__device__ __forceinline__ float tap_next(const EdgeArgs &a, int64_t b, int64_t j, int64_t c, int k) {
    if (a.kind == EDGE_STATIC) return ldf<T>(a.w, c * a.W + k);
    const int64_t g = c / a.H;
    const int64_t row = b * (a.W - 1) + j;
    if (a.kind == EDGE_HEADWISE) return ldf<T>(a.f_next, (row * a.G + g) * a.W + k);
    float s = 0.f;
    for (int r = 0; r < a.R; ++r) s = fmaf(ldf<T>(a.f_next, row * a.R + r), ldf<T>(a.U, r * a.GW + g * a.W + k), s);
    return s;
}

// x at position u < s (left of segment i's start), as the definition reads
// it (`want`: zero for a document, the previous chunk's row for a chunk) and
// as the zero-padded pass read it (`had`: the previous document's token, or
// zero before the row start).
template <typename T>
__device__ __forceinline__ void x_left(const EdgeArgs &a, int64_t b, int64_t s, int64_t u, int64_t c, float &want,
                                       float &had) {
    if (a.cu) {
        want = 0.f;
        had = u >= 0 ? ldf<T>(a.x, (b * a.T + u) * a.D + c) : 0.f;
    } else {
        want = ldf<T>(a.x_prev, (b * (a.W - 1) + (u - s + a.W - 1)) * a.D + c);
        had = 0.f;
    }
}

// ---------------------------------------------------------------- forward ---
// y of the first W-1 tokens of each segment with a wrong left edge.
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_y(const EdgeArgs a, int64_t cblocks) {
    if (!a.early) pdl_wait();  // no row pass in this call: inputs may come from the stream's previous kernel
    pdl_trigger();             // the next fix-up kernel may start its loads
    const int64_t row = blockIdx.x / cblocks;
    const int64_t c = (blockIdx.x % cblocks) * ED_THREADS + threadIdx.x;
    const int64_t i = row / (a.W - 1);
    const int j = (int)(row % (a.W - 1));
    if (c >= a.D || !left_edge(a, i)) return;
    int64_t b, s, e;
    segment(a, i, b, s, e);
    const int64_t t = s + j;
    if (t >= e) return;
    const float xt = ldf<T>(a.x, (b * a.T + t) * a.D + c);
    float acc = a.residual ? xt : 0.f;
    for (int k = 0; k < a.W; ++k) {
        const int64_t u = t - k;
        float xv, unused;
        if (u >= s) xv = ldf<T>(a.x, (b * a.T + u) * a.D + c);
        else x_left<T>(a, b, s, u, c, xv, unused);
        acc = fmaf(tap<T>(a, b, t, c, k), xv, acc);
    }
    pdl_wait();  // the row pass, which wrote y here first, is done
    static_cast<T *>(a.y)[(b * a.T + t) * a.D + c] = from_f<T>(acc);
}

// --------------------------------------------------------------- backward ---
// dx of the last W-1 tokens of each segment with a wrong right edge.
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_dx(const EdgeArgs a, int64_t cblocks) {
    if (!a.early) pdl_wait();  // no row pass in this call: inputs may come from the stream's previous kernel
    pdl_trigger();             // the next fix-up kernel may start its loads
    const int64_t row = blockIdx.x / cblocks;
    const int64_t c = (blockIdx.x % cblocks) * ED_THREADS + threadIdx.x;
    const int64_t i = row / (a.W - 1);
    const int j = (int)(row % (a.W - 1));
    if (c >= a.D || !right_edge(a, i)) return;
    int64_t b, s, e;
    segment(a, i, b, s, e);
    const int64_t t = e - (a.W - 1) + j;
    if (t < s) return;
    float acc = a.residual ? ldf<T>(a.dy, (b * a.T + t) * a.D + c) : 0.f;
    for (int k = 0; k < a.W; ++k) {
        const int64_t u = t + k;
        if (u < e) {
            acc = fmaf(tap<T>(a, b, u, c, k), ldf<T>(a.dy, (b * a.T + u) * a.D + c), acc);
        } else if (!a.cu) {  // the next chunk's token u - e (a document takes nothing past its end)
            const int64_t jn = u - e;
            acc = fmaf(tap_next<T>(a, b, jn, c, k), ldf<T>(a.dy_next, (b * (a.W - 1) + jn) * a.D + c), acc);
        }
    }
    pdl_wait();  // the row pass, which wrote dx here first, is done
    static_cast<T *>(a.dx)[(b * a.T + t) * a.D + c] = from_f<T>(acc);
}

// Filter gradients of the first W-1 tokens after a wrong left edge: one
// thread per (segment, token j, group g).  Taps k <= j read x inside the
// segment and were right; taps k > j reach across the edge.
//   head-wise: dw[t, g, k] for k > j overwritten with the definition's value;
//   low-rank:  fixed row (i, j) of the scratch gets the token's whole dw row
//              (dwfull) and, for k > j, the definition's value minus the
//              zero-padded pass's (dwdelta); rows with nothing to fix are
//              zero in both.
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_dw(const EdgeArgs a) {
    if (!a.early) pdl_wait();  // no row pass in this call: inputs may come from the stream's previous kernel
    pdl_trigger();             // the next fix-up kernel may start its loads
    const int64_t idx = (int64_t)blockIdx.x * ED_THREADS + threadIdx.x;
    const int64_t nrows = a.nseg * (a.W - 1);
    if (idx >= nrows * a.G) return;
    const int64_t rowi = idx / a.G, g = idx % a.G;
    const int64_t i = rowi / (a.W - 1);
    const int j = (int)(rowi % (a.W - 1));
    int64_t b, s, e;
    segment(a, i, b, s, e);
    const int64_t t = s + j;
    const bool live = left_edge(a, i) && t < e;
    float want[8], had[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) want[k] = had[k] = 0.f;
    if (live) {
        // Unrolled so that several channels' loads are in flight at once (the
        // loop is latency-bound: a few hundred threads, each reading H rows).
#pragma unroll 8
        for (int64_t c = g * a.H; c < (g + 1) * a.H; ++c) {
            const float d = ldf<T>(a.dy, (b * a.T + t) * a.D + c);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (k >= a.W) break;
                const int64_t u = t - k;
                if (u >= s) {
                    const float xv = ldf<T>(a.x, (b * a.T + u) * a.D + c);
                    want[k] = fmaf(d, xv, want[k]);
                    had[k] = fmaf(d, xv, had[k]);
                } else {
                    float xw, xh;
                    x_left<T>(a, b, s, u, c, xw, xh);
                    want[k] = fmaf(d, xw, want[k]);
                    had[k] = fmaf(d, xh, had[k]);
                }
            }
        }
    }
    pdl_wait();  // the row pass (dw) and the previous call's readers of the scratch are done
    if (a.kind == EDGE_HEADWISE) {
        if (!live) return;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < a.W && k > j) static_cast<T *>(a.dw)[((b * a.T + t) * a.G + g) * a.W + k] = from_f<T>(want[k]);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k >= a.W) break;
            a.dwfull[rowi * a.GW + g * a.W + k] = want[k];
            a.dwdelta[rowi * a.GW + g * a.W + k] = k > j ? want[k] - had[k] : 0.f;
        }
    }
}

// Low-rank: dz of each fixed token from its whole dw row, dz[t, r] =
// sum_n dwfull[row, n] U[r, n]; one block per fixed row, a warp per rank,
// lanes along the G*W columns.
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_dz(const EdgeArgs a) {
    const int64_t rowi = blockIdx.x;
    const int64_t i = rowi / (a.W - 1);
    const int j = (int)(rowi % (a.W - 1));
    pdl_wait();
    int64_t b, s, e;
    segment(a, i, b, s, e);
    const int64_t t = s + j;
    if (!left_edge(a, i) || t >= e) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *dwr = a.dwfull + rowi * a.GW;
    for (int r = warp; r < a.R; r += ED_THREADS / 32) {
        float acc = 0.f;
        for (int64_t n = lane; n < a.GW; n += 32) acc = fmaf(dwr[n], ldf<T>(a.U, r * a.GW + n), acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL_MASK, acc, o);
        if (lane == 0) static_cast<T *>(a.dz)[(b * a.T + t) * a.R + r] = from_f<T>(acc);
    }
}

// Low-rank: dU[r, n] += sum over fixed rows of z[t, r] dwdelta[row, n]
// (rows with nothing to fix are zero).  Thread per column n and 16 ranks.
constexpr int ED_RC = 16;
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_dU(const EdgeArgs a) {
    const int64_t n = (int64_t)blockIdx.x * ED_THREADS + threadIdx.x;
    const int r0 = blockIdx.y * ED_RC;
    pdl_wait();
    if (n >= a.GW) return;
    float acc[ED_RC];
#pragma unroll
    for (int q = 0; q < ED_RC; ++q) acc[q] = 0.f;
    const int64_t nrows = a.nseg * (a.W - 1);
    for (int64_t rowi = 0; rowi < nrows; ++rowi) {
        const int64_t i = rowi / (a.W - 1);
        const int j = (int)(rowi % (a.W - 1));
        int64_t b, s, e;
        segment(a, i, b, s, e);
        const int64_t t = s + j;
        if (!left_edge(a, i) || t >= e) continue;
        const float d = a.dwdelta[rowi * a.GW + n];
        const int64_t zo = (b * a.T + t) * a.R;
#pragma unroll
        for (int q = 0; q < ED_RC; ++q)
            if (r0 + q < a.R) acc[q] = fmaf(ldf<T>(a.z, zo + r0 + q), d, acc[q]);
    }
#pragma unroll
    for (int q = 0; q < ED_RC; ++q)
        if (r0 + q < a.R) a.dU[(int64_t)(r0 + q) * a.GW + n] += acc[q];
}

// Static: dws[c, k] += sum over fixed tokens of dy_t (x_want - x_had)(t-k),
// for the taps that reach across a left edge.  Thread per channel.
template <typename T> __global__ void __launch_bounds__(ED_THREADS) k_edge_dws(const EdgeArgs a) {
    const int64_t c = (int64_t)blockIdx.x * ED_THREADS + threadIdx.x;
    if (c >= a.D) return;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    for (int64_t i = 0; i < a.nseg; ++i) {
        if (!left_edge(a, i)) continue;
        int64_t b, s, e;
        segment(a, i, b, s, e);
        for (int j = 0; j < a.W - 1 && s + j < e; ++j) {
            const int64_t t = s + j;
            const float d = ldf<T>(a.dy, (b * a.T + t) * a.D + c);
#pragma unroll
            for (int k = 1; k < 8; ++k) {
                if (k >= a.W || k <= j) continue;
                float xw, xh;
                x_left<T>(a, b, s, t - k, c, xw, xh);
                acc[k] = fmaf(d, xw - xh, acc[k]);
            }
        }
    }
    pdl_wait();  // dws is complete (the row pass and its partial sums)
#pragma unroll
    for (int k = 1; k < 8; ++k)
        if (k < a.W) a.dws[c * a.W + k] += acc[k];
}

template <typename T> cudaError_t fwd_t(const Ctx &c, const EdgeArgs &a) {
    const int64_t cb = (a.D + ED_THREADS - 1) / ED_THREADS;
    cudaError_t e = launch_pdl(k_edge_y<T>, dim3((unsigned)(a.nseg * (a.W - 1) * cb)), dim3(ED_THREADS), 0, c.stream, a,
                               cb);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename T> cudaError_t bwd_t(const Ctx &c, const EdgeArgs &a) {
    const int64_t cb = (a.D + ED_THREADS - 1) / ED_THREADS;
    const int64_t nrows = a.nseg * (a.W - 1);
    cudaError_t e = launch_pdl(k_edge_dx<T>, dim3((unsigned)(nrows * cb)), dim3(ED_THREADS), 0, c.stream, a, cb);
    if (e != cudaSuccess) return e;
    if (a.kind == EDGE_STATIC) {
        e = launch_pdl(k_edge_dws<T>, dim3((unsigned)cb), dim3(ED_THREADS), 0, c.stream, a);
        return e != cudaSuccess ? e : cudaGetLastError();
    }
    e = launch_pdl(k_edge_dw<T>, dim3((unsigned)((nrows * a.G + ED_THREADS - 1) / ED_THREADS)), dim3(ED_THREADS), 0,
                   c.stream, a);
    if (e != cudaSuccess || a.kind == EDGE_HEADWISE) return e != cudaSuccess ? e : cudaGetLastError();
    e = launch_pdl(k_edge_dz<T>, dim3((unsigned)nrows), dim3(ED_THREADS), 0, c.stream, a);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_edge_dU<T>, dim3((unsigned)((a.GW + ED_THREADS - 1) / ED_THREADS), (unsigned)((a.R + ED_RC - 1) / ED_RC)),
                   dim3(ED_THREADS), 0, c.stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t edge_scratch_bytes(const dsc_problem &p, int kind, int64_t nseg) {
    if (kind != EDGE_LOWRANK || p.W < 2) return 0;
    return 2 * (size_t)nseg * (size_t)(p.W - 1) * (size_t)((p.D / p.H) * p.W) * sizeof(float);
}

void edge_args(const dsc_problem &p, int kind, EdgeArgs &a) {
    a.B = p.B; a.T = p.T; a.D = p.D; a.H = kind == EDGE_STATIC ? 1 : p.H;
    a.G = p.D / a.H; a.R = p.R; a.GW = a.G * p.W;
    a.W = (int)p.W;
    a.residual = p.residual ? 1 : 0;
    a.kind = kind;
}

cudaError_t launch_edges_fwd(const Ctx &c, const dsc_problem &p, const EdgeArgs &a) {
    if (a.W < 2 || a.nseg < 1) return cudaSuccess;
    return p.dtype == DSC_BF16 ? fwd_t<bf16>(c, a) : fwd_t<float>(c, a);
}

cudaError_t launch_edges_bwd(const Ctx &c, const dsc_problem &p, const EdgeArgs &a) {
    if (a.W < 2 || a.nseg < 1) return cudaSuccess;
    return p.dtype == DSC_BF16 ? bwd_t<bf16>(c, a) : bwd_t<float>(c, a);
}

}  // namespace dsc
