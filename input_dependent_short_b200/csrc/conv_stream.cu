// Time-streaming kernels of the head-wise and static dynamic short convolution.
//
// Operation: "Dynamic Short Convolutions Improve Transformers", technical
// summary, Methodology ("Mechanism": y_t = sum_k w(t)_k (.) x_{t-k};
// "Parameterisation" 2: one filter per H consecutive channels; "Placement":
// residual X + conv(X)), and the static short convolution of the authors'
// thread (one fixed filter per channel).  The pages' own kernels (Triton,
// H100) read activations and filters, convolve on chip and write only the
// result; these kernels keep that property and are laid out for sm_100a.
//
// Design.  The op is HBM-bound (a few FMAs per byte), so each kernel is one
// pass over memory with 16-byte, fully coalesced accesses:
//  - a thread owns one 16-byte vector of channels and walks Tt tokens of one
//    sequence; the W-1 previous x rows live in registers (a sliding window),
//    so x is read once, plus a (W-1)-row halo at the tile start (an L2 hit:
//    the neighbouring tile streams the same rows at the same time);
//  - loads of U_LD consecutive tokens are issued together before any of them
//    is used, so each thread keeps several 16-byte requests in flight;
//  - backward walks forward in time too: dx rows are finished W-1 tokens
//    late from an accumulator window (row s collects w(s+k)_k dy_{s+k} as
//    token s+k streams by), and the tile runs W-1 tokens past its end (right
//    halo of dy and w) to finish its last rows; dw(t) needs dy_t and the
//    x window, and is reduced over the H channels of a group with shuffles
//    inside the warp (no shared memory, no atomics);
//  - the grid is sized from the measured residency so that all tiles are in
//    flight at once (one wave), avoiding a tail of partially filled SMs.
#include "kernels.cuh"

namespace dsc {

constexpr int STREAM_THREADS = 256;

__host__ __device__ constexpr int ld_batch(int wwords) { return wwords >= 16 ? 2 : (wwords >= 8 ? 4 : 8); }

struct Pos {
    int64_t b;
    int t_start, t_end;
    int64_t c0;
    bool active;
    int lane;
};

template <int V>
__device__ __forceinline__ bool locate(const StreamMap &m, Pos &q) {
    q.lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= m.n_warps) return false;
    const int wc = (int)(gw % m.nWc);
    const int64_t bt = gw / m.nWc;
    const int tile = (int)(bt % m.nTiles);
    q.b = bt / m.nTiles;
    q.t_start = tile * m.Tt;
    q.t_end = min((int64_t)q.t_start + m.Tt, m.T);
    q.c0 = (int64_t)wc * m.CW + (int64_t)q.lane * V;
    q.active = q.lane < m.lanes_used && q.c0 < m.D;
    return true;
}

// ---------------------------------------------------------------- forward ---

// WSTATIC = false: head-wise filters w[b,t,g,k] read per token.
// WSTATIC = true : static filters ws[c,k] read once per thread.
template <typename T, int W, int GPT, bool WSTATIC>
__global__ void __launch_bounds__(STREAM_THREADS) k_stream_fwd(const HwArgs a) {
    constexpr int V = VecOf<T>::V;
    constexpr int NW = WSTATIC ? V * W : GPT * W;  // filter taps a thread needs per token
    constexpr int CPG = WSTATIC ? 1 : V / GPT;      // channels per filter (within the thread)
    constexpr int UL = ld_batch(Row<T, NW>::WORDS);
    constexpr int WIN = W > 1 ? W - 1 : 1;
    const StreamMap &m = a.m;
    Pos q;
    if (!locate<V>(m, q) || !q.active) return;

    const int64_t row0 = q.b * m.T;
    const T *xb = static_cast<const T *>(a.x) + row0 * m.D + q.c0;
    T *yb = static_cast<T *>(a.y) + row0 * m.D + q.c0;
    const T *wb = WSTATIC ? static_cast<const T *>(a.w) + q.c0 * W
                          : static_cast<const T *>(a.w) + row0 * m.G * W + (q.c0 / m.H) * W;
    const int64_t wstride = WSTATIC ? 0 : m.G * W;

    Row<T, NW> wst;
    if constexpr (WSTATIC) wst.load(wb);

    float win[WIN][V];
#pragma unroll
    for (int j = 0; j < WIN; ++j) {
        const int t = q.t_start - 1 - j;
        if (W > 1 && t >= 0) {
            unpack(ld16(xb + (int64_t)t * m.D), win[j]);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) win[j][v] = 0.f;
        }
    }
    const float res = m.residual ? 1.f : 0.f;

    for (int t = q.t_start; t < q.t_end; t += UL) {
        uint4 xr[UL];
        Row<T, NW> wr[UL];
#pragma unroll
        for (int u = 0; u < UL; ++u) {
            if (t + u < q.t_end) {
                xr[u] = ld16(xb + (int64_t)(t + u) * m.D);
                if constexpr (!WSTATIC) wr[u].load(wb + (int64_t)(t + u) * wstride);
            } else {
                xr[u] = make_uint4(0, 0, 0, 0);
                if constexpr (!WSTATIC) wr[u].zero();
            }
        }
#pragma unroll
        for (int u = 0; u < UL; ++u) {
            const Row<T, NW> &wv = WSTATIC ? wst : wr[u];
            float xc[V], acc[V];
            unpack(xr[u], xc);
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int f = WSTATIC ? v * W : (v / CPG) * W;
                float s = res * xc[v];
                s = fmaf(wv.get(f), xc[v], s);
#pragma unroll
                for (int k = 1; k < W; ++k) s = fmaf(wv.get(f + k), win[k - 1][v], s);
                acc[v] = s;
            }
            if (t + u < q.t_end) st16(yb + (int64_t)(t + u) * m.D, pack(acc));
#pragma unroll
            for (int j = WIN - 1; j > 0; --j)
#pragma unroll
                for (int v = 0; v < V; ++v) win[j][v] = win[j - 1][v];
#pragma unroll
            for (int v = 0; v < V; ++v) win[0][v] = xc[v];
        }
    }
}

// --------------------------------------------------------------- backward ---

template <typename T, int W, int GPT, bool WSTATIC>
__global__ void __launch_bounds__(STREAM_THREADS) k_stream_bwd(const HwArgs a) {
    constexpr int V = VecOf<T>::V;
    constexpr int NW = WSTATIC ? V * W : GPT * W;
    constexpr int CPG = WSTATIC ? 1 : V / GPT;
    constexpr int UL = ld_batch(Row<T, NW>::WORDS) > 4 ? 4 : ld_batch(Row<T, NW>::WORDS);
    constexpr int WIN = W > 1 ? W - 1 : 1;
    const StreamMap &m = a.m;
    Pos q;
    if (!locate<V>(m, q)) return;  // whole warp out of range
    const bool act = q.active;
    const int L = m.L;
    const int pos = q.lane % (L > 0 ? L : 1);

    const int64_t row0 = q.b * m.T;
    const int64_t c0 = act ? q.c0 : 0;
    const T *xb = static_cast<const T *>(a.x) + row0 * m.D + c0;
    const T *dyb = static_cast<const T *>(a.dy) + row0 * m.D + c0;
    T *dxb = static_cast<T *>(a.dx) + row0 * m.D + c0;
    const int64_t g0 = c0 / m.H;
    const T *wb = WSTATIC ? static_cast<const T *>(a.w) + c0 * W
                          : static_cast<const T *>(a.w) + row0 * m.G * W + g0 * W;
    T *dwb = WSTATIC ? nullptr : static_cast<T *>(a.dw) + row0 * m.G * W + g0 * W;
    const int64_t wstride = WSTATIC ? 0 : m.G * W;

    Row<T, NW> wst;
    if constexpr (WSTATIC) {
        if (act) wst.load(wb); else wst.zero();
    }
    float dws[WSTATIC ? V : 1][WSTATIC ? W : 1];
    if constexpr (WSTATIC) {
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int k = 0; k < W; ++k) dws[v][k] = 0.f;
    }

    float xw[WIN][V];   // xw[j] = x[t-1-j]
    float acc[WIN][V];  // acc[j] = partial dx of row t-1-j
#pragma unroll
    for (int j = 0; j < WIN; ++j) {
        const int t = q.t_start - 1 - j;
        if (W > 1 && act && t >= 0) {
            unpack(ld16(xb + (int64_t)t * m.D), xw[j]);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) xw[j][v] = 0.f;
        }
#pragma unroll
        for (int v = 0; v < V; ++v) acc[j][v] = 0.f;
    }
    const float res = m.residual ? 1.f : 0.f;
    const int t_stop = q.t_end + W - 1;  // right halo: W-1 extra tokens finish the last rows
    const int t_lim = (int)min((int64_t)t_stop, m.T);

    for (int t = q.t_start; t < t_stop; t += UL) {
        uint4 xr[UL], dr[UL];
        Row<T, NW> wr[UL];
#pragma unroll
        for (int u = 0; u < UL; ++u) {
            const int tt = t + u;
            xr[u] = (act && tt < q.t_end) ? ld16(xb + (int64_t)tt * m.D) : make_uint4(0, 0, 0, 0);
            dr[u] = (act && tt < t_lim) ? ld16(dyb + (int64_t)tt * m.D) : make_uint4(0, 0, 0, 0);
            if constexpr (!WSTATIC) {
                if (act && tt < t_lim) wr[u].load(wb + (int64_t)tt * wstride); else wr[u].zero();
            }
        }
#pragma unroll
        for (int u = 0; u < UL; ++u) {
            const int tt = t + u;
            const Row<T, NW> &wv = WSTATIC ? wst : wr[u];
            float xc[V], dyc[V], r0[V];
            unpack(xr[u], xc);
            unpack(dr[u], dyc);
            const bool main = tt < q.t_end;
            // dx: token tt feeds row tt-k through tap k of w(tt).
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int f = WSTATIC ? v * W : (v / CPG) * W;
                r0[v] = fmaf(wv.get(f), dyc[v], main ? res * dyc[v] : 0.f);
#pragma unroll
                for (int k = 1; k < W; ++k) acc[k - 1][v] = fmaf(wv.get(f + k), dyc[v], acc[k - 1][v]);
            }
            // row tt-(W-1) is complete
            const int done = tt - (W - 1);
            if (act && done >= q.t_start && done < q.t_end) {
                if constexpr (W > 1) st16(dxb + (int64_t)done * m.D, pack(acc[WIN - 1]));
                else st16(dxb + (int64_t)done * m.D, pack(r0));
            }
            // dw(tt)_k = sum over the group's channels of dy_tt * x_{tt-k}
            if (tt < q.t_end) {
                if constexpr (WSTATIC) {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        dws[v][0] = fmaf(dyc[v], xc[v], dws[v][0]);
#pragma unroll
                        for (int k = 1; k < W; ++k) dws[v][k] = fmaf(dyc[v], xw[k - 1][v], dws[v][k]);
                    }
                } else {
                    float part[GPT * W];
#pragma unroll
                    for (int gi = 0; gi < GPT; ++gi) {
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            float s = 0.f;
#pragma unroll
                            for (int v = gi * CPG; v < (gi + 1) * CPG; ++v) s = fmaf(dyc[v], k == 0 ? xc[v] : xw[k - 1][v], s);
                            part[gi * W + k] = s;
                        }
                    }
                    if (GPT == 1 && L > 1) {
#pragma unroll
                        for (int k = 0; k < W; ++k) part[k] = segment_sum(part[k], L, pos);
                        if (act && pos == 0) store_row<T, GPT * W>(dwb + (int64_t)tt * wstride, part);
                    } else if (act) {
                        store_row<T, GPT * W>(dwb + (int64_t)tt * wstride, part);
                    }
                }
            }
            // shift windows
#pragma unroll
            for (int j = WIN - 1; j > 0; --j)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    acc[j][v] = acc[j - 1][v];
                    xw[j][v] = xw[j - 1][v];
                }
#pragma unroll
            for (int v = 0; v < V; ++v) {
                acc[0][v] = r0[v];
                xw[0][v] = xc[v];
            }
        }
    }
    if constexpr (WSTATIC) {
        if (act) {
            const int64_t s = q.b * m.nTiles + q.t_start / m.Tt;
            float *pp = a.partial + (s * m.D + c0) * W;
#pragma unroll
            for (int v = 0; v < V; ++v)
#pragma unroll
                for (int k = 0; k < W; ++k) pp[v * W + k] = dws[v][k];
        }
    }
}

// dws[i] = sum_s partial[s][i], in order of s (deterministic).
__global__ void k_reduce_partials(const float *__restrict__ partial, int64_t S, int64_t n, float *__restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float s = 0.f;
    for (int64_t j = 0; j < S; ++j) s += partial[j * n + i];
    out[i] = s;
}

// ------------------------------------------------------------------- host ---

int resident_blocks(const void *kernel, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
    }
    return n;
}

bool stream_map(const dsc_problem &p, int V, StreamMap &m) {
    m = StreamMap{};
    m.B = p.B; m.T = p.T; m.D = p.D; m.H = p.H; m.G = p.D / p.H;
    m.W = (int)p.W;
    m.residual = p.residual ? 1 : 0;
    if (p.D % V) return false;
    if (V % p.H == 0) {
        m.gpt = (int)(V / p.H);
        m.L = 1;
        m.lanes_used = 32;
        m.CW = 32 * V;
    } else if (p.H % V == 0 && p.H / V <= 32) {
        m.gpt = 1;
        m.L = (int)(p.H / V);
        const int gpw = 32 / m.L;
        m.lanes_used = gpw * m.L;
        m.CW = (int)(gpw * p.H);
    } else {
        return false;
    }
    m.nWc = (int)((p.D + m.CW - 1) / m.CW);
    return true;
}

// Pick the tile length so that all warps are resident at once (one wave),
// with at least 32 tokens per tile to keep the (W-1)-row halo small.
void finish_map(StreamMap &m, int64_t target_warps) {
    const int64_t cols = m.B * m.nWc;
    int64_t tt = (m.T * cols + target_warps - 1) / target_warps;
    tt = ((tt + 7) / 8) * 8;
    if (tt < 32) tt = 32;
    if (tt > m.T) tt = m.T;
    m.Tt = (int)tt;
    m.nTiles = (int)((m.T + tt - 1) / tt);
    m.n_warps = m.B * m.nTiles * (int64_t)m.nWc;
}

template <typename T, int W, int GPT, bool WS, bool BWD>
static const void *stream_kernel() {
    if constexpr (BWD) return (const void *)k_stream_bwd<T, W, GPT, WS>;
    else return (const void *)k_stream_fwd<T, W, GPT, WS>;
}

template <typename T, int W, int GPT, bool WS, bool BWD>
static cudaError_t run_stream(const Ctx &c, HwArgs a) {
    const void *k = stream_kernel<T, W, GPT, WS, BWD>();
    const int per_sm = resident_blocks(k, STREAM_THREADS, 0) * (STREAM_THREADS / 32);
    finish_map(a.m, (int64_t)per_sm * c.sms);
    const int64_t blocks = (a.m.n_warps + STREAM_THREADS / 32 - 1) / (STREAM_THREADS / 32);
    if constexpr (BWD) { k_stream_bwd<T, W, GPT, WS><<<(unsigned)blocks, STREAM_THREADS, 0, c.stream>>>(a); count_launch(); }
    else { k_stream_fwd<T, W, GPT, WS><<<(unsigned)blocks, STREAM_THREADS, 0, c.stream>>>(a); count_launch(); }
    return cudaGetLastError();
}

template <typename T, bool WS, bool BWD, int GPT>
static cudaError_t by_w(const Ctx &c, int W, HwArgs a) {
    switch (W) {
    case 1: return run_stream<T, 1, GPT, WS, BWD>(c, a);
    case 2: return run_stream<T, 2, GPT, WS, BWD>(c, a);
    case 3: return run_stream<T, 3, GPT, WS, BWD>(c, a);
    case 4: return run_stream<T, 4, GPT, WS, BWD>(c, a);
    case 5: return run_stream<T, 5, GPT, WS, BWD>(c, a);
    case 6: return run_stream<T, 6, GPT, WS, BWD>(c, a);
    case 7: return run_stream<T, 7, GPT, WS, BWD>(c, a);
    case 8: return run_stream<T, 8, GPT, WS, BWD>(c, a);
    }
    return cudaErrorInvalidValue;
}

template <typename T, bool BWD>
static cudaError_t hw_dispatch(const Ctx &c, const dsc_problem &p, HwArgs a) {
    switch (a.m.gpt) {
    case 1: return by_w<T, false, BWD, 1>(c, (int)p.W, a);
    case 2: return by_w<T, false, BWD, 2>(c, (int)p.W, a);
    case 4: return by_w<T, false, BWD, 4>(c, (int)p.W, a);
    case 8:
        if constexpr (VecOf<T>::V == 8) return by_w<T, false, BWD, 8>(c, (int)p.W, a);
        break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_hw_fwd(const Ctx &c, const dsc_problem &p, HwArgs a) {
    return p.dtype == DSC_BF16 ? hw_dispatch<bf16, false>(c, p, a) : hw_dispatch<float, false>(c, p, a);
}
cudaError_t launch_hw_bwd(const Ctx &c, const dsc_problem &p, HwArgs a) {
    return p.dtype == DSC_BF16 ? hw_dispatch<bf16, true>(c, p, a) : hw_dispatch<float, true>(c, p, a);
}
cudaError_t launch_st_fwd(const Ctx &c, const dsc_problem &p, HwArgs a) {
    return p.dtype == DSC_BF16 ? by_w<bf16, true, false, 1>(c, (int)p.W, a) : by_w<float, true, false, 1>(c, (int)p.W, a);
}

// Static backward: the streaming kernel writes one partial filter gradient
// per (sequence, tile); a second kernel sums them in a fixed order.
cudaError_t launch_st_bwd(const Ctx &c, const dsc_problem &p, HwArgs a, float *dws) {
    cudaError_t e = p.dtype == DSC_BF16 ? by_w<bf16, true, true, 1>(c, (int)p.W, a)
                                        : by_w<float, true, true, 1>(c, (int)p.W, a);
    if (e != cudaSuccess) return e;
    return launch_reduce_partials(c, a.partial, st_partial_count(c, p), p.D * p.W, dws);
}

template <typename T> static int64_t st_tiles(const Ctx &c, const dsc_problem &p) {
    StreamMap m;
    stream_map(p, VecOf<T>::V, m);
    const void *k = nullptr;
    switch (p.W) {
    case 1: k = stream_kernel<T, 1, 1, true, true>(); break;
    case 2: k = stream_kernel<T, 2, 1, true, true>(); break;
    case 3: k = stream_kernel<T, 3, 1, true, true>(); break;
    case 4: k = stream_kernel<T, 4, 1, true, true>(); break;
    case 5: k = stream_kernel<T, 5, 1, true, true>(); break;
    case 6: k = stream_kernel<T, 6, 1, true, true>(); break;
    case 7: k = stream_kernel<T, 7, 1, true, true>(); break;
    default: k = stream_kernel<T, 8, 1, true, true>(); break;
    }
    const int per_sm = resident_blocks(k, STREAM_THREADS, 0) * (STREAM_THREADS / 32);
    finish_map(m, (int64_t)per_sm * c.sms);
    return m.B * m.nTiles;
}

// Number of partial gradients the static backward writes (fast path).
size_t st_partial_count(const Ctx &c, const dsc_problem &p) {
    return (size_t)(p.dtype == DSC_BF16 ? st_tiles<bf16>(c, p) : st_tiles<float>(c, p));
}

cudaError_t launch_reduce_partials(const Ctx &c, const float *partial, int64_t S, int64_t n, float *out) {
    const int threads = 256;
    { k_reduce_partials<<<(unsigned)((n + threads - 1) / threads), threads, 0, c.stream>>>(partial, S, n, out); count_launch(); }
    return cudaGetLastError();
}

}  // namespace dsc
