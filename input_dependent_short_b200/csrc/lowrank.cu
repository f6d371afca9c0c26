// Fused low-rank dynamic short convolution (CUDA-core kernels, any shape).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 (low-rank factorisation of rank R of the
// filter generator) and "Efficient training implementation" (the fused
// low-rank kernel reads z and U, forms zU on chip and convolves at once,
// without writing the dynamic filter tensor to HBM).  Here the filters are
// w[b,t,g,k] = sum_r z[b,t,r] U[r, g*W+k] with head-wise groups of H channels.
//
// One CTA owns a tile of Tt tokens of one sequence and walks the channels in
// chunks of whole filter groups:
//   1. the chunk's filters for the tile (plus a (W-1)-token right halo in the
//      backward) are formed in shared memory from the z tile and U columns;
//   2. a streaming pass over the chunk's channels (one 16-byte channel vector
//      per thread, register sliding windows as in the head-wise kernels) reads
//      x (and dy) once and writes y (or dx and the chunk's dw into shared
//      memory, reduced over each group's H channels with shuffles);
//   3. backward only: a CTA owns one column chunk and a contiguous range of
//      token tiles.  The chunk's dU accumulator (R x chunk columns) stays in
//      shared memory over the whole range and is written once as a per-range
//      partial; dz[t,r] = sum_j dw[t,j] U[r,j] gets one contribution per chunk
//      (written directly when one chunk covers all channels, otherwise added
//      into an fp32 accumulator).  A small kernel then sums the dU partials in
//      a fixed order and rounds dz.
// w and dw never leave the SM; the workspace holds only the R x (G*W) dU
// partials of the token ranges and, with several chunks, dz in fp32.  When the
// token tile is split across warps (narrow chunks), each warp streams a
// sub-tile of TS tokens.
#include "kernels.cuh"

namespace dsc {

constexpr int LR_THREADS = 256;
constexpr int LR_WARPS = LR_THREADS / 32;

// Device status word of this library on each device: 0 = OK, otherwise the
// dsc_status a kernel recorded when one of its bounded waits expired.
__device__ int g_dsc_status = 0;

int take_device_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

struct LrMap {
    int64_t B, T, D, H, G, R, GW;
    int W;
    int CW, lanes_used, L, gpt;  // lane mapping inside a warp (as for the head-wise kernels)
    int SUB, TS, Tt, nTiles;     // token sub-tiles per tile, tokens per sub-tile / tile
    int CHC, CGc, CC, nChunks;   // channels, groups and columns per chunk
    int nRanges, tilesPerRange;  // backward: token ranges (each CTA: one range x one chunk)
    int64_t totalTiles;
    int residual;
};

struct LrArgs {
    LrMap m;
    const void *x, *z, *U, *dy;
    void *y, *dx, *dz;
    float *dU;
    float *dz_acc;   // fp32 [B*T][R] accumulator of dz (several column chunks)
    float *dU_part;  // fp32 [nRanges][R][G*W] per-range partials of dU
};

// w_s[i][j] = sum_r z_s[i][r] U[r][col0 + j] for i < rows, j < cols: each work
// item is one column and 8 rows.
template <typename T>
__device__ __forceinline__ void form_filters(const LrMap &m, const float *z_s, float *w_s, const T *U, int64_t col0,
                                             int rows, int cols) {
    const int rb = (rows + 7) / 8;
    for (int item = threadIdx.x; item < cols * rb; item += LR_THREADS) {
        const int j = item % cols, i0 = (item / cols) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const T *u = U + col0 + j;
        for (int r = 0; r < m.R; ++r) {
            const float uv = to_f<T>(__ldg(u + (int64_t)r * m.GW));
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(z_s[(i0 + q) * m.R + r], uv, acc[q]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (i0 + q < rows) w_s[(i0 + q) * m.CC + j] = acc[q];
    }
}

// ------------------------------------------------------------------ forward ---

template <typename T, int W, int GPT>
__global__ void __launch_bounds__(LR_THREADS) k_lr_fwd(const LrArgs a) {
    constexpr int V = VecOf<T>::V, CPG = V / GPT, WIN = W - 1, XW = W > 1 ? W - 1 : 1;
    extern __shared__ float sm[];
    const LrMap &m = a.m;
    const int tile = blockIdx.x % m.nTiles;
    const int64_t b = blockIdx.x / m.nTiles;
    const int t0 = tile * m.Tt;
    const int rows = (int)min((int64_t)m.Tt, m.T - t0);
    float *z_s = sm;                                  // [Tt rounded up to 8][R]
    float *w_s = z_s + ((m.Tt + 7) / 8) * 8 * m.R;    // [Tt][CC]
    const T *z = static_cast<const T *>(a.z) + (b * m.T + t0) * m.R;
    for (int i = threadIdx.x; i < rows * m.R; i += LR_THREADS) z_s[i] = to_f<T>(z[i]);
    for (int i = rows * m.R + threadIdx.x; i < ((rows + 7) / 8) * 8 * m.R; i += LR_THREADS) z_s[i] = 0.f;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpr = LR_WARPS / m.SUB;  // warps per chunk row
    const int sub = warp / wpr, wrow = warp % wpr;
    const int ts0 = t0 + sub * m.TS, ts1 = (int)min((int64_t)ts0 + m.TS, (int64_t)t0 + rows);
    const float res = m.residual ? 1.f : 0.f;
    const int64_t row0 = b * m.T;

    for (int ch = 0; ch < m.nChunks; ++ch) {
        const int64_t c_lo = (int64_t)ch * m.CHC;
        const int64_t g_lo = c_lo / m.H;
        const int cols = (int)min((int64_t)m.CC, m.GW - g_lo * W);
        __syncthreads();
        form_filters<T>(m, z_s, w_s, static_cast<const T *>(a.U), g_lo * W, rows, cols);
        __syncthreads();
        const int64_t c0 = c_lo + (int64_t)wrow * m.CW + (int64_t)lane * V;
        if (lane >= m.lanes_used || c0 >= m.D || c0 >= c_lo + m.CHC || ts0 >= ts1) continue;
        const int jg = (int)((c0 / m.H - g_lo) * W);  // first filter column of this thread
        const T *xp = static_cast<const T *>(a.x) + row0 * m.D + c0;
        T *yp = static_cast<T *>(a.y) + row0 * m.D + c0;
        float xs[XW][V];
#pragma unroll
        for (int j = 0; j < XW; ++j) {
            const int t = ts0 - 1 - j;
            if (WIN > 0 && t >= 0) unpack(ld16(xp + (int64_t)t * m.D), xs[j]);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) xs[j][v] = 0.f;
        }
        for (int tb = ts0; tb < ts1; tb += 4) {
            uint4 xr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) xr[u] = tb + u < ts1 ? ld16(xp + (int64_t)(tb + u) * m.D) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = tb + u;
                if (t >= ts1) break;
                float xc[V], acc[V];
                unpack(xr[u], xc);
                const float *wr = w_s + (t - t0) * m.CC + jg;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int f = (v / CPG) * W;
                    float s = fmaf(wr[f], xc[v], res * xc[v]);
#pragma unroll
                    for (int k = 1; k < W; ++k) s = fmaf(wr[f + k], xs[k - 1][v], s);
                    acc[v] = s;
                }
                st16(yp + (int64_t)t * m.D, pack(acc));
#pragma unroll
                for (int j = XW - 1; j > 0; --j)
#pragma unroll
                    for (int v = 0; v < V; ++v) xs[j][v] = xs[j - 1][v];
#pragma unroll
                for (int v = 0; v < V; ++v) xs[0][v] = xc[v];
            }
        }
    }
}

// ----------------------------------------------------------------- backward ---

// One CTA per (token range, column chunk): it walks the tiles of its range,
// keeping the chunk of U (fp32, padded rows) and the chunk's dU accumulator in
// shared memory; dz per tile is summed over chunks in an fp32 accumulator.
template <typename T, int W, int GPT>
__global__ void __launch_bounds__(LR_THREADS) k_lr_bwd(const LrArgs a) {
    constexpr int V = VecOf<T>::V, CPG = V / GPT, WIN = W - 1, XW = W > 1 ? W - 1 : 1;
    extern __shared__ float sm[];
    const LrMap &m = a.m;
    const int ch = blockIdx.x % m.nChunks;
    const int range = blockIdx.x / m.nChunks;
    const int R = (int)m.R, RP = R + 1;
    const int RW = ((m.Tt + WIN + 7) / 8) * 8;
    float *z_s = sm;                    // [RW][R]
    float *w_s = z_s + RW * R;          // [RW][CC]
    float *dw_s = w_s + RW * m.CC;      // [Tt][CC]
    float *dU_s = dw_s + m.Tt * m.CC;   // [R][CC]
    float *u_s = dU_s + R * m.CC;       // [CC][R+1]  (U chunk, transposed, padded)

    const int64_t c_lo = (int64_t)ch * m.CHC;
    const int64_t g_lo = c_lo / m.H;
    const int64_t col0 = g_lo * W;
    const int cols = (int)min((int64_t)m.CC, m.GW - col0);
    const T *U = static_cast<const T *>(a.U);
    for (int i = threadIdx.x; i < R * m.CC; i += LR_THREADS) {
        const int r = i / m.CC, j = i % m.CC;
        u_s[j * RP + r] = j < cols ? to_f<T>(U[(int64_t)r * m.GW + col0 + j]) : 0.f;
        dU_s[i] = 0.f;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpr = LR_WARPS / m.SUB;
    const int sub = warp / wpr, wrow = warp % wpr;
    const float res = m.residual ? 1.f : 0.f;
    const int L = m.L, pos = lane % L;
    const int64_t c0r = c_lo + (int64_t)wrow * m.CW + (int64_t)lane * V;
    const bool act = lane < m.lanes_used && c0r < m.D && c0r < c_lo + m.CHC;
    const int64_t c0 = act ? c0r : c_lo;  // inactive lanes stream an in-bounds vector, never stored
    const int jg = (int)((c0 / m.H - g_lo) * W);

    const int64_t tile_lo = (int64_t)range * m.tilesPerRange;
    const int64_t tile_hi = min(tile_lo + m.tilesPerRange, m.totalTiles);
    for (int64_t ti = tile_lo; ti < tile_hi; ++ti) {
        const int64_t b = ti / m.nTiles;
        const int t0 = (int)(ti % m.nTiles) * m.Tt;
        const int rows = (int)min((int64_t)m.Tt, m.T - t0);
        const int rows_w = (int)min((int64_t)m.Tt + WIN, m.T - t0);
        const int64_t row0 = b * m.T;
        __syncthreads();  // previous tile fully consumed
        const T *z = static_cast<const T *>(a.z) + (row0 + t0) * R;
        for (int i = threadIdx.x; i < RW * R; i += LR_THREADS) z_s[i] = i < rows_w * R ? to_f<T>(z[i]) : 0.f;
        __syncthreads();
        // filters of the tile (+ right halo): w_s[i][j] = sum_r z_s[i][r] u(r, j)
        {
            const int rb = (rows_w + 7) / 8;
            for (int item = threadIdx.x; item < cols * rb; item += LR_THREADS) {
                const int j = item % cols, i0 = (item / cols) * 8;
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int r = 0; r < R; ++r) {
                    const float uv = u_s[j * RP + r];
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[q] = fmaf(z_s[(i0 + q) * R + r], uv, acc[q]);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (i0 + q < rows_w) w_s[(i0 + q) * m.CC + j] = acc[q];
            }
        }
        __syncthreads();

        // streaming pass over this warp's token sub-tile: dx rows and dw (into dw_s)
        const int ts0 = t0 + sub * m.TS, ts1 = (int)min((int64_t)ts0 + m.TS, (int64_t)t0 + rows);
        const int tl1 = (int)min((int64_t)ts1 + WIN, m.T);
        if (ts0 < ts1) {  // warp-uniform
            const T *xp = static_cast<const T *>(a.x) + row0 * m.D + c0;
            const T *dyp = static_cast<const T *>(a.dy) + row0 * m.D + c0;
            T *dxp = static_cast<T *>(a.dx) + row0 * m.D + c0;
            float xs[XW][V], acc[XW][V];
#pragma unroll
            for (int j = 0; j < XW; ++j) {
                const int t = ts0 - 1 - j;
                if (WIN > 0 && t >= 0) unpack(ld16(xp + (int64_t)t * m.D), xs[j]);
                else
#pragma unroll
                    for (int v = 0; v < V; ++v) xs[j][v] = 0.f;
#pragma unroll
                for (int v = 0; v < V; ++v) acc[j][v] = 0.f;
            }
            for (int tb = ts0; tb < ts1 + WIN; tb += 4) {
                uint4 xr[4], dr[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    xr[u] = tb + u < ts1 ? ld16(xp + (int64_t)(tb + u) * m.D) : make_uint4(0, 0, 0, 0);
                    dr[u] = tb + u < tl1 ? ld16(dyp + (int64_t)(tb + u) * m.D) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = tb + u;
                    if (t >= ts1 + WIN) break;
                    const bool hx = t < ts1, hd = t < tl1;
                    float xc[V], dyc[V], r0[V], wv[GPT * W];
                    unpack(xr[u], xc);
                    unpack(dr[u], dyc);
                    if (hd) {
                        const float *wr = w_s + (t - t0) * m.CC + jg;
#pragma unroll
                        for (int f = 0; f < GPT * W; ++f) wv[f] = wr[f];
                    } else {
#pragma unroll
                        for (int f = 0; f < GPT * W; ++f) wv[f] = 0.f;
                    }
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const int f = (v / CPG) * W;
                        r0[v] = (wv[f] + res) * dyc[v];
#pragma unroll
                        for (int k = 1; k < W; ++k) acc[k - 1][v] = fmaf(wv[f + k], dyc[v], acc[k - 1][v]);
                    }
                    const int done = t - WIN;
                    if (act && done >= ts0) {
                        if constexpr (W > 1) st16(dxp + (int64_t)done * m.D, pack(acc[XW - 1]));
                        else st16(dxp + (int64_t)done * m.D, pack(r0));
                    }
                    if (hx) {
                        float part[GPT * W];
#pragma unroll
                        for (int gi = 0; gi < GPT; ++gi)
#pragma unroll
                            for (int k = 0; k < W; ++k) {
                                float s2 = 0.f;
#pragma unroll
                                for (int v = gi * CPG; v < (gi + 1) * CPG; ++v)
                                    s2 = fmaf(dyc[v], k == 0 ? xc[v] : xs[k - 1][v], s2);
                                part[gi * W + k] = s2;
                            }
                        float *dwr = dw_s + (t - t0) * m.CC + jg;
                        if (GPT == 1 && L > 1) {
                            for (int o = 1; o < L; o <<= 1)
#pragma unroll
                                for (int k = 0; k < W; ++k) {
                                    const float o2 = __shfl_down_sync(FULL_MASK, part[k], o);
                                    if (pos + o < L) part[k] += o2;
                                }
                            if (act && pos == 0)
#pragma unroll
                                for (int k = 0; k < W; ++k) dwr[k] = part[k];
                        } else if (act) {
#pragma unroll
                            for (int f = 0; f < GPT * W; ++f) dwr[f] = part[f];
                        }
                    }
#pragma unroll
                    for (int j = XW - 1; j > 0; --j)
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            acc[j][v] = acc[j - 1][v];
                            xs[j][v] = xs[j - 1][v];
                        }
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        acc[0][v] = r0[v];
                        xs[0][v] = xc[v];
                    }
                }
            }
        }
        __syncthreads();
        // dz rows of this tile: sum over the chunk's columns of dw[t][j] U[r][j]
        for (int item = threadIdx.x; item < rows * R; item += LR_THREADS) {
            const int t = item / R, r = item % R;
            const float *dwr = dw_s + t * m.CC;
            float s2 = 0.f;
            for (int j = 0; j < cols; ++j) s2 = fmaf(dwr[j], u_s[j * RP + r], s2);
            const int64_t o = (row0 + t0 + t) * R + r;
            if (m.nChunks == 1) static_cast<T *>(a.dz)[o] = from_f<T>(s2);
            else atomicAdd(a.dz_acc + o, s2);
        }
        // dU accumulator of the chunk: sum over the tile's tokens of z[t][r] dw[t][j]
        for (int item = threadIdx.x; item < R * cols; item += LR_THREADS) {
            const int r = item / cols, j = item % cols;
            float s2 = 0.f;
            for (int t = 0; t < rows; ++t) s2 = fmaf(z_s[t * R + r], dw_s[t * m.CC + j], s2);
            dU_s[r * m.CC + j] += s2;
        }
    }
    __syncthreads();
    float *part = a.dU_part + (int64_t)range * R * m.GW;
    for (int i = threadIdx.x; i < R * cols; i += LR_THREADS) {
        const int r = i / cols, j = i % cols;
        part[(int64_t)r * m.GW + col0 + j] = dU_s[r * m.CC + j];
    }
}

// dU = sum of the per-range partials (fixed order); dz = the fp32 accumulator
// rounded to the output type (when several chunks contributed).
template <typename T>
__global__ void k_lr_finalize(const LrArgs a) {
    const LrMap &m = a.m;
    const int64_t nU = m.R * m.GW, nz = a.m.B * a.m.T * m.R;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nU + nz; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nU) {
            float s = 0.f;
            for (int q = 0; q < m.nRanges; ++q) s += a.dU_part[(int64_t)q * nU + i];
            a.dU[i] = s;
        } else if (m.nChunks > 1) {
            static_cast<T *>(a.dz)[i - nU] = from_f<T>(a.dz_acc[i - nU]);
        }
    }
}

__global__ void k_zero(float *p, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = 0.f;
}

// ------------------------------------------------------------------- host ---

static size_t lr_smem(const LrMap &m, bool bwd) {
    const int WIN = m.W - 1;
    if (!bwd) return (size_t)(((m.Tt + 7) / 8) * 8 * m.R + m.Tt * m.CC) * sizeof(float);
    const int RW = ((m.Tt + WIN + 7) / 8) * 8;
    return (size_t)(RW * m.R + RW * m.CC + m.Tt * m.CC + m.R * m.CC + m.CC * (m.R + 1)) * sizeof(float);
}

static bool lr_map(const dsc_problem &p, bool bwd, LrMap &m) {
    const int V = p.dtype == DSC_BF16 ? 8 : 4;
    m = LrMap{};
    m.B = p.B; m.T = p.T; m.D = p.D; m.H = p.H; m.G = p.D / p.H; m.R = p.R; m.W = (int)p.W;
    m.GW = m.G * p.W;
    m.residual = p.residual ? 1 : 0;
    if (p.D % V) return false;
    if (V % p.H == 0) {
        m.gpt = (int)(V / p.H); m.L = 1; m.lanes_used = 32; m.CW = 32 * V;
    } else if (p.H % V == 0 && p.H / V <= 32) {
        m.gpt = 1; m.L = (int)(p.H / V);
        const int gpw = 32 / m.L;
        m.lanes_used = gpw * m.L; m.CW = (int)(gpw * p.H);
    } else {
        return false;
    }
    int wpr = LR_WARPS;
    while (wpr > 1 && (int64_t)(wpr / 2) * m.CW >= p.D) wpr /= 2;  // no idle warps beyond D
    int Tt = 64;
    // Shrink until the shared-memory tiles fit: first the tile length (to 32),
    // then the warps per chunk row, then the lanes (filter groups) per warp,
    // then the tile length again.
    auto fit = [&](size_t cap) {
        for (;;) {
            m.SUB = LR_WARPS / wpr;
            m.CHC = wpr * m.CW;
            m.CGc = (int)(m.CHC / p.H);
            m.CC = m.CGc * (int)p.W;
            m.Tt = Tt;
            if (lr_smem(m, bwd) <= cap) return true;
            if (Tt > 32) Tt /= 2;
            else if (wpr > 1) wpr /= 2;
            else if (m.L == 1 && m.lanes_used > 4) { m.lanes_used /= 2; m.CW = m.lanes_used * V; }
            else if (m.L > 1 && m.lanes_used >= 2 * m.L) {
                const int gpw = (m.lanes_used / m.L) / 2;
                m.lanes_used = gpw * m.L;
                m.CW = (int)(gpw * p.H);
            }
            else if (Tt > 8) Tt /= 2;
            else return false;
        }
    };
    if (!fit(100 * 1024) && !fit(200 * 1024)) return false;
    if (Tt < m.SUB) return false;
    m.TS = m.Tt / m.SUB;
    m.nTiles = (int)((p.T + m.Tt - 1) / m.Tt);
    m.nChunks = (int)((p.D + m.CHC - 1) / m.CHC);
    m.totalTiles = p.B * (int64_t)m.nTiles;
    // backward: about two CTAs per SM in one wave, each over a contiguous range of tiles
    int64_t ranges = (2 * 148 + m.nChunks - 1) / m.nChunks;
    if (ranges > m.totalTiles) ranges = m.totalTiles;
    if (ranges < 1) ranges = 1;
    m.tilesPerRange = (int)((m.totalTiles + ranges - 1) / ranges);
    m.nRanges = (int)((m.totalTiles + m.tilesPerRange - 1) / m.tilesPerRange);
    return true;
}

// Workspace of the fused backward: per-range dU partials, plus the fp32 dz
// accumulator when the channels span several chunks.
static size_t lr_ws_bytes(const LrMap &m) {
    size_t n = (size_t)m.nRanges * m.R * m.GW;
    if (m.nChunks > 1) n += (size_t)m.B * m.T * m.R;
    return n * sizeof(float);
}

bool lowrank_fused_ok(const dsc_problem &p) {
    LrMap f, b;
    return lr_map(p, false, f) && lr_map(p, true, b);
}

template <typename T, int W, int GPT, bool BWD>
static cudaError_t lr_launch(const Ctx &c, const LrArgs &a, size_t smem) {
    const void *k = BWD ? (const void *)k_lr_bwd<T, W, GPT> : (const void *)k_lr_fwd<T, W, GPT>;
    static const cudaError_t attr =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (attr != cudaSuccess) return attr;
    const unsigned grid = BWD ? (unsigned)(a.m.nRanges * a.m.nChunks) : (unsigned)(a.m.B * a.m.nTiles);
    if constexpr (BWD) k_lr_bwd<T, W, GPT><<<grid, LR_THREADS, smem, c.stream>>>(a);
    else k_lr_fwd<T, W, GPT><<<grid, LR_THREADS, smem, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename T, int GPT, bool BWD>
static cudaError_t lr_by_w(const Ctx &c, const LrArgs &a, size_t smem) {
    switch (a.m.W) {
    case 1: return lr_launch<T, 1, GPT, BWD>(c, a, smem);
    case 2: return lr_launch<T, 2, GPT, BWD>(c, a, smem);
    case 3: return lr_launch<T, 3, GPT, BWD>(c, a, smem);
    case 4: return lr_launch<T, 4, GPT, BWD>(c, a, smem);
    case 5: return lr_launch<T, 5, GPT, BWD>(c, a, smem);
    case 6: return lr_launch<T, 6, GPT, BWD>(c, a, smem);
    case 7: return lr_launch<T, 7, GPT, BWD>(c, a, smem);
    case 8: return lr_launch<T, 8, GPT, BWD>(c, a, smem);
    }
    return cudaErrorInvalidValue;
}

template <typename T, bool BWD>
static cudaError_t lr_dispatch(const Ctx &c, const LrArgs &a, size_t smem) {
    switch (a.m.gpt) {
    case 1: return lr_by_w<T, 1, BWD>(c, a, smem);
    case 2: return lr_by_w<T, 2, BWD>(c, a, smem);
    case 4: return lr_by_w<T, 4, BWD>(c, a, smem);
    case 8:
        if constexpr (VecOf<T>::V == 8) return lr_by_w<T, 8, BWD>(c, a, smem);
        break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_lr_fwd_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                void *y) {
    LrArgs a{};
    if (!lr_map(p, false, a.m)) return cudaErrorNotSupported;
    a.x = x; a.z = z; a.U = U; a.y = y;
    const size_t smem = lr_smem(a.m, false);
    return p.dtype == DSC_BF16 ? lr_dispatch<bf16, false>(c, a, smem) : lr_dispatch<float, false>(c, a, smem);
}

cudaError_t launch_lr_bwd_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                const void *dy, void *dx, void *dz, float *dU, void *ws, size_t ws_bytes) {
    LrArgs a{};
    if (!lr_map(p, true, a.m)) return cudaErrorNotSupported;
    if (ws_bytes < lr_ws_bytes(a.m) || !ws) return cudaErrorInvalidValue;
    a.x = x; a.z = z; a.U = U; a.dy = dy; a.dx = dx; a.dz = dz; a.dU = dU;
    a.dU_part = static_cast<float *>(ws);
    a.dz_acc = a.dU_part + (size_t)a.m.nRanges * a.m.R * a.m.GW;
    if (a.m.nChunks > 1) {
        const int64_t n = a.m.B * a.m.T * a.m.R;
        k_zero<<<(unsigned)min((int64_t)1024, (n + 255) / 256), 256, 0, c.stream>>>(a.dz_acc, n);
        count_launch();
    }
    const size_t smem = lr_smem(a.m, true);
    cudaError_t e = p.dtype == DSC_BF16 ? lr_dispatch<bf16, true>(c, a, smem) : lr_dispatch<float, true>(c, a, smem);
    if (e != cudaSuccess) return e;
    const int64_t n = a.m.R * a.m.GW + (a.m.nChunks > 1 ? a.m.B * a.m.T * a.m.R : 0);
    const unsigned g = (unsigned)min((int64_t)2048, (n + 255) / 256);
    if (p.dtype == DSC_BF16) k_lr_finalize<bf16><<<g, 256, 0, c.stream>>>(a);
    else k_lr_finalize<float><<<g, 256, 0, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

size_t lr_bwd_fused_ws_bytes(const Ctx &, const dsc_problem &p) {
    LrMap m;
    return lr_map(p, true, m) ? lr_ws_bytes(m) : 0;
}

}  // namespace dsc
