// Generic (fallback) kernels: any D, any H dividing D, any W <= 8.
//
// These handle the shapes the vectorised streaming kernels do not (D not a
// multiple of the 16-byte vector, groups wider than a warp's channels, ...)
// and the unfused low-rank path used when the fused kernels do not apply:
// there the filters w = zU and their gradient dw are held in a caller-given
// fp32 workspace and dz = dw U^T, dU = z^T dw are small tiled GEMMs.
// One thread per channel walks the tokens of a tile with the same
// sliding-window scheme as the fast kernels.
#include "kernels.cuh"

namespace dsc {

constexpr int GEN_THREADS = 256;
constexpr int GEN_TT = 64;

template <typename TW>
__device__ __forceinline__ float filt(const GenArgs &a, const TW *w, int64_t b, int64_t t, int64_t c, int k) {
    if (a.wmode == WMODE_STATIC) return to_f<TW>(w[c * a.W + k]);
    return to_f<TW>(w[((b * a.T + t) * a.G + c / a.H) * a.W + k]);
}

template <typename T, typename TW>
__global__ void __launch_bounds__(GEN_THREADS) k_gen_fwd(const GenArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.z;
    const int t0 = blockIdx.y * a.Tt;
    if (c >= a.D) return;
    const int t1 = (int)min((int64_t)t0 + a.Tt, a.T);
    const T *x = static_cast<const T *>(a.x) + b * a.T * a.D + c;
    T *y = static_cast<T *>(a.y) + b * a.T * a.D + c;
    const TW *w = static_cast<const TW *>(a.w);
    float win[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int t = t0 - 1 - j;
        win[j] = (j < a.W - 1 && t >= 0) ? to_f<T>(x[(int64_t)t * a.D]) : 0.f;
    }
    for (int t = t0; t < t1; ++t) {
        const float xc = to_f<T>(x[(int64_t)t * a.D]);
        float s = a.residual ? xc : 0.f;
        s = fmaf(filt(a, w, b, t, c, 0), xc, s);
#pragma unroll
        for (int k = 1; k < 8; ++k)
            if (k < a.W) s = fmaf(filt(a, w, b, t, c, k), win[k - 1], s);
        y[(int64_t)t * a.D] = from_f<T>(s);
#pragma unroll
        for (int j = 7; j > 0; --j) win[j] = win[j - 1];
        win[0] = xc;
    }
}

// dx[s] = r dy_s + sum_k w(s+k)_k dy_{s+k}; rows are finished W-1 tokens late.
template <typename T, typename TW>
__global__ void __launch_bounds__(GEN_THREADS) k_gen_dx(const GenArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.z;
    const int t0 = blockIdx.y * a.Tt;
    if (c >= a.D) return;
    const int t1 = (int)min((int64_t)t0 + a.Tt, a.T);
    const int tlim = (int)min((int64_t)t1 + a.W - 1, a.T);
    const T *dy = static_cast<const T *>(a.dy) + b * a.T * a.D + c;
    T *dx = static_cast<T *>(a.dx) + b * a.T * a.D + c;
    const TW *w = static_cast<const TW *>(a.w);
    float acc[8];  // acc[j]: partial of row t-j (after token t)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int t = t0; t < t1 + a.W - 1; ++t) {
        const float d = t < tlim ? to_f<T>(dy[(int64_t)t * a.D]) : 0.f;
#pragma unroll
        for (int j = 7; j > 0; --j) acc[j] = acc[j - 1];
        acc[0] = (a.residual && t < t1) ? d : 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < a.W && t < tlim) acc[k] = fmaf(filt(a, w, b, t, c, k), d, acc[k]);
        const int done = t - (a.W - 1);
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k == a.W - 1) v = acc[k];
        if (done >= t0 && done < t1) dx[(int64_t)done * a.D] = from_f<T>(v);
    }
}

// dw[b,t,g,k] = sum_{c in g} dy[b,t,c] x[b,t-k,c]: one warp per (token, group).
template <typename T, typename TO>
__global__ void __launch_bounds__(GEN_THREADS) k_gen_dw(const GenArgs a) {
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t N = a.B * a.T;
    if (wid >= N * a.G) return;
    const int64_t g = wid % a.G, n = wid / a.G;
    const int64_t t = n % a.T;
    const T *x = static_cast<const T *>(a.x);
    const T *dy = static_cast<const T *>(a.dy);
    float s[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] = 0.f;
    for (int64_t c = g * a.H + lane; c < (g + 1) * a.H; c += 32) {
        const float d = to_f<T>(dy[n * a.D + c]);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < a.W && t - k >= 0) s[k] = fmaf(d, to_f<T>(x[(n - k) * a.D + c]), s[k]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
        for (int o = 16; o > 0; o >>= 1) s[k] += __shfl_xor_sync(FULL_MASK, s[k], o);
    if (lane < a.W) {
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k == lane) v = s[k];
        static_cast<TO *>(a.dw)[(n * a.G + g) * a.W + lane] = from_f<TO>(v);
    }
}

// Static filter gradient partials: one per (sequence, tile), channel per thread.
template <typename T>
__global__ void __launch_bounds__(GEN_THREADS) k_gen_dws_partial(const GenArgs a, float *partial) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.z;
    const int t0 = blockIdx.y * a.Tt;
    if (c >= a.D) return;
    const int t1 = (int)min((int64_t)t0 + a.Tt, a.T);
    const T *x = static_cast<const T *>(a.x) + b * a.T * a.D + c;
    const T *dy = static_cast<const T *>(a.dy) + b * a.T * a.D + c;
    float win[8], s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int t = t0 - 1 - j;
        win[j] = (j < a.W - 1 && t >= 0) ? to_f<T>(x[(int64_t)t * a.D]) : 0.f;
        s[j] = 0.f;
    }
    for (int t = t0; t < t1; ++t) {
        const float xc = to_f<T>(x[(int64_t)t * a.D]);
        const float d = to_f<T>(dy[(int64_t)t * a.D]);
        s[0] = fmaf(d, xc, s[0]);
#pragma unroll
        for (int k = 1; k < 8; ++k) s[k] = fmaf(d, win[k - 1], s[k]);
#pragma unroll
        for (int j = 7; j > 0; --j) win[j] = win[j - 1];
        win[0] = xc;
    }
    const int64_t si = b * a.nTiles + blockIdx.y;
    for (int k = 0; k < a.W; ++k) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j == k) v = s[j];
        partial[(si * a.D + c) * a.W + k] = v;
    }
}

// Low-rank filters w[n, j] = sum_r z[n, r] U[r, j] into a fp32 workspace.
template <typename T>
__global__ void __launch_bounds__(256) k_lr_filters(const T *__restrict__ z, const T *__restrict__ U, float *wf,
                                                    int64_t N, int R, int64_t GW) {
    constexpr int TB = 16;
    __shared__ __align__(16) float zs[256][TB];  // [r][token]: one 16-byte load gives four tokens' z_r
    const int64_t n0 = (int64_t)blockIdx.y * TB;
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = threadIdx.x; i < TB * R; i += blockDim.x) {
        const int tn = i / R, r = i % R;
        zs[r][tn] = (n0 + tn < N) ? to_f<T>(z[(n0 + tn) * R + r]) : 0.f;
    }
    __syncthreads();
    if (j >= GW) return;
    float acc[TB];
#pragma unroll
    for (int i = 0; i < TB; ++i) acc[i] = 0.f;
    for (int r = 0; r < R; ++r) {
        const float u = to_f<T>(U[(int64_t)r * GW + j]);
#pragma unroll
        for (int i = 0; i < TB; i += 4) {
            const float4 zq = *reinterpret_cast<const float4 *>(&zs[r][i]);
            acc[i] = fmaf(zq.x, u, acc[i]);
            acc[i + 1] = fmaf(zq.y, u, acc[i + 1]);
            acc[i + 2] = fmaf(zq.z, u, acc[i + 2]);
            acc[i + 3] = fmaf(zq.w, u, acc[i + 3]);
        }
    }
#pragma unroll
    for (int i = 0; i < TB; ++i)
        if (n0 + i < N) wf[(n0 + i) * GW + j] = acc[i];
}

// C[i][j] = sum_k A(i,k) B(j,k), 64x64 tiles, 16-deep k steps, 4x4 per thread.
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) k_gemm(int M, int N, int K, const TA *A, int64_t sai, int64_t sak, const TB *B,
                                              int64_t sbj, int64_t sbk, TC *C, int64_t ldc) {
    __shared__ float As[16][64 + 1];
    __shared__ float Bs[16][64 + 1];
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int kk = e / 64, ii = e % 64;
            const int64_t k = k0 + kk;
            As[kk][ii] = (i0 + ii < M && k < K) ? to_f<TA>(A[(int64_t)(i0 + ii) * sai + k * sak]) : 0.f;
            Bs[kk][ii] = (j0 + ii < N && k < K) ? to_f<TB>(B[(int64_t)(j0 + ii) * sbj + k * sbk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                av[q] = As[kk][ty * 4 + q];
                bv[q] = Bs[kk][tx * 4 + q];
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = i0 + ty * 4 + p, j = j0 + tx * 4 + q;
            if (i < M && j < N) C[(int64_t)i * ldc + j] = from_f<TC>(acc[p][q]);
        }
}

// ------------------------------------------------------------------- host ---

static dim3 gen_grid(const dsc_problem &p, GenArgs &a) {
    a.Tt = GEN_TT;
    a.nTiles = (int)((p.T + GEN_TT - 1) / GEN_TT);
    return dim3((unsigned)((p.D + GEN_THREADS - 1) / GEN_THREADS), (unsigned)a.nTiles, (unsigned)p.B);
}

cudaError_t launch_gen_fwd(const Ctx &c, const dsc_problem &p, GenArgs a, bool w_f32) {
    dim3 g = gen_grid(p, a);
    if (p.dtype == DSC_BF16) {
        if (w_f32) { k_gen_fwd<bf16, float><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
        else { k_gen_fwd<bf16, bf16><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    } else {
        { k_gen_fwd<float, float><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    }
    return cudaGetLastError();
}

cudaError_t launch_gen_dx(const Ctx &c, const dsc_problem &p, GenArgs a, bool w_f32) {
    dim3 g = gen_grid(p, a);
    if (p.dtype == DSC_BF16) {
        if (w_f32) { k_gen_dx<bf16, float><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
        else { k_gen_dx<bf16, bf16><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    } else {
        { k_gen_dx<float, float><<<g, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    }
    return cudaGetLastError();
}

cudaError_t launch_gen_dw(const Ctx &c, const dsc_problem &p, GenArgs a, bool out_f32) {
    const int64_t warps = p.B * p.T * (p.D / p.H);
    const int64_t blocks = (warps * 32 + GEN_THREADS - 1) / GEN_THREADS;
    if (p.dtype == DSC_BF16) {
        if (out_f32) { k_gen_dw<bf16, float><<<(unsigned)blocks, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
        else { k_gen_dw<bf16, bf16><<<(unsigned)blocks, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    } else {
        { k_gen_dw<float, float><<<(unsigned)blocks, GEN_THREADS, 0, c.stream>>>(a); count_launch(); }
    }
    return cudaGetLastError();
}

// Static backward, generic: per-channel dx plus partials reduced in order.
cudaError_t launch_gen_dws(const Ctx &c, const dsc_problem &p, GenArgs a, float *dws, float *partial, int) {
    dim3 g = gen_grid(p, a);
    if (p.dtype == DSC_BF16) { k_gen_dws_partial<bf16><<<g, GEN_THREADS, 0, c.stream>>>(a, partial); count_launch(); }
    else { k_gen_dws_partial<float><<<g, GEN_THREADS, 0, c.stream>>>(a, partial); count_launch(); }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_reduce_partials(c, partial, p.B * (int64_t)a.nTiles, p.D * p.W, dws);
}

cudaError_t launch_lr_filters(const Ctx &c, const dsc_problem &p, const void *z, const void *U, float *wf) {
    const int64_t N = p.B * p.T, GW = (p.D / p.H) * p.W;
    dim3 g((unsigned)((GW + 255) / 256), (unsigned)((N + 15) / 16));
    if (p.dtype == DSC_BF16)
        { k_lr_filters<bf16><<<g, 256, 0, c.stream>>>((const bf16 *)z, (const bf16 *)U, wf, N, (int)p.R, GW); count_launch(); }
    else
        { k_lr_filters<float><<<g, 256, 0, c.stream>>>((const float *)z, (const float *)U, wf, N, (int)p.R, GW); count_launch(); }
    return cudaGetLastError();
}

cudaError_t launch_gemm(const Ctx &c, int M, int N, int K, const void *A, bool a_f32, int64_t sai, int64_t sak,
                        const void *B, bool b_f32, int64_t sbj, int64_t sbk, void *C, bool c_f32, int64_t ldc,
                        bool bf16_io) {
    dim3 g((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64));
    // A is the fp32 workspace or the bf16/fp32 input; B likewise; C fp32 or io type.
#define DSC_GEMM(TA, TB, TC)                                                                                   \
    k_gemm<TA, TB, TC><<<g, 256, 0, c.stream>>>(M, N, K, (const TA *)A, sai, sak, (const TB *)B, sbj, sbk, (TC *)C, ldc)
    if (!bf16_io) {
        DSC_GEMM(float, float, float);
    } else if (a_f32 && !b_f32) {
        if (c_f32) DSC_GEMM(float, bf16, float); else DSC_GEMM(float, bf16, bf16);
    } else if (!a_f32 && b_f32) {
        if (c_f32) DSC_GEMM(bf16, float, float); else DSC_GEMM(bf16, float, bf16);
    } else if (a_f32 && b_f32) {
        if (c_f32) DSC_GEMM(float, float, float); else DSC_GEMM(float, float, bf16);
    } else {
        if (c_f32) DSC_GEMM(bf16, bf16, float); else DSC_GEMM(bf16, bf16, bf16);
    }
    count_launch();
#undef DSC_GEMM
    return cudaGetLastError();
}

}  // namespace dsc
