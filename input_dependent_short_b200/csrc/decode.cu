// Decode step of the dynamic short convolution: one new token per sequence,
// with a rolling state of the sequence's last W-1 inputs.
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Mechanism" (y_t = sum_k w(t)_k x_{t-k}), "Placement" (the
// residual X + conv(X)) and "Parameterisation" 1-2 (low-rank and head-wise
// filters).  At inference a causal short convolution only ever needs the last
// W-1 inputs of each sequence, so a step reads them from a state instead of
// the whole history:
//   y[b,c]   = r x[b,c] + w_0 x[b,c] + sum_{k=1}^{W-1} w_k state[b, W-1-k, c]
//   state'   = state rows 1 .. W-2, then x   (row j holds x_{t-W+1+j})
// with the filters of the new token (head-wise w [B,G,W], static ws [D,W], or
// low-rank w = z U formed first by k_lr_filters into a [B,G,W] fp32 scratch:
// for one token per sequence that is B*G*W values, not a per-token tensor of
// the whole sequence).
//
// Thread = (sequence, vector of V channels): it reads x and the W-1 state
// rows of its channels once, writes y and the shifted state rows in place
// (no other thread touches them), all with 16-byte accesses when D allows.
// The step moves (2 + 2(W-1)) D elements per sequence plus the filters; it is
// bound by HBM bandwidth at large B and by launch latency at small B.
#include <algorithm>

#include "kernels.cuh"

namespace dsc {
namespace {

struct DecArgs {
    int64_t B, D, H, G;
    int residual;
    const void *x;  // [B, D]
    const void *w;  // head-wise [B, G, W] / low-rank fp32 [B, G, W] / static [D, W]
    void *state;    // [B, W-1, D]
    void *y;        // [B, D]
};

enum { DEC_HEADWISE = 0, DEC_LOWRANK = 1, DEC_STATIC = 2 };

template <typename T, int V> __device__ __forceinline__ void load_v(const T *p, float (&f)[V], bool nc) {
    if constexpr (V == VecOf<T>::V) {
        uint4 u;
        if (nc) {
            u = ld16(p);
        } else {
            u = *reinterpret_cast<const uint4 *>(p);
        }
        unpack(u, f);
    } else {
        static_assert(V == 1, "a 16-byte vector or one element");
        f[0] = to_f<T>(*p);
    }
}

template <typename T, int V> __device__ __forceinline__ void store_v(T *p, const float (&f)[V]) {
    if constexpr (V == VecOf<T>::V) {
        st16(p, pack(f));
    } else {
        *p = from_f<T>(f[0]);
    }
}

// WT: filter element type (T, or float for the low-rank scratch).
template <typename T, typename WT, int W, int V, int MODE>
__global__ void __launch_bounds__(256) k_decode(const DecArgs a) {
    constexpr int S = W - 1;
    const int64_t nv = a.D / V;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.B * nv) return;
    const int64_t b = i / nv, c0 = (i - b * nv) * V;
    const T *xp = static_cast<const T *>(a.x) + b * a.D + c0;
    T *sp = static_cast<T *>(a.state) + b * S * a.D + c0;
    const WT *wp = static_cast<const WT *>(a.w);
    float xf[V], st[S > 0 ? S : 1][V];
    load_v<T, V>(xp, xf, true);
#pragma unroll
    for (int j = 0; j < S; ++j) load_v<T, V>(sp + j * a.D, st[j], false);
    float y[V];
    Row<WT, W> taps;  // the W taps of the current channel's filter, reloaded when the filter changes
    int64_t cur = -1;
#pragma unroll
    for (int e = 0; e < V; ++e) {
        const int64_t c = c0 + e;
        const int64_t fi = MODE == DEC_STATIC ? c : b * a.G + c / a.H;  // filter row of channel c
        if (fi != cur) {
            taps.load(wp + fi * W);
            cur = fi;
        }
        float acc = a.residual ? xf[e] : 0.f;
        acc = fmaf(taps.get(0), xf[e], acc);
#pragma unroll
        for (int k = 1; k < W; ++k) acc = fmaf(taps.get(k), st[S - k][e], acc);
        y[e] = acc;
    }
    store_v<T, V>(static_cast<T *>(a.y) + b * a.D + c0, y);
#pragma unroll
    for (int j = 0; j + 1 < S; ++j) store_v<T, V>(sp + j * a.D, st[j + 1]);
    if constexpr (S > 0) store_v<T, V>(sp + (S - 1) * a.D, xf);
}

// Low-rank decode with the new token's filters formed on chip.  A CTA takes
// DL_NV vectors of V channels (a channel chunk) for DL_SLOTS*QS sequences.
// It stages, in shared memory, the U columns of its chunk (fp32, laid out
// [r][column quad][vector][4] so that the chunk's vectors read adjacent
// 16-byte words) and the z rows of its sequences ([r][sequence]).  Thread
// (vector v, slot q) forms the GPV*W filter taps of its vector for QS
// sequences, w = sum_r z[b,r] U[r, g*W+k], in registers, then takes the
// decode step of each.  No filter value reaches HBM.
constexpr int DL_NV = 8;          // vectors per CTA
constexpr int DL_SLOTS = 32;      // sequence slots per CTA (DL_NV * DL_SLOTS = 256 threads)
constexpr int DL_SMEM_MAX = 96 * 1024;

struct DecLrArgs {
    int64_t B, D, H, G, GW;
    int R, residual;
    const void *x, *z, *U;
    void *state, *y;
};

template <typename T, int W, int GPV, int QS>
__global__ void __launch_bounds__(256) k_decode_lr(const DecLrArgs a) {
    constexpr int V = VecOf<T>::V;
    constexpr int S = W - 1;
    constexpr int NC = GPV * W;          // filter taps of one vector
    constexpr int NQ = (NC + 3) / 4;     // column quads
    constexpr int SB = DL_SLOTS * QS;    // sequences per CTA
    extern __shared__ __align__(16) float dl_shared[];
    float *us = dl_shared;                        // [R][NQ][DL_NV][4]
    float *zs = dl_shared + (size_t)a.R * NQ * DL_NV * 4;  // [R][SB]
    const int tid = threadIdx.x, v = tid % DL_NV, q = tid / DL_NV;
    const int64_t c_lo = (int64_t)blockIdx.x * DL_NV * V;
    const int64_t b_lo = (int64_t)blockIdx.y * SB;
    const T *U = static_cast<const T *>(a.U);
    const T *z = static_cast<const T *>(a.z);
    // staging: unrolled so that each thread's global loads are in flight together
#pragma unroll 8
    for (int i = tid; i < a.R * NQ * DL_NV * 4; i += blockDim.x) {
        const int e = i & 3, vv = (i >> 2) % DL_NV, jq = (i >> 2) / DL_NV % NQ, r = (i >> 2) / DL_NV / NQ;
        const int cc = jq * 4 + e;  // tap index within the vector's taps
        const int64_t c = c_lo + (int64_t)vv * V;
        float u = 0.f;
        if (cc < NC && c < a.D) {
            const int64_t g = c / a.H + cc / W;  // the vector's (cc/W)-th group
            u = to_f<T>(U[(int64_t)r * a.GW + g * W + cc % W]);
        }
        us[i] = u;
    }
#pragma unroll 8
    for (int i = tid; i < a.R * SB; i += blockDim.x) {
        const int r = i / SB, sq = i % SB;
        zs[i] = b_lo + sq < a.B ? to_f<T>(z[(b_lo + sq) * a.R + r]) : 0.f;
    }
    __syncthreads();
    const int64_t c0 = c_lo + (int64_t)v * V;
    if (c0 >= a.D) return;
    float acc[QS][NC];
#pragma unroll
    for (int s = 0; s < QS; ++s)
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[s][j] = 0.f;
    for (int r = 0; r < a.R; ++r) {
        float u[NQ * 4];
#pragma unroll
        for (int jq = 0; jq < NQ; ++jq) {
            const float4 f = *reinterpret_cast<const float4 *>(us + (((size_t)r * NQ + jq) * DL_NV + v) * 4);
            u[4 * jq] = f.x; u[4 * jq + 1] = f.y; u[4 * jq + 2] = f.z; u[4 * jq + 3] = f.w;
        }
#pragma unroll
        for (int s = 0; s < QS; ++s) {
            const float zr = zs[r * SB + q * QS + s];
#pragma unroll
            for (int j = 0; j < NC; ++j) acc[s][j] = fmaf(zr, u[j], acc[s][j]);
        }
    }
#pragma unroll
    for (int s = 0; s < QS; ++s) {
        const int64_t b = b_lo + q * QS + s;
        if (b >= a.B) break;
        const T *xp = static_cast<const T *>(a.x) + b * a.D + c0;
        T *sp = static_cast<T *>(a.state) + b * S * a.D + c0;
        float xf[V], st[S > 0 ? S : 1][V], y[V];
        load_v<T, V>(xp, xf, true);
#pragma unroll
        for (int j = 0; j < S; ++j) load_v<T, V>(sp + j * a.D, st[j], false);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const int gi = GPV == 1 ? 0 : e / (V / GPV);  // the channel's group among the vector's
            float acc2 = a.residual ? xf[e] : 0.f;
            acc2 = fmaf(acc[s][gi * W], xf[e], acc2);
#pragma unroll
            for (int k = 1; k < W; ++k) acc2 = fmaf(acc[s][gi * W + k], st[S - k][e], acc2);
            y[e] = acc2;
        }
        store_v<T, V>(static_cast<T *>(a.y) + b * a.D + c0, y);
#pragma unroll
        for (int j = 0; j + 1 < S; ++j) store_v<T, V>(sp + j * a.D, st[j + 1]);
        if constexpr (S > 0) store_v<T, V>(sp + (S - 1) * a.D, xf);
    }
}

// state[b, j, c] = x[b, T-S+j, c] for T-S+j >= 0, else 0 (S = W-1).
template <typename T>
__global__ void __launch_bounds__(256) k_decode_state(const T *__restrict__ x, T *__restrict__ state, int64_t B,
                                                      int64_t T_, int64_t D, int S) {
    const int64_t n = B * S * D;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = i % D, j = (i / D) % S, b = i / (D * S);
        const int64_t t = T_ - S + j;
        state[i] = t >= 0 ? x[(b * T_ + t) * D + c] : from_f<T>(0.f);
    }
}

template <typename T, typename WT, int W, int MODE>
cudaError_t dec_by_v(const Ctx &c, const DecArgs &a) {
    constexpr int VV = VecOf<T>::V;
    const bool vec = a.D % VV == 0;
    const int64_t n = a.B * (vec ? a.D / VV : a.D);
    const unsigned grid = (unsigned)((n + 255) / 256);
    if (vec) k_decode<T, WT, W, VV, MODE><<<grid, 256, 0, c.stream>>>(a);
    else k_decode<T, WT, W, 1, MODE><<<grid, 256, 0, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename T, typename WT, int MODE>
cudaError_t dec_by_w(const Ctx &c, int W, const DecArgs &a) {
    switch (W) {
    case 1: return dec_by_v<T, WT, 1, MODE>(c, a);
    case 2: return dec_by_v<T, WT, 2, MODE>(c, a);
    case 3: return dec_by_v<T, WT, 3, MODE>(c, a);
    case 4: return dec_by_v<T, WT, 4, MODE>(c, a);
    case 5: return dec_by_v<T, WT, 5, MODE>(c, a);
    case 6: return dec_by_v<T, WT, 6, MODE>(c, a);
    case 7: return dec_by_v<T, WT, 7, MODE>(c, a);
    case 8: return dec_by_v<T, WT, 8, MODE>(c, a);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dec_dispatch(const Ctx &c, int W, int mode, const DecArgs &a) {
    switch (mode) {
    case DEC_HEADWISE: return dec_by_w<T, T, DEC_HEADWISE>(c, W, a);
    case DEC_LOWRANK: return dec_by_w<T, float, DEC_LOWRANK>(c, W, a);
    case DEC_STATIC: return dec_by_w<T, T, DEC_STATIC>(c, W, a);
    }
    return cudaErrorInvalidValue;
}

// Groups per vector of the fused low-rank decode (0: not taken).
template <typename T> int dl_gpv(const dsc_problem &p) {
    constexpr int V = VecOf<T>::V;
    if (p.D % V) return 0;
    if (V % p.H == 0) return (int)(V / p.H);
    if (p.H % V == 0) return 1;
    return 0;
}

template <int GPV, int W> constexpr int dl_qs() { return GPV * W <= 32 ? 2 : 1; }

size_t dl_smem(int R, int gpv, int W) {
    const int nc = gpv * W, nq = (nc + 3) / 4, qs = nc <= 32 ? 2 : 1;
    return ((size_t)R * nq * DL_NV * 4 + (size_t)R * DL_SLOTS * qs) * sizeof(float);
}

template <typename T, int W, int GPV>
cudaError_t dl_launch(const Ctx &c, const DecLrArgs &a) {
    constexpr int QS = dl_qs<GPV, W>();
    const size_t smem = dl_smem(a.R, GPV, W);
    static const cudaError_t attr =
        cudaFuncSetAttribute(k_decode_lr<T, W, GPV, QS>, cudaFuncAttributeMaxDynamicSharedMemorySize, DL_SMEM_MAX);
    if (attr != cudaSuccess) return attr;
    constexpr int V = VecOf<T>::V;
    const dim3 grid((unsigned)((a.D + DL_NV * V - 1) / (DL_NV * V)), (unsigned)((a.B + DL_SLOTS * QS - 1) / (DL_SLOTS * QS)));
    k_decode_lr<T, W, GPV, QS><<<grid, 256, smem, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <typename T, int W>
cudaError_t dl_by_gpv(const Ctx &c, int gpv, const DecLrArgs &a) {
    switch (gpv) {
    case 1: return dl_launch<T, W, 1>(c, a);
    case 2: return dl_launch<T, W, 2>(c, a);
    case 4: return dl_launch<T, W, 4>(c, a);
    case 8:
        if constexpr (VecOf<T>::V == 8) return dl_launch<T, W, 8>(c, a);
        break;
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t dl_dispatch(const Ctx &c, const dsc_problem &p, const DecLrArgs &a) {
    const int gpv = dl_gpv<T>(p);
    switch (p.W) {
    case 1: return dl_by_gpv<T, 1>(c, gpv, a);
    case 2: return dl_by_gpv<T, 2>(c, gpv, a);
    case 3: return dl_by_gpv<T, 3>(c, gpv, a);
    case 4: return dl_by_gpv<T, 4>(c, gpv, a);
    case 5: return dl_by_gpv<T, 5>(c, gpv, a);
    case 6: return dl_by_gpv<T, 6>(c, gpv, a);
    case 7: return dl_by_gpv<T, 7>(c, gpv, a);
    case 8: return dl_by_gpv<T, 8>(c, gpv, a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// lowrank_tc_dec.cu: the tensor-core decode (bf16 shapes the tensor-core map takes).
bool decode_lowrank_tc_ok(const dsc_problem &p);
cudaError_t launch_decode_lowrank_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                     void *state, void *y);

static bool decode_lowrank_cc_ok(const dsc_problem &p) {
    const int gpv = p.dtype == DSC_BF16 ? dl_gpv<bf16>(p) : dl_gpv<float>(p);
    return gpv > 0 && dl_smem((int)p.R, gpv, (int)p.W) <= (size_t)DL_SMEM_MAX;
}

bool decode_lowrank_fused_ok(const dsc_problem &p) { return decode_lowrank_tc_ok(p) || decode_lowrank_cc_ok(p); }

cudaError_t launch_decode_lowrank_fused(const Ctx &c, const dsc_problem &p, const void *x, const void *z,
                                        const void *U, void *state, void *y) {
    if (decode_lowrank_tc_ok(p)) return launch_decode_lowrank_tc(c, p, x, z, U, state, y);
    if (!decode_lowrank_cc_ok(p)) return cudaErrorNotSupported;
    DecLrArgs a{};
    a.B = p.B;
    a.D = p.D;
    a.H = p.H;
    a.G = p.D / p.H;
    a.GW = a.G * p.W;
    a.R = (int)p.R;
    a.residual = p.residual ? 1 : 0;
    a.x = x;
    a.z = z;
    a.U = U;
    a.state = state;
    a.y = y;
    return p.dtype == DSC_BF16 ? dl_dispatch<bf16>(c, p, a) : dl_dispatch<float>(c, p, a);
}

cudaError_t launch_decode(const Ctx &c, const dsc_problem &p, int mode, const void *x, const void *w, void *state,
                          void *y) {
    DecArgs a{};
    a.B = p.B;
    a.D = p.D;
    a.H = mode == DEC_STATIC ? 1 : p.H;
    a.G = p.D / a.H;
    a.residual = p.residual ? 1 : 0;
    a.x = x;
    a.w = w;
    a.state = state;
    a.y = y;
    return p.dtype == DSC_BF16 ? dec_dispatch<bf16>(c, (int)p.W, mode, a) : dec_dispatch<float>(c, (int)p.W, mode, a);
}

cudaError_t launch_decode_state(const Ctx &c, const dsc_problem &p, const void *x, void *state) {
    const int S = (int)p.W - 1;
    const int64_t n = p.B * S * p.D;
    if (n == 0) return cudaSuccess;
    const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 4096);
    if (p.dtype == DSC_BF16)
        k_decode_state<bf16><<<grid, 256, 0, c.stream>>>(static_cast<const bf16 *>(x), static_cast<bf16 *>(state), p.B,
                                                          p.T, p.D, S);
    else
        k_decode_state<float><<<grid, 256, 0, c.stream>>>(static_cast<const float *>(x), static_cast<float *>(state),
                                                           p.B, p.T, p.D, S);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsc
