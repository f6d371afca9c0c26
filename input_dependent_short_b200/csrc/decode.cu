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

}  // namespace

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
