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
//  - each thread keeps its next tokens' loads in flight through a private
//    ring of shared-memory slots filled by cp.async (see "async copy ring");
//  - the arithmetic runs on fp32 pairs (fma.rn.f32x2), two channels per
//    instruction, and the residual is folded into tap 0 (w_0 + 1);
//  - backward walks forward in time too: dx rows are finished W-1 tokens
//    late from an accumulator window (row s collects w(s+k)_k dy_{s+k} as
//    token s+k streams by), and the tile runs W-1 tokens past its end (right
//    halo of dy and w) to finish its last rows; dw(t) needs dy_t and the
//    x window, and is reduced over the H channels of a group with shuffles
//    inside the warp (no shared memory, no atomics);
//  - the grid is sized from the measured residency: a whole number of waves
//    of resident warps (one, or for the head-wise kernels two or three waves
//    of shorter tiles, which even out the warps' unequal progress; see
//    stream_waves).
#include "kernels.cuh"

namespace dsc {

constexpr int STREAM_THREADS = 256;

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

// ------------------------------------------------------- async copy ring ---
// Each thread streams its own tokens through a private ring of NS slots in
// shared memory, filled with cp.async (LDGSTS) NS-1 tokens ahead of use, so
// its next tokens' loads stay in flight while it computes without holding
// registers.  A thread only reads slots it filled itself, so cp.async.wait_group
// is the only synchronisation needed (no barriers, no spin loops).

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint4 lds16(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

// A thread's channel vector: 16 bytes, or 8 bytes for wide filters (W >= 5),
// where holding the W-1 previous rows and the filter taps of 16 bytes' worth
// of channels would leave registers for one block of 256 threads per SM.
template <int VB> struct VIO;
template <> struct VIO<16> {
    using U = uint4;
    __device__ __forceinline__ static U ld(const void *p) { return ld16(p); }
    __device__ __forceinline__ static void st(void *p, const U &v) { st16(p, v); }
    __device__ __forceinline__ static U lds(uint32_t a) { return lds16(a); }
    __device__ __forceinline__ static void cp(uint32_t dst, const void *src) { cp_async16(dst, src); }
};
template <> struct VIO<8> {
    using U = uint2;
    __device__ __forceinline__ static U ld(const void *p) {
        U r;
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
        return r;
    }
    __device__ __forceinline__ static void st(void *p, const U &v) {
        asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
    }
    __device__ __forceinline__ static U lds(uint32_t a) {
        U r;
        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
        return r;
    }
    __device__ __forceinline__ static void cp(uint32_t dst, const void *src) { cp_async8(dst, src); }
};

// VB bytes of T <-> P pairs of fp32 (pair p holds the vector's channels 2p, 2p+1).
template <typename T, int VB> struct PairsV {
    static constexpr int P = VB / (2 * (int)sizeof(T));
    using U = typename VIO<VB>::U;
    __device__ __forceinline__ static void unpack(const U &u, u64 (&p)[P]) {
        if constexpr (VB == 16) {
            Pairs<T>::unpack(u, p);
        } else if constexpr (sizeof(T) == 2) {
            p[0] = mk2(bf_lo(u.x), bf_hi(u.x));
            p[1] = mk2(bf_lo(u.y), bf_hi(u.y));
        } else {
            p[0] = mk2(__uint_as_float(u.x), __uint_as_float(u.y));
        }
    }
    __device__ __forceinline__ static U pack(const u64 (&p)[P]) {
        if constexpr (VB == 16) {
            return Pairs<T>::pack(p);
        } else if constexpr (sizeof(T) == 2) {
            return make_uint2(pack_bf2(lo2(p[0]), hi2(p[0])), pack_bf2(lo2(p[1]), hi2(p[1])));
        } else {
            return make_uint2(__float_as_uint(lo2(p[0])), __float_as_uint(hi2(p[0])));
        }
    }
};

constexpr int gcd_c(int a, int b) { return b == 0 ? a : gcd_c(b, a % b); }

// The filter taps a thread needs per token (NW elements of T).  The start of
// every such row is a multiple of AL = gcd(16, row bytes): the base pointer is
// 16-byte aligned and both the token stride G*W and a thread's group offset
// are multiples of the row length.  Rows with AL >= 4 travel through the ring
// with cp.async; 2-byte aligned rows (odd W, bf16, one group per thread) are
// read into a register ring instead.
template <typename T, int NW> struct FiltRow {
    static constexpr int BYTES = NW * (int)sizeof(T);
    static constexpr int AL = gcd_c(16, BYTES);
    static constexpr bool IN_SMEM = AL >= 4;
    static constexpr int SLOTS = IN_SMEM ? (BYTES + 15) / 16 : 0;  // 16-byte ring slots
    static constexpr int WORDS = (BYTES + 3) / 4;

    __device__ __forceinline__ static void copy(uint32_t dst, uint32_t stride, const char *src) {
        if constexpr (AL == 16) {
#pragma unroll
            for (int i = 0; i < BYTES / 16; ++i) cp_async16(dst + i * stride, src + 16 * i);
        } else if constexpr (AL == 8) {
#pragma unroll
            for (int i = 0; i < BYTES / 8; ++i) cp_async8(dst + (i / 2) * stride + 8 * (i % 2), src + 8 * i);
        } else if constexpr (AL == 4) {
#pragma unroll
            for (int i = 0; i < BYTES / 4; ++i) cp_async4(dst + (i / 4) * stride + 4 * (i % 4), src + 4 * i);
        }
    }

    // Read back the words of a row that went through the ring.
    __device__ __forceinline__ static void read(uint32_t src, uint32_t stride, uint32_t (&w)[WORDS]) {
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) {
            uint4 v = lds16(src + i * stride);
            if (4 * i + 0 < WORDS) w[4 * i + 0] = v.x;
            if (4 * i + 1 < WORDS) w[4 * i + 1] = v.y;
            if (4 * i + 2 < WORDS) w[4 * i + 2] = v.z;
            if (4 * i + 3 < WORDS) w[4 * i + 3] = v.w;
        }
    }

    // Direct read of a row with plain loads (element by element).
    __device__ __forceinline__ static void load_direct(const char *src, uint32_t (&w)[WORDS]) {
        if constexpr (sizeof(T) == 4) {
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
        } else {
            const unsigned short *q = reinterpret_cast<const unsigned short *>(src);
#pragma unroll
            for (int i = 0; i < WORDS; ++i) w[i] = 0u;
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i >> 1] |= (uint32_t)__ldg(q + i) << (16 * (i & 1));
        }
    }

    __device__ __forceinline__ static float get(const uint32_t (&w)[WORDS], int i) {
        if constexpr (sizeof(T) == 4) return __uint_as_float(w[i]);
        else return (i & 1) ? bf_hi(w[i >> 1]) : bf_lo(w[i >> 1]);
    }
};

// Ring depth (tokens) for a given number of 16-byte slots per token, keeping
// the ring at <= 96 KB for a 256-thread block (two blocks per SM).
__host__ __device__ constexpr int ring_depth(int slots) {
    return slots * 16 * 8 <= 384 ? 8 : (384 / (slots * 16) < 2 ? 2 : 384 / (slots * 16));
}

template <typename T, int W, int GPT, bool WS, bool BWD, int VB = 16> struct StreamCfg {
    static constexpr int V = VB / (int)sizeof(T);
    static constexpr int NW = WS ? V * W : GPT * W;  // filter taps per token per thread
    static constexpr int CPG = WS ? 1 : V / GPT;      // channels sharing one filter inside a thread
    static constexpr int WIN = W - 1;
    using F = FiltRow<T, NW>;
    static constexpr bool WRING = !WS && F::IN_SMEM;  // filter rows through the shared ring
    static constexpr bool WREG = !WS && !F::IN_SMEM;  // filter rows through a register ring
    // Ring slots per token (16 bytes x STREAM_THREADS each): the x (and, in
    // the backward, dy) vectors, then the filter row.  8-byte vectors of one
    // token share a slot, each row contiguous over the block's threads, so a
    // warp's 8-byte accesses cover 256 consecutive bytes (no bank conflicts).
    static constexpr int NV = BWD ? 2 : 1;
    static constexpr int VSLOTS = VB == 16 ? NV : (NV * 8 + 15) / 16;
    static constexpr int SUB = VSLOTS + (WRING ? F::SLOTS : 0);  // 16-byte slots per token
    static constexpr int NS = ring_depth(SUB);
    static constexpr size_t SMEM = (size_t)NS * SUB * 16 * STREAM_THREADS;
    // Blocks per SM the register budget is sized for: the narrow head-wise
    // filters fit 3 (forward) / 2 (backward) blocks of 256 threads; wider or
    // per-channel (static) filters need more registers per thread.
    // With 8-byte vectors a thread holds half the state: two blocks per SM,
    // except the static backward at W >= 6, whose filters, filter-gradient
    // sums and two windows still need more than the 128 registers that two
    // blocks leave a thread (one block: no spills).
    static constexpr int MINB = VB == 8 ? (WS && BWD && W >= 6 ? 1 : 2)
                                : BWD ? ((!WS && W <= 4) || (WS && W <= 2) ? 2 : 1)
                                      : ((!WS && W <= 4) ? 3 : (W <= 3 ? 2 : 1));
};

template <typename T, int W, int GPT, bool WS, bool BWD, int VB>
size_t stream_smem() { return StreamCfg<T, W, GPT, WS, BWD, VB>::SMEM; }

template <bool B> struct BoolC { static constexpr bool value = B; };

// Tap k of the filters of channel pair p (channels 2p, 2p+1 of the thread's
// vector) as an fp32 pair; `add` is added to both (the residual on tap 0).
template <typename F, int W, int CPG>
__device__ __forceinline__ u64 tap2(const uint32_t (&wv)[F::WORDS], int p, int k, float add) {
    const int g0 = (2 * p) / CPG, g1 = (2 * p + 1) / CPG;
    const float a = F::get(wv, g0 * W + k) + add;
    if (g0 == g1) return mk2(a, a);
    return mk2(a, F::get(wv, g1 * W + k) + add);
}
// The same pair without an added constant (x + 0.f is not x for x = -0, so a
// default of 0 would cost an add per tap).
template <typename F, int W, int CPG>
__device__ __forceinline__ u64 tap2(const uint32_t (&wv)[F::WORDS], int p, int k) {
    const int g0 = (2 * p) / CPG, g1 = (2 * p + 1) / CPG;
    const float a = F::get(wv, g0 * W + k);
    if (g0 == g1) return mk2(a, a);
    return mk2(a, F::get(wv, g1 * W + k));
}

// Sum part[k] (k < N) over the L lanes of a filter group; afterwards the
// group's first lane holds the sums (every lane, when L is a power of two).
template <int N>
__device__ __forceinline__ void group_reduce(float (&part)[N], int L, int pos) {
    if ((L & (L - 1)) == 0) {
        for (int o = 1; o < L; o <<= 1)
#pragma unroll
            for (int k = 0; k < N; ++k) part[k] += __shfl_xor_sync(FULL_MASK, part[k], o);
    } else {
        for (int o = 1; o < L; o <<= 1)
#pragma unroll
            for (int k = 0; k < N; ++k) {
                const float t = __shfl_down_sync(FULL_MASK, part[k], o);
                if (pos + o < L) part[k] += t;
            }
    }
}

// Taps padded to a power of two for the reduce-scatter below.
template <int W> struct Pow2Taps {
    static constexpr int NP = W <= 1 ? 1 : (W <= 2 ? 2 : (W <= 4 ? 4 : 8));
};

// Lane `pos` of a group ends the reduce-scatter holding tap rs_tap(pos):
// at the level of lane bit j it kept the upper half of its taps when bit j
// was set, i.e. NP/2^(j+1) more.
template <int W> __device__ __forceinline__ int rs_tap(int pos) {
    constexpr int NP = Pow2Taps<W>::NP;
    int t = 0;
#pragma unroll
    for (int j = 0, c = NP / 2; c >= 1; ++j, c >>= 1)
        if ((pos >> j) & 1) t += c;
    return t;
}

// Sum part[k] (k < W) over the L lanes of a filter group, L a power of two
// with L >= NP (the taps padded to NP): recursive halving.  At the level of
// lane bit o each lane sends the half of its remaining taps it does not keep
// and adds the half its partner sends, so after log2(NP) levels each lane
// holds one tap summed over NP lanes, and the remaining levels add that value
// across the group: NP-1 + log2(L/NP) shuffles per token instead of
// W*log2(L).  Returns this lane's total, of tap rs_tap<W>(pos).
template <int W>
__device__ __forceinline__ float group_reduce_scatter(float (&part)[W], int L, int pos) {
    constexpr int NP = Pow2Taps<W>::NP;
    // taps padded with zeros to NP (in place when W is already a power of two)
    float pad[NP == W ? 1 : NP];
    float *v = part;
    if constexpr (NP != W) {
#pragma unroll
        for (int k = 0; k < NP; ++k) pad[k] = k < W ? part[k] : 0.f;
        v = pad;
    }
#pragma unroll
    for (int o = 1, cnt = NP / 2; o < NP; o <<= 1, cnt >>= 1) {
        const bool up = (pos & o) != 0;
#pragma unroll
        for (int i = 0; i < NP / 2; ++i) {
            if (i < cnt) {
                const float send = up ? v[i] : v[i + cnt];
                const float keep = up ? v[i + cnt] : v[i];
                v[i] = keep + __shfl_xor_sync(FULL_MASK, send, o);
            }
        }
    }
    float r = v[0];
    for (int o = NP; o < L; o <<= 1) r += __shfl_xor_sync(FULL_MASK, r, o);
    return r;
}

// ---------------------------------------------------------------- forward ---

// WS = false: head-wise filters w[b,t,g,k] read per token.
// WS = true : static filters ws[c,k] read once per thread.
template <typename T, int W, int GPT, bool WS, int VB>
__global__ void __launch_bounds__(STREAM_THREADS, (StreamCfg<T, W, GPT, WS, false, VB>::MINB)) k_stream_fwd(const HwArgs a) {
    using C = StreamCfg<T, W, GPT, WS, false, VB>;
    using F = typename C::F;
    using PR = PairsV<T, VB>;
    using IO = VIO<VB>;
    constexpr int P = PR::P, NS = C::NS, WIN = C::WIN, XW = WIN > 0 ? WIN : 1, CPG = C::CPG;
    extern __shared__ uint4 ring[];
    const StreamMap &m = a.m;
    Pos q;
    if (!locate<C::V>(m, q) || !q.active) return;
    pdl_wait();  // inputs may come from the previous kernel of the stream
    pdl_trigger();

    const int n = q.t_end - q.t_start;
    const int64_t xstep = m.D * (int64_t)sizeof(T);
    const int64_t wstep = WS ? 0 : m.G * W * (int64_t)sizeof(T);
    const int64_t row = q.b * m.T + q.t_start;
    const char *xp = static_cast<const char *>(a.x) + (row * m.D + q.c0) * (int64_t)sizeof(T);
    char *yp = static_cast<char *>(a.y) + (row * m.D + q.c0) * (int64_t)sizeof(T);
    const char *wp = WS ? static_cast<const char *>(a.w) + q.c0 * W * (int64_t)sizeof(T)
                        : static_cast<const char *>(a.w) + (row * m.G + q.c0 / m.H) * W * (int64_t)sizeof(T);
    const float res = m.residual ? 1.f : 0.f;

    const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(ring);
    const uint32_t base = ring0 + 16u * threadIdx.x;
    constexpr uint32_t SUBSTRIDE = 16u * STREAM_THREADS;
    auto slot = [&](int s, int sub) { return base + (uint32_t)(s * C::SUB + sub) * SUBSTRIDE; };
    // Vector row r (0: x, 1: dy) of ring token s.
    auto vslot = [&](int s, int r) {
        if constexpr (VB == 16) return slot(s, r);
        else return ring0 + 8u * threadIdx.x + (uint32_t)(s * C::SUB) * SUBSTRIDE + (uint32_t)r * (8u * STREAM_THREADS);
    };

    u64 wsp[WS ? P : 1][WS ? W : 1];  // static filters as pairs (tap 0 carries the residual)
    if constexpr (WS) {
        uint32_t wst[F::WORDS];
        F::load_direct(wp, wst);
#pragma unroll
        for (int pp = 0; pp < P; ++pp)
#pragma unroll
            for (int k = 0; k < W; ++k) wsp[pp][k] = k == 0 ? tap2<F, W, CPG>(wst, pp, 0, res) : tap2<F, W, CPG>(wst, pp, k);
    }
    uint32_t wreg[C::WREG ? NS : 1][F::WORDS];

    auto issue = [&](int i, int s, bool full) {
        if (full || i < n) {
            IO::cp(vslot(s, 0), xp + i * xstep);
            if constexpr (C::WRING) F::copy(slot(s, C::VSLOTS), SUBSTRIDE, wp + i * wstep);
            if constexpr (C::WREG) F::load_direct(wp + i * wstep, wreg[s]);
        }
        cp_commit();
    };

    u64 xs[XW][P];  // xs[j] = x[t-1-j]
#pragma unroll
    for (int j = 0; j < XW; ++j) {
        const int t = q.t_start - 1 - j;
        if (WIN > 0 && t >= 0) PR::unpack(IO::ld(xp - (int64_t)(1 + j) * xstep), xs[j]);
        else
#pragma unroll
            for (int pp = 0; pp < P; ++pp) xs[j][pp] = 0ull;
    }
#pragma unroll
    for (int j = 0; j < NS - 1; ++j) issue(j, j, false);

    auto group = [&](int i0, auto fulltag) {
        constexpr bool FULL = decltype(fulltag)::value;
#pragma unroll
        for (int u = 0; u < NS; ++u) {
            const int i = i0 + u;
            if (!FULL && i >= n) break;
            issue(i + NS - 1, (u + NS - 1) % NS, FULL);
            cp_wait<NS - 1>();
            u64 xc[P], acc[P];
            PR::unpack(IO::lds(vslot(u, 0)), xc);
            uint32_t wv[F::WORDS];
            if constexpr (C::WRING) F::read(slot(u, C::VSLOTS), SUBSTRIDE, wv);
            if constexpr (C::WREG)
#pragma unroll
                for (int k = 0; k < F::WORDS; ++k) wv[k] = wreg[u][k];
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                u64 s = mul2(WS ? wsp[pp][0] : tap2<F, W, CPG>(wv, pp, 0, res), xc[pp]);
#pragma unroll
                for (int k = 1; k < W; ++k) s = fma2(WS ? wsp[pp][k] : tap2<F, W, CPG>(wv, pp, k), xs[k - 1][pp], s);
                acc[pp] = s;
            }
            IO::st(yp + i * xstep, PR::pack(acc));
#pragma unroll
            for (int j = XW - 1; j > 0; --j)
#pragma unroll
                for (int pp = 0; pp < P; ++pp) xs[j][pp] = xs[j - 1][pp];
#pragma unroll
            for (int pp = 0; pp < P; ++pp) xs[0][pp] = xc[pp];
        }
    };
    int i0 = 0;
    for (; i0 + 2 * NS - 1 <= n; i0 += NS) group(i0, BoolC<true>{});
    for (; i0 < n; i0 += NS) group(i0, BoolC<false>{});
    cp_wait<0>();
}

// --------------------------------------------------------------- backward ---

// RS: wide filter groups (one per thread, L >= NP lanes, L a power of two)
// reduce their filter gradients by reduce-scatter (a separate instance, so
// that the other instances keep their registers).
template <typename T, int W, int GPT, bool WS, int VB, bool RS = false>
__global__ void __launch_bounds__(STREAM_THREADS, (StreamCfg<T, W, GPT, WS, true, VB>::MINB)) k_stream_bwd(const HwArgs a) {
    using C = StreamCfg<T, W, GPT, WS, true, VB>;
    using F = typename C::F;
    using PR = PairsV<T, VB>;
    using IO = VIO<VB>;
    constexpr int P = PR::P, NS = C::NS, WIN = C::WIN, XW = WIN > 0 ? WIN : 1, CPG = C::CPG;
    constexpr int PPG = CPG >= 2 ? CPG / 2 : 1;  // channel pairs per filter group (CPG >= 2)
    extern __shared__ uint4 ring[];
    const StreamMap &m = a.m;
    Pos q;
    if (!locate<C::V>(m, q)) return;  // whole warp out of range; partial warps stay for the shuffles
    pdl_wait();  // inputs may come from the previous kernel of the stream
    pdl_trigger();
    // Inactive lanes (no channels of their own) stream channel 0 of the same rows: in bounds, never
    // stored, and never in a filter group with an active lane.
    const bool act = q.active;
    const int L = m.L;
    const int pos = q.lane % L;

    const int n = q.t_end - q.t_start;                                   // tokens owned
    const int nl = (int)(min((int64_t)q.t_end + WIN, m.T) - q.t_start);  // tokens with dy and w
    const int niter = n + WIN;                                            // tokens streamed
    const int64_t c0 = act ? q.c0 : 0;
    const int64_t xstep = m.D * (int64_t)sizeof(T);
    const int64_t wstep = WS ? 0 : m.G * W * (int64_t)sizeof(T);
    const int64_t row = q.b * m.T + q.t_start;
    const char *xp = static_cast<const char *>(a.x) + (row * m.D + c0) * (int64_t)sizeof(T);
    const char *dyp = static_cast<const char *>(a.dy) + (row * m.D + c0) * (int64_t)sizeof(T);
    char *dxp = static_cast<char *>(a.dx) + (row * m.D + c0) * (int64_t)sizeof(T);
    const char *wp = WS ? static_cast<const char *>(a.w) + c0 * W * (int64_t)sizeof(T)
                        : static_cast<const char *>(a.w) + (row * m.G + c0 / m.H) * W * (int64_t)sizeof(T);
    char *dwp = WS ? nullptr : static_cast<char *>(a.dw) + (row * m.G + c0 / m.H) * W * (int64_t)sizeof(T);
    const float res = m.residual ? 1.f : 0.f;

    const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(ring);
    const uint32_t base = ring0 + 16u * threadIdx.x;
    constexpr uint32_t SUBSTRIDE = 16u * STREAM_THREADS;
    auto slot = [&](int s, int sub) { return base + (uint32_t)(s * C::SUB + sub) * SUBSTRIDE; };
    // Vector row r (0: x, 1: dy) of ring token s.
    auto vslot = [&](int s, int r) {
        if constexpr (VB == 16) return slot(s, r);
        else return ring0 + 8u * threadIdx.x + (uint32_t)(s * C::SUB) * SUBSTRIDE + (uint32_t)r * (8u * STREAM_THREADS);
    };

    // Static filters: fp32 pairs, or (bf16 with 8-byte vectors, where the
    // registers are tightest) taps 1 .. W-1 as packed bf16 pairs, unpacked at
    // each use; exact, the taps being bf16 values.  Tap 0 carries the residual.
    constexpr bool WPK = WS && VB == 8 && sizeof(T) == 2;
    u64 wsp[WS && !WPK ? P : 1][WS && !WPK ? W : 1];
    uint32_t wpk[WPK ? P : 1][WPK ? W : 1];
    u64 w0p[WPK ? P : 1];
    u64 dws[WS ? P : 1][WS ? W : 1];
    if constexpr (WS) {
        uint32_t wst[F::WORDS];
        F::load_direct(wp, wst);
#pragma unroll
        for (int pp = 0; pp < P; ++pp)
#pragma unroll
            for (int k = 0; k < W; ++k) {
                if constexpr (WPK) {
                    if (k == 0) w0p[pp] = tap2<F, W, CPG>(wst, pp, 0, res);
                    else wpk[pp][k] = pack_bf2(F::get(wst, (2 * pp) * W + k), F::get(wst, (2 * pp + 1) * W + k));
                } else {
                    wsp[pp][k] = k == 0 ? tap2<F, W, CPG>(wst, pp, 0, res) : tap2<F, W, CPG>(wst, pp, k);
                }
                dws[pp][k] = 0ull;
            }
    }
    auto stap = [&](int pp, int k) -> u64 {  // static filters only
        if constexpr (WPK) return k == 0 ? w0p[pp] : mk2(bf_lo(wpk[pp][k]), bf_hi(wpk[pp][k]));
        else if constexpr (WS) return wsp[pp][k];
        else return 0ull;
    };
    uint32_t wreg[C::WREG ? NS : 1][F::WORDS];

    auto issue = [&](int i, int s, bool full) {
        if (full || i < n) IO::cp(vslot(s, 0), xp + i * xstep);
        if (full || i < nl) {
            IO::cp(vslot(s, 1), dyp + i * xstep);
            if constexpr (C::WRING) F::copy(slot(s, C::VSLOTS), SUBSTRIDE, wp + i * wstep);
            if constexpr (C::WREG) F::load_direct(wp + i * wstep, wreg[s]);
        }
        cp_commit();
    };

    u64 xs[XW][P];   // xs[j] = x[t-1-j]
    u64 acc[XW][P];  // acc[j] = partial dx of row t-1-j
#pragma unroll
    for (int j = 0; j < XW; ++j) {
        const int t = q.t_start - 1 - j;
        if (WIN > 0 && t >= 0) PR::unpack(IO::ld(xp - (int64_t)(1 + j) * xstep), xs[j]);
        else
#pragma unroll
            for (int pp = 0; pp < P; ++pp) xs[j][pp] = 0ull;
#pragma unroll
        for (int pp = 0; pp < P; ++pp) acc[j][pp] = 0ull;
    }
#pragma unroll
    for (int j = 0; j < NS - 1; ++j) issue(j, j, false);

    auto group = [&](int i0, auto fulltag) {
        constexpr bool FULL = decltype(fulltag)::value;
#pragma unroll
        for (int u = 0; u < NS; ++u) {
            const int i = i0 + u;
            if (!FULL && i >= niter) break;
            issue(i + NS - 1, (u + NS - 1) % NS, FULL);
            cp_wait<NS - 1>();
            const bool hx = FULL || i < n, hd = FULL || i < nl;
            u64 xc[P], dyc[P], r0[P];
            uint32_t wv[F::WORDS];
            if (hx) PR::unpack(IO::lds(vslot(u, 0)), xc);
            else
#pragma unroll
                for (int pp = 0; pp < P; ++pp) xc[pp] = 0ull;
            if (hd) {
                PR::unpack(IO::lds(vslot(u, 1)), dyc);
                if constexpr (C::WRING) F::read(slot(u, C::VSLOTS), SUBSTRIDE, wv);
                if constexpr (C::WREG)
#pragma unroll
                    for (int k = 0; k < F::WORDS; ++k) wv[k] = wreg[u][k];
            } else {
#pragma unroll
                for (int pp = 0; pp < P; ++pp) dyc[pp] = 0ull;
#pragma unroll
                for (int k = 0; k < F::WORDS; ++k) wv[k] = 0u;
            }
            // dx: token i feeds row i-k through tap k of w(i); row i itself starts
            // with the residual (rows past the tile are never stored).
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                r0[pp] = mul2(WS ? stap(pp, 0) : tap2<F, W, CPG>(wv, pp, 0, res), dyc[pp]);
#pragma unroll
                for (int k = 1; k < W; ++k)
                    acc[k - 1][pp] = fma2(WS ? stap(pp, k) : tap2<F, W, CPG>(wv, pp, k), dyc[pp], acc[k - 1][pp]);
            }
            if (act && i >= WIN) {  // row i-WIN is complete
                if constexpr (W > 1) IO::st(dxp + (i - WIN) * xstep, PR::pack(acc[XW - 1]));
                else IO::st(dxp + (i - WIN) * xstep, PR::pack(r0));
            }
            // dw(i)_k = sum over the group's channels of dy_i * x_{i-k}
            if (FULL || i < n) {
                if constexpr (WS) {
#pragma unroll
                    for (int pp = 0; pp < P; ++pp)
#pragma unroll
                        for (int k = 0; k < W; ++k) dws[pp][k] = fma2(dyc[pp], k == 0 ? xc[pp] : xs[k - 1][pp], dws[pp][k]);
                } else if constexpr (CPG == 1) {
                    float part[GPT * W];
#pragma unroll
                    for (int pp = 0; pp < P; ++pp)
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            const u64 d = mul2(dyc[pp], k == 0 ? xc[pp] : xs[k - 1][pp]);
                            part[(2 * pp) * W + k] = lo2(d);
                            part[(2 * pp + 1) * W + k] = hi2(d);
                        }
                    if (act) store_row<T, GPT * W>(reinterpret_cast<T *>(dwp + i * wstep), part);
                } else {
                    float part[GPT * W];
#pragma unroll
                    for (int gi = 0; gi < GPT; ++gi)
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            u64 s2 = mul2(dyc[gi * PPG], k == 0 ? xc[gi * PPG] : xs[k - 1][gi * PPG]);
#pragma unroll
                            for (int pp = gi * PPG + 1; pp < (gi + 1) * PPG; ++pp)
                                s2 = fma2(dyc[pp], k == 0 ? xc[pp] : xs[k - 1][pp], s2);
                            part[gi * W + k] = lo2(s2) + hi2(s2);
                        }
                    if constexpr (RS) {
                        // wide groups: each of the first NP lanes ends with one tap's total and stores it
                        const float tot = group_reduce_scatter<W>(*reinterpret_cast<float(*)[W]>(part), L, pos);
                        const int tap = rs_tap<W>(pos);
                        if (act && pos < Pow2Taps<W>::NP && tap < W)
                            reinterpret_cast<T *>(dwp + i * wstep)[tap] = from_f<T>(tot);
                    } else if (GPT == 1 && L > 1) {
                        group_reduce<GPT * W>(part, L, pos);
                        if (act && pos == 0) store_row<T, GPT * W>(reinterpret_cast<T *>(dwp + i * wstep), part);
                    } else if (act) {
                        store_row<T, GPT * W>(reinterpret_cast<T *>(dwp + i * wstep), part);
                    }
                }
            }
#pragma unroll
            for (int j = XW - 1; j > 0; --j)
#pragma unroll
                for (int pp = 0; pp < P; ++pp) {
                    acc[j][pp] = acc[j - 1][pp];
                    xs[j][pp] = xs[j - 1][pp];
                }
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                acc[0][pp] = r0[pp];
                xs[0][pp] = xc[pp];
            }
        }
    };
    int i0 = 0;
    for (; i0 + 2 * NS - 1 <= n; i0 += NS) group(i0, BoolC<true>{});
    for (; i0 < niter; i0 += NS) group(i0, BoolC<false>{});
    cp_wait<0>();
    if constexpr (WS) {
        if (act) {
            const int64_t s = q.b * m.nTiles + q.t_start / m.Tt;
            float *pp = a.partial + (s * m.D + c0) * W;
#pragma unroll
            for (int p2 = 0; p2 < P; ++p2)
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    pp[(2 * p2) * W + k] = lo2(dws[p2][k]);
                    pp[(2 * p2 + 1) * W + k] = hi2(dws[p2][k]);
                }
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

// Pick the tile length for `target_warps` warps (a whole number of waves of
// resident warps): the largest number of time tiles whose warps fit.
void finish_map(StreamMap &m, int64_t target_warps) {
    const int64_t cols = m.B * m.nWc;
    int64_t tiles = target_warps / cols;
    if (tiles < 1) tiles = 1;
    if (tiles > m.T) tiles = m.T;
    const int64_t tt = (m.T + tiles - 1) / tiles;
    m.Tt = (int)tt;
    m.nTiles = (int)((m.T + tt - 1) / tt);
    m.n_warps = m.B * m.nTiles * (int64_t)m.nWc;
}

// The plan: 8-byte vectors for W >= 5 when that mapping keeps every filter
// group inside one thread (two blocks per SM instead of one, and no cross-lane
// reduction), else 16-byte vectors; false when neither exists (the generic
// kernels take the shape).  Groups that span lanes keep 16-byte vectors:
// halving the vector would double the lanes of a group and with them the
// shuffle levels of its dw reduction per byte, which costs more than the
// second block gains (measured at W = 8, H = 16 and 128).
bool stream_plan(const dsc_problem &p, StreamMap &m) {
    const int V16 = p.dtype == DSC_BF16 ? 8 : 4;
    if (p.W >= 5 && stream_map(p, V16 / 2, m) && m.L == 1) {
        m.vb = 8;
        return true;
    }
    if (stream_map(p, V16, m)) {
        m.vb = 16;
        return true;
    }
    return false;
}

template <typename T, int W, int GPT, bool WS, bool BWD, int VB, bool RS = false>
static const void *stream_kernel() {
    if constexpr (BWD) return (const void *)k_stream_bwd<T, W, GPT, WS, VB, RS>;
    else return (const void *)k_stream_fwd<T, W, GPT, WS, VB>;
}

// Dynamic shared memory of one instantiation, set up once (thread-safe).
template <typename T, int W, int GPT, bool WS, bool BWD, int VB, bool RS = false>
static size_t stream_setup(int &per_sm_warps) {
    static const size_t smem = stream_smem<T, W, GPT, WS, BWD, VB>();
    static const int blocks = [] {
        const void *k = stream_kernel<T, W, GPT, WS, BWD, VB, RS>();
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cudaGetLastError();
        return resident_blocks(k, STREAM_THREADS, smem);
    }();
    per_sm_warps = blocks * (STREAM_THREADS / 32);
    return smem;
}

// Waves of tiles.  With one wave (every tile in flight at once) the kernel
// ends with its slowest warp, and per-warp finish times spread widely: in the
// Q/K/V head-wise backward from 58 to 138 us around a mean of 104 us, by
// where the block ran rather than by its data (moving the tensors by half
// their size left the slow sequences the same).  Several waves of shorter
// tiles let the SMs whose blocks finish early take new ones; each extra tile
// costs a ring start-up and, backward, a W-1 token right halo.  Measured per
// kernel on one box at W = 4: Q/K/V forward -7 % with 3 waves, backward -5 %
// with 2 (-8 % with 3, but the all-linear backward then +5 %), all-linear
// forward -4 %, packed-document row -3 %.  They lost elsewhere, so those keep
// one wave: at W = 2 and W = 8 (+4 to +9 % on the B = 1, T = 16384 widths,
// where the lighter or register-heavier tokens make a tile's start-up a
// larger share), with tiles under 32 tokens (forward) or 64 (backward), and
// in the static kernels, whose filter-gradient partials grow with the tiles.
template <bool BWD, bool WS> static int stream_waves(StreamMap m, int64_t one_wave) {
    if constexpr (WS) return 1;
    if (m.W != 4) return 1;
    const int f = BWD ? 2 : 3;
    finish_map(m, one_wave * f);
    return m.Tt >= (BWD ? 64 : 32) ? f : 1;
}

template <typename T, int W, int GPT, bool WS, bool BWD, int VB, bool RS = false>
static cudaError_t run_stream(const Ctx &c, HwArgs a) {
    int per_sm = 0;
    const size_t smem = stream_setup<T, W, GPT, WS, BWD, VB, RS>(per_sm);
    const int64_t one_wave = (int64_t)per_sm * c.sms;
    finish_map(a.m, one_wave * stream_waves<BWD, WS>(a.m, one_wave));
    const int64_t blocks = (a.m.n_warps + STREAM_THREADS / 32 - 1) / (STREAM_THREADS / 32);
    cudaError_t e;
    if constexpr (BWD)
        e = launch_pdl(k_stream_bwd<T, W, GPT, WS, VB, RS>, dim3((unsigned)blocks), dim3(STREAM_THREADS), smem, c.stream, a);
    else
        e = launch_pdl(k_stream_fwd<T, W, GPT, WS, VB>, dim3((unsigned)blocks), dim3(STREAM_THREADS), smem, c.stream, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// W <= 4: 16-byte vectors only; W >= 5: the vector width of the plan.
template <typename T, bool WS, bool BWD, int GPT>
static cudaError_t by_w(const Ctx &c, int W, HwArgs a) {
    constexpr int V16 = VecOf<T>::V;
    const bool half = a.m.vb == 8;
    if constexpr (!WS && BWD && GPT == 1) {
        // a filter group over L >= 16 lanes (L a power of two, L >= NP): the
        // reduce-scatter instance.  Measured on one box against the butterfly:
        // L = 16 backward 26 % (W = 8) and 15 % (W = 4) faster; L = 8, W = 4
        // 3 % slower (the taps' single-element stores outweigh the shuffles saved).
        const int L = a.m.L, np = W <= 1 ? 1 : (W <= 2 ? 2 : (W <= 4 ? 4 : 8));
        if (!half && L >= 16 && L >= np && (L & (L - 1)) == 0) {
            switch (W) {
            case 2: return run_stream<T, 2, 1, false, true, 16, true>(c, a);
            case 3: return run_stream<T, 3, 1, false, true, 16, true>(c, a);
            case 4: return run_stream<T, 4, 1, false, true, 16, true>(c, a);
            case 5: return run_stream<T, 5, 1, false, true, 16, true>(c, a);
            case 6: return run_stream<T, 6, 1, false, true, 16, true>(c, a);
            case 7: return run_stream<T, 7, 1, false, true, 16, true>(c, a);
            case 8: return run_stream<T, 8, 1, false, true, 16, true>(c, a);
            }
        }
    }
    switch (W) {
    case 1: return run_stream<T, 1, GPT, WS, BWD, 16>(c, a);
    case 2: return run_stream<T, 2, GPT, WS, BWD, 16>(c, a);
    case 3: return run_stream<T, 3, GPT, WS, BWD, 16>(c, a);
    case 4: return run_stream<T, 4, GPT, WS, BWD, 16>(c, a);
    }
    if (half) {
        if constexpr (GPT <= V16 / 2) {
            switch (W) {
            case 5: return run_stream<T, 5, GPT, WS, BWD, 8>(c, a);
            case 6: return run_stream<T, 6, GPT, WS, BWD, 8>(c, a);
            case 7: return run_stream<T, 7, GPT, WS, BWD, 8>(c, a);
            case 8: return run_stream<T, 8, GPT, WS, BWD, 8>(c, a);
            }
        }
        return cudaErrorInvalidValue;
    }
    switch (W) {
    case 5: return run_stream<T, 5, GPT, WS, BWD, 16>(c, a);
    case 6: return run_stream<T, 6, GPT, WS, BWD, 16>(c, a);
    case 7: return run_stream<T, 7, GPT, WS, BWD, 16>(c, a);
    case 8: return run_stream<T, 8, GPT, WS, BWD, 16>(c, a);
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

template <typename T, int W, int VB> static int64_t st_tiles_w(const Ctx &c, StreamMap m) {
    int per_sm = 0;
    stream_setup<T, W, 1, true, true, VB>(per_sm);
    finish_map(m, (int64_t)per_sm * c.sms);
    return m.B * m.nTiles;
}

template <typename T> static int64_t st_tiles(const Ctx &c, const dsc_problem &p) {
    StreamMap m;
    stream_plan(p, m);
    if (m.vb == 8) {
        switch (p.W) {
        case 5: return st_tiles_w<T, 5, 8>(c, m);
        case 6: return st_tiles_w<T, 6, 8>(c, m);
        case 7: return st_tiles_w<T, 7, 8>(c, m);
        default: return st_tiles_w<T, 8, 8>(c, m);
        }
    }
    switch (p.W) {
    case 1: return st_tiles_w<T, 1, 16>(c, m);
    case 2: return st_tiles_w<T, 2, 16>(c, m);
    case 3: return st_tiles_w<T, 3, 16>(c, m);
    case 4: return st_tiles_w<T, 4, 16>(c, m);
    case 5: return st_tiles_w<T, 5, 16>(c, m);
    case 6: return st_tiles_w<T, 6, 16>(c, m);
    case 7: return st_tiles_w<T, 7, 16>(c, m);
    default: return st_tiles_w<T, 8, 16>(c, m);
    }
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
