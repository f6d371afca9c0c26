// Shared device helpers of the dynamic short convolution kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsc.h"

namespace dsc {

using bf16 = __nv_bfloat16;

constexpr unsigned FULL_MASK = 0xffffffffu;

// Elements of T in one 16-byte vector: each thread of the streaming kernels
// owns one such vector of channels.
template <typename T> struct VecOf;
template <> struct VecOf<float> { static constexpr int V = 4; };
template <> struct VecOf<bf16> { static constexpr int V = 8; };

// ------------------------------------------------------------ raw memory ---

// 16-byte read-only streaming load (inputs are never written by the call).
__device__ __forceinline__ uint4 ld16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st16(void *p, const uint4 &v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------ conversion ---

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 16 bytes -> V floats.
__device__ __forceinline__ void unpack(const uint4 &u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack(const uint4 &u, float (&f)[8]) {
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x);
    f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    f[4] = bf_lo(u.z); f[5] = bf_hi(u.z);
    f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
}

// V floats -> 16 bytes (bf16: round to nearest even).
__device__ __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf2(f[0], f[1]), pack_bf2(f[2], f[3]), pack_bf2(f[4], f[5]), pack_bf2(f[6], f[7]));
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// ------------------------------------------------- short contiguous rows ---
// A row of N elements of T (N*sizeof(T) bytes, e.g. the W taps of one or more
// filter groups) read with the widest accesses its address allows.

template <typename T, int N> struct Row {
    static constexpr int BYTES = N * (int)sizeof(T);
    static constexpr int WORDS = (BYTES + 3) / 4;
    uint32_t w[WORDS];

    __device__ __forceinline__ float get(int i) const {
        if constexpr (sizeof(T) == 4) {
            return __uint_as_float(w[i]);
        } else {
            return (i & 1) ? bf_hi(w[i >> 1]) : bf_lo(w[i >> 1]);
        }
    }

    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < WORDS; ++i) w[i] = 0u;
    }

    __device__ __forceinline__ void load(const T *p) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p);
        if constexpr (BYTES % 16 == 0) {
            if ((a & 15) == 0) {
#pragma unroll
                for (int i = 0; i < BYTES / 16; ++i) {
                    uint4 v = ld16(reinterpret_cast<const char *>(p) + 16 * i);
                    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                }
                return;
            }
        }
        if constexpr (BYTES % 8 == 0) {
            if ((a & 7) == 0) {
#pragma unroll
                for (int i = 0; i < BYTES / 8; ++i) {
                    uint2 v = __ldg(reinterpret_cast<const uint2 *>(p) + i);
                    w[2 * i] = v.x; w[2 * i + 1] = v.y;
                }
                return;
            }
        }
        if constexpr (BYTES % 4 == 0) {
            if ((a & 3) == 0) {
#pragma unroll
                for (int i = 0; i < BYTES / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(p) + i);
                return;
            }
        }
        if constexpr (sizeof(T) == 2) {
            const unsigned short *q = reinterpret_cast<const unsigned short *>(p);
            zero();
#pragma unroll
            for (int i = 0; i < N; ++i) w[i >> 1] |= (uint32_t)__ldg(q + i) << (16 * (i & 1));
        } else {
#pragma unroll
            for (int i = 0; i < N; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(p) + i);
        }
    }
};

// Store N floats as a row of T with the widest accesses the address allows.
template <typename T, int N> __device__ __forceinline__ void store_row(T *p, const float (&f)[N]) {
    constexpr int BYTES = N * (int)sizeof(T);
    constexpr int WORDS = (BYTES + 3) / 4;
    uint32_t w[WORDS];
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < N; ++i) w[i] = __float_as_uint(f[i]);
    } else {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) w[i] = pack_bf2(f[2 * i], f[2 * i + 1]);
        if constexpr (N & 1) w[N / 2] = pack_bf2(f[N - 1], 0.f);
    }
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if constexpr (BYTES % 16 == 0) {
        if ((a & 15) == 0) {
#pragma unroll
            for (int i = 0; i < BYTES / 16; ++i)
                st16(reinterpret_cast<char *>(p) + 16 * i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
            return;
        }
    }
    if constexpr (BYTES % 8 == 0) {
        if ((a & 7) == 0) {
#pragma unroll
            for (int i = 0; i < BYTES / 8; ++i) reinterpret_cast<uint2 *>(p)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
            return;
        }
    }
    if constexpr (BYTES % 4 == 0) {
        if ((a & 3) == 0) {
#pragma unroll
            for (int i = 0; i < BYTES / 4; ++i) reinterpret_cast<uint32_t *>(p)[i] = w[i];
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < N; ++i) p[i] = from_f<T>(f[i]);
}

// ------------------------------------------------------------ f32 pairs ---
// sm_100 executes fma/mul/add on pairs of fp32 values in one instruction
// (fma.rn.f32x2): each lane of the pair is an ordinary fp32 operation with
// round-to-nearest, so results equal the scalar ones.

typedef unsigned long long u64;

__device__ __forceinline__ u64 mk2(float lo, float hi) {
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float lo2(u64 v) {
    float a;
    asm("{ .reg .f32 hi; mov.b64 {%0, hi}, %1; }" : "=f"(a) : "l"(v));
    return a;
}
__device__ __forceinline__ float hi2(u64 v) {
    float b;
    asm("{ .reg .f32 lo; mov.b64 {lo, %0}, %1; }" : "=f"(b) : "l"(v));
    return b;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
    u64 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
    u64 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
    u64 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 16 bytes of T <-> P pairs of fp32 (pair p holds channels 2p and 2p+1).
template <typename T> struct Pairs;
template <> struct Pairs<bf16> {
    static constexpr int P = 4;
    __device__ __forceinline__ static void unpack(const uint4 &u, u64 (&p)[4]) {
        p[0] = mk2(bf_lo(u.x), bf_hi(u.x));
        p[1] = mk2(bf_lo(u.y), bf_hi(u.y));
        p[2] = mk2(bf_lo(u.z), bf_hi(u.z));
        p[3] = mk2(bf_lo(u.w), bf_hi(u.w));
    }
    __device__ __forceinline__ static uint4 pack(const u64 (&p)[4]) {
        return make_uint4(pack_bf2(lo2(p[0]), hi2(p[0])), pack_bf2(lo2(p[1]), hi2(p[1])),
                          pack_bf2(lo2(p[2]), hi2(p[2])), pack_bf2(lo2(p[3]), hi2(p[3])));
    }
};
template <> struct Pairs<float> {
    static constexpr int P = 2;
    __device__ __forceinline__ static void unpack(const uint4 &u, u64 (&p)[2]) {
        p[0] = mk2(__uint_as_float(u.x), __uint_as_float(u.y));
        p[1] = mk2(__uint_as_float(u.z), __uint_as_float(u.w));
    }
    __device__ __forceinline__ static uint4 pack(const u64 (&p)[2]) {
        return make_uint4(__float_as_uint(lo2(p[0])), __float_as_uint(hi2(p[0])), __float_as_uint(lo2(p[1])),
                          __float_as_uint(hi2(p[1])));
    }
};

// Sum of v over the L consecutive lanes of this lane's segment (segments start
// at multiples of L and lie inside the warp); the result is valid on the
// segment's first lane.  Any 1 <= L <= 32.
__device__ __forceinline__ float segment_sum(float v, int L, int pos) {
    for (int o = 1; o < L; o <<= 1) {
        float other = __shfl_down_sync(FULL_MASK, v, o);
        if (pos + o < L) v += other;
    }
    return v;
}

}  // namespace dsc
