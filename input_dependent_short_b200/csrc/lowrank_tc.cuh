// Shared pieces of the tensor-core low-rank kernels (lowrank_tc_fwd.cu,
// lowrank_tc_bwd.cu): the problem map, the kernel arguments, tensor-map
// encoding and small device helpers.
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 (rank-R factorisation of the filter
// generator, w[b,t,g,k] = sum_r z[b,t,r] U[r, g*W + k]) and "Efficient
// training implementation" (the fused kernels form zU on chip and convolve at
// once; the filter tensor never reaches HBM).
//
// Used for bf16 with R a multiple of 8 up to 64, H a divisor of 64 and D a
// multiple of 32*H (any W from 1 to 8); the CUDA-core kernels cover every
// other shape.
#pragma once

#include <cuda.h>

#include "kernels.cuh"
#include "tc.cuh"

namespace dsc {
namespace lrtc {

constexpr int TC_M = 128;                            // tokens per tile (TMEM lanes)
constexpr int TC_GROUPS = 32;                        // filter groups per forward unit block
constexpr long long TC_WAIT_LIMIT = 2000000000ll;    // ~1 s of clock cycles

struct TcMap {
    int64_t B, T, D, H, R, GW;
    int W, RP;           // RP: R padded to a multiple of 16
    int tilesPerSeq;     // tiles of 128 tokens per sequence
    int lgH;             // log2 H
    int residual;
    // forward: item = (tile, block of CF channels) -> NF TMEM columns; sub-tiles of SF channels
    int CF, NF, SF, nSubF, nBlkF, NSF, NOPF;
    int NFS;             // TMEM columns per filter buffer: NF rounded up to a power of two
    int64_t nItemsF;
    int zsw;             // forward z tile: one TMA box with this row swizzle (2R bytes: R = 16, 32, 64), or 0: 8-column boxes
    // backward: block of CB channels = GB groups -> NBW = W*GB <= 128 filter columns;
    // sub-tiles of SB channels; CTA = (range of tiles) x (group of CPC blocks)
    int CB, GB, NBW, SB, nSubB, nBlkB;
    int CPC, nGroups, nRanges, tilesPerRange;
    int splitUnits;      // > 0: one block per CTA, ranges of this many (tile, sub-tile) units
    int dzAcc;           // dz through an fp32 accumulator (several CTAs add to a token's dz)
    int NSB, DWB, NOP;   // sub-tile ring slots, dw tile buffers, operand buffers
    int64_t totalTiles;
};

struct TcArgs {
    TcMap m;
    const bf16 *x, *z, *U, *dy;
    bf16 *y, *dx, *dz;
    float *dU, *dz_acc, *dU_part;
    bf16 *Up;    // backward: U blocks as shared-memory images (columns tap-major, rows padded to RP)
    bf16 *zimg;  // backward: z tiles (136 rows) as shared-memory images
    bf16 *Uf;    // forward, H < 8: U [R, G*W] with each 8/H groups' columns tap-major (k*GPV + g)
};

// Fills the common part of the map; false when the tensor-core kernels do not take the shape.
bool tc_map(const dsc_problem &p, TcMap &m);

// bf16 tensor map of `rank` dimensions (innermost first): extents `dims`,
// byte strides of dimensions 1.. in `strides_bytes`, box `box`, zeros outside.
bool make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
              const uint32_t *box, CUtensorMapSwizzle swz, CUtensorMapL2promotion l2);

// Status word of the backward's bounded waits (read and cleared).
int take_tc_bwd_status(cudaStream_t stream);

__host__ __device__ constexpr uint32_t up1024(uint32_t v) { return (v + 1023u) & ~1023u; }

// 32 lanes x N consecutive fp32 TMEM columns (any N: loads of 8, then 4, 2, 1).
template <int N> __device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]) {
    uint32_t r[N];
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[8 * i]), "=r"(r[8 * i + 1]), "=r"(r[8 * i + 2]), "=r"(r[8 * i + 3]),
                       "=r"(r[8 * i + 4]), "=r"(r[8 * i + 5]), "=r"(r[8 * i + 6]), "=r"(r[8 * i + 7])
                     : "r"(taddr + 8 * i));
    constexpr int o4 = N / 8 * 8, o2 = o4 + (N & 4), o1 = o2 + (N & 2);
    if constexpr ((N & 4) != 0)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[o4]), "=r"(r[o4 + 1]), "=r"(r[o4 + 2]), "=r"(r[o4 + 3])
                     : "r"(taddr + o4));
    if constexpr ((N & 2) != 0)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[o2]), "=r"(r[o2 + 1]) : "r"(taddr + o2));
    if constexpr ((N & 1) != 0)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[o1]) : "r"(taddr + o1));
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint4 lds16(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Packed bf16 products a.lo*b.lo, a.hi*b.hi, each rounded once to bf16 (the
// exact product of two bf16 values, as fp32 would hold it, rounded to nearest).
__device__ __forceinline__ uint32_t mul_bf2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// acc + a.lo*b.lo and acc + a.hi*b.hi straight from packed bf16 words
// (exact bf16 products, fp32 round-to-nearest adds).
__device__ __forceinline__ float fma_bf16_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{ .reg .b16 al, ah, bl, bh;\n\t mov.b32 {al, ah}, %1;\n\t mov.b32 {bl, bh}, %2;\n\t"
        " fma.rn.f32.bf16 %0, al, bl, %3; }"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{ .reg .b16 al, ah, bl, bh;\n\t mov.b32 {al, ah}, %1;\n\t mov.b32 {bl, bh}, %2;\n\t"
        " fma.rn.f32.bf16 %0, ah, bh, %3; }"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}

}  // namespace lrtc
}  // namespace dsc
