// Shared pieces of the tensor-core low-rank kernels (lowrank_tc_fwd.cu,
// lowrank_tc_bwd.cu, lowrank_tc_dec.cu): the problem map, the kernel
// arguments, tensor-map encoding, small device helpers, and the filter-forming
// pipeline that the training forward and the decode step share.
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

// ------------------------------------------------ filter-forming pipeline ---
// The protocol the training forward (lowrank_tc_fwd.cu) and the decode step
// (lowrank_tc_dec.cu) share.  A producer thread fills NOP operand buffers (a
// z tile and a U block each); one thread issues the zU MMAs of consecutive
// items into two TMEM filter buffers; the sub-tiles the epilogue reads pass
// through a ring of NS slots.  Each hand-off is a full/empty mbarrier pair:
// OPF/OPE per operand buffer, WF/WE per filter buffer, XF/XE per slot.
constexpr int TP_MAXOP = 4;  // most operand buffers
constexpr int TP_MAXNS = 8;  // most ring slots

struct PipeBars {
    uint32_t base;
    static constexpr uint32_t BYTES = (2 * TP_MAXOP + 4 + 2 * TP_MAXNS) * 8;
    __device__ uint32_t opf(int b) const { return base + 8u * (uint32_t)b; }
    __device__ uint32_t ope(int b) const { return base + 8u * TP_MAXOP + 8u * (uint32_t)b; }
    __device__ uint32_t wf(int b) const { return base + 16u * TP_MAXOP + 8u * (uint32_t)b; }
    __device__ uint32_t we(int b) const { return base + 16u * TP_MAXOP + 16u + 8u * (uint32_t)b; }
    __device__ uint32_t xf(int s) const { return base + 16u * TP_MAXOP + 32u + 8u * (uint32_t)s; }
    __device__ uint32_t xe(int s) const { return base + 16u * TP_MAXOP + 32u + 8u * TP_MAXNS + 8u * (uint32_t)s; }
    // One thread, before the block synchronises: OPF, OPE, WF and XF take one
    // arrival (a transaction count or an MMA commit); WE and XE take the
    // counts of their consumers.
    __device__ void init(int ns, uint32_t we_count, uint32_t xe_count) const {
        for (int i = 0; i < TP_MAXOP; ++i) {
            tc::mbar_init(opf(i), 1);
            tc::mbar_init(ope(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(wf(i), 1);
            tc::mbar_init(we(i), we_count);
        }
        for (int i = 0; i < ns; ++i) {
            tc::mbar_init(xf(i), 1);
            tc::mbar_init(xe(i), xe_count);
        }
        tc::fence_mbar_init();
    }
};

// Zeroes the k-chunks R/8 .. RP/8-1 of every z buffer (the MMA reads them,
// nothing loads them); a no-op when R = RP.  All threads of the block.
__device__ __forceinline__ void zero_z_padding(unsigned char *smem, uint32_t opsize, int nop, const TcMap &m, int tid,
                                               int nthreads) {
    const int kz = m.R / 8;
    const int zpad = (m.RP / 8 - kz) * 128;
    for (int i = tid; i < nop * zpad; i += nthreads) {
        const int b = i / zpad, r = i % zpad;
        *reinterpret_cast<uint4 *>(smem + (uint32_t)b * opsize + (uint32_t)kz * 2048 + (uint32_t)r * 16) =
            make_uint4(0, 0, 0, 0);
    }
}

// One item's operands into the buffer at (zb, ub), completing on `bar`: the
// z tile of rows t0 .. t0+127 of sequence `bseq` (one box of 2R-byte rows
// with a 2R-byte swizzle for R = 16, 32 or 64, else R/8 boxes of 8 columns in
// the no-swizzle core-matrix layout) and, when `newu`, the NF columns of U
// block `blk` as boxes of 8 columns.  The producer thread.
__device__ __forceinline__ void load_operands(const TcMap &m, const CUtensorMap *tmz, const CUtensorMap *tmu,
                                              uint32_t zb, uint32_t ub, uint32_t ubytes, int t0, int bseq, int blk,
                                              int NF, bool newu, uint32_t bar) {
    const int kz = m.R / 8;
    tc::mbar_expect_tx(bar, (uint32_t)kz * 2048u + (newu ? ubytes : 0u));
    if (m.zsw) {
        tc::tma_load_3d(zb, tmz, 0, t0, bseq, bar);
    } else {
        for (int j = 0; j < kz; ++j) tc::tma_load_3d(zb + (uint32_t)j * 2048u, tmz, 8 * j, t0, bseq, bar);
    }
    if (newu) {
        const int col0 = blk * NF;
        for (int j = 0; j < NF / 8; ++j) tc::tma_load_2d(ub + (uint32_t)(j * m.RP * 16), tmu, col0 + 8 * j, 0, bar);
    }
}

// The zU MMAs of nI consecutive items, issued by one thread: item li waits
// for its operands (OPF) and for its TMEM buffer li & 1 to be read (WE, from
// item li-2), forms all NF filter columns of 128 rows with RP/16 MMAs, and
// commits to WF (filters ready) and OPE (operand buffer free).  `wait` is the
// kernel's bounded wait.
template <typename Wait>
__device__ __forceinline__ void filter_mma_loop(const TcMap &m, const PipeBars &bars, uint32_t sbase, uint32_t opsize,
                                                uint32_t zbytes, uint32_t tmem, int NF, int NFS, int nI, int NOP,
                                                Wait &&wait) {
    const uint32_t id_w = tc::idesc_bf16(TC_M, NF, 0, 1);
    int ob = 0;
    uint32_t oph = 0;
    for (int li = 0; li < nI; ++li) {
        const int b = li & 1;
        wait(bars.opf(ob), oph);
        if (li >= 2) wait(bars.we(b), (uint32_t)(((li - 2) >> 1) & 1));
        tc::fence_after_sync();
        const uint32_t zb = sbase + (uint32_t)ob * opsize, ub = zb + zbytes;
        for (int ks = 0; ks < m.RP / 16; ++ks) {
            const uint64_t ad = m.zsw ? tc::smem_desc_swz(zb + (uint32_t)ks * 32u, 16, 8u * (uint32_t)m.zsw, m.zsw)
                                      : tc::smem_desc(zb + (uint32_t)ks * 4096u, 2048, 128);
            const uint64_t bd = tc::smem_desc(ub + (uint32_t)ks * 256u, 128, (uint32_t)(m.RP * 16));
            tc::mma_bf16(tmem + (uint32_t)(b * NFS), ad, bd, id_w, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(bars.wf(b));
        tc::mma_commit(bars.ope(ob));
        if (++ob == NOP) {
            ob = 0;
            oph ^= 1u;
        }
    }
}

// Teardown, bounded (also after a time-out): the producer thread waits for
// the last loads into each of the NS slots (nG sub-tiles in all), the MMA
// thread for the MMAs that last read each of the NOP operand buffers (nI
// items), before the shared memory and TMEM are given back.
__device__ __forceinline__ void drain_loads(const PipeBars &bars, int NS, int nG) {
    for (int s = 0; s < NS && s < nG; ++s) {
        const int lastl = s + ((nG - 1 - s) / NS) * NS;
        tc::mbar_wait(bars.xf(s), (uint32_t)((lastl / NS) & 1), TC_WAIT_LIMIT);
    }
}
__device__ __forceinline__ void drain_mmas(const PipeBars &bars, int NOP, int nI) {
    for (int b = 0; b < NOP && b < nI; ++b) {
        const int lastli = b + ((nI - 1 - b) / NOP) * NOP;
        tc::mbar_wait(bars.ope(b), (uint32_t)((lastli / NOP) & 1), TC_WAIT_LIMIT);
    }
}

}  // namespace lrtc
}  // namespace dsc
