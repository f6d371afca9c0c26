// Tensor-core backward of the low-rank dynamic short convolution (sm_100a).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 and "Efficient training implementation"
// (the backward forms the filters on chip as the forward does):
//   dx[t,c]   = (w[t,g,0] + r) dy[t,c] + sum_{k>=1} w[t+k,g,k] dy[t+k,c]
//   dw[t,g,k] = sum_{c in g} dy[t,c] x[t-k,c]
//   dz[t,:]   = sum_{g,k} dw[t,g,k] U[:, g*W+k]      dU[:, g*W+k] = sum_t z[t,:] dw[t,g,k]
// (g = g(c) the channel's group; x, dy zero outside [0, T)).
//
// Block = GB groups = CB = GB*H channels, GB the largest power of two with
// NBW = W*GB <= 128 filter columns whose block divides D (128/W for W = 1, 2,
// 4, 8, 32 for W = 3 and 16 for W = 5 .. 7, unless D is too narrow for that;
// columns NBW .. 127 of the filter and dw tiles stay unused).  A prep kernel
// writes each block's U columns tap-major (column k*GB + g) and each z tile
// (136 rows) in the byte order of their shared-memory images, so per tap k one MMA
// z[t0+k .. t0+k+127] . U_block[:, k-th GB columns] puts w[t+k, g, k] -- the
// filter dx of token t needs -- on TMEM lane t: the shift by k tokens is only
// a start address in the z image.  Work item = (tile of 128 tokens, block).
// Per item:
//   W * RP/16 MMAs  filters into one of two TMEM buffers (128 columns);
//   epilogue        per sub-tile of SB = 16, 32 or 64 channels: dx (staged, TMA store) and dw
//                   (bf16, tap-major, into a [128 x 128] shared tile);
//   NBW/16 + 8 MMAs dz[tile] += dw . U_block^T   (TMEM, over the CTA's blocks),
//                   dU[block] += dw^T . z         (TMEM, over the CTA's tiles).
// CTA = (range of tiles) x (group of CPC blocks), or for long items with one
// block per CTA an equal range of (tile, sub-tile) units.  dz leaves TMEM after
// a tile's last block (bf16, or fp32 adds into an accumulator when several
// CTAs add to the same token), dU after the range (directly, or as a
// per-range partial summed by a finalize kernel).
//
// Warp roles (640 threads): warp 16 x/dy TMA producer, warp 17 TMEM owner and
// filter-MMA issuer, warp 18 operand loads and dU MMAs, warp 19 dz MMAs, warps
// 0-15 epilogue (thread part p of token t: VPT 8-channel vectors of each
// sub-tile, or 4 channels of a 16-channel sub-tile).  Groups wider than a
// part's channels (PPG parts per group) add their dw partial sums through a
// small exchange buffer.
#include "lowrank_tc.cuh"

namespace dsc {

// Status word of the backward's bounded waits on each device.
__device__ int g_dsc_status_tcb = 0;

namespace lrtc {

int take_tc_bwd_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status_tcb, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status_tcb, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

namespace {

constexpr int TB_EPI = 512;              // epilogue threads
constexpr int TB_THREADS = TB_EPI + 128;  // + x/dy producer, filter-MMA, operand/dU-MMA and dz-MMA warps
constexpr int TB_MAXNS = 8;              // most sub-tiles in flight
constexpr int TB_SMEM = 220 * 1024;
constexpr int TB_NB = 128;               // columns of a filter buffer and a dw tile (W * GB of them in use)
constexpr int TB_ZROWS = 136;            // z rows per tile: 128 + up to 7 for the shifted filters
constexpr uint32_t TB_ZR = TB_ZROWS * 16;  // bytes per 8-wide k-chunk of the z tile
constexpr int TB_MAXOP = 4;              // most operand (z, U) buffers
constexpr int TB_NBARS = 2 * TB_MAXOP + 13 + 2 * TB_MAXNS;

struct BwdSmem {
    uint32_t zbytes, ubytes, opsize, dw, dwsize, xch, ystage, ybox, ring, boxb, slot, bars, tmem, total;
    __host__ __device__ BwdSmem(const TcMap &m, int nop, int ns, int dwb, bool xchg) {
        const int rb = 2 * m.SB;  // box row bytes
        boxb = up1024((uint32_t)(rb * (TC_M + m.W - 1)));
        slot = 2 * boxb;  // x box + dy box
        ybox = (uint32_t)(rb * TC_M);
        zbytes = (uint32_t)(m.RP / 8) * TB_ZR;
        ubytes = (uint32_t)(m.RP * TB_NB * 2);
        opsize = up1024(zbytes + ubytes);
        dw = (uint32_t)nop * opsize;
        dwsize = (uint32_t)(TC_M * TB_NB * 2);
        ystage = dw + (uint32_t)dwb * dwsize;  // two dx staging tiles (TMA store sources)
        xch = ystage + 2 * ybox;
        ring = up1024(xch + (xchg ? (uint32_t)(2 * 4 * TC_M * m.W * 4) : 0u));
        bars = ring + (uint32_t)ns * slot;
        tmem = bars + TB_NBARS * 8;
        total = tmem + 16 + 1024;  // + slack to align the base to 1024 bytes
    }
};

// OPF[4] OPE[4] WF[2] WE[2] DWF[2] DWE[2] DZF[2] DZE[2] DUF XF[MAXNS] XE[MAXNS]
struct BwdBars {
    uint32_t base;
    __device__ uint32_t opf(int b) const { return base + 8u * (uint32_t)b; }
    __device__ uint32_t ope(int b) const { return base + 32u + 8u * (uint32_t)b; }
    __device__ uint32_t wf(int b) const { return base + 64u + 8u * (uint32_t)b; }
    __device__ uint32_t we(int b) const { return base + 80u + 8u * (uint32_t)b; }
    __device__ uint32_t dwf(int b) const { return base + 96u + 8u * (uint32_t)b; }
    __device__ uint32_t dwe(int b) const { return base + 112u + 8u * (uint32_t)b; }
    __device__ uint32_t dzf(int b) const { return base + 128u + 8u * (uint32_t)b; }
    __device__ uint32_t dze(int b) const { return base + 144u + 8u * (uint32_t)b; }
    __device__ uint32_t duf() const { return base + 160u; }
    __device__ uint32_t xf(int s) const { return base + 168u + 8u * (uint32_t)s; }
    __device__ uint32_t xe(int s) const { return base + 168u + 8u * TB_MAXNS + 8u * (uint32_t)s; }
};

// Items of a CTA in order (tile-major, block-minor), advanced without divisions.
struct BwdWalk {
    int tl, cl, t0, b, blk;
    __device__ void init(const TcMap &m, int64_t tile_lo, int chunk_lo) {
        tl = 0;
        cl = 0;
        b = (int)(tile_lo / m.tilesPerSeq);
        t0 = (int)(tile_lo % m.tilesPerSeq) * TC_M;
        blk = chunk_lo;
    }
    __device__ void next(const TcMap &m, int chunk_lo, int ncl) {
        if (++cl == ncl) {
            cl = 0;
            ++tl;
            t0 += TC_M;
            if (t0 >= m.T) {
                t0 = 0;
                ++b;
            }
        }
        blk = chunk_lo + cl;
    }
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(TB_EPI) : "memory"); }

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Stores n = 1, 2, 4, 8 or 16 consecutive bf16 values (from fp32) at a dw tile address.
template <int N> __device__ __forceinline__ void st_dw(unsigned char *p, const float *v) {
    if constexpr (N == 1) {
        *reinterpret_cast<bf16 *>(p) = __float2bfloat16_rn(v[0]);
    } else if constexpr (N == 2) {
        *reinterpret_cast<uint32_t *>(p) = pack_bf2(v[0], v[1]);
    } else if constexpr (N == 4) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf2(v[0], v[1]), pack_bf2(v[2], v[3]));
    } else if constexpr (N == 8) {
        *reinterpret_cast<uint4 *>(p) =
            make_uint4(pack_bf2(v[0], v[1]), pack_bf2(v[2], v[3]), pack_bf2(v[4], v[5]), pack_bf2(v[6], v[7]));
    } else {
        static_assert(N == 16, "dw run length");
        st_dw<8>(p, v);
        st_dw<8>(p + 128, v + 8);  // the next core matrix along the columns
    }
}

// dw[t, g, k] of groups of several channels: fp32 sums over the thread's
// channels, then across the PPG parts that share a group.
template <int W, int VPT, int GPT, int PPG, int RB>
__device__ __forceinline__ void bwd_dw_groups(const TcMap &m, const unsigned char *xb, const uint4 (&dyv)[VPT][W],
                                              unsigned char *dwt, float *xch, int part, int t_loc, int s, int g0) {
    constexpr int WIN = W - 1;
    constexpr int CT = 8 * VPT;
    constexpr int GPV = GPT >= VPT ? GPT / VPT : 1;
    constexpr int CPG = 8 / GPV;
    const int cs0 = part * CT;
    float pk[W][GPT];
#pragma unroll
    for (int k = 0; k < W; ++k)
#pragma unroll
        for (int g = 0; g < GPT; ++g) pk[k][g] = 0.f;
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int cs = cs0 + 8 * v;
        const int bo = (cs % (RB / 2)) / 8;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xb + tc::swz<RB>(t_loc + WIN - k, bo));
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
                const uint32_t dyw = word_of(dyv[v][0], wd), xwd = word_of(xv, wd);
                const int ga = GPT >= VPT ? v * GPV + (2 * wd) / CPG : (v * GPT) / VPT;
                const int gb = GPT >= VPT ? v * GPV + (2 * wd + 1) / CPG : (v * GPT) / VPT;
                pk[k][ga] = fma_bf16_lo(dyw, xwd, pk[k][ga]);
                pk[k][gb] = fma_bf16_hi(dyw, xwd, pk[k][gb]);
            }
        }
    }
    if constexpr (PPG == 1) {
#pragma unroll
        for (int k = 0; k < W; ++k)
            st_dw<GPT>(dwt + tc::core_off(t_loc, k * m.GB + g0, TB_NB), pk[k]);
    } else {
        // parts p0 .. p0+PPG-1 share the group; part p finishes the taps k = p (mod PPG)
        float *mine = xch + ((s & 1) * 4 * TC_M + part * TC_M + t_loc) * W;
#pragma unroll
        for (int k = 0; k < W; ++k) mine[k] = pk[k][0];
        epi_bar();
        const int p0 = part - part % PPG;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            if (k % PPG != part % PPG) continue;
            float tot = 0.f;
#pragma unroll
            for (int q = 0; q < PPG; ++q) tot += xch[((s & 1) * 4 * TC_M + (p0 + q) * TC_M + t_loc) * W + k];
            st_dw<1>(dwt + tc::core_off(t_loc, k * m.GB + g0, TB_NB), &tot);
        }
    }
}

// One sub-tile of the epilogue for token t_loc, thread part `part`.
//   VPT vectors of 8 channels; GPT groups among the thread's 8*VPT channels
//   (1 when the group is wider: PPG parts then share it).  With one vector
//   (VPT = 1) the thread's swizzled row offsets ro[k] (box row t_loc + k; the
//   x, dy and dx staging boxes share them) are computed once per thread.
template <int W, int VPT, int GPT, int PPG, int RB>
__device__ __forceinline__ void bwd_subtile(const TcMap &m, const unsigned char *xs, uint32_t boxb, uint32_t tb,
                                            unsigned char *dwt, float *xch, int part, int t_loc, int s,
                                            unsigned char *ys, float res, uint32_t release_w,
                                            const uint32_t (&ro)[W]) {
    constexpr int WIN = W - 1;
    constexpr int CT = 8 * VPT;                      // the thread's channels
    constexpr int GPV = GPT >= VPT ? GPT / VPT : 1;  // groups inside one vector
    constexpr int CPG = 8 / GPV;                     // a group's channels inside one vector
    const int cs0 = part * CT;                       // sub-tile channel of the thread's first vector
    const int ci0 = s * m.SB + cs0;                  // block channel
    const int g0 = ci0 >> m.lgH;                     // block group of the thread's first channel
    // filters w[t+k, g0 .. g0+GPT-1, k] (tap-major TMEM columns k*GB + g)
    float wt[W][GPT];
#pragma unroll
    for (int k = 0; k < W; ++k) tmem_ld<GPT>(tb + (uint32_t)(k * m.GB + g0), wt[k]);
    const unsigned char *xb = xs;          // x rows t0-WIN .. t0+127
    const unsigned char *yb = xs + boxb;   // dy rows t0 .. t0+127+WIN
    uint4 dyv[VPT][W];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int cs = cs0 + 8 * v;
        const int bo = (cs % (RB / 2)) / 8;
#pragma unroll
        for (int k = 0; k < W; ++k)
            dyv[v][k] = *reinterpret_cast<const uint4 *>(yb + (VPT == 1 ? ro[k] : tc::swz<RB>(t_loc + k, bo)));
    }
    tc::tmem_wait_ld();
    if (release_w) {  // the item's last filter read: its TMEM buffer is free for the next MMA
        tc::fence_before_sync();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) tc::mbar_arrive(release_w);
    }
#pragma unroll
    for (int g = 0; g < GPT; ++g) wt[0][g] += res;
    // dx
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        float dxv[8];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const int ga = GPT >= VPT ? v * GPV + (2 * pp) / CPG : (v * GPT) / VPT;
            const int gb = GPT >= VPT ? v * GPV + (2 * pp + 1) / CPG : (v * GPT) / VPT;
            if constexpr (GPV == 1) {
                u64 acc2 = 0ull;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const uint32_t word = word_of(dyv[v][k], pp);
                    const u64 dp = mk2(bf_lo(word), bf_hi(word));
                    const float wk = wt[k][ga];
                    acc2 = k == 0 ? mul2(mk2(wk, wk), dp) : fma2(mk2(wk, wk), dp, acc2);
                }
                dxv[2 * pp] = lo2(acc2);
                dxv[2 * pp + 1] = hi2(acc2);
            } else if constexpr (CPG == 1) {  // a group per channel: the two channels' filters as a pair
                u64 acc2 = 0ull;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const uint32_t word = word_of(dyv[v][k], pp);
                    const u64 wp = mk2(wt[k][ga], wt[k][gb]), dp = mk2(bf_lo(word), bf_hi(word));
                    acc2 = k == 0 ? mul2(wp, dp) : fma2(wp, dp, acc2);
                }
                dxv[2 * pp] = lo2(acc2);
                dxv[2 * pp + 1] = hi2(acc2);
            } else {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const uint32_t word = word_of(dyv[v][k], pp);
                    a0 = k == 0 ? wt[k][ga] * bf_lo(word) : fmaf(wt[k][ga], bf_lo(word), a0);
                    a1 = k == 0 ? wt[k][gb] * bf_hi(word) : fmaf(wt[k][gb], bf_hi(word), a1);
                }
                dxv[2 * pp] = a0;
                dxv[2 * pp + 1] = a1;
            }
        }
        *reinterpret_cast<uint4 *>(ys + (VPT == 1 ? ro[0] : tc::swz<RB>(t_loc, ((cs0 + 8 * v) % (RB / 2)) / 8))) =
            make_uint4(pack_bf2(dxv[0], dxv[1]), pack_bf2(dxv[2], dxv[3]), pack_bf2(dxv[4], dxv[5]),
                       pack_bf2(dxv[6], dxv[7]));
    }
    if constexpr (GPT == CT) {
        // one channel per group (H = 1): dw[t, g, k] = dy[t, c] x[t-k, c], rounded once to bf16
        const uint32_t gb16 = (uint32_t)m.GB * 16u;  // bytes between the taps' column blocks of a dw row
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            const int bo = ((cs0 + 8 * v) % (RB / 2)) / 8;
            unsigned char *dwv = dwt + tc::core_off(t_loc, g0 + 8 * v, TB_NB);
#pragma unroll
            for (int k = 0; k < W; ++k) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(
                    xb + (VPT == 1 ? ro[WIN - k] : tc::swz<RB>(t_loc + WIN - k, bo)));
                *reinterpret_cast<uint4 *>(dwv + (uint32_t)k * gb16) =
                    make_uint4(mul_bf2(dyv[v][0].x, xv.x), mul_bf2(dyv[v][0].y, xv.y), mul_bf2(dyv[v][0].z, xv.z),
                               mul_bf2(dyv[v][0].w, xv.w));
            }
        }
    } else {
        bwd_dw_groups<W, VPT, GPT, PPG, RB>(m, xb, dyv, dwt, xch, part, t_loc, s, g0);
    }
}

// The same for sub-tiles of 16 channels (blocks of 16 groups, H = 1): the
// thread's 4 channels are the 8 bytes at `off` in 16-byte chunk `chunk` of
// each 32-byte row; channel i of the thread is its group g0 + i.
template <int W>
__device__ __forceinline__ void bwd_subtile_q(const TcMap &m, const unsigned char *xs, uint32_t boxb, uint32_t tb,
                                              unsigned char *dwt, int part, int t_loc, int s, unsigned char *ys,
                                              float res, uint32_t release_w) {
    constexpr int WIN = W - 1;
    const int g0 = s * m.SB + part * 4;  // block group = block channel of the thread's first channel
    const int chunk = part >> 1;
    const uint32_t off = (uint32_t)(part & 1) * 8u;
    float wt[W][4];
#pragma unroll
    for (int k = 0; k < W; ++k) tmem_ld<4>(tb + (uint32_t)(k * m.GB + g0), wt[k]);
    const unsigned char *xb = xs;         // x rows t0-WIN .. t0+127
    const unsigned char *yb = xs + boxb;  // dy rows t0 .. t0+127+WIN
    uint2 dyv[W];
#pragma unroll
    for (int k = 0; k < W; ++k) dyv[k] = *reinterpret_cast<const uint2 *>(yb + tc::swz<32>(t_loc + k, chunk) + off);
    tc::tmem_wait_ld();
    if (release_w) {  // the item's last filter read: its TMEM buffer is free for the next MMA
        tc::fence_before_sync();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) tc::mbar_arrive(release_w);
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) wt[0][g] += res;
    // dx
    uint32_t dxw[2];
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
        u64 acc2 = 0ull;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const uint32_t word = pp ? dyv[k].y : dyv[k].x;
            const u64 wp = mk2(wt[k][2 * pp], wt[k][2 * pp + 1]), dp = mk2(bf_lo(word), bf_hi(word));
            acc2 = k == 0 ? mul2(wp, dp) : fma2(wp, dp, acc2);
        }
        dxw[pp] = pack_bf2(lo2(acc2), hi2(acc2));
    }
    *reinterpret_cast<uint2 *>(ys + tc::swz<32>(t_loc, chunk) + off) = make_uint2(dxw[0], dxw[1]);
    // dw[t, g0+i, k] = dy[t, c] x[t-k, c] (one channel per group), rounded once to bf16
#pragma unroll
    for (int k = 0; k < W; ++k) {
        const uint2 xv = *reinterpret_cast<const uint2 *>(xb + tc::swz<32>(t_loc + WIN - k, chunk) + off);
        *reinterpret_cast<uint2 *>(dwt + tc::core_off(t_loc, k * m.GB + g0, TB_NB)) =
            make_uint2(mul_bf2(dyv[0].x, xv.x), mul_bf2(dyv[0].y, xv.y));
    }
}

template <int W, int VPT, int GPT, int PPG>
__global__ void __launch_bounds__(TB_THREADS, 1)
    k_lr_tc_bwd(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmdy,
                const __grid_constant__ CUtensorMap tmdx, const TcArgs a) {
    constexpr int WIN = W - 1;
    constexpr int RB = VPT == 0 ? 32 : (VPT == 1 ? 64 : 128);  // box row bytes (16, 32 or 64 channels)
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const TcMap &m = a.m;
    const int NS = m.NSB, NOP = m.NOP, DWB = m.DWB;
    const BwdSmem S(m, NOP, NS, DWB, PPG > 1);
    const int group = blockIdx.x % m.nGroups;
    const int range = blockIdx.x / m.nGroups;
    const int chunk_lo = group * m.CPC;
    const int ncl = min(m.CPC, m.nBlkB - chunk_lo);
    int64_t tile_lo;
    int ntl, s_first = 0, s_last = m.nSubB;  // sub-tiles of the first and last item
    if (m.splitUnits > 0) {  // a range of (tile, sub-tile) units of one block
        const int64_t u_lo = (int64_t)range * m.splitUnits;
        const int64_t u_hi = min(u_lo + m.splitUnits, m.totalTiles * m.nSubB);
        if (u_lo >= u_hi) return;
        tile_lo = u_lo / m.nSubB;
        ntl = (int)((u_hi - 1) / m.nSubB - tile_lo + 1);
        s_first = (int)(u_lo % m.nSubB);
        s_last = (int)((u_hi - 1) % m.nSubB) + 1;
    } else {
        tile_lo = (int64_t)range * m.tilesPerRange;
        ntl = (int)min((int64_t)m.tilesPerRange, m.totalTiles - tile_lo);
    }
    if (ncl <= 0 || ntl <= 0) return;
    const int nI = ntl * ncl;
    auto s_begin = [&](int li) { return li == 0 ? s_first : 0; };
    auto s_end = [&](int li) { return li == nI - 1 ? s_last : m.nSubB; };
    const int nG = nI == 1 ? s_last - s_first : (m.nSubB - s_first) + (nI - 2) * m.nSubB + s_last;

    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const BwdBars bars{sbase + S.bars};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t col_dz = 2 * TB_NB, col_dU = 2 * TB_NB + 2 * m.RP;

    if (tid == 0) {
        for (int i = 0; i < TB_MAXOP; ++i) {
            tc::mbar_init(bars.opf(i), 1);
            tc::mbar_init(bars.ope(i), 2);  // dz and dU MMAs of the item, from two threads
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bars.wf(i), 1);
            tc::mbar_init(bars.we(i), TB_EPI / 32);
            tc::mbar_init(bars.dwf(i), TB_EPI / 32);
            tc::mbar_init(bars.dwe(i), 2);
            tc::mbar_init(bars.dzf(i), 1);
            tc::mbar_init(bars.dze(i), TB_EPI / 32);
        }
        tc::mbar_init(bars.duf(), 1);
        for (int i = 0; i < NS; ++i) {
            tc::mbar_init(bars.xf(i), 1);
            tc::mbar_init(bars.xe(i), TB_EPI / 32);
        }
        tc::fence_mbar_init();
    }
    if (warp == 17) tc::tmem_alloc(sbase + S.tmem, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S.tmem);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;  // sticky: later waits skip
    };
    pdl_wait();  // inputs and operand images come from earlier kernels of the stream
    pdl_trigger();

    if (warp == 18) {
        // --------------------------- operand loads and dU MMAs (one lane)
        // The tile's z image and the block's U image arrive by one bulk copy each;
        // a buffer is refilled once the dz and dU MMAs of its previous item are done.
        if (lane == 0) {
            const uint32_t id_dU = tc::idesc_bf16(TC_M, m.RP, 1, 1);
            BwdWalk it, pf;
            it.init(m, tile_lo, chunk_lo);
            pf.init(m, tile_lo, chunk_lo);
            constexpr int PF = 6;  // operand images are prefetched into L2 this many items ahead
            for (int li = 0; li < PF && li < nI; ++li, pf.next(m, chunk_lo, ncl)) {
                tc::bulk_prefetch_l2(a.zimg + (size_t)(tile_lo + pf.tl) * (S.zbytes / 2), S.zbytes);
                tc::bulk_prefetch_l2(a.Up + (size_t)pf.blk * (S.ubytes / 2), S.ubytes);
            }
            auto load_op = [&](int ob) {
                const uint32_t zb = sbase + (uint32_t)ob * S.opsize, ub = zb + S.zbytes;
                tc::mbar_expect_tx(bars.opf(ob), S.zbytes + S.ubytes);
                tc::bulk_load(zb, a.zimg + (size_t)(tile_lo + it.tl) * (S.zbytes / 2), S.zbytes, bars.opf(ob));
                tc::bulk_load(ub, a.Up + (size_t)it.blk * (S.ubytes / 2), S.ubytes, bars.opf(ob));
                if (pf.tl < ntl) {
                    tc::bulk_prefetch_l2(a.zimg + (size_t)(tile_lo + pf.tl) * (S.zbytes / 2), S.zbytes);
                    tc::bulk_prefetch_l2(a.Up + (size_t)pf.blk * (S.ubytes / 2), S.ubytes);
                    pf.next(m, chunk_lo, ncl);
                }
                it.next(m, chunk_lo, ncl);
            };
            int nload = 0;
            for (; nload < NOP && nload < nI; ++nload) load_op(nload);
            int fob = 0, fdb = 0, ftl = 0, fcl = 0;
            uint32_t fdph = 0, foph = 0;
            for (int li = 0; li < nI; ++li) {
                wait(bars.dwf(fdb), fdph);  // item li's dw tile is complete
                tc::fence_after_sync();
                const uint32_t zb = sbase + (uint32_t)fob * S.opsize;
                const uint32_t dwb = sbase + S.dw + (uint32_t)fdb * S.dwsize;
                for (int ks = 0; ks < TC_M / 16; ++ks) {
                    const uint64_t ad =
                        tc::smem_desc(dwb + (uint32_t)ks * 2u * ((TB_NB / 8) * 128), (TB_NB / 8) * 128, 128);
                    const uint64_t bd = tc::smem_desc(zb + (uint32_t)ks * 256u, 128, TB_ZR);
                    tc::mma_bf16(tmem + col_dU + (uint32_t)(fcl * m.RP), ad, bd, id_dU, (ftl > 0 || ks > 0) ? 1u : 0u);
                }
                tc::mma_commit(bars.dwe(fdb));
                tc::mma_commit(bars.ope(fob));
                if (nload < nI) {  // refill this buffer for item li + NOP
                    wait(bars.ope(fob), foph);
                    load_op(fob);
                    ++nload;
                }
                if (++fob == NOP) {
                    fob = 0;
                    foph ^= 1u;
                }
                if (++fdb == DWB) {
                    fdb = 0;
                    fdph ^= 1u;
                }
                if (++fcl == ncl) {
                    fcl = 0;
                    ++ftl;
                }
            }
            tc::mma_commit(bars.duf());
            for (int b = 0; b < NOP && b < nI; ++b) {  // the last loads have landed
                const int last = b + ((nI - 1 - b) / NOP) * NOP;
                tc::mbar_wait(bars.opf(b), (uint32_t)((last / NOP) & 1), TC_WAIT_LIMIT);
            }
        }
    } else if (warp == 16) {
        // ------------------------------------------------- x / dy producer
        if (lane == 0) {
            tc::tma_prefetch_desc(&tmx);            tc::tma_prefetch_desc(&tmdy);
            BwdWalk it;
            it.init(m, tile_lo, chunk_lo);
            int slot = 0, l = 0;
            uint32_t xph = 0;
            for (int li = 0; li < nI; ++li, it.next(m, chunk_lo, ncl)) {
                for (int s = s_begin(li); s < s_end(li); ++s, ++l) {
                    if (l >= NS) wait(bars.xe(slot), xph ^ 1u);
                    const uint32_t xb = sbase + S.ring + (uint32_t)slot * S.slot;
                    tc::mbar_expect_tx(bars.xf(slot), (uint32_t)(2 * RB * (TC_M + WIN)));
                    const int c = it.blk * m.CB + s * m.SB;
                    tc::tma_load_3d(xb, &tmx, c, it.t0 - WIN, it.b, bars.xf(slot));
                    tc::tma_load_3d(xb + S.boxb, &tmdy, c, it.t0, it.b, bars.xf(slot));
                    if (++slot == NS) {
                        slot = 0;
                        xph ^= 1u;
                    }
                }
            }
            for (int s = 0; s < NS && s < nG; ++s) {  // the last loads have landed
                const int lastl = s + ((nG - 1 - s) / NS) * NS;
                tc::mbar_wait(bars.xf(s), (uint32_t)((lastl / NS) & 1), TC_WAIT_LIMIT);
            }
        }
    } else if (warp == 17) {
        // ------------------------------------------------- filter MMAs (w)
        // One lane issues each item's per-tap MMAs; the dz / dU MMAs come from
        // warp 19, so the two streams of instructions overlap (a commit tracks
        // only the MMAs of the thread that issues it).
        if (lane == 0) {
            const uint32_t id_w = tc::idesc_bf16(TC_M, m.GB, 0, 1);
            int ob = 0;
            uint32_t oph = 0;
            for (int li = 0; li < nI; ++li) {
                const int b = li & 1;
                wait(bars.opf(ob), oph);
                if (li >= 2) wait(bars.we(b), (uint32_t)(((li - 2) >> 1) & 1));
                tc::fence_after_sync();
                const uint32_t zb = sbase + (uint32_t)ob * S.opsize, ub = zb + S.zbytes;
                for (int k = 0; k < W; ++k)
                    for (int ks = 0; ks < m.RP / 16; ++ks) {
                        const uint64_t ad = tc::smem_desc(zb + (uint32_t)(k * 16) + (uint32_t)ks * 2u * TB_ZR, TB_ZR, 128);
                        const uint64_t bd = tc::smem_desc(ub + (uint32_t)((k * m.GB / 8) * m.RP * 16) + (uint32_t)ks * 256u,
                                                          128, (uint32_t)(m.RP * 16));
                        tc::mma_bf16(tmem + (uint32_t)(b * TB_NB + k * m.GB), ad, bd, id_w, ks > 0 ? 1u : 0u);
                    }
                tc::mma_commit(bars.wf(b));
                if (++ob == NOP) {
                    ob = 0;
                    oph ^= 1u;
                }
            }
        }
    } else if (warp == 19) {
        // ---------------------------------------------------- dz MMAs
        if (lane == 0) {
            const uint32_t id_dz = tc::idesc_bf16(TC_M, m.RP, 0, 0);
            int fob = 0, fdb = 0, ftl = 0, fcl = 0;
            uint32_t fdph = 0;
            for (int li = 0; li < nI; ++li) {
                const int tp = ftl & 1;
                wait(bars.dwf(fdb), fdph);  // item li's dw tile is complete (so are its filter MMAs)
                if (fcl == 0 && ftl >= 2) wait(bars.dze(tp), (uint32_t)(((ftl - 2) >> 1) & 1));
                tc::fence_after_sync();
                const uint32_t ub = sbase + (uint32_t)fob * S.opsize + S.zbytes;
                const uint32_t dwb = sbase + S.dw + (uint32_t)fdb * S.dwsize;
                for (int ks = 0; ks < m.NBW / 16; ++ks) {  // dw columns NBW .. 127 are never written
                    const uint64_t ad = tc::smem_desc(dwb + (uint32_t)ks * 256u, 128, (TB_NB / 8) * 128);
                    const uint64_t bd = tc::smem_desc(ub + (uint32_t)(ks * 2 * m.RP * 16), (uint32_t)(m.RP * 16), 128);
                    tc::mma_bf16(tmem + col_dz + (uint32_t)(tp * m.RP), ad, bd, id_dz, (fcl > 0 || ks > 0) ? 1u : 0u);
                }
                tc::mma_commit(bars.dwe(fdb));
                tc::mma_commit(bars.ope(fob));
                if (fcl == ncl - 1) tc::mma_commit(bars.dzf(tp));
                if (++fob == NOP) fob = 0;
                if (++fdb == DWB) {
                    fdb = 0;
                    fdph ^= 1u;
                }
                if (++fcl == ncl) {
                    fcl = 0;
                    ++ftl;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int t_loc = tid & (TC_M - 1), part = tid >> 7, quarter = warp & 3;
        const float res = m.residual ? 1.f : 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        float *xch = reinterpret_cast<float *>(smem + S.xch);
        uint32_t ro[W];  // swizzled offsets of box rows t_loc .. t_loc+W-1 (one-vector parts)
#pragma unroll
        for (int k = 0; k < W; ++k) ro[k] = tc::swz<RB>(t_loc + k, VPT == 1 ? ((part * 8) % (RB / 2)) / 8 : 0);
        // dz of CTA-local tile j (its last block's MMAs are done) leaves TMEM
        auto dz_out = [&](int j, int bseq, int t0) {
            const int tp = j & 1;
            wait(bars.dzf(tp), (uint32_t)((j >> 1) & 1));
            tc::fence_after_sync();
            const int t = t0 + t_loc;
            for (int r = 8 * part; r < m.RP; r += 32) {  // 8-column chunks, dealt round the parts
                float v[8];
                tmem_ld<8>(tlane + col_dz + (uint32_t)(tp * m.RP + r), v);
                tc::tmem_wait_ld();
                if (t < m.T && r < m.R) {  // R is a multiple of 8
                    const int64_t o = ((int64_t)bseq * m.T + t) * m.R + r;
                    if (!m.dzAcc) {
                        st16(a.dz + o, make_uint4(pack_bf2(v[0], v[1]), pack_bf2(v[2], v[3]), pack_bf2(v[4], v[5]),
                                                  pack_bf2(v[6], v[7])));
                    } else {
                        red_add_v4(a.dz_acc + o, v[0], v[1], v[2], v[3]);
                        red_add_v4(a.dz_acc + o + 4, v[4], v[5], v[6], v[7]);
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bars.dze(tp));
        };
        BwdWalk it;
        it.init(m, tile_lo, chunk_lo);
        int slot = 0, db = 0, pb = 0, pt0 = 0, ybuf = 0;
        uint32_t xph = 0, dph = 0;
        for (int li = 0; li < nI; ++li) {
            const int b = li & 1;
            wait(bars.wf(b), (uint32_t)((li >> 1) & 1));
            if (li >= DWB) wait(bars.dwe(db), dph ^ 1u);
            tc::fence_after_sync();
            const uint32_t tb = tlane + (uint32_t)(b * TB_NB);
            unsigned char *dwt = smem + S.dw + (uint32_t)db * S.dwsize;
            const int sb = s_begin(li), se = s_end(li);
            if (sb > 0 || se < m.nSubB) {
                // part of the block's groups only: the other dw columns must read as zero
                for (int i = tid; i < TC_M * TB_NB * 2 / 16; i += TB_EPI)
                    *reinterpret_cast<uint4 *>(dwt + 16 * i) = make_uint4(0, 0, 0, 0);
                epi_bar();
            }
            for (int s = sb; s < se; ++s) {
                wait(bars.xf(slot), xph);
                if constexpr (VPT == 0)
                    bwd_subtile_q<W>(m, smem + S.ring + (uint32_t)slot * S.slot, S.boxb, tb, dwt, part, t_loc, s,
                                     smem + S.ystage + (uint32_t)ybuf * S.ybox, res, s == se - 1 ? bars.we(b) : 0u);
                else
                    bwd_subtile<W, VPT, GPT, PPG, RB>(m, smem + S.ring + (uint32_t)slot * S.slot, S.boxb, tb, dwt, xch,
                                                      part, t_loc, s, smem + S.ystage + (uint32_t)ybuf * S.ybox, res,
                                                      s == se - 1 ? bars.we(b) : 0u, ro);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bars.xe(slot));
                // dx rows of this lane quarter (32 tokens) -> global by TMA, issued by the
                // quarter's first thread after a barrier of its 4 warps only; the staging
                // rows the next sub-tile writes were read by the store this thread issued one
                // sub-tile ago, waited for before the barrier
                tc::fence_proxy_async();
                const bool qlead = warp == quarter && lane == 0;
                if (qlead) tc::bulk_wait_read_all();
                asm volatile("bar.sync %0, %1;" ::"r"(2 + quarter), "n"(TB_EPI / 4) : "memory");
                if (qlead) {
                    tc::tma_store_3d(&tmdx, sbase + S.ystage + (uint32_t)ybuf * S.ybox + (uint32_t)(quarter * 32 * RB),
                                     it.blk * m.CB + s * m.SB, it.t0 + quarter * 32, it.b);
                    tc::bulk_commit();
                }
                ybuf ^= 1;
                if (++slot == NS) {
                    slot = 0;
                    xph ^= 1u;
                }
            }
            tc::fence_proxy_async();  // dw tile (generic stores) -> MMA operand
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bars.dwf(db));
            if (++db == DWB) {
                db = 0;
                dph ^= 1u;
            }
            // the previous tile's dz (its last MMAs have had this whole item to finish)
            if (li >= 1 && it.cl == 0) dz_out(it.tl - 1, pb, pt0);
            pb = it.b;
            pt0 = it.t0;
            it.next(m, chunk_lo, ncl);
        }
        dz_out(ntl - 1, pb, pt0);
        // dU of the CTA's blocks over its tile range: TMEM lane = block column k*GB + g
        // (lanes NBW .. 127 hold no filter column)
        wait(bars.duf(), 0);
        tc::fence_after_sync();
        const int k = t_loc / m.GB, gl = t_loc % m.GB;
        for (int cl = 0; cl < ncl; ++cl) {
            const int64_t col = (int64_t)(chunk_lo + cl) * m.NBW + gl * W + k;
            for (int r8 = 8 * part; r8 < m.RP; r8 += 32) {  // 8-column chunks, dealt round the parts
                float v[8];
                tmem_ld<8>(tlane + col_dU + (uint32_t)(cl * m.RP + r8), v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = r8 + j;
                    if (r < m.R && k < W) {
                        if (m.nRanges == 1) a.dU[(int64_t)r * m.GW + col] = v[j];
                        else a.dU_part[((int64_t)range * m.R + r) * m.GW + col] = v[j];
                    }
                }
            }
        }
        if (warp == quarter && lane == 0) tc::bulk_wait_all();  // each quarter's own dx stores
    }

    // teardown: every load and MMA this CTA issued has landed before the
    // shared memory and TMEM are given back (bounded, also after a time-out)
    if (warp == 18 && lane == 0) tc::mbar_wait(bars.duf(), 0, TC_WAIT_LIMIT);
    if (timed_out) atomicExch(&g_dsc_status_tcb, (int)DSC_ERR_TIMEOUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 17) tc::tmem_dealloc(tmem, 512);
}

// Operand images the backward loads with one bulk copy each:
//   U image of block blk: element (j, r) at (j/8)*(RP*8) + r*8 + j%8, column
//     j = k*GB + g holding U[r][(blk*GB + g)*W + k] (tap-major), rows r >= R and
//     columns j >= NBW zero;
//   z image of tile i (sequence b, first token t0): element (t, r) at
//     (r/8)*(136*8) + t*8 + r%8 holding z[b][t0+t][r], zero for r >= R or t0+t >= T.
// One thread per 16-byte chunk of the images (8 consecutive elements):
//   U image chunk (blk, jc, r): columns j = 8*jc .. 8*jc+7 of rank row r, one
//     tap k and 8 consecutive groups (GB is a multiple of 8), gathered with
//     stride W from U;
//   z image chunk (tile, rc, t): ranks 8*rc .. 8*rc+7 of token t, one 16-byte
//     load of z (R is a multiple of 8).
__global__ void k_bwd_prep(const TcArgs a) {
    pdl_wait();
    pdl_trigger();
    const TcMap &m = a.m;
    const int uper = 16 * m.RP;                  // chunks per U block image
    const int zper = (m.RP / 8) * TB_ZROWS;      // chunks per z tile image
    const int64_t nU = (int64_t)m.nBlkB * uper;
    const int64_t nZ = m.totalTiles * zper;
    for (int64_t ci = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; ci < nU + nZ; ci += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ci < nU) {
            // thread order (block, rank row, column chunk): a warp's gathers stay
            // inside the 256-byte run of U that holds a block's row
            const int64_t blk = ci / uper;
            const int rem = (int)(ci - blk * uper);
            const int r = rem >> 4, jc = rem & 15;
            const int j0 = 8 * jc, k = j0 / m.GB, g0 = j0 - k * m.GB;
            if (r < m.R && k < m.W) {
                const bf16 *src = a.U + (int64_t)r * m.GW + (blk * m.GB + g0) * m.W + k;
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = (uint32_t)__bfloat16_as_ushort(src[(2 * e) * m.W]) |
                           ((uint32_t)__bfloat16_as_ushort(src[(2 * e + 1) * m.W]) << 16);
                v = make_uint4(w[0], w[1], w[2], w[3]);
            }
            st16(a.Up + ((blk * 16 + jc) * m.RP + r) * 8, v);
        } else {
            const int64_t i2 = ci - nU;
            const int64_t tile = i2 / zper;
            const int rem = (int)(i2 - tile * zper);
            const int rc = rem / TB_ZROWS, t = rem - rc * TB_ZROWS;
            const int64_t b = tile / m.tilesPerSeq;
            const int64_t tt = (tile - b * m.tilesPerSeq) * TC_M + t;
            if (8 * rc < m.R && tt < m.T) v = ld16(a.z + (b * m.T + tt) * m.R + 8 * rc);
            st16(a.zimg + i2 * 8, v);
        }
    }
}

// n is a multiple of 4 and p 16-byte aligned.
__global__ void k_tc_zero(float *p, int64_t n) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += (int64_t)gridDim.x * blockDim.x)
        reinterpret_cast<float4 *>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dU = sum of the per-range partials (fixed order); dz = the fp32 accumulator in
// bf16.  Four elements per thread (R and R*GW are multiples of 8).
__global__ void k_tc_finalize(const TcArgs a) {
    pdl_wait();
    pdl_trigger();
    const TcMap &m = a.m;
    const int64_t nU = m.nRanges > 1 ? m.R * m.GW / 4 : 0;
    const int64_t nz = m.dzAcc ? m.B * m.T * m.R / 4 : 0;
    const int64_t qs = m.R * m.GW / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nU + nz; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nU) {
            const float4 *part = reinterpret_cast<const float4 *>(a.dU_part);
            float4 sacc = part[i];
            for (int q = 1; q < m.nRanges; ++q) {
                const float4 v = part[(int64_t)q * qs + i];
                sacc.x += v.x;
                sacc.y += v.y;
                sacc.z += v.z;
                sacc.w += v.w;
            }
            reinterpret_cast<float4 *>(a.dU)[i] = sacc;
        } else {
            const float4 v = reinterpret_cast<const float4 *>(a.dz_acc)[i - nU];
            reinterpret_cast<uint2 *>(a.dz)[i - nU] = make_uint2(pack_bf2(v.x, v.y), pack_bf2(v.z, v.w));
        }
    }
}

// CTA split and shared-memory layout for a chosen sub-tile width m.SB.  TMEM
// holds two filter buffers (2 x 128 columns), two dz accumulators (2 x RP) and
// one dU accumulator per block of the CTA (RP each).  Among the block-group
// sizes that fit, take the one with the fewest items on the busiest SM, then
// the least partial-sum traffic (dU partials of the token ranges, dz
// contributions of the block groups).  Shared memory: operand buffers (up to
// 4 when items are short), dw tiles (2 when items are short and they fit),
// the exchange buffer, and as deep a sub-tile ring as fits.
static bool bwd_layout(TcMap &m, int sms) {
    m.nSubB = m.CB / m.SB;
    const int cpc_max = (512 - 2 * TB_NB - 2 * m.RP) / m.RP;
    if (cpc_max < 1) return false;
    double best_work = -1, best_cost = 0;
    for (int cpc = 1; cpc <= cpc_max && cpc <= m.nBlkB; ++cpc) {
        const int ng = (m.nBlkB + cpc - 1) / cpc;
        int64_t nr = sms / ng;
        if (nr < 1) nr = 1;
        if (nr > m.totalTiles) nr = m.totalTiles;
        const int64_t tpr = (m.totalTiles + nr - 1) / nr;
        const int64_t waves = (ng * nr + sms - 1) / sms;
        const double work = (double)waves * tpr * cpc;  // items on the busiest SM
        const double nz = (double)m.B * m.T * m.R;
        const double cost = (nr > 1 ? 2.0 * nr * m.R * m.GW : 0.0) + (ng > 1 ? (2.0 + 0.25 * ng) * nz : 0.0);
        if (best_work < 0 || work < best_work * 0.97 || (work <= best_work * 1.03 && cost < best_cost)) {
            best_work = work;
            best_cost = cost;
            m.CPC = cpc;
            m.nGroups = ng;
            m.nRanges = (int)nr;
        }
    }
    m.tilesPerRange = (int)((m.totalTiles + m.nRanges - 1) / m.nRanges);
    m.nRanges = (int)((m.totalTiles + m.tilesPerRange - 1) / m.tilesPerRange);
    m.splitUnits = 0;
    if (m.CPC == 1 && m.nSubB >= 8) {
        // long items, one block per CTA: split the (tile, sub-tile) units evenly so
        // that every SM gets the same share even when tiles do not divide evenly
        const int64_t units = m.totalTiles * m.nSubB;
        const int64_t nr = max((int64_t)1, (int64_t)(sms / m.nGroups));
        const int64_t per = (units + nr - 1) / nr;
        if (per < (int64_t)m.tilesPerRange * m.nSubB) {
            m.splitUnits = (int)per;
            m.nRanges = (int)((units + per - 1) / per);
        }
    }
    m.dzAcc = (m.nGroups > 1 || m.splitUnits > 0) ? 1 : 0;
    const int ct = m.SB / 4;  // a thread's channels per sub-tile
    const bool xchg = m.H > ct;
    const bool short_items = m.nSubB < 4;
    // short items: two dw tiles when they fit, else one
    for (m.DWB = short_items ? 2 : 1; m.DWB >= 1; --m.DWB)
        for (int nop = short_items ? TB_MAXOP : 2; nop >= 2; --nop)
            for (m.NSB = TB_MAXNS; m.NSB >= (nop > 2 ? 4 : 2); --m.NSB) {
                m.NOP = nop;
                if (BwdSmem(m, nop, m.NSB, m.DWB, xchg).total <= TB_SMEM) return true;
            }
    return false;
}

// Backward plan: blocks of GB groups, the largest power of two with W*GB <= 128
// whose CB = GB*H channels divide D (GB >= 16: the filter MMAs are GB wide).
bool tc_bwd_plan(TcMap &m, int sms) {
    m.totalTiles = m.B * (int64_t)m.tilesPerSeq;
    for (m.GB = TB_NB; m.GB * m.W > TB_NB;) m.GB /= 2;
    for (; m.GB >= 16; m.GB /= 2) {
        m.NBW = m.GB * m.W;
        m.CB = (int)(m.GB * m.H);
        if (m.D % m.CB) continue;
        m.nBlkB = (int)(m.D / m.CB);
        // sub-tiles of 64 channels (32 for W >= 5, whose wider filters take more
        // registers), or of 32 where the wider ring does not fit (a group never
        // spans two sub-tiles); 16 for blocks of 16 channels (W >= 5, H = 1)
        if (m.CB == 16) {
            m.SB = 16;
            if (m.W >= 5 && m.H == 1 && bwd_layout(m, sms)) return true;
            continue;
        }
        const int sb_max = m.W >= 5 && m.H <= 32 ? 32 : 64;
        for (m.SB = m.CB < sb_max ? m.CB : sb_max; m.SB >= 32 && m.SB >= m.H; m.SB /= 2)
            if (bwd_layout(m, sms)) return true;
    }
    return false;
}

size_t up_bytes(const TcMap &m) { return ((size_t)m.nBlkB * m.RP * TB_NB * 2 + 255) & ~(size_t)255; }
size_t zimg_bytes(const TcMap &m) { return ((size_t)m.totalTiles * (m.RP / 8) * TB_ZR + 255) & ~(size_t)255; }

size_t tc_bwd_ws_bytes(const TcMap &m) {
    size_t n = up_bytes(m) + zimg_bytes(m);
    if (m.nRanges > 1) n += (size_t)m.nRanges * m.R * m.GW * 4;
    if (m.dzAcc) n += (size_t)m.B * m.T * m.R * 4;
    return n;
}

struct BwdMaps {
    CUtensorMap x, dy, dx;
};

bool bwd_maps(const TcArgs &a, BwdMaps &f) {
    const TcMap &m = a.m;
    const int rb = 2 * m.SB;
    const uint64_t xd[3] = {(uint64_t)m.D, (uint64_t)m.T, (uint64_t)m.B};
    const uint64_t xs[2] = {(uint64_t)m.D * 2, (uint64_t)(m.T * m.D * 2)};
    const uint32_t xb[3] = {(uint32_t)(rb / 2), (uint32_t)(TC_M + m.W - 1), 1};
    const uint32_t yb[3] = {(uint32_t)(rb / 2), 32, 1};  // a lane quarter's 32 rows
    const CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    return make_map(&f.x, a.x, 3, xd, xs, xb, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
           make_map(&f.dy, a.dy, 3, xd, xs, xb, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
           make_map(&f.dx, a.dx, 3, xd, xs, yb, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

template <int W, int VPT, int GPT, int PPG>
cudaError_t launch_bwd(const Ctx &c, const TcArgs &a) {
    const BwdSmem S(a.m, a.m.NOP, a.m.NSB, a.m.DWB, PPG > 1);
    static const cudaError_t attr = cudaFuncSetAttribute(k_lr_tc_bwd<W, VPT, GPT, PPG>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, TB_SMEM);
    if (attr != cudaSuccess) return attr;
    if (S.total > TB_SMEM) return cudaErrorInvalidValue;
    BwdMaps f;
    if (!bwd_maps(a, f)) return cudaErrorNotSupported;
    // the whole of TMEM per CTA: enough shared memory that no second CTA shares the SM
    const uint32_t smem = S.total < 120 * 1024 ? 120 * 1024 : S.total;
    const cudaError_t e = launch_pdl(k_lr_tc_bwd<W, VPT, GPT, PPG>, dim3((unsigned)(a.m.nGroups * a.m.nRanges)),
                                     dim3(TB_THREADS), smem, c.stream, f.x, f.dy, f.dx, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Thread channels per sub-tile: CT = 8*VPT (SB = 32 or 64, four parts).
template <int W, int VPT> cudaError_t bwd_by_h(const Ctx &c, const TcArgs &a) {
    constexpr int CT = 8 * VPT;
    if constexpr (W >= 5 && VPT == 2) {  // the plan takes 64-channel sub-tiles for W >= 5 only when H = 64
        if (a.m.H == 64) return launch_bwd<W, VPT, 1, 64 / CT>(c, a);
        return cudaErrorNotSupported;
    }
    switch (a.m.H) {
    case 1: if constexpr (CT * W <= 32) return launch_bwd<W, VPT, CT, 1>(c, a); break;
    case 2: if constexpr (CT / 2 * W <= 32) return launch_bwd<W, VPT, CT / 2, 1>(c, a); break;
    case 4: return launch_bwd<W, VPT, CT / 4, 1>(c, a);
    case 8: return launch_bwd<W, VPT, CT / 8, 1>(c, a);
    case 16: if constexpr (CT >= 16) return launch_bwd<W, VPT, 1, 1>(c, a); else return launch_bwd<W, VPT, 1, 2>(c, a);
    case 32: return launch_bwd<W, VPT, 1, 32 / CT>(c, a);
    case 64: return launch_bwd<W, VPT, 1, 64 / CT>(c, a);
    }
    return cudaErrorNotSupported;
}

template <int W> cudaError_t bwd_by_vpt(const Ctx &c, const TcArgs &a) {
    if (a.m.SB == 16) {  // blocks of 16 single-channel groups (W >= 5, H = 1)
        if constexpr (W >= 5) return launch_bwd<W, 0, 4, 1>(c, a);
        return cudaErrorNotSupported;
    }
    return a.m.SB == 32 ? bwd_by_h<W, 1>(c, a) : bwd_by_h<W, 2>(c, a);
}

}  // namespace
}  // namespace lrtc

bool lowrank_tc_bwd_ok(const dsc_problem &p, int sms) {
    lrtc::TcMap m;
    return lrtc::tc_map(p, m) && lrtc::tc_bwd_plan(m, sms);
}

size_t lr_tc_bwd_ws_bytes(const dsc_problem &p, int sms) {
    lrtc::TcMap m;
    if (!lrtc::tc_map(p, m) || !lrtc::tc_bwd_plan(m, sms)) return 0;
    return lrtc::tc_bwd_ws_bytes(m);
}

cudaError_t launch_lr_bwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                             const void *dy, void *dx, void *dz, float *dU, void *ws, size_t ws_bytes) {
    using namespace lrtc;
    TcArgs a{};
    if (!tc_map(p, a.m) || !tc_bwd_plan(a.m, c.sms)) return cudaErrorNotSupported;
    if (!ws || ws_bytes < tc_bwd_ws_bytes(a.m)) return cudaErrorInvalidValue;
    a.x = static_cast<const bf16 *>(x);
    a.z = static_cast<const bf16 *>(z);
    a.U = static_cast<const bf16 *>(U);
    a.dy = static_cast<const bf16 *>(dy);
    a.dx = static_cast<bf16 *>(dx);
    a.dz = static_cast<bf16 *>(dz);
    a.dU = dU;
    unsigned char *w = static_cast<unsigned char *>(ws);
    a.Up = reinterpret_cast<bf16 *>(w);
    w += up_bytes(a.m);
    a.zimg = reinterpret_cast<bf16 *>(w);
    w += zimg_bytes(a.m);
    if (a.m.nRanges > 1) {
        a.dU_part = reinterpret_cast<float *>(w);
        w += (size_t)a.m.nRanges * a.m.R * a.m.GW * 4;
    }
    const int64_t nprep = (int64_t)a.m.nBlkB * 16 * a.m.RP + a.m.totalTiles * (a.m.RP / 8) * TB_ZROWS;  // chunks
    cudaError_t e = launch_pdl(k_bwd_prep, dim3((unsigned)min((int64_t)2048, (nprep + 255) / 256)), dim3(256), 0,
                               c.stream, a);
    if (e != cudaSuccess) return e;
    if (a.m.dzAcc) {
        a.dz_acc = reinterpret_cast<float *>(w);
        const int64_t n = a.m.B * a.m.T * a.m.R;
        e = launch_pdl(k_tc_zero, dim3((unsigned)min((int64_t)1024, (n / 4 + 255) / 256)), dim3(256), 0, c.stream, a.dz_acc, n);
        if (e != cudaSuccess) return e;
    }
    e = cudaErrorNotSupported;
    switch (a.m.W) {
    case 1: e = bwd_by_vpt<1>(c, a); break;
    case 2: e = bwd_by_vpt<2>(c, a); break;
    case 3: e = bwd_by_vpt<3>(c, a); break;
    case 4: e = bwd_by_vpt<4>(c, a); break;
    case 5: e = bwd_by_vpt<5>(c, a); break;
    case 6: e = bwd_by_vpt<6>(c, a); break;
    case 7: e = bwd_by_vpt<7>(c, a); break;
    case 8: e = bwd_by_vpt<8>(c, a); break;
    }
    if (e != cudaSuccess) return e;
    if (a.m.nRanges > 1 || a.m.dzAcc) {
        const int64_t n = ((a.m.nRanges > 1 ? a.m.R * a.m.GW : 0) + (a.m.dzAcc ? a.m.B * a.m.T * a.m.R : 0)) / 4;
        e = launch_pdl(k_tc_finalize, dim3((unsigned)min((int64_t)2048, (n + 255) / 256)), dim3(256), 0, c.stream, a);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace dsc
