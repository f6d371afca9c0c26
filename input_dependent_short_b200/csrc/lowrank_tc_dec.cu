// Tensor-core decode step of the low-rank dynamic short convolution (sm_100a).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 (w = z U) and "Efficient training
// implementation" (the filters formed on chip, never written to HBM), applied
// to one new token per sequence: the token's filters w[b,g,k] = z[b,:] .
// U[:, g*W+k] come from one tcgen05 MMA per tile of 128 sequences and block
// of CF channels (TMEM lane = sequence), and the step
//   y[b,c] = r x[b,c] + w_0 x[b,c] + sum_{k>=1} w_k state[b, W-1-k, c]
// reads x and the W-1 state rows of the tile's sequences from shared memory.
// The state box is loaded row-major ([row][sequence][channels]: the tensor
// map lists the state's dimensions as channels, sequence, row), so each row
// of the tile is one contiguous slab, and the new state (rows 1 .. W-2 of
// the old one, then x) leaves by W-1 TMA stores straight from those slabs.
// The ring slot is released once the stores have read it.
//
// This is the training forward's kernel structure (the pipeline of
// lowrank_tc.cuh that lowrank_tc_fwd.cu also runs) with a
// tile of 128 sequences in place of 128 tokens of one sequence: z [B,R] and
// U [R,G*W] arrive by TMA into the MMA's operand layouts (z as one swizzled box when
// R is 16, 32 or 64, as in the forward); per sub-tile of
// SF channels one TMA box brings x [128 sequences x SF] and one the state
// [128 sequences x (W-1) rows x SF] (rows of 64 or 128 bytes, swizzled); y
// leaves through a swizzled staging tile and a TMA store.  Warp roles (576
// threads): warp 16 TMA producer, warp 17 TMEM owner and MMA issuer, warps
// 0-15 epilogue.  Every wait is bounded (about 1 s) and records
// DSC_ERR_TIMEOUT in a status word that dsc_check reads.
#include "lowrank_tc.cuh"

namespace dsc {

__device__ int g_dsc_status_tcd = 0;

int take_tc_dec_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status_tcd, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status_tcd, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

namespace lrtc {
namespace {

constexpr int TD_EPI = 512;
constexpr int TD_THREADS = TD_EPI + 64;
constexpr int TD_MAXNS = TP_MAXNS;
constexpr int TD_MAXOP = TP_MAXOP;
constexpr int TD_SMEM = 220 * 1024;

// Decode plan: the channel blocks of the training forward (CF channels, NF =
// CF/H*W <= 256 filter columns, buffers NFS apart in TMEM), sub-tiles of SF
// channels; a ring slot holds the x box and the state box of a sub-tile.
struct DecPlan {
    int CF, NF, NFS, SF, nSubF, nBlkF, NS, NOP;
    int64_t nItems;
};

struct DecSmem {
    uint32_t zbytes, ubytes, opsize, boxb, slot, ybox, ystage, ring, bars, tmem, total;
    __host__ __device__ DecSmem(const TcMap &m, const DecPlan &d, int nop, int ns) {
        const int rb = d.SF == 32 ? 64 : 128;
        const int nbx = d.SF == 128 ? 2 : 1;
        boxb = up1024((uint32_t)(rb * TC_M * m.W));  // x rows, then the state rows
        slot = (uint32_t)nbx * boxb;
        ybox = (uint32_t)(rb * TC_M);
        zbytes = (uint32_t)(TC_M * m.RP * 2);
        ubytes = (uint32_t)(m.RP * d.NF * 2);
        opsize = up1024(zbytes + ubytes);
        ystage = (uint32_t)nop * opsize;
        ring = ystage + 2 * (uint32_t)nbx * ybox;
        bars = ring + (uint32_t)ns * slot;  // PipeBars
        tmem = bars + PipeBars::BYTES;
        total = tmem + 16 + 1024;
    }
};

struct DecArgsTc {
    TcMap m;
    DecPlan d;
    int64_t B;        // sequences
    const bf16 *x;    // [B, D]
    bf16 *state;      // [B, W-1, D]
};

// Item i = (block i / tiles, tile i % tiles): a CTA keeps one U block for many tiles.
struct DecWalk {
    int blk, t0;
    int64_t tiles;
    __device__ void init(int64_t ntiles, int64_t item) {
        tiles = ntiles;
        blk = (int)(item / ntiles);
        t0 = (int)(item % ntiles) * TC_M;
    }
    __device__ void next() {
        t0 += TC_M;
        if (t0 >= tiles * TC_M) {
            t0 = 0;
            ++blk;
        }
    }
};

// Epilogue of one sub-tile for sequence t_loc (row t_loc of the tile): y for
// VPT vectors of 8 channels (the new state leaves by TMA from the slabs).
template <int W, int GPV, int VPT, int NGT, int RB>
__device__ __forceinline__ void dec_subtile(const TcMap &m, const unsigned char *xs, uint32_t boxb, uint32_t tb,
                                            int part, int t_loc, int ci0, unsigned char *ys, uint32_t ybox, float res) {
    constexpr int S = W - 1;
    constexpr int NT = GPV * W;
    constexpr int CPG = 8 / GPV;
    const int cs0 = part * (8 * VPT);
    float wt[GPV == 1 ? W : NT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int cs = cs0 + 8 * v;
        const unsigned char *bx = xs + (uint32_t)(cs / (RB / 2)) * boxb;
        const int chunk = (cs % (RB / 2)) / 8;
        // slab 0: x; slabs 1 .. S: the state rows j = 0 .. S-1 (x_{t-S+j}); row t_loc of each
        uint4 xw[W];
        const uint32_t so = tc::swz<RB>(t_loc, chunk);
#pragma unroll
        for (int q = 0; q < W; ++q) xw[q] = *reinterpret_cast<const uint4 *>(bx + (uint32_t)q * (RB * TC_M) + so);
        const int ci = ci0 + 8 * v;
        if constexpr (GPV == 1) {  // one group per vector: its W taps, reloaded when the group changes
            if (v == 0 || ((ci >> m.lgH) != ((ci - 8) >> m.lgH))) {
                tmem_ld<W>(tb + (uint32_t)((ci >> m.lgH) * W), *reinterpret_cast<float(*)[W]>(wt));
                tc::tmem_wait_ld();
            }
        } else {
            tmem_ld<NT>(tb + (uint32_t)((ci >> m.lgH) * W), *reinterpret_cast<float(*)[NT]>(wt));
            tc::tmem_wait_ld();
        }
        float y[8];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const int g0 = GPV == 1 ? 0 : (2 * pp) / CPG, g1 = GPV == 1 ? 0 : (2 * pp + 1) / CPG;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int k = 0; k < W; ++k) {
                // tap 0 takes x (row 0); tap k >= 1 takes state row S-k (row 1 + S - k)
                const uint32_t word = word_of(xw[k == 0 ? 0 : 1 + S - k], pp);
                if (k == 0) {  // tap 0 carries the residual
                    a0 = (wt[g0 * W] + res) * bf_lo(word);
                    a1 = (wt[g1 * W] + res) * bf_hi(word);
                } else {
                    a0 = fmaf(wt[g0 * W + k], bf_lo(word), a0);
                    a1 = fmaf(wt[g1 * W + k], bf_hi(word), a1);
                }
            }
            y[2 * pp] = a0;
            y[2 * pp + 1] = a1;
        }
        *reinterpret_cast<uint4 *>(ys + (uint32_t)(cs / (RB / 2)) * ybox + tc::swz<RB>(t_loc, (cs % (RB / 2)) / 8)) =
            make_uint4(pack_bf2(y[0], y[1]), pack_bf2(y[2], y[3]), pack_bf2(y[4], y[5]), pack_bf2(y[6], y[7]));
    }
}

template <int W, int GPV, int VPT, int NGT>
__global__ void __launch_bounds__(TD_THREADS, 1)
    k_lr_tc_dec(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tms,
                const __grid_constant__ CUtensorMap tmz, const __grid_constant__ CUtensorMap tmu,
                const __grid_constant__ CUtensorMap tmy, const __grid_constant__ CUtensorMap tmsr, const DecArgsTc a) {
    constexpr int S = W - 1;
    constexpr int RB = VPT == 1 ? 64 : 128;
    constexpr int NBX = VPT == 4 ? 2 : 1;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const TcMap &m = a.m;
    const DecPlan &d = a.d;
    const int NS = d.NS, NOP = d.NOP;
    const DecSmem Sm(m, d, NOP, NS);
    const int64_t total = d.nItems * d.nSubF;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t g_lo = (int64_t)blockIdx.x * per;
    const int64_t g_hi = min(total, g_lo + per);
    if (g_lo >= g_hi) return;
    const int64_t i_lo = g_lo / d.nSubF;
    const int nI = (int)((g_hi - 1) / d.nSubF - i_lo + 1);
    const int nG = (int)(g_hi - g_lo);
    const int s_first = (int)(g_lo % d.nSubF);
    const int s_last = (int)((g_hi - 1) % d.nSubF) + 1;
    const int64_t ntiles = m.tilesPerSeq;

    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const PipeBars bars{sbase + Sm.bars};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // WE: one arrival per epilogue warp; XE: thread 0, once the slot's state stores have read it
    if (tid == 0) bars.init(NS, TD_EPI / 32, 1);
    zero_z_padding(smem, Sm.opsize, NOP, m, tid, TD_THREADS);
    tc::fence_proxy_async();
    if (warp == 17) tc::tmem_alloc(sbase + Sm.tmem, (uint32_t)(2 * d.NFS));
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Sm.tmem);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;
    };

    if (warp == 16) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch_desc(&tmx);
            if constexpr (S > 0) tc::tma_prefetch_desc(&tms);
            if constexpr (S > 0) tc::tma_prefetch_desc(&tmsr);
            tc::tma_prefetch_desc(&tmz);
            tc::tma_prefetch_desc(&tmu);
            DecWalk it;
            it.init(ntiles, i_lo);
            int slot = 0, l = 0, ob = 0;
            uint32_t xph = 0, oph = 0;
            int ublk[TD_MAXOP];
#pragma unroll
            for (int i = 0; i < TD_MAXOP; ++i) ublk[i] = -1;
            for (int li = 0; li < nI; ++li, it.next()) {
                if (li >= NOP) wait(bars.ope(ob), oph ^ 1u);
                const uint32_t zb = sbase + (uint32_t)ob * Sm.opsize, ub = zb + Sm.zbytes;
                int held = -1;
#pragma unroll
                for (int i = 0; i < TD_MAXOP; ++i)
                    if (i == ob) held = ublk[i];
                const bool newu = held != it.blk;
                if (newu) {
#pragma unroll
                    for (int i = 0; i < TD_MAXOP; ++i)
                        if (i == ob) ublk[i] = it.blk;
                }
                load_operands(m, &tmz, &tmu, zb, ub, Sm.ubytes, it.t0, 0, it.blk, d.NF, newu, bars.opf(ob));
                if (++ob == NOP) {
                    ob = 0;
                    oph ^= 1u;
                }
                const int se = li == nI - 1 ? s_last : d.nSubF;
                for (int s = li == 0 ? s_first : 0; s < se; ++s, ++l) {
                    if (l >= NS) wait(bars.xe(slot), xph ^ 1u);
                    const uint32_t xb = sbase + Sm.ring + (uint32_t)slot * Sm.slot;
                    tc::mbar_expect_tx(bars.xf(slot), (uint32_t)(NBX * RB * TC_M * W));
                    const int c = it.blk * d.CF + s * d.SF;
#pragma unroll
                    for (int bx = 0; bx < NBX; ++bx) {
                        tc::tma_load_3d(xb + (uint32_t)bx * Sm.boxb, &tmx, c + bx * (RB / 2), it.t0, 0, bars.xf(slot));
                        if constexpr (S > 0)
                            tc::tma_load_3d(xb + (uint32_t)bx * Sm.boxb + RB * TC_M, &tms, c + bx * (RB / 2), it.t0, 0,
                                            bars.xf(slot));
                    }
                    if (++slot == NS) {
                        slot = 0;
                        xph ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 17) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) filter_mma_loop(m, bars, sbase, Sm.opsize, Sm.zbytes, tmem, d.NF, d.NFS, nI, NOP, wait);
    } else {
        // ------------------------------------------------------------ epilogue
        const int t_loc = tid & (TC_M - 1), part = tid >> 7, quarter = warp & 3;
        const float res = m.residual ? 1.f : 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        DecWalk it;
        it.init(ntiles, i_lo);
        int slot = 0, ybuf = 0, pslot = -1;
        uint32_t xph = 0;
        for (int li = 0; li < nI; ++li, it.next()) {
            const int b = li & 1;
            wait(bars.wf(b), (uint32_t)((li >> 1) & 1));
            tc::fence_after_sync();
            const uint32_t tb = tlane + (uint32_t)(b * d.NFS);
            const int se = li == nI - 1 ? s_last : d.nSubF;
            for (int s = li == 0 ? s_first : 0; s < se; ++s) {
                wait(bars.xf(slot), xph);
                unsigned char *ys = smem + Sm.ystage + (uint32_t)ybuf * NBX * Sm.ybox;
                dec_subtile<W, GPV, VPT, NGT, RB>(m, smem + Sm.ring + (uint32_t)slot * Sm.slot, Sm.boxb, tb, part,
                                                  t_loc, s * d.SF + part * (8 * VPT), ys, Sm.ybox, res);
                tc::fence_proxy_async();
                if (tid == 0) {
                    // the previous sub-tile's stores (y staging tile, state slabs) have read
                    // shared memory: its ring slot goes back to the producer
                    tc::bulk_wait_read_all();
                    if (pslot >= 0) tc::mbar_arrive(bars.xe(pslot));
                }
                asm volatile("bar.sync 1, %0;" ::"n"(TD_EPI) : "memory");
                if (tid == 0) {
                    const int c = it.blk * d.CF + s * d.SF;
                    const uint32_t xb = sbase + Sm.ring + (uint32_t)slot * Sm.slot;
#pragma unroll
                    for (int bx = 0; bx < NBX; ++bx) {
                        tc::tma_store_3d(&tmy, sbase + Sm.ystage + (uint32_t)(ybuf * NBX + bx) * Sm.ybox,
                                         c + bx * (RB / 2), it.t0, 0);
                        // new state row j: old row j+1 (slab j+2) for j < S-1, x (slab 0) for j = S-1;
                        // rows of sequences past B are clipped by the store
#pragma unroll
                        for (int jr = 0; jr < S; ++jr)
                            tc::tma_store_3d(&tmsr, xb + (uint32_t)bx * Sm.boxb + (uint32_t)(jr + 1 < S ? jr + 2 : 0) * (RB * TC_M),
                                             c + bx * (RB / 2), it.t0, jr);
                    }
                    tc::bulk_commit();
                }
                pslot = slot;
                ybuf ^= 1;
                if (++slot == NS) {
                    slot = 0;
                    xph ^= 1u;
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bars.we(b));
        }
        if (tid == 0) tc::bulk_wait_all();
    }

    // teardown (bounded): the loads and MMAs issued have landed before the
    // shared memory and TMEM are given back
    if (warp == 16 && lane == 0) drain_loads(bars, NS, nG);
    if (warp == 17 && lane == 0) drain_mmas(bars, NOP, nI);
    if (timed_out) atomicExch(&g_dsc_status_tcd, (int)DSC_ERR_TIMEOUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 17) tc::tmem_dealloc(tmem, (uint32_t)(2 * d.NFS));
}

bool dec_plan(const TcMap &m, DecPlan &d) {
    int mm = 1;
    while (TC_GROUPS * 2 * mm * m.W <= 256 && m.D % (TC_GROUPS * m.H * 2 * mm) == 0) mm *= 2;
    while (mm > 1 && (TC_GROUPS * m.H * mm / 2) / 128 >= 8) mm /= 2;
    d.CF = (int)(TC_GROUPS * m.H * mm);
    d.NF = TC_GROUPS * mm * m.W;
    for (d.NFS = 32; d.NFS < d.NF;) d.NFS *= 2;
    d.SF = d.CF < 64 ? d.CF : 64;
    d.nSubF = d.CF / d.SF;
    d.nBlkF = (int)(m.D / d.CF);
    d.nItems = (int64_t)m.tilesPerSeq * d.nBlkF;
    for (d.NOP = d.nSubF <= 2 ? TD_MAXOP : 2; d.NOP >= 2; --d.NOP)
        for (d.NS = TD_MAXNS; d.NS >= 2; --d.NS)
            if (DecSmem(m, d, d.NOP, d.NS).total <= TD_SMEM) return true;
    return false;
}

// The problem as the tensor-core map sees it: one "sequence" whose tokens are
// the B sequences (z [B,R] is z [1,B,R]).
bool dec_map(const dsc_problem &p, TcMap &m, DecPlan &d) {
    dsc_problem q = p;
    q.B = 1;
    q.T = p.B;
    return tc_map(q, m) && dec_plan(m, d);
}

struct DecMaps {
    CUtensorMap x, s, z, u, y, sr;  // sr: one state row of a tile, for the stores
};

bool dec_maps(const DecArgsTc &a, const void *z, const void *U, void *y, DecMaps &f) {
    const TcMap &m = a.m;
    const int rb = a.d.SF == 32 ? 64 : 128;
    const CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const uint64_t xd[3] = {(uint64_t)m.D, (uint64_t)a.B, 1};
    const uint64_t xs[2] = {(uint64_t)m.D * 2, (uint64_t)(a.B * m.D * 2)};
    const uint32_t xbx[3] = {(uint32_t)(rb / 2), (uint32_t)TC_M, 1};
    const uint64_t zd[3] = {(uint64_t)m.R, (uint64_t)a.B, 1};
    const uint64_t zs[2] = {(uint64_t)m.R * 2, (uint64_t)(a.B * m.R * 2)};
    const uint32_t zb[3] = {m.zsw ? (uint32_t)m.R : 8u, (uint32_t)TC_M, 1};
    const CUtensorMapSwizzle zsw = m.zsw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : m.zsw == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : m.zsw == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
    const uint64_t ud[2] = {(uint64_t)m.GW, (uint64_t)m.R};
    const uint64_t us[1] = {(uint64_t)m.GW * 2};
    const uint32_t ub[2] = {8, (uint32_t)m.RP};
    bool ok = make_map(&f.x, a.x, 3, xd, xs, xbx, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
              make_map(&f.y, y, 3, xd, xs, xbx, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE) &&
              make_map(&f.z, z, 3, zd, zs, zb, zsw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) &&
              make_map(&f.u, U, 2, ud, us, ub, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
    if (!ok) return false;
    f.s = f.x;  // unused for W = 1
    f.sr = f.x;
    if (m.W > 1) {
        // the state [B][W-1][D] seen as channels, sequence, row (strides out of order), so that a
        // box lands row-major: one [128 sequences x SF] slab per row
        const uint64_t sd[3] = {(uint64_t)m.D, (uint64_t)a.B, (uint64_t)(m.W - 1)};
        const uint64_t ss[2] = {(uint64_t)((m.W - 1) * m.D * 2), (uint64_t)m.D * 2};
        const uint32_t sb[3] = {(uint32_t)(rb / 2), (uint32_t)TC_M, (uint32_t)(m.W - 1)};
        const uint32_t sb1[3] = {(uint32_t)(rb / 2), (uint32_t)TC_M, 1};
        ok = make_map(&f.s, a.state, 3, sd, ss, sb, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
             make_map(&f.sr, a.state, 3, sd, ss, sb1, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE);
    }
    return ok;
}

template <int W, int GPV, int VPT, int NGT>
cudaError_t launch_dec(const Ctx &c, const DecArgsTc &a, const DecMaps &f) {
    const DecSmem S(a.m, a.d, a.d.NOP, a.d.NS);
    static const cudaError_t attr =
        cudaFuncSetAttribute(k_lr_tc_dec<W, GPV, VPT, NGT>, cudaFuncAttributeMaxDynamicSharedMemorySize, TD_SMEM);
    if (attr != cudaSuccess) return attr;
    if (S.total > TD_SMEM) return cudaErrorInvalidValue;
    const int64_t total = a.d.nItems * a.d.nSubF;
    const int64_t per = (total + c.sms - 1) / c.sms;
    const int64_t grid = (total + per - 1) / per;
    const uint32_t smem = 2 * a.d.NFS > 256 && S.total < 120 * 1024 ? 120 * 1024 : S.total;
    k_lr_tc_dec<W, GPV, VPT, NGT><<<(unsigned)grid, TD_THREADS, smem, c.stream>>>(f.x, f.s, f.z, f.u, f.y, f.sr, a);
    count_launch();
    return cudaGetLastError();
}

template <int W, int GPV, int VPT> cudaError_t dec_by_ngt(const Ctx &c, const DecArgsTc &a, const DecMaps &f) {
    if constexpr (GPV > 1) {
        return launch_dec<W, GPV, VPT, 1>(c, a, f);
    } else {
        const int ngt = (8 * VPT) >> a.m.lgH;
        if (ngt <= 1) return launch_dec<W, 1, VPT, 1>(c, a, f);
        if constexpr (VPT >= 2)
            if (ngt == 2) return launch_dec<W, 1, VPT, 2>(c, a, f);
        return cudaErrorNotSupported;
    }
}

template <int W, int GPV> cudaError_t dec_by_vpt(const Ctx &c, const DecArgsTc &a, const DecMaps &f) {
    switch (a.d.SF) {
    case 32: return dec_by_ngt<W, GPV, 1>(c, a, f);
    case 64:
        if constexpr (GPV * W <= 32) return dec_by_ngt<W, GPV, 2>(c, a, f);
        break;
    }
    return cudaErrorNotSupported;
}

template <int W> cudaError_t dec_by_gpv(const Ctx &c, const DecArgsTc &a, const DecMaps &f) {
    switch (a.m.H) {
    case 1: return dec_by_vpt<W, 8>(c, a, f);
    case 2: return dec_by_vpt<W, 4>(c, a, f);
    case 4: return dec_by_vpt<W, 2>(c, a, f);
    default: return dec_by_vpt<W, 1>(c, a, f);
    }
}

}  // namespace
}  // namespace lrtc

bool decode_lowrank_tc_ok(const dsc_problem &p) {
    if (p.dtype != DSC_BF16) return false;
    lrtc::TcMap m;
    lrtc::DecPlan d;
    if (!lrtc::dec_map(p, m, d)) return false;
    // instances: SF = 64 needs GPV*W <= 32 (per-vector filters in registers)
    const int gpv = p.H == 1 ? 8 : (p.H == 2 ? 4 : (p.H == 4 ? 2 : 1));
    return d.SF == 32 || gpv * p.W <= 32;
}

cudaError_t launch_decode_lowrank_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                                     void *state, void *y) {
    lrtc::DecArgsTc a{};
    if (!decode_lowrank_tc_ok(p) || !lrtc::dec_map(p, a.m, a.d)) return cudaErrorNotSupported;
    a.B = p.B;
    a.x = static_cast<const bf16 *>(x);
    a.state = static_cast<bf16 *>(state);
    lrtc::DecMaps f;
    if (!lrtc::dec_maps(a, z, U, y, f)) return cudaErrorNotSupported;
    switch (p.W) {
    case 1: return lrtc::dec_by_gpv<1>(c, a, f);
    case 2: return lrtc::dec_by_gpv<2>(c, a, f);
    case 3: return lrtc::dec_by_gpv<3>(c, a, f);
    case 4: return lrtc::dec_by_gpv<4>(c, a, f);
    case 5: return lrtc::dec_by_gpv<5>(c, a, f);
    case 6: return lrtc::dec_by_gpv<6>(c, a, f);
    case 7: return lrtc::dec_by_gpv<7>(c, a, f);
    case 8: return lrtc::dec_by_gpv<8>(c, a, f);
    }
    return cudaErrorNotSupported;
}

}  // namespace dsc
