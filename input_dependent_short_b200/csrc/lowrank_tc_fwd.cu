// Tensor-core forward of the low-rank dynamic short convolution (sm_100a).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 and "Efficient training implementation":
//     y[b,t,c] = r x[b,t,c] + sum_k w[b,t,g(c),k] x[b,t-k,c],
//     w[b,t,g,k] = sum_r z[b,t,r] U[r, g*W + k],
// with the filters formed on chip (tcgen05 MMA into tensor memory) and never
// written to HBM.
//
// Item = (tile of 128 tokens, block of CF channels); the block's filters are
// NF = CF/H*W TMEM columns (NF <= 256) formed by one zU MMA.  TMEM holds two
// such buffers (NFS columns apart, NF rounded up to a power of two), so the MMA of item i+1 runs while item i's outputs are formed.
// A CTA takes a contiguous range of (item, sub-tile) pairs, so every CTA gets
// the same number of sub-tiles; an item split between two CTAs has its MMA
// issued by both.  Warp roles (576 threads):
//   warp 16    TMA producer: z tile and U block of each item (two buffers),
//              x sub-tiles of SF channels x (128 + W-1) rows (a ring of NS);
//   warp 17    TMEM owner and MMA issuer;
//   warps 0-15 epilogue: thread part p of token t forms y for VPT 8-channel
//              vectors of each sub-tile from its own TMEM lane.
// Every hand-off is an mbarrier (full / empty pairs); nothing waits on the
// whole block inside the loop.
//
// Operand layouts written by TMA:
//   z tile  (A, K-major):  for R = 16, 32 or 64 one box of 128 rows of 2R
//                          bytes with a 2R-byte swizzle (a few long rows move
//                          faster than many 16-byte ones); otherwise 8-element
//                          boxes, element (t, k) at (k/8)*2048 + t*16 + (k%8)*2
//   U block (B, MN-major): element (k, n) at (n/8)*(RP*16) + k*16 + (n%8)*2
//                          (no swizzle, 8-element boxes)
// x sub-tiles: boxes of 64 channels (128-byte rows, 128-byte swizzle) or of
// 32 channels (64-byte rows, 64-byte swizzle).
#include "lowrank_tc.cuh"

namespace dsc {

// Status word of the forward's bounded waits on each device: 0 = OK,
// otherwise the dsc_status of a wait that gave up.
__device__ int g_dsc_status_tcf = 0;

int take_tc_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status_tcf, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status_tcf, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    const int vb = lrtc::take_tc_bwd_status(stream);
    if (vb < 0) return -1;
    return v ? v : vb;
}

// One thread waits on an mbarrier that nothing arrives at; the bounded wait
// gives up and the time-out is recorded as in the tensor-core kernels.
__global__ void k_wait_selftest(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = tc::smem_u32(&bar);
    tc::mbar_init(a, 1);
    tc::fence_mbar_init();
    if (!tc::mbar_wait(a, 0, limit)) atomicExch(&g_dsc_status_tcf, (int)DSC_ERR_TIMEOUT);
}

cudaError_t launch_wait_selftest(cudaStream_t stream) {
    k_wait_selftest<<<1, 1, 0, stream>>>(10000000ll);
    count_launch();
    return cudaGetLastError();
}

namespace lrtc {

// ------------------------------------------------------------------ common ---

bool tc_map(const dsc_problem &p, TcMap &m) {
    if (p.dtype != DSC_BF16) return false;
    if (p.R < 8 || p.R > 64 || p.R % 8) return false;  // 16-byte z rows
    if (p.W < 1 || p.W > 8) return false;
    if (p.H > 64 || (64 % p.H) != 0) return false;
    if (p.D % (TC_GROUPS * p.H)) return false;
    m = TcMap{};
    m.B = p.B; m.T = p.T; m.D = p.D; m.H = p.H; m.R = p.R; m.W = (int)p.W;
    m.GW = (p.D / p.H) * p.W;
    m.RP = (int)((p.R + 15) / 16) * 16;
    m.tilesPerSeq = (int)((p.T + TC_M - 1) / TC_M);
    m.lgH = 0;
    while ((1 << m.lgH) < m.H) ++m.lgH;
    m.residual = p.residual ? 1 : 0;
    m.zsw = (m.R == 16 || m.R == 32 || m.R == 64) ? (int)(2 * m.R) : 0;  // then R == RP: no padded k-chunks
    return true;
}

// cuTensorMapEncodeTiled, looked up once through the runtime.
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    static EncodeTiled fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiled>(p);
    }();
    return fn;
}

bool make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
              const uint32_t *box, CUtensorMapSwizzle swz, CUtensorMapL2promotion l2) {
    const EncodeTiled fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bd[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bd[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) gs[i] = strides_bytes[i];
    }
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), gd, gs, bd, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// ----------------------------------------------------------------- forward ---

constexpr int TF_EPI = 512;               // epilogue threads
constexpr int TF_THREADS = TF_EPI + 64;   // + producer warp + MMA warp
constexpr int TF_MAXNS = TP_MAXNS;        // most x sub-tiles in flight
constexpr int TF_MAXOP = TP_MAXOP;        // most operand (z, U) buffers
constexpr int TF_SMEM = 220 * 1024;

struct FwdSmem {
    uint32_t zbytes, ubytes, opsize, ring, boxb, slot, ystage, ybox, bars, tmem, total;
    __host__ __device__ FwdSmem(const TcMap &m, int nop, int ns) {
        const int rb = m.SF == 32 ? 64 : 128;
        const int nbx = m.SF == 128 ? 2 : 1;
        boxb = up1024((uint32_t)(rb * (TC_M + m.W - 1)));
        slot = (uint32_t)nbx * boxb;
        ybox = (uint32_t)(rb * TC_M);
        zbytes = (uint32_t)(TC_M * m.RP * 2);
        ubytes = (uint32_t)(m.RP * m.NF * 2);
        opsize = up1024(zbytes + ubytes);
        ystage = (uint32_t)nop * opsize;          // two y staging tiles (TMA store sources)
        ring = ystage + 2 * (uint32_t)nbx * ybox;
        bars = ring + (uint32_t)ns * slot;        // PipeBars
        tmem = bars + PipeBars::BYTES;
        total = tmem + 16 + 1024;                 // + slack to align the base to 1024 bytes
    }
};

// Coordinates of consecutive items (block-major, tile-minor: a CTA keeps one
// U block for many items), advanced without divisions.
struct ItemWalk {
    int blk, t0, b;
    __device__ void init(const TcMap &m, int64_t item) {
        const int64_t ntiles = m.B * (int64_t)m.tilesPerSeq;
        blk = (int)(item / ntiles);
        const int64_t tile = item % ntiles;
        b = (int)(tile / m.tilesPerSeq);
        t0 = (int)(tile % m.tilesPerSeq) * TC_M;
    }
    __device__ void next(const TcMap &m) {
        t0 += TC_M;
        if (t0 >= m.T) {
            t0 = 0;
            if (++b == m.B) {
                b = 0;
                ++blk;
            }
        }
    }
};

// Epilogue of one sub-tile: y for VPT vectors of 8 channels of token t.
// GPV: filter groups inside one vector (8/H for H < 8, else 1).  NGT (only
// for GPV == 1): groups among the thread's 8*VPT channels.  HOFF: the
// thread's shared-memory offsets (x rows xo[v][k], staging row yo[v]) were
// computed once per thread (they do not depend on the item or sub-tile).
constexpr int FWD_HOFF_MAX = 8;  // most hoisted x-row offsets per thread (VPT * W)
template <int W, int GPV, int VPT, int NGT, int RB, bool HOFF>
__device__ __forceinline__ void fwd_subtile(const TcMap &m, const unsigned char *xs, uint32_t boxb, uint32_t tb,
                                            int part, int t_loc, int ci0, unsigned char *ys, uint32_t ybox, float res,
                                            const uint32_t (&xo)[HOFF ? VPT : 1][HOFF ? W : 1],
                                            const uint32_t (&yo)[HOFF ? VPT : 1]) {
    constexpr int WIN = W - 1;
    constexpr int NT = GPV * W;
    constexpr int CPG = 8 / GPV;
    constexpr int VBW = W > 4 ? 1 : (W > 2 ? 2 : 4);
    constexpr int VB = VBW < VPT ? VBW : VPT;  // vectors whose x rows are loaded together
    const int cs0 = part * (8 * VPT);  // sub-tile channel of the thread's first vector
    float wt[GPV == 1 ? NGT * W : 2 * NT];
    if constexpr (GPV == 1) {
        // one TMEM load covers the thread's NGT groups
        tmem_ld<NGT * W>(tb + (uint32_t)((ci0 >> m.lgH) * W), *reinterpret_cast<float(*)[NGT * W]>(wt));
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < NGT * W; k += W) wt[k] += res;
    } else {
        tmem_ld<NT>(tb + (uint32_t)((ci0 >> m.lgH) * W), *reinterpret_cast<float(*)[NT]>(wt));
    }
#pragma unroll
    for (int v0 = 0; v0 < VPT; v0 += VB) {
        uint4 xw[VB][W];
#pragma unroll
        for (int vv = 0; vv < VB; ++vv) {
            const int cs = cs0 + 8 * (v0 + vv);
            const unsigned char *bx = xs + (uint32_t)(cs / (RB / 2)) * boxb;
            const int chunk = (cs % (RB / 2)) / 8;
#pragma unroll
            for (int k = 0; k < W; ++k) {
                if constexpr (HOFF) xw[vv][k] = *reinterpret_cast<const uint4 *>(xs + xo[v0 + vv][k]);
                else xw[vv][k] = *reinterpret_cast<const uint4 *>(bx + tc::swz<RB>(t_loc + WIN - k, chunk));
            }
        }
#pragma unroll
        for (int vv = 0; vv < VB; ++vv) {
            const int v = v0 + vv;
            if constexpr (GPV == 1) {
                const int gi = (v * NGT) / VPT;  // the vector's group among the thread's
                u64 yp[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    u64 acc2 = 0ull;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const uint32_t word = word_of(xw[vv][k], pp);
                        const u64 xp = mk2(bf_lo(word), bf_hi(word));
                        const float wk = wt[gi * W + k];
                        acc2 = k == 0 ? mul2(mk2(wk, wk), xp) : fma2(mk2(wk, wk), xp, acc2);
                    }
                    yp[pp] = acc2;
                }
                const int cs = cs0 + 8 * v;
                *reinterpret_cast<uint4 *>(ys + (HOFF ? yo[v] : (uint32_t)(cs / (RB / 2)) * ybox + tc::swz<RB>(t_loc, (cs % (RB / 2)) / 8))) =
                    make_uint4(pack_bf2(lo2(yp[0]), hi2(yp[0])), pack_bf2(lo2(yp[1]), hi2(yp[1])),
                               pack_bf2(lo2(yp[2]), hi2(yp[2])), pack_bf2(lo2(yp[3]), hi2(yp[3])));
            } else {
                // several groups per vector: per-vector loads, the next one in flight while this one computes.
                // The vector's GPV groups have their filters tap-major (column k*GPV + g, from the
                // permuted U image), so the filters of a channel pair at tap k sit in adjacent
                // registers and one fma.rn.f32x2 applies a tap to both channels.
                tc::tmem_wait_ld();
                float *w = wt + (v & 1) * NT;
                if (v + 1 < VPT)
                    tmem_ld<NT>(tb + (uint32_t)(((ci0 + 8 * (v + 1)) >> m.lgH) * W),
                                *reinterpret_cast<float(*)[NT]>(wt + ((v + 1) & 1) * NT));
                u64 y2[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const int g0 = (2 * pp) / CPG, g1 = (2 * pp + 1) / CPG;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const uint32_t word = word_of(xw[vv][k], pp);
                        const u64 xp = mk2(bf_lo(word), bf_hi(word));
                        u64 wp = mk2(w[k * GPV + g0], w[k * GPV + g1]);
                        if (k == 0) {  // tap 0 carries the residual
                            wp = add2(wp, mk2(res, res));
                            y2[pp] = mul2(wp, xp);
                        } else {
                            y2[pp] = fma2(wp, xp, y2[pp]);
                        }
                    }
                }
                const int cs = cs0 + 8 * v;
                *reinterpret_cast<uint4 *>(ys + (HOFF ? yo[v] : (uint32_t)(cs / (RB / 2)) * ybox + tc::swz<RB>(t_loc, (cs % (RB / 2)) / 8))) =
                    make_uint4(pack_bf2(lo2(y2[0]), hi2(y2[0])), pack_bf2(lo2(y2[1]), hi2(y2[1])),
                               pack_bf2(lo2(y2[2]), hi2(y2[2])), pack_bf2(lo2(y2[3]), hi2(y2[3])));
            }
        }
    }
}

template <int W, int GPV, int VPT, int NGT>
__global__ void __launch_bounds__(TF_THREADS, 1)
    k_lr_tc_fwd(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmz,
                const __grid_constant__ CUtensorMap tmu, const __grid_constant__ CUtensorMap tmy, const TcArgs a) {
    constexpr int WIN = W - 1;
    constexpr int RB = VPT == 1 ? 64 : 128;  // x box row bytes
    constexpr int NBX = VPT == 4 ? 2 : 1;    // x boxes per sub-tile
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const TcMap &m = a.m;
    const int NS = m.NSF, NOP = m.NOPF;
    const FwdSmem S(m, NOP, NS);
    const int64_t total = m.nItemsF * m.nSubF;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t g_lo = (int64_t)blockIdx.x * per;
    const int64_t g_hi = min(total, g_lo + per);
    if (g_lo >= g_hi) return;
    const int64_t i_lo = g_lo / m.nSubF;
    const int nI = (int)((g_hi - 1) / m.nSubF - i_lo + 1);
    const int nG = (int)(g_hi - g_lo);
    const int s_first = (int)(g_lo % m.nSubF);          // first sub-tile of the first item
    const int s_last = (int)((g_hi - 1) % m.nSubF) + 1;  // end of the last item's sub-tiles

    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const PipeBars bars{sbase + S.bars};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) bars.init(NS, TF_EPI / 32, TF_EPI / 32);  // WE, XE: one arrival per epilogue warp
    zero_z_padding(smem, S.opsize, NOP, m, tid, TF_THREADS);
    tc::fence_proxy_async();
    if (warp == 17) tc::tmem_alloc(sbase + S.tmem, (uint32_t)(2 * m.NFS));
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S.tmem);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;  // sticky: later waits skip
    };
    pdl_wait();  // inputs may come from the previous kernel of the stream
    pdl_trigger();

    if (warp == 16) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::tma_prefetch_desc(&tmx);
            tc::tma_prefetch_desc(&tmz);
            tc::tma_prefetch_desc(&tmu);
            ItemWalk it;
            it.init(m, i_lo);
            int slot = 0, l = 0;
            uint32_t xph = 0;
            int ublk[TF_MAXOP];  // U block held by each operand buffer
#pragma unroll
            for (int i = 0; i < TF_MAXOP; ++i) ublk[i] = -1;
            int ob = 0;
            uint32_t oph = 0;
            for (int li = 0; li < nI; ++li, it.next(m)) {
                if (li >= NOP) wait(bars.ope(ob), oph ^ 1u);
                const uint32_t zb = sbase + (uint32_t)ob * S.opsize, ub = zb + S.zbytes;
                int held = -1;
#pragma unroll
                for (int i = 0; i < TF_MAXOP; ++i)
                    if (i == ob) held = ublk[i];
                const bool newu = held != it.blk;
                if (newu) {
#pragma unroll
                    for (int i = 0; i < TF_MAXOP; ++i)
                        if (i == ob) ublk[i] = it.blk;
                }
                load_operands(m, &tmz, &tmu, zb, ub, S.ubytes, it.t0, it.b, it.blk, m.NF, newu, bars.opf(ob));
                if (++ob == NOP) {
                    ob = 0;
                    oph ^= 1u;
                }
                const int se = li == nI - 1 ? s_last : m.nSubF;
                for (int s = li == 0 ? s_first : 0; s < se; ++s, ++l) {
                    if (l >= NS) wait(bars.xe(slot), xph ^ 1u);
                    const uint32_t xb = sbase + S.ring + (uint32_t)slot * S.slot;
                    tc::mbar_expect_tx(bars.xf(slot), (uint32_t)(NBX * RB * (TC_M + WIN)));
                    const int c = it.blk * m.CF + s * m.SF;
#pragma unroll
                    for (int bx = 0; bx < NBX; ++bx)
                        tc::tma_load_3d(xb + (uint32_t)bx * S.boxb, &tmx, c + bx * (RB / 2), it.t0 - WIN, it.b,
                                        bars.xf(slot));
                    if (++slot == NS) {
                        slot = 0;
                        xph ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 17) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) filter_mma_loop(m, bars, sbase, S.opsize, S.zbytes, tmem, m.NF, m.NFS, nI, NOP, wait);
    } else {
        // ------------------------------------------------------------ epilogue
        const int t_loc = tid & (TC_M - 1), part = tid >> 7, quarter = warp & 3;
        // the thread's x-row and staging offsets, the same for every item and sub-tile
        constexpr bool HOFF = VPT * W <= FWD_HOFF_MAX;
        uint32_t xo[HOFF ? VPT : 1][HOFF ? W : 1], yo[HOFF ? VPT : 1];
        if constexpr (HOFF) {
#pragma unroll
            for (int v = 0; v < VPT; ++v) {
                const int cs = part * (8 * VPT) + 8 * v;
                const uint32_t bxo = (uint32_t)(cs / (RB / 2)) * S.boxb;
#pragma unroll
                for (int k = 0; k < W; ++k) xo[v][k] = bxo + tc::swz<RB>(t_loc + WIN - k, (cs % (RB / 2)) / 8);
                yo[v] = (uint32_t)(cs / (RB / 2)) * S.ybox + tc::swz<RB>(t_loc, (cs % (RB / 2)) / 8);
            }
        } else {
            xo[0][0] = 0;
            yo[0] = 0;
        }
        const float res = m.residual ? 1.f : 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        ItemWalk it;
        it.init(m, i_lo);
        int slot = 0, ybuf = 0;
        uint32_t xph = 0;
        for (int li = 0; li < nI; ++li, it.next(m)) {
            const int b = li & 1;
            wait(bars.wf(b), (uint32_t)((li >> 1) & 1));
            tc::fence_after_sync();
            const uint32_t tb = tlane + (uint32_t)(b * m.NFS);
            const int se = li == nI - 1 ? s_last : m.nSubF;
            for (int s = li == 0 ? s_first : 0; s < se; ++s) {
                wait(bars.xf(slot), xph);
                unsigned char *ys = smem + S.ystage + (uint32_t)ybuf * NBX * S.ybox;
                fwd_subtile<W, GPV, VPT, NGT, RB, HOFF>(m, smem + S.ring + (uint32_t)slot * S.slot, S.boxb, tb, part,
                                                        t_loc, s * m.SF + part * (8 * VPT), ys, S.ybox, res, xo, yo);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bars.xe(slot));
                // y tile -> global by TMA: the staging tile the next sub-tile writes was
                // read by the store issued one sub-tile ago, waited for before the barrier
                tc::fence_proxy_async();
                if (tid == 0) tc::bulk_wait_read_all();
                asm volatile("bar.sync 1, %0;" ::"n"(TF_EPI) : "memory");
                if (tid == 0) {
                    const int c = it.blk * m.CF + s * m.SF;
#pragma unroll
                    for (int bx = 0; bx < NBX; ++bx)
                        tc::tma_store_3d(&tmy, sbase + S.ystage + (uint32_t)(ybuf * NBX + bx) * S.ybox, c + bx * (RB / 2),
                                         it.t0, it.b);
                    tc::bulk_commit();
                }
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

    // teardown: every load and MMA this CTA issued has landed before the
    // shared memory and TMEM are given back (bounded, also after a time-out)
    if (warp == 16 && lane == 0) drain_loads(bars, NS, nG);
    if (warp == 17 && lane == 0) drain_mmas(bars, NOP, nI);
    if (timed_out) atomicExch(&g_dsc_status_tcf, (int)DSC_ERR_TIMEOUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 17) tc::tmem_dealloc(tmem, (uint32_t)(2 * m.NFS));
}

// U with the columns of every GPV = 8/H consecutive groups tap-major: column
// c*GPV*W + k*GPV + g of the image holds U column (c*GPV + g)*W + k.  With
// it, the MMA leaves a vector's filters with the taps outermost, so the two
// channels of a pair find tap k in adjacent registers.
// One thread per chunk of GPV*W columns (a row's chunks are contiguous in
// both U and the image, GW being a multiple of GPV*W): the chunk is read whole,
// transposed from group-major to tap-major in registers (GPV and W are
// compile-time, so the chunk stays in registers) and written whole, with
// 16-byte accesses when the chunk is a multiple of 16 bytes.
template <int GPV, int W>
__global__ void k_fwd_uperm(const bf16 *__restrict__ U, bf16 *__restrict__ Uf, int64_t R, int64_t GW) {
    pdl_wait();
    pdl_trigger();
    constexpr int CH = GPV * W;
    constexpr bool VEC = (CH * 2) % 16 == 0;
    const int64_t nck = R * (GW / CH);
    for (int64_t ci = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; ci < nck; ci += (int64_t)gridDim.x * blockDim.x) {
        const bf16 *src = U + ci * CH;
        bf16 *dst = Uf + ci * CH;
        unsigned short in[CH], out[CH];
        if constexpr (VEC) {
#pragma unroll
            for (int v = 0; v < CH / 8; ++v) {
                const uint4 q = ld16(src + 8 * v);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) in[8 * v + e] = (unsigned short)(w4[e / 2] >> (16 * (e & 1)));
            }
        } else {
#pragma unroll
            for (int q = 0; q < CH; ++q) in[q] = __bfloat16_as_ushort(src[q]);
        }
#pragma unroll
        for (int g = 0; g < GPV; ++g)
#pragma unroll
            for (int k = 0; k < W; ++k) out[k * GPV + g] = in[g * W + k];
        if constexpr (VEC) {
#pragma unroll
            for (int v = 0; v < CH / 8; ++v) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) w4[e] = (uint32_t)out[8 * v + 2 * e] | ((uint32_t)out[8 * v + 2 * e + 1] << 16);
                st16(dst + 8 * v, make_uint4(w4[0], w4[1], w4[2], w4[3]));
            }
        } else {
#pragma unroll
            for (int q = 0; q < CH; ++q) dst[q] = __ushort_as_bfloat16(out[q]);
        }
    }
}

template <int GPV>
cudaError_t launch_uperm_w(const Ctx &c, int W, const bf16 *U, bf16 *Uf, int64_t R, int64_t GW) {
    const int64_t n = R * (GW / (GPV * W));  // chunks
    const dim3 grid((unsigned)min((int64_t)1024, (n + 127) / 128));
    switch (W) {
    case 1: return launch_pdl(k_fwd_uperm<GPV, 1>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 2: return launch_pdl(k_fwd_uperm<GPV, 2>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 3: return launch_pdl(k_fwd_uperm<GPV, 3>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 4: return launch_pdl(k_fwd_uperm<GPV, 4>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 5: return launch_pdl(k_fwd_uperm<GPV, 5>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 6: return launch_pdl(k_fwd_uperm<GPV, 6>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 7: return launch_pdl(k_fwd_uperm<GPV, 7>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    case 8: return launch_pdl(k_fwd_uperm<GPV, 8>, grid, dim3(128), 0, c.stream, U, Uf, R, GW);
    }
    return cudaErrorNotSupported;
}

// Forward plan: the widest channel block whose filters fit half of TMEM
// (NF <= 256 columns; a buffer takes NFS = NF rounded up to a power of two),
// narrowed while it still spans 8 or more sub-tiles of 128 channels;
// sub-tiles of up to 64 channels (128-byte rows, one TMA box); as many x
// sub-tiles in flight as shared memory holds (2 .. 8).
bool tc_fwd_plan(TcMap &m) {
    int mm = 1;
    while (TC_GROUPS * 2 * mm * m.W <= 256 && m.D % (TC_GROUPS * m.H * 2 * mm) == 0) mm *= 2;
    while (mm > 1 && (TC_GROUPS * m.H * mm / 2) / 128 >= 8) mm /= 2;
    m.CF = (int)(TC_GROUPS * m.H * mm);
    m.NF = TC_GROUPS * mm * m.W;
    for (m.NFS = 32; m.NFS < m.NF;) m.NFS *= 2;  // TMEM is allocated in powers of two
    m.SF = m.CF < 64 ? m.CF : 64;
    m.nSubF = m.CF / m.SF;
    m.nBlkF = (int)(m.D / m.CF);
    m.nItemsF = m.B * (int64_t)m.tilesPerSeq * m.nBlkF;
    // short items (few sub-tiles each) keep more operand loads in flight
    for (m.NOPF = m.nSubF <= 2 ? TF_MAXOP : 2; m.NOPF >= 2; --m.NOPF)
        for (m.NSF = TF_MAXNS; m.NSF >= (m.NOPF > 2 ? 4 : 2); --m.NSF)
            if (FwdSmem(m, m.NOPF, m.NSF).total <= TF_SMEM) return true;
    return false;
}

struct FwdMaps {
    CUtensorMap x, z, u, y;
};

bool fwd_maps(const TcArgs &a, FwdMaps &f) {
    const TcMap &m = a.m;
    const int rb = m.SF == 32 ? 64 : 128;
    const uint64_t xd[3] = {(uint64_t)m.D, (uint64_t)m.T, (uint64_t)m.B};
    const uint64_t xs[2] = {(uint64_t)m.D * 2, (uint64_t)(m.T * m.D * 2)};
    const uint32_t xb[3] = {(uint32_t)(rb / 2), (uint32_t)(TC_M + m.W - 1), 1};
    const uint32_t yb[3] = {(uint32_t)(rb / 2), (uint32_t)TC_M, 1};
    const uint64_t zd[3] = {(uint64_t)m.R, (uint64_t)m.T, (uint64_t)m.B};
    const uint64_t zs[2] = {(uint64_t)m.R * 2, (uint64_t)(m.T * m.R * 2)};
    const uint32_t zb[3] = {m.zsw ? (uint32_t)m.R : 8u, (uint32_t)TC_M, 1};
    const CUtensorMapSwizzle zsw = m.zsw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : m.zsw == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : m.zsw == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
    const uint64_t ud[2] = {(uint64_t)m.GW, (uint64_t)m.R};
    const uint64_t us[1] = {(uint64_t)m.GW * 2};
    const uint32_t ub[2] = {8, (uint32_t)m.RP};
    const CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return make_map(&f.x, a.x, 3, xd, xs, xb, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
           make_map(&f.y, a.y, 3, xd, xs, yb, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE) &&
           make_map(&f.z, a.z, 3, zd, zs, zb, zsw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) &&
           make_map(&f.u, a.Uf ? a.Uf : a.U, 2, ud, us, ub, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
}

template <int W, int GPV, int VPT, int NGT>
cudaError_t launch_fwd(const Ctx &c, const TcArgs &a) {
    const FwdSmem S(a.m, a.m.NOPF, a.m.NSF);
    static const cudaError_t attr = cudaFuncSetAttribute(k_lr_tc_fwd<W, GPV, VPT, NGT>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, TF_SMEM);
    if (attr != cudaSuccess) return attr;
    if (S.total > TF_SMEM) return cudaErrorInvalidValue;
    FwdMaps f;
    if (!fwd_maps(a, f)) return cudaErrorNotSupported;
    const int64_t total = a.m.nItemsF * a.m.nSubF;
    const int64_t per = (total + c.sms - 1) / c.sms;
    const int64_t grid = (total + per - 1) / per;
    // More than half of TMEM per CTA: enough shared memory that no second CTA shares the SM.
    const uint32_t smem = 2 * a.m.NFS > 256 && S.total < 120 * 1024 ? 120 * 1024 : S.total;
    const cudaError_t e =
        launch_pdl(k_lr_tc_fwd<W, GPV, VPT, NGT>, dim3((unsigned)grid), dim3(TF_THREADS), smem, c.stream, f.x, f.z, f.u, f.y, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// A sub-tile's filters fit one block (4 * VPT * GPV * W <= NF <= 256); other
// combinations never come out of the plan and are not instantiated.
template <int W, int GPV, int VPT> cudaError_t fwd_by_ngt(const Ctx &c, const TcArgs &a) {
    if constexpr (GPV > 1) {
        return launch_fwd<W, GPV, VPT, 1>(c, a);
    } else {
        const int ngt = (8 * VPT) >> a.m.lgH;  // groups among the thread's 8*VPT channels (H >= 8)
        if (ngt <= 1) return launch_fwd<W, 1, VPT, 1>(c, a);
        if constexpr (VPT >= 2)
            if (ngt == 2) return launch_fwd<W, 1, VPT, 2>(c, a);
        if constexpr (VPT == 4)
            if (ngt == 4) return launch_fwd<W, 1, VPT, 4>(c, a);
        return cudaErrorNotSupported;
    }
}

template <int W, int GPV> cudaError_t fwd_by_vpt(const Ctx &c, const TcArgs &a) {
    switch (a.m.SF) {
    case 32: return fwd_by_ngt<W, GPV, 1>(c, a);
    case 64:
        if constexpr (2 * GPV * W <= 64) return fwd_by_ngt<W, GPV, 2>(c, a);
        break;
    }
    return cudaErrorNotSupported;
}

template <int W> cudaError_t fwd_by_gpv(const Ctx &c, const TcArgs &a) {
    switch (a.m.H) {
    case 1: return fwd_by_vpt<W, 8>(c, a);
    case 2: return fwd_by_vpt<W, 4>(c, a);
    case 4: return fwd_by_vpt<W, 2>(c, a);
    default: return fwd_by_vpt<W, 1>(c, a);
    }
}

}  // namespace
}  // namespace lrtc

bool lowrank_tc_ok(const dsc_problem &p) {
    lrtc::TcMap m;
    return lrtc::tc_map(p, m) && lrtc::tc_fwd_plan(m);
}

// Scratch of the tensor-core forward: the permuted U image when several
// groups share a vector (H < 8), else nothing.
size_t lr_tc_fwd_ws_bytes(const dsc_problem &p) {
    if (!lowrank_tc_ok(p) || p.H >= 8) return 0;
    return ((size_t)p.R * (size_t)((p.D / p.H) * p.W) * 2 + 255) & ~(size_t)255;
}

cudaError_t launch_lr_fwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U, void *y,
                             void *ws, size_t ws_bytes) {
    lrtc::TcArgs a{};
    if (!lrtc::tc_map(p, a.m) || !lrtc::tc_fwd_plan(a.m)) return cudaErrorNotSupported;
    a.x = static_cast<const bf16 *>(x);
    a.z = static_cast<const bf16 *>(z);
    a.U = static_cast<const bf16 *>(U);
    a.y = static_cast<bf16 *>(y);
    if (p.H < 8) {
        if (!ws || ws_bytes < lr_tc_fwd_ws_bytes(p)) return cudaErrorInvalidValue;
        a.Uf = static_cast<bf16 *>(ws);
        const int gpv = (int)(8 / p.H);
        const cudaError_t e = gpv == 8   ? lrtc::launch_uperm_w<8>(c, (int)p.W, a.U, a.Uf, p.R, a.m.GW)
                              : gpv == 4 ? lrtc::launch_uperm_w<4>(c, (int)p.W, a.U, a.Uf, p.R, a.m.GW)
                                         : lrtc::launch_uperm_w<2>(c, (int)p.W, a.U, a.Uf, p.R, a.m.GW);
        if (e != cudaSuccess) return e;
    }
    switch (a.m.W) {
    case 1: return lrtc::fwd_by_gpv<1>(c, a);
    case 2: return lrtc::fwd_by_gpv<2>(c, a);
    case 3: return lrtc::fwd_by_gpv<3>(c, a);
    case 4: return lrtc::fwd_by_gpv<4>(c, a);
    case 5: return lrtc::fwd_by_gpv<5>(c, a);
    case 6: return lrtc::fwd_by_gpv<6>(c, a);
    case 7: return lrtc::fwd_by_gpv<7>(c, a);
    case 8: return lrtc::fwd_by_gpv<8>(c, a);
    }
    return cudaErrorNotSupported;
}

}  // namespace dsc
