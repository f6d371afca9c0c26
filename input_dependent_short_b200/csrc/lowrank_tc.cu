// Fused low-rank dynamic short convolution on the tensor cores (sm_100a).
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1 (rank-R factorisation of the filter
// generator) and "Efficient training implementation" (the fused low-rank
// kernel forms zU on chip and convolves at once; the filter tensor never
// reaches HBM).  Filters: w[b,t,g,k] = sum_r z[b,t,r] U[r, g*W + k].
//
// Work item = (tile of 128 tokens of one sequence, chunk of 32 filter groups,
// i.e. NB = 32*W columns of U and 32*H channels).  Per item:
//   1. the z tile [128 x R] and the U chunk [R x NB] go to shared memory in the
//      core-matrix layout of tc.cuh (bf16; R padded with zeros to a multiple
//      of 16);
//   2. one thread issues the tcgen05 MMAs  w[128 x NB] = z . U_chunk  into
//      tensor memory, so TMEM lane t holds the filters of token t;
//   3. the chunk's channels stream through shared memory in sub-tiles of SC
//      channels x (128 + W - 1) rows (cp.async, double-buffered), and thread t
//      forms y for token t from its own TMEM row and the x rows t-W+1 .. t.
// 256 threads: thread t (< 128) and t + 128 share token t and split each
// sub-tile's channels in halves.  Persistent CTAs walk the work items.
//
// Used for bf16 with R <= 64, W in {1, 2, 4, 8}, H in {1, 2, ..., 64} and D a
// multiple of 32*H; the CUDA-core kernels cover every other shape.
#include "kernels.cuh"
#include "tc.cuh"

namespace dsc {

namespace {

constexpr int TC_THREADS = 256;
constexpr int TC_M = 128;          // tokens per tile (TMEM lanes)
constexpr int TC_GROUPS = 32;      // filter groups per chunk
constexpr long long TC_WAIT_LIMIT = 2000000000ll;  // ~1 s of clock cycles

}  // namespace

// Status word of this file's bounded waits on each device: 0 = OK, otherwise
// the dsc_status of a wait that gave up.
__device__ int g_dsc_status_tc = 0;

int take_tc_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status_tc, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status_tc, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

namespace {

struct TcMap {
    int64_t B, T, D, H, R, GW;
    int W, RP;          // RP: R padded to a multiple of 16
    int NB;             // columns per chunk (32*W)
    int CH;             // channels per chunk (32*H)
    int SC;             // channels per sub-tile
    int nSub;           // sub-tiles per chunk
    int nChunks, tilesPerSeq;
    int64_t nItems;
    int residual;
    // backward plan: CTA = (range of token tiles) x (group of CPC chunks)
    int CPC, nGroups, nRanges, tilesPerRange, MH, tcols;
    int64_t totalTiles;
};

struct TcArgs {
    TcMap m;
    const bf16 *x, *z, *U, *dy;
    bf16 *y, *dx, *dz;
    float *dU, *dz_acc, *dU_part;
};

// 32 lanes x N consecutive fp32 TMEM columns (N in 1..32, power of two).
template <int N> __device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]) {
    uint32_t r[N];
    if constexpr (N == 1) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
    } else if constexpr (N == 2) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
    } else if constexpr (N == 4) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(taddr));
    } else {
        static_assert(N % 8 == 0, "TMEM loads of 8 columns at a time");
#pragma unroll
        for (int i = 0; i < N / 8; ++i)
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(r[8 * i]), "=r"(r[8 * i + 1]), "=r"(r[8 * i + 2]), "=r"(r[8 * i + 3]),
                           "=r"(r[8 * i + 4]), "=r"(r[8 * i + 5]), "=r"(r[8 * i + 6]), "=r"(r[8 * i + 7])
                         : "r"(taddr + 8 * i));
    }
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint4 lds16(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

// Shared-memory plan of the forward kernel (bytes).
struct FwdSmem {
    uint32_t z, u, xs, bar, tmem, total;
    __host__ __device__ FwdSmem(const TcMap &m) {
        const uint32_t row = (uint32_t)(m.SC * 2 + 16);         // padded x row
        const uint32_t xtile = row * (uint32_t)(TC_M + m.W - 1);  // one sub-tile
        z = 0;
        u = z + (uint32_t)(TC_M * m.RP * 2);
        xs = u + (uint32_t)(m.RP * m.NB * 2);
        xs = (xs + 127u) & ~127u;
        bar = xs + 2 * xtile;
        bar = (bar + 15u) & ~15u;
        tmem = bar + 16;
        total = tmem + 16;
    }
};

// Copy one x sub-tile (rows t0-W+1 .. t0+127, SC channels from c_first) with
// zero fill outside the sequence.
__device__ __forceinline__ void load_rows(const TcMap &m, const bf16 *src, int64_t row0, int t_first, int nrows,
                                          int64_t c_first, uint32_t dst, uint32_t rowbytes) {
    const int pieces = m.SC / 8;  // 16-byte pieces per row
    for (int i = threadIdx.x; i < nrows * pieces; i += TC_THREADS) {
        const int r = i / pieces, pc = i % pieces;
        const int t = t_first + r;
        const bool valid = t >= 0 && t < m.T;
        const bf16 *p = src + (row0 + (valid ? t : 0)) * m.D + c_first + pc * 8;
        cp16_zfill(dst + (uint32_t)r * rowbytes + (uint32_t)pc * 16, p, valid);
    }
}

template <int W, int GPV>
__global__ void __launch_bounds__(TC_THREADS, 1) k_lr_tc_fwd(const TcArgs a) {
    constexpr int WIN = W - 1;
    constexpr int NT = GPV * W;  // filter taps per 8-channel vector
    extern __shared__ __align__(1024) unsigned char smem[];
    const TcMap &m = a.m;
    const FwdSmem S(m);
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t bar = sbase + S.bar;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int t_loc = tid & (TC_M - 1), half = tid >> 7, quarter = warp & 3;
    const uint32_t rowbytes = (uint32_t)(m.SC * 2 + 16);
    const uint32_t xtile = rowbytes * (uint32_t)(TC_M + WIN);

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    const uint32_t ncols = (uint32_t)m.NB;  // a power of two >= 32
    if (warp == 0) tc::tmem_alloc(sbase + S.tmem, ncols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S.tmem);
    const uint32_t tmem_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const float res = m.residual ? 1.f : 0.f;
    const uint32_t idesc = tc::idesc_bf16(TC_M, m.NB, 0, 1);
    uint32_t phase = 0;
    bool timed_out = false;

    for (int64_t item = blockIdx.x; item < m.nItems; item += gridDim.x) {
        const int chunk = (int)(item % m.nChunks);
        const int64_t tile = item / m.nChunks;
        const int64_t b = tile / m.tilesPerSeq;
        const int t0 = (int)(tile % m.tilesPerSeq) * TC_M;
        const int64_t row0 = b * m.T;
        const int64_t c_chunk = (int64_t)chunk * m.CH;
        const int64_t col0 = (int64_t)chunk * m.NB;

        // z tile and U chunk -> core-matrix layout (bf16, zero padding)
        for (int i = tid; i < TC_M * m.RP; i += TC_THREADS) {
            const int p = i / m.RP, r = i % m.RP;
            const int t = t0 + p;
            bf16 v = __float2bfloat16_rn(0.f);
            if (r < m.R && t < m.T) v = a.z[(row0 + t) * m.R + r];
            *reinterpret_cast<bf16 *>(smem + S.z + tc::core_off(p, r, m.RP)) = v;
        }
        for (int i = tid; i < m.RP * m.NB; i += TC_THREADS) {
            const int r = i / m.NB, j = i % m.NB;
            bf16 v = __float2bfloat16_rn(0.f);
            if (r < m.R) v = a.U[(int64_t)r * m.GW + col0 + j];
            *reinterpret_cast<bf16 *>(smem + S.u + tc::core_off(r, j, m.NB)) = v;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        if (tid == 0) {
            for (int ks = 0; ks < m.RP / 16; ++ks) {
                const uint64_t ad = tc::smem_desc(sbase + S.z + ks * 256, 128, (uint32_t)(m.RP / 8) * 128);
                const uint64_t bd = tc::smem_desc(sbase + S.u + ks * 2 * (m.NB / 8) * 128, (uint32_t)(m.NB / 8) * 128, 128);
                tc::mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
            tc::mma_commit(bar);
        }
        // first x sub-tile while the MMA runs
        load_rows(m, a.x, row0, t0 - WIN, TC_M + WIN, c_chunk, sbase + S.xs, rowbytes);
        cp_commit();
        if (!tc::mbar_wait(bar, phase, TC_WAIT_LIMIT)) timed_out = true;
        phase ^= 1;
        tc::fence_after_sync();

        for (int s = 0; s < m.nSub; ++s) {
            if (s + 1 < m.nSub)
                load_rows(m, a.x, row0, t0 - WIN, TC_M + WIN, c_chunk + (int64_t)(s + 1) * m.SC,
                          sbase + S.xs + (uint32_t)((s + 1) & 1) * xtile, rowbytes);
            cp_commit();
            cp_wait<1>();
            __syncthreads();
            const uint32_t xb = sbase + S.xs + (uint32_t)(s & 1) * xtile;
            const int t = t0 + t_loc;
            const int nvec = m.SC / 16;  // vectors per half
            for (int v = 0; v < nvec; ++v) {
                const int cl = s * m.SC + half * (m.SC / 2) + 8 * v;  // channel within the chunk
                const int gl = cl / (int)m.H;                          // first group of the vector
                float wt[NT];
                tmem_ld<NT>(tmem_lane + (uint32_t)(gl * W), wt);
                tc::tmem_wait_ld();
                float xr[W][8];
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const uint4 u = lds16(xb + (uint32_t)(t_loc + WIN - k) * rowbytes + (uint32_t)(half * (m.SC / 2) + 8 * v) * 2);
                    unpack(u, xr[k]);
                }
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int f = (j / (8 / GPV)) * W;
                    float sacc = (wt[f] + res) * xr[0][j];
#pragma unroll
                    for (int k = 1; k < W; ++k) sacc = fmaf(wt[f + k], xr[k][j], sacc);
                    acc[j] = sacc;
                }
                if (t < m.T) st16(a.y + (row0 + t) * m.D + c_chunk + cl, pack(acc));
            }
            __syncthreads();  // sub-tile buffer free for the load two steps ahead
        }
        tc::fence_before_sync();
        __syncthreads();  // TMEM and the z/U tiles free for the next item
        tc::fence_after_sync();
    }
    cp_wait<0>();
    if (timed_out && (tid & 31) == 0) atomicExch(&g_dsc_status_tc, (int)DSC_ERR_TIMEOUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, ncols);
}


// ------------------------------------------------------------------ backward ---
//
// CTA = (a contiguous range of token tiles) x (a group of CPC chunks).  Per
// (tile, chunk):
//   zU MMA -> w in TMEM (lane = token); the W-1 filter rows of the next tile's
//   first tokens are formed on CUDA cores, and the first W-1 rows of each
//   32-lane quarter are copied to shared memory, so that token t can read
//   w(t+k)_k for dx: from lane t+k by shuffle, or from those rows;
//   x and dy stream in sub-tiles of 32 channels (cp.async, double-buffered);
//   thread t forms dx for token t and the dw values of its groups, written as
//   bf16 into a core-matrix tile [128 tokens x NB];
//   dz += dw . U^T   (MMA, TMEM, accumulated over the CTA's chunks of the tile),
//   dU += dw^T . z   (MMA, TMEM, one accumulator per chunk, over the range).
// dz is written after the tile's last chunk (directly, or added into an fp32
// accumulator when several chunk groups exist); dU after the range (directly
// or as a per-range partial).

constexpr int TC_SC = 32;  // channels per backward sub-tile

struct BwdSmem {
    uint32_t z, u, zh, edge, ring, dw, xch, bar, tmem, total, rowbytes, tile;
    __host__ __device__ BwdSmem(const TcMap &m) {
        const int WIN = m.W - 1;
        rowbytes = (uint32_t)(TC_SC * 2 + 16);
        tile = rowbytes * (uint32_t)(TC_M + WIN);
        z = 0;
        u = z + (uint32_t)(TC_M * m.RP * 2);
        zh = u + (uint32_t)(m.RP * m.NB * 2);
        edge = (zh + (uint32_t)(8 * m.RP * 2) + 15u) & ~15u;
        ring = (edge + (uint32_t)(4 * 8 * m.NB * 4) + 127u) & ~127u;
        dw = ring + 4 * tile;  // 2 stages x (x tile, dy tile)
        xch = dw + (uint32_t)(TC_M * m.NB * 2);
        bar = (xch + (uint32_t)(TC_M * 8 * 4) + 15u) & ~15u;
        tmem = bar + 16;
        total = tmem + 16;
    }
};

// x rows t0-WIN .. t0+127 and dy rows t0 .. t0+127+WIN of one 32-channel
// sub-tile, zero outside the sequence.
__device__ __forceinline__ void load_sub_bwd(const TcMap &m, const TcArgs &a, int64_t row0, int t0, int64_t c_first,
                                             uint32_t xdst, uint32_t dydst, uint32_t rowbytes) {
    const int WIN = m.W - 1;
    const int nrows = TC_M + WIN;
    for (int i = threadIdx.x; i < 2 * nrows * (TC_SC / 8); i += TC_THREADS) {
        const int which = i / (nrows * (TC_SC / 8));
        const int j = i % (nrows * (TC_SC / 8));
        const int r = j / (TC_SC / 8), pc = j % (TC_SC / 8);
        const int t = which == 0 ? t0 - WIN + r : t0 + r;
        const bool valid = t >= 0 && t < m.T;
        const bf16 *src = (which == 0 ? a.x : a.dy) + (row0 + (valid ? t : 0)) * m.D + c_first + pc * 8;
        cp16_zfill((which == 0 ? xdst : dydst) + (uint32_t)r * rowbytes + (uint32_t)pc * 16, src, valid);
    }
}

// z tile [128 x RP] and U chunk [RP x NB] in the core-matrix layout, plus the
// WIN z rows after the tile (row-major, for the halo filters).
__device__ __forceinline__ void load_item_bwd(const TcMap &m, const TcArgs &a, int64_t row0, int t0, int64_t col0,
                                              uint32_t zdst, uint32_t udst, uint32_t zhdst) {
    const int WIN = m.W - 1;
    const int zp = m.RP / 8, up = m.NB / 8;
    for (int i = threadIdx.x; i < TC_M * zp; i += TC_THREADS) {
        const int p = i / zp, pc = i % zp;
        const int t = t0 + p;
        const bool valid = t < m.T && pc * 8 < m.R;
        cp16_zfill(zdst + tc::core_off(p, pc * 8, m.RP), a.z + (row0 + (valid ? t : 0)) * m.R + (valid ? pc * 8 : 0), valid);
    }
    for (int i = threadIdx.x; i < m.RP * up; i += TC_THREADS) {
        const int r = i / up, pc = i % up;
        const bool valid = r < m.R;
        cp16_zfill(udst + tc::core_off(r, pc * 8, m.NB), a.U + (int64_t)(valid ? r : 0) * m.GW + col0 + pc * 8, valid);
    }
    for (int i = threadIdx.x; i < WIN * zp; i += TC_THREADS) {
        const int h = i / zp, pc = i % zp;
        const int t = t0 + TC_M + h;
        const bool valid = t < m.T && pc * 8 < m.R;
        cp16_zfill(zhdst + (uint32_t)(h * m.RP + pc * 8) * 2, a.z + (row0 + (valid ? t : 0)) * m.R + (valid ? pc * 8 : 0),
                   valid);
    }
}

// HM: how dw is reduced over a group's channels.  0: H <= 8 (groups inside
// one 8-channel vector); 1: H = 16 (both vectors of a half); 2: H = 32 (a whole
// sub-tile: the two halves combine through shared memory); 3: H = 64 (two
// sub-tiles, then the halves combine).
template <int W, int GPV, int HM>
__global__ void __launch_bounds__(TC_THREADS, 1) k_lr_tc_bwd(const TcArgs a) {
    constexpr int WIN = W - 1;
    constexpr int NT = GPV * W;
    extern __shared__ __align__(1024) unsigned char smem[];
    const TcMap &m = a.m;
    const BwdSmem S(m);
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t bar = sbase + S.bar;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t_loc = tid & (TC_M - 1), half = tid >> 7, quarter = warp & 3;
    const uint32_t rowbytes = S.rowbytes;
    float *edge = reinterpret_cast<float *>(smem + S.edge);  // [4][8][NB]
    float *xch = reinterpret_cast<float *>(smem + S.xch);    // [128][8]
    const int nSub = m.CH / TC_SC;

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(sbase + S.tmem, (uint32_t)m.tcols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S.tmem);
    const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t col_dz = (uint32_t)m.NB;
    const uint32_t col_dU = (uint32_t)(m.NB + m.RP);
    const float res = m.residual ? 1.f : 0.f;
    const uint32_t id_w = tc::idesc_bf16(TC_M, m.NB, 0, 1);
    const uint32_t id_dz = tc::idesc_bf16(TC_M, m.RP, 0, 0);
    const uint32_t id_dU = tc::idesc_bf16(TC_M, m.RP, 1, 1);
    uint32_t phase = 0;
    bool timed_out = false;

    const int group = blockIdx.x % m.nGroups;
    const int range = blockIdx.x / m.nGroups;
    const int chunk_lo = group * m.CPC;
    const int ncl = min(m.CPC, m.nChunks - chunk_lo);
    const int64_t tile_lo = (int64_t)range * m.tilesPerRange;
    const int ntl = (int)min((int64_t)m.tilesPerRange, m.totalTiles - tile_lo);

    for (int tl = 0; tl < ntl; ++tl) {
        const int64_t tile = tile_lo + tl;
        const int64_t b = tile / m.tilesPerSeq;
        const int t0 = (int)(tile % m.tilesPerSeq) * TC_M;
        const int64_t row0 = b * m.T;
        const int t = t0 + t_loc;
        for (int cl = 0; cl < ncl; ++cl) {
            const int chunk = chunk_lo + cl;
            const int64_t c_chunk = (int64_t)chunk * m.CH;
            const int64_t col0 = (int64_t)chunk * m.NB;
            // A. operands of the item and its first two sub-tiles
            load_item_bwd(m, a, row0, t0, col0, sbase + S.z, sbase + S.u, sbase + S.zh);
            load_sub_bwd(m, a, row0, t0, c_chunk, sbase + S.ring, sbase + S.ring + S.tile, rowbytes);
            cp_commit();
            if (nSub > 1)
                load_sub_bwd(m, a, row0, t0, c_chunk + TC_SC, sbase + S.ring + 2 * S.tile, sbase + S.ring + 3 * S.tile,
                             rowbytes);
            cp_commit();
            cp_wait<1>();
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            // B. w = z . U_chunk into TMEM columns [0, NB)
            if (tid == 0) {
                for (int ks = 0; ks < m.RP / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc(sbase + S.z + ks * 256, 128, (uint32_t)(m.RP / 8) * 128);
                    const uint64_t bd = tc::smem_desc(sbase + S.u + ks * 2 * (m.NB / 8) * 128, (uint32_t)(m.NB / 8) * 128, 128);
                    tc::mma_bf16(tmem, ad, bd, id_w, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(bar);
            }
            if (!tc::mbar_wait(bar, phase, TC_WAIT_LIMIT)) timed_out = true;
            phase ^= 1;
            tc::fence_after_sync();
            // C. rows w(t+k) that live outside this thread's warp quarter:
            //    edge[q][h] = w of token 32(q+1)+h (q < 3: from TMEM; q = 3: next tile, CUDA cores)
            if (WIN > 0) {
                const bf16 *zh = reinterpret_cast<const bf16 *>(smem + S.zh);
                for (int i = tid; i < WIN * m.NB; i += TC_THREADS) {
                    const int h = i / m.NB, col = i % m.NB;
                    float sacc = 0.f;
                    for (int r = 0; r < m.R; ++r)
                        sacc = fmaf(__bfloat162float(zh[h * m.RP + r]),
                                    __bfloat162float(*reinterpret_cast<const bf16 *>(smem + S.u + tc::core_off(r, col, m.NB))),
                                    sacc);
                    edge[(3 * 8 + h) * m.NB + col] = sacc;
                }
                if (half == 0 && quarter > 0) {
                    for (int c8 = 0; c8 < m.NB; c8 += 8) {
                        float v[8];
                        tc::tmem_ld8(tlane + (uint32_t)c8, v);
                        tc::tmem_wait_ld();
                        if (lane < WIN)
#pragma unroll
                            for (int j = 0; j < 8; ++j) edge[((quarter - 1) * 8 + lane) * m.NB + c8 + j] = v[j];
                    }
                }
            }
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();

            // D. sub-tiles
            float dacc[W];
#pragma unroll
            for (int k = 0; k < W; ++k) dacc[k] = 0.f;
            for (int sI = 0; sI < nSub; ++sI) {
                cp_wait<1>();
                __syncthreads();
                const uint32_t xb = sbase + S.ring + (uint32_t)(sI & 1) * 2 * S.tile;
                const uint32_t yb = xb + S.tile;
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    const int clc = sI * TC_SC + half * 16 + 8 * v;  // chunk-local channel
                    const int gl = clc / (int)m.H;                  // chunk-local group
                    float wt[NT], wsft[NT];
                    tmem_ld<NT>(tlane + (uint32_t)(gl * W), wt);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int f = 0; f < NT; ++f) wsft[f] = 0.f;
#pragma unroll
                    for (int gi = 0; gi < GPV; ++gi)
#pragma unroll
                        for (int k = 1; k < W; ++k) {
                            const float o = __shfl_down_sync(FULL_MASK, wt[gi * W + k], k);
                            wsft[gi * W + k] = lane + k < 32 ? o : edge[(quarter * 8 + lane + k - 32) * m.NB + (gl + gi) * W + k];
                        }
                    float xr[W][8], dr[W][8];
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        unpack(lds16(xb + (uint32_t)(t_loc + WIN - k) * rowbytes + (uint32_t)(half * 16 + 8 * v) * 2), xr[k]);
                        unpack(lds16(yb + (uint32_t)(t_loc + k) * rowbytes + (uint32_t)(half * 16 + 8 * v) * 2), dr[k]);
                    }
                    float dxv[8];
                    float pk[GPV][W];
#pragma unroll
                    for (int gi = 0; gi < GPV; ++gi)
#pragma unroll
                        for (int k = 0; k < W; ++k) pk[gi][k] = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int gi = j / (8 / GPV);
                        const int f = gi * W;
                        float sacc = (wt[f] + res) * dr[0][j];
#pragma unroll
                        for (int k = 1; k < W; ++k) sacc = fmaf(wsft[f + k], dr[k][j], sacc);
                        dxv[j] = sacc;
#pragma unroll
                        for (int k = 0; k < W; ++k) pk[gi][k] = fmaf(dr[0][j], xr[k][j], pk[gi][k]);
                    }
                    if (t < m.T) st16(a.dx + (row0 + t) * m.D + c_chunk + clc, pack(dxv));
                    if constexpr (HM == 0) {
#pragma unroll
                        for (int gi = 0; gi < GPV; ++gi)
#pragma unroll
                            for (int k = 0; k < W; ++k)
                                *reinterpret_cast<bf16 *>(smem + S.dw + tc::core_off(t_loc, (gl + gi) * W + k, m.NB)) =
                                    __float2bfloat16_rn(pk[gi][k]);
                    } else {
#pragma unroll
                        for (int k = 0; k < W; ++k) dacc[k] += pk[0][k];
                    }
                }
                if constexpr (HM == 1) {  // the half's two vectors form one group
                    const int gl = (sI * TC_SC + half * 16) / 16;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        *reinterpret_cast<bf16 *>(smem + S.dw + tc::core_off(t_loc, gl * W + k, m.NB)) =
                            __float2bfloat16_rn(dacc[k]);
                        dacc[k] = 0.f;
                    }
                }
                const bool group_done = HM == 2 || (HM == 3 && (sI & 1));
                if ((HM == 2 || HM == 3) && group_done && half == 1) {
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        xch[t_loc * 8 + k] = dacc[k];
                        dacc[k] = 0.f;
                    }
                }
                __syncthreads();  // sub-tile buffers consumed; halves' partials visible
                if ((HM == 2 || HM == 3) && group_done && half == 0) {
                    const int gl = (sI * TC_SC) / (int)m.H;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        *reinterpret_cast<bf16 *>(smem + S.dw + tc::core_off(t_loc, gl * W + k, m.NB)) =
                            __float2bfloat16_rn(dacc[k] + xch[t_loc * 8 + k]);
                        dacc[k] = 0.f;
                    }
                }
                if (sI + 2 < nSub) {
                    const uint32_t xn = sbase + S.ring + (uint32_t)(sI & 1) * 2 * S.tile;
                    load_sub_bwd(m, a, row0, t0, c_chunk + (int64_t)(sI + 2) * TC_SC, xn, xn + S.tile, rowbytes);
                }
                cp_commit();
            }
            // E. dz += dw U^T and dU[cl] += dw^T z
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
            if (tid == 0) {
                for (int ks = 0; ks < m.NB / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc(sbase + S.dw + ks * 256, 128, (uint32_t)(m.NB / 8) * 128);
                    const uint64_t bd = tc::smem_desc(sbase + S.u + ks * 256, 128, (uint32_t)(m.NB / 8) * 128);
                    tc::mma_bf16(tmem + col_dz, ad, bd, id_dz, (cl > 0 || ks > 0) ? 1u : 0u);
                }
                for (int mh = 0; mh < m.MH; ++mh)
                    for (int ks = 0; ks < TC_M / 16; ++ks) {
                        const uint64_t ad = tc::smem_desc(sbase + S.dw + mh * 16 * 128 + ks * 2 * (m.NB / 8) * 128,
                                                          (uint32_t)(m.NB / 8) * 128, 128);
                        const uint64_t bd = tc::smem_desc(sbase + S.z + ks * 2 * (m.RP / 8) * 128, (uint32_t)(m.RP / 8) * 128, 128);
                        tc::mma_bf16(tmem + col_dU + (uint32_t)((cl * m.MH + mh) * m.RP), ad, bd, id_dU,
                                     (tl > 0 || ks > 0) ? 1u : 0u);
                    }
                tc::mma_commit(bar);
            }
            if (!tc::mbar_wait(bar, phase, TC_WAIT_LIMIT)) timed_out = true;
            phase ^= 1;
            tc::fence_after_sync();
            // F. dz of the tile after the group's last chunk
            if (cl == ncl - 1 && half == 0) {
                for (int r8 = 0; r8 < m.RP; r8 += 8) {
                    float v[8];
                    tc::tmem_ld8(tlane + col_dz + (uint32_t)r8, v);
                    tc::tmem_wait_ld();
                    if (t < m.T)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int r = r8 + j;
                            if (r < m.R) {
                                const int64_t o = (row0 + t) * m.R + r;
                                if (m.nGroups == 1) a.dz[o] = __float2bfloat16_rn(v[j]);
                                else atomicAdd(a.dz_acc + o, v[j]);
                            }
                        }
                }
            }
            tc::fence_before_sync();
            __syncthreads();
            tc::fence_after_sync();
        }
    }
    // dU of the CTA's chunks over its token range (TMEM lane = U column)
    if (half == 0) {
        for (int cl = 0; cl < ncl; ++cl)
            for (int mh = 0; mh < m.MH; ++mh) {
                const int64_t col = (int64_t)(chunk_lo + cl) * m.NB + mh * TC_M + t_loc;
                for (int r8 = 0; r8 < m.RP; r8 += 8) {
                    float v[8];
                    tc::tmem_ld8(tlane + col_dU + (uint32_t)((cl * m.MH + mh) * m.RP + r8), v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r = r8 + j;
                        if (r < m.R && mh * TC_M + t_loc < m.NB) {
                            if (m.nRanges == 1) a.dU[(int64_t)r * m.GW + col] = v[j];
                            else a.dU_part[((int64_t)range * m.R + r) * m.GW + col] = v[j];
                        }
                    }
                }
            }
    }
    cp_wait<0>();
    if (timed_out && lane == 0) atomicExch(&g_dsc_status_tc, (int)DSC_ERR_TIMEOUT);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, (uint32_t)m.tcols);
}

__global__ void k_tc_zero(float *p, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) p[i] = 0.f;
}

// dU = sum of the per-range partials (fixed order); dz = the fp32 accumulator in bf16.
__global__ void k_tc_finalize(const TcArgs a) {
    const TcMap &m = a.m;
    const int64_t nU = m.nRanges > 1 ? m.R * m.GW : 0;
    const int64_t nz = m.nGroups > 1 ? m.B * m.T * m.R : 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nU + nz; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < nU) {
            float sacc = 0.f;
            for (int q = 0; q < m.nRanges; ++q) sacc += a.dU_part[(int64_t)q * m.R * m.GW + i];
            a.dU[i] = sacc;
        } else {
            a.dz[i - nU] = __float2bfloat16_rn(a.dz_acc[i - nU]);
        }
    }
}

bool tc_map(const dsc_problem &p, TcMap &m) {
    if (p.dtype != DSC_BF16) return false;
    if (p.R < 8 || p.R > 64 || p.R % 8) return false;  // 16-byte z rows
    if (!(p.W == 1 || p.W == 2 || p.W == 4 || p.W == 8)) return false;
    if (p.H > 64 || (64 % p.H) != 0) return false;
    if (p.D % (TC_GROUPS * p.H)) return false;
    m = TcMap{};
    m.B = p.B; m.T = p.T; m.D = p.D; m.H = p.H; m.R = p.R; m.W = (int)p.W;
    m.GW = (p.D / p.H) * p.W;
    m.RP = (int)((p.R + 15) / 16) * 16;
    m.NB = TC_GROUPS * (int)p.W;
    m.CH = TC_GROUPS * (int)p.H;
    m.SC = m.CH < 64 ? m.CH : 64;
    if (m.SC < 16) return false;  // each half needs at least one 8-channel vector
    m.nSub = m.CH / m.SC;
    m.nChunks = (int)(p.D / m.CH);
    m.tilesPerSeq = (int)((p.T + TC_M - 1) / TC_M);
    m.nItems = p.B * (int64_t)m.tilesPerSeq * m.nChunks;
    m.residual = p.residual ? 1 : 0;
    return true;
}

// Backward plan.  TMEM holds w (NB columns), dz (RP) and one dU accumulator
// per chunk of the CTA (MH * RP each); among the chunk-group sizes that fit,
// take the one with the least partial-sum traffic (dU partials of the token
// ranges, dz contributions of the chunk groups) for about one CTA per SM.
bool tc_bwd_plan(TcMap &m, int sms) {
    if (m.W < 4) return false;  // the dU MMA needs M = NB >= 128
    if (m.CH % TC_SC) return false;
    m.MH = m.NB / TC_M;
    m.totalTiles = m.B * (int64_t)m.tilesPerSeq;
    const int cpc_max = (512 - m.NB - m.RP) / (m.MH * m.RP);
    if (cpc_max < 1) return false;
    double best = -1;
    for (int cpc = 1; cpc <= cpc_max && cpc <= m.nChunks; ++cpc) {
        const int ng = (m.nChunks + cpc - 1) / cpc;
        int64_t nr = sms / ng;
        if (nr < 1) nr = 1;
        if (nr > m.totalTiles) nr = m.totalTiles;
        // DRAM floats: dU partials are written and read back once; dz goes
        // through one fp32 accumulator (written back and read once) that
        // takes ng reductions per element in L2 (counted at a quarter each).
        const double nz = (double)m.B * m.T * m.R;
        const double cost = (nr > 1 ? 2.0 * nr * m.R * m.GW : 0.0) + (ng > 1 ? (2.0 + 0.25 * ng) * nz : 0.0);
        if (best < 0 || cost < best) {
            best = cost;
            m.CPC = cpc;
            m.nGroups = ng;
            m.nRanges = (int)nr;
        }
    }
    m.tilesPerRange = (int)((m.totalTiles + m.nRanges - 1) / m.nRanges);
    m.nRanges = (int)((m.totalTiles + m.tilesPerRange - 1) / m.tilesPerRange);
    const int cols = m.NB + m.RP + m.CPC * m.MH * m.RP;
    m.tcols = 32;
    while (m.tcols < cols) m.tcols *= 2;
    return m.tcols <= 512;
}

size_t tc_bwd_ws_bytes(const TcMap &m) {
    size_t n = 0;
    if (m.nRanges > 1) n += (size_t)m.nRanges * m.R * m.GW;
    if (m.nGroups > 1) n += (size_t)m.B * m.T * m.R;
    return n * sizeof(float);
}

template <int W, int GPV>
cudaError_t launch_fwd(const Ctx &c, const TcArgs &a) {
    const FwdSmem S(a.m);
    static const cudaError_t attr = cudaFuncSetAttribute(k_lr_tc_fwd<W, GPV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                         200 * 1024);
    if (attr != cudaSuccess) return attr;
    const int64_t grid = a.m.nItems < c.sms ? a.m.nItems : c.sms;
    k_lr_tc_fwd<W, GPV><<<(unsigned)grid, TC_THREADS, S.total, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <int W> cudaError_t fwd_by_gpv(const Ctx &c, const TcArgs &a) {
    switch (a.m.H) {
    case 1: return launch_fwd<W, 8>(c, a);
    case 2: return launch_fwd<W, 4>(c, a);
    case 4: return launch_fwd<W, 2>(c, a);
    default: return launch_fwd<W, 1>(c, a);
    }
}


template <int W, int GPV, int HM>
cudaError_t launch_bwd(const Ctx &c, const TcArgs &a) {
    const BwdSmem S(a.m);
    static const cudaError_t attr = cudaFuncSetAttribute(k_lr_tc_bwd<W, GPV, HM>,
                                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    if (attr != cudaSuccess) return attr;
    if (S.total > 220 * 1024) return cudaErrorInvalidValue;
    // More than half of TMEM per CTA: reserve enough shared memory that a
    // second CTA never lands on the same SM (it would wait for the TMEM).
    const uint32_t smem = a.m.tcols > 256 && S.total < 120 * 1024 ? 120 * 1024 : S.total;
    k_lr_tc_bwd<W, GPV, HM><<<(unsigned)(a.m.nGroups * a.m.nRanges), TC_THREADS, smem, c.stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <int W> cudaError_t bwd_by_h(const Ctx &c, const TcArgs &a) {
    switch (a.m.H) {
    case 1: return launch_bwd<W, 8, 0>(c, a);
    case 2: return launch_bwd<W, 4, 0>(c, a);
    case 4: return launch_bwd<W, 2, 0>(c, a);
    case 8: return launch_bwd<W, 1, 0>(c, a);
    case 16: return launch_bwd<W, 1, 1>(c, a);
    case 32: return launch_bwd<W, 1, 2>(c, a);
    case 64: return launch_bwd<W, 1, 3>(c, a);
    }
    return cudaErrorNotSupported;
}

}  // namespace

bool lowrank_tc_ok(const dsc_problem &p) {
    TcMap m;
    return tc_map(p, m);
}

bool lowrank_tc_bwd_ok(const dsc_problem &p, int sms) {
    TcMap m;
    return tc_map(p, m) && tc_bwd_plan(m, sms);
}

size_t lr_tc_bwd_ws_bytes(const dsc_problem &p, int sms) {
    TcMap m;
    if (!tc_map(p, m) || !tc_bwd_plan(m, sms)) return 0;
    return tc_bwd_ws_bytes(m);
}

cudaError_t launch_lr_bwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U,
                             const void *dy, void *dx, void *dz, float *dU, void *ws, size_t ws_bytes) {
    TcArgs a{};
    if (!tc_map(p, a.m) || !tc_bwd_plan(a.m, c.sms)) return cudaErrorNotSupported;
    if (ws_bytes < tc_bwd_ws_bytes(a.m)) return cudaErrorInvalidValue;
    a.x = static_cast<const bf16 *>(x);
    a.z = static_cast<const bf16 *>(z);
    a.U = static_cast<const bf16 *>(U);
    a.dy = static_cast<const bf16 *>(dy);
    a.dx = static_cast<bf16 *>(dx);
    a.dz = static_cast<bf16 *>(dz);
    a.dU = dU;
    float *w = static_cast<float *>(ws);
    if (a.m.nRanges > 1) {
        a.dU_part = w;
        w += (size_t)a.m.nRanges * a.m.R * a.m.GW;
    }
    if (a.m.nGroups > 1) {
        a.dz_acc = w;
        const int64_t n = a.m.B * a.m.T * a.m.R;
        k_tc_zero<<<(unsigned)min((int64_t)1024, (n + 255) / 256), 256, 0, c.stream>>>(a.dz_acc, n);
        count_launch();
    }
    cudaError_t e = cudaErrorNotSupported;
    switch (a.m.W) {
    case 4: e = bwd_by_h<4>(c, a); break;
    case 8: e = bwd_by_h<8>(c, a); break;
    }
    if (e != cudaSuccess) return e;
    if (a.m.nRanges > 1 || a.m.nGroups > 1) {
        const int64_t n = (a.m.nRanges > 1 ? a.m.R * a.m.GW : 0) + (a.m.nGroups > 1 ? a.m.B * a.m.T * a.m.R : 0);
        k_tc_finalize<<<(unsigned)min((int64_t)2048, (n + 255) / 256), 256, 0, c.stream>>>(a);
        count_launch();
    }
    return cudaGetLastError();
}

cudaError_t launch_lr_fwd_tc(const Ctx &c, const dsc_problem &p, const void *x, const void *z, const void *U, void *y) {
    TcArgs a{};
    if (!tc_map(p, a.m)) return cudaErrorNotSupported;
    a.x = static_cast<const bf16 *>(x);
    a.z = static_cast<const bf16 *>(z);
    a.U = static_cast<const bf16 *>(U);
    a.y = static_cast<bf16 *>(y);
    switch (a.m.W) {
    case 1: return fwd_by_gpv<1>(c, a);
    case 2: return fwd_by_gpv<2>(c, a);
    case 4: return fwd_by_gpv<4>(c, a);
    case 8: return fwd_by_gpv<8>(c, a);
    }
    return cudaErrorNotSupported;
}

}  // namespace dsc
