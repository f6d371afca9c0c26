// The first low-rank projection z = h V on the tensor cores, and its
// gradients dh = dz V^T and dV = sum_t h^T dz.
//
// "Dynamic Short Convolutions Improve Transformers", technical summary,
// Methodology, "Parameterisation" 1: the filter is a linear map of the
// current hidden state factorised at rank R, w(t) = h_t V U.  The fused
// convolution kernels take z = hV and U; the calls in this file take h and V
// and form z themselves, on tcgen05 tensor cores with fp32 accumulation in
// TMEM, inside the same call (z leaves as an output: the backward needs it).
//
// Why z is formed by its own kernel and not inside the convolution's items:
// the convolution's work items are (128-token tile, channel block); a tile's
// z is needed by every block of the tile (192 of them on the Q/K/V shape), so
// forming it per item would repeat the d_model-long contraction per block,
// and forming it per CTA would re-read h by the number of CTAs sharing a
// tile.  One persistent pass forms each tile's z once, reading h once; the
// convolution then reads z (R*2 bytes per token, from L2) through the same
// stream, its prologue overlapping this kernel's tail (programmatic
// dependent launch).
//
// Kernels (bf16, R a multiple of 8 up to 64, d_model a multiple of 128):
//   k_proj_z   persistent; per 128-token tile a K loop over d_model in steps
//              of 64 (TMA ring of h and V chunks), MMA M=128 N=RP into one of
//              two TMEM accumulators; 4 epilogue warps store z rows.
//   k_proj_dh  persistent; per (tile, 256 model columns): dz tile x V^T chunk
//              (K = R) into one of two TMEM accumulators, staged in one of two
//              shared-memory tiles and stored by TMA while the next item runs.
//   k_proj_dV  per (128 model rows, token range): h^T x dz over the range,
//              accumulated in TMEM, written as a per-range partial; a second
//              kernel sums the partials in a fixed order (deterministic).
// h travels as TMA boxes of 64 model columns (128-byte rows, 128-byte
// swizzle: one copy per 16 KB stage, full 128-byte requests), read by the MMA
// through swizzled descriptors (K-major for z, MN-major for dV); the small
// operands (V, dz) are boxes of 8 columns (16-byte rows) laid out as the
// MMA's core matrices, as in the convolution kernels.
#include "lowrank_tc.cuh"

namespace dsc {

__device__ int g_dsc_status_proj = 0;

int take_proj_status(cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_dsc_status_proj, sizeof v, 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return -1;
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_dsc_status_proj, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return -1;
    return v;
}

namespace {

using lrtc::TC_M;
using lrtc::TC_WAIT_LIMIT;
using lrtc::make_map;

constexpr int PJ_THREADS = 192;  // warps 0-3 epilogue (TMEM lanes), warp 4 TMA producer, warp 5 MMA + TMEM owner
constexpr int PJ_KC = 64;        // model columns per pipeline stage of k_proj_z
constexpr int PJ_NST = 6;        // stages of k_proj_z
constexpr int PV_NST = 4;        // stages of k_proj_dV
constexpr int PH_NC = 256;       // model columns per k_proj_dh item

struct ProjArgs {
    int64_t N, d, R;  // tokens, model width, rank
    int RP;           // R rounded up to 16
    int64_t ntiles;
    bf16 *z, *dh;
    float *part;  // dV partials [nranges][d][R]
    int64_t tilesPerRange;
};

__device__ __forceinline__ uint32_t pow2_cols(int n) {
    uint32_t c = 32;
    while ((int)c < n) c <<= 1;
    return c;
}

__device__ __forceinline__ void record_timeout() { atomicExch(&g_dsc_status_proj, (int)DSC_ERR_TIMEOUT); }

// ------------------------------------------------------------- z = h V ---
__global__ void __launch_bounds__(PJ_THREADS, 1)
    k_proj_z(const __grid_constant__ CUtensorMap tmh, const __grid_constant__ CUtensorMap tmv, const ProjArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const int RP = a.RP, kz = (int)(a.R / 8);
    const uint32_t abytes = TC_M * PJ_KC * 2, bbytes = (uint32_t)(PJ_KC * RP * 2), sbytes = abytes + bbytes;
    const uint32_t bars = PJ_NST * sbytes;  // full[NST] empty[NST] accf[2] acce[2]
    auto full = [&](int s) { return sbase + bars + 8u * s; };
    auto empty = [&](int s) { return sbase + bars + 8u * (PJ_NST + s); };
    auto accf = [&](int b) { return sbase + bars + 8u * (2 * PJ_NST + b); };
    auto acce = [&](int b) { return sbase + bars + 8u * (2 * PJ_NST + 2 + b); };
    const uint32_t tslot = bars + 8u * (2 * PJ_NST + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntl = a.ntiles > blockIdx.x ? (int)((a.ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
    const int nK = (int)((a.d + PJ_KC - 1) / PJ_KC);
    const uint32_t ncols = pow2_cols(2 * RP);

    if (tid == 0) {
        for (int s = 0; s < PJ_NST; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(accf(b), 1);
            tc::mbar_init(acce(b), 4);
        }
        tc::fence_mbar_init();
    }
    // V columns R .. RP-1 are never loaded: zero them once in every stage
    for (int i = tid; i < PJ_NST * (RP / 8 - kz) * PJ_KC; i += PJ_THREADS) {
        const int s = i / ((RP / 8 - kz) * PJ_KC), rem = i % ((RP / 8 - kz) * PJ_KC);
        *reinterpret_cast<uint4 *>(smem + s * sbytes + abytes + (uint32_t)(kz + rem / PJ_KC) * (PJ_KC * 16) +
                                   (uint32_t)(rem % PJ_KC) * 16) = make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async();
    if (warp == 5) tc::tmem_alloc(sbase + tslot, ncols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + tslot);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;
    };
    pdl_wait();
    pdl_trigger();  // the convolution may start its prologue

    if (warp == 4) {
        if (lane == 0 && ntl > 0) {
            tc::tma_prefetch_desc(&tmh);
            tc::tma_prefetch_desc(&tmv);
            int s = 0, it = 0;
            uint32_t ph = 0;
            for (int tl = 0; tl < ntl; ++tl) {
                const int64_t tile = blockIdx.x + (int64_t)tl * gridDim.x;
                for (int kc = 0; kc < nK; ++kc, ++it) {
                    if (it >= PJ_NST) wait(empty(s), ph ^ 1u);
                    const uint32_t st = sbase + (uint32_t)s * sbytes;
                    tc::mbar_expect_tx(full(s), abytes + (uint32_t)kz * (PJ_KC * 16));
                    tc::tma_load_2d(st, &tmh, kc * PJ_KC, (int)(tile * TC_M), full(s));
                    for (int j = 0; j < kz; ++j)
                        tc::tma_load_2d(st + abytes + (uint32_t)j * (PJ_KC * 16), &tmv, 8 * j, kc * PJ_KC, full(s));
                    if (++s == PJ_NST) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the last loads have landed before the block may exit
            const int total = ntl * nK;
            for (int q = 0; q < PJ_NST && q < total; ++q) {
                const int last = q + ((total - 1 - q) / PJ_NST) * PJ_NST;
                if (!tc::mbar_wait(full(q), (uint32_t)((last / PJ_NST) & 1), TC_WAIT_LIMIT)) timed_out = true;
            }
        }
    } else if (warp == 5) {
        if (lane == 0 && ntl > 0) {
            const uint32_t id = tc::idesc_bf16(TC_M, RP, 0, 1);
            int s = 0;
            uint32_t ph = 0;
            for (int tl = 0; tl < ntl; ++tl) {
                const int b = tl & 1;
                if (tl >= 2) wait(acce(b), (uint32_t)(((tl - 2) >> 1) & 1));
                tc::fence_after_sync();
                for (int kc = 0; kc < nK; ++kc) {
                    wait(full(s), ph);
                    tc::fence_after_sync();
                    const uint32_t st = sbase + (uint32_t)s * sbytes;
                    for (int ks = 0; ks < PJ_KC / 16; ++ks) {
                        const uint64_t ad = tc::smem_desc_sw128(st + (uint32_t)ks * 32u, 16, 1024);
                        const uint64_t bd = tc::smem_desc(st + abytes + (uint32_t)ks * 256u, 128, PJ_KC * 16);
                        tc::mma_bf16(tmem + (uint32_t)(b * RP), ad, bd, id, (kc > 0 || ks > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(empty(s));
                    if (++s == PJ_NST) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                tc::mma_commit(accf(b));
            }
            const int lb = (ntl - 1) & 1;  // the last accumulator's MMAs are done before TMEM is freed
            if (!tc::mbar_wait(accf(lb), (uint32_t)(((ntl - 1) >> 1) & 1), TC_WAIT_LIMIT)) timed_out = true;
        }
    } else {
        // epilogue: warp q reads TMEM lanes 32q .. 32q+31 = tokens of the tile
        const uint32_t tl_base = tmem + ((uint32_t)(warp * 32) << 16);
        for (int tl = 0; tl < ntl; ++tl) {
            const int b = tl & 1;
            wait(accf(b), (uint32_t)((tl >> 1) & 1));
            tc::fence_after_sync();
            const int64_t tile = blockIdx.x + (int64_t)tl * gridDim.x;
            const int64_t tok = tile * TC_M + warp * 32 + lane;
            for (int c = 0; c < kz; ++c) {
                float v[8];
                tc::tmem_ld8(tl_base + (uint32_t)(b * RP + 8 * c), v);
                tc::tmem_wait_ld();
                if (tok < a.N)
                    st16(a.z + tok * a.R + 8 * c, make_uint4(pack_bf2(v[0], v[1]), pack_bf2(v[2], v[3]),
                                                             pack_bf2(v[4], v[5]), pack_bf2(v[6], v[7])));
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(acce(b));
        }
    }
    if (timed_out) record_timeout();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 5) tc::tmem_dealloc(tmem, ncols);
}

// ---------------------------------------------------------- dh = dz V^T ---
// Persistent.  Item = (tile of 128 tokens, PH_NC model columns): A = dz tile
// [128 x RP] (K-major), B = V rows [PH_NC x RP] read as V^T (K-major), K = RP.
// Two operand stages, two TMEM accumulators (2 x 256 columns) and two staging
// tiles, so that one item's store leaves while the next item's MMAs and
// epilogue run.  Warp 8 (one lane) loads and issues the MMAs; warps 0-7 drain
// the accumulator (warp w: TMEM lanes 32*(w%4).., columns 128*(w/4)..) into
// 128-byte-swizzled staging boxes that thread 0 stores by TMA.
constexpr int PH_BOX = PH_NC / 64;  // staging boxes of 64 columns
constexpr int PH_EPI = 256;         // epilogue threads
constexpr int PH_THREADS = PH_EPI + 32;

struct DhSmem {
    uint32_t abytes, bbytes, stage, stg, bars, tslot, total;
    __host__ __device__ explicit DhSmem(int RP) {
        abytes = (uint32_t)(TC_M * RP * 2);
        bbytes = (uint32_t)(PH_NC * RP * 2);
        stage = abytes + bbytes;                                                 // multiple of 1024
        stg = 2 * stage;                                                         // two staging tiles
        bars = stg + 2 * PH_BOX * TC_M * 128;                                    // opf[2] ope[2] accf[2] acce[2]
        tslot = bars + 8 * 8;
        total = tslot + 16 + 1024;
    }
};

__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

__global__ void __launch_bounds__(PH_THREADS, 1)
    k_proj_dh(const __grid_constant__ CUtensorMap tmdz, const __grid_constant__ CUtensorMap tmv,
              const __grid_constant__ CUtensorMap tmdh, const ProjArgs a, int nchunks) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const int RP = a.RP, kz = (int)(a.R / 8);
    const DhSmem S(RP);
    auto opf = [&](int s) { return sbase + S.bars + 8u * s; };
    auto ope = [&](int s) { return sbase + S.bars + 16u + 8u * s; };
    auto accf = [&](int s) { return sbase + S.bars + 32u + 8u * s; };
    auto acce = [&](int s) { return sbase + S.bars + 48u + 8u * s; };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t nitems = a.ntiles * nchunks;
    const int nit = nitems > blockIdx.x ? (int)((nitems - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (tid == 0) {
        for (int q = 0; q < 2; ++q) {
            tc::mbar_init(opf(q), 1);
            tc::mbar_init(ope(q), 1);
            tc::mbar_init(accf(q), 1);
            tc::mbar_init(acce(q), 1);
        }
        tc::fence_mbar_init();
    }
    // rank columns R .. RP-1 of both operands of both stages stay zero (never loaded)
    for (int i = tid; i < 2 * (RP / 8 - kz) * (TC_M + PH_NC); i += PH_THREADS) {
        const int st = i / ((RP / 8 - kz) * (TC_M + PH_NC)), i1 = i % ((RP / 8 - kz) * (TC_M + PH_NC));
        const int j = kz + i1 / (TC_M + PH_NC), r = i1 % (TC_M + PH_NC);
        const uint32_t off = r < TC_M ? (uint32_t)j * (TC_M * 16) + (uint32_t)r * 16
                                      : S.abytes + (uint32_t)j * (PH_NC * 16) + (uint32_t)(r - TC_M) * 16;
        *reinterpret_cast<uint4 *>(smem + (uint32_t)st * S.stage + off) = make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async();
    if (warp == 0) tc::tmem_alloc(sbase + S.tslot, 2 * PH_NC);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + S.tslot);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;
    };
    pdl_wait();
    pdl_trigger();
    // item it of this CTA: tile-minor, so that neighbouring CTAs share a V chunk
    auto item = [&](int it, int64_t &tile, int &chunk) {
        const int64_t g = blockIdx.x + (int64_t)it * gridDim.x;
        chunk = (int)(g / a.ntiles);
        tile = g - (int64_t)chunk * a.ntiles;
    };

    if (warp == PH_EPI / 32) {
        if (lane == 0 && nit > 0) {
            tc::tma_prefetch_desc(&tmdz);
            tc::tma_prefetch_desc(&tmv);
            auto load = [&](int it) {
                const int st = it & 1;
                int64_t tile;
                int chunk;
                item(it, tile, chunk);
                const uint32_t base = sbase + (uint32_t)st * S.stage;
                tc::mbar_expect_tx(opf(st), (uint32_t)kz * (TC_M * 16 + PH_NC * 16));
                for (int j = 0; j < kz; ++j) {
                    tc::tma_load_2d(base + (uint32_t)j * (TC_M * 16), &tmdz, 8 * j, (int)(tile * TC_M), opf(st));
                    tc::tma_load_2d(base + S.abytes + (uint32_t)j * (PH_NC * 16), &tmv, 8 * j, chunk * PH_NC, opf(st));
                }
            };
            for (int it = 0; it < 2 && it < nit; ++it) load(it);
            const uint32_t id = tc::idesc_bf16(TC_M, PH_NC, 0, 0);
            for (int it = 0; it < nit; ++it) {
                const int st = it & 1;
                const uint32_t ph = (uint32_t)((it >> 1) & 1);
                wait(opf(st), ph);
                if (it >= 2) wait(acce(st), ph ^ 1u);
                tc::fence_after_sync();
                const uint32_t base = sbase + (uint32_t)st * S.stage;
                for (int ks = 0; ks < RP / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc(base + (uint32_t)ks * 2u * (TC_M * 16), TC_M * 16, 128);
                    const uint64_t bd = tc::smem_desc(base + S.abytes + (uint32_t)ks * 2u * (PH_NC * 16), PH_NC * 16, 128);
                    tc::mma_bf16(tmem + (uint32_t)(st * PH_NC), ad, bd, id, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(accf(st));
                tc::mma_commit(ope(st));
                if (it + 2 < nit) {  // refill this stage once its MMAs have read it
                    wait(ope(st), ph);
                    load(it + 2);
                }
            }
        }
    } else {
        const int q4 = warp & 3, half = warp >> 2;
        const int t = q4 * 32 + lane;  // token row of the tile = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        for (int it = 0; it < nit; ++it) {
            const int st = it & 1;
            const uint32_t ph = (uint32_t)((it >> 1) & 1);
            int64_t tile;
            int chunk;
            item(it, tile, chunk);
            wait(accf(st), ph);
            tc::fence_after_sync();
            // the store that last used this staging tile (item it-2) has read it;
            // the one of item it-1 may still be in flight
            if (tid == 0) bulk_wait_read_1();
            asm volatile("bar.sync 1, %0;" ::"n"(PH_EPI) : "memory");
            unsigned char *stg = smem + S.stg + (uint32_t)st * (PH_BOX * TC_M * 128);
            for (int c0 = half * (PH_NC / 2); c0 < (half + 1) * (PH_NC / 2); c0 += 32) {
                float v[32];
                lrtc::tmem_ld<32>(tl + (uint32_t)(st * PH_NC + c0), v);
                tc::tmem_wait_ld();
                unsigned char *box = stg + (uint32_t)(c0 / 64) * (TC_M * 128);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(box + tc::swz<128>(t, (c0 % 64) / 8 + q)) =
                        make_uint4(pack_bf2(v[8 * q], v[8 * q + 1]), pack_bf2(v[8 * q + 2], v[8 * q + 3]),
                                   pack_bf2(v[8 * q + 4], v[8 * q + 5]), pack_bf2(v[8 * q + 6], v[8 * q + 7]));
            }
            tc::fence_before_sync();
            tc::fence_proxy_async();
            asm volatile("bar.sync 1, %0;" ::"n"(PH_EPI) : "memory");
            if (tid == 0) {
                tc::mbar_arrive(acce(st));
                for (int bx = 0; bx < PH_BOX; ++bx)
                    if (chunk * PH_NC + bx * 64 < a.d)
                        tc::tma_store_3d(&tmdh, sbase + S.stg + (uint32_t)(st * PH_BOX + bx) * (TC_M * 128),
                                         chunk * PH_NC + bx * 64, (int)(tile * TC_M), 0);
                tc::bulk_commit();
            }
        }
        if (tid == 0) tc::bulk_wait_all();
    }
    if (timed_out) record_timeout();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 2 * PH_NC);
}

// ---------------------------------------------------- dV = sum_t h^T dz ---
// CTA = (128 model rows, range of token tiles).  Per tile: A = h^T [128 rows
// x 128 tokens] (MN-major: two swizzled h boxes of 64 model columns), B = dz
// tile [128 tokens x RP] (MN-major), 8 MMAs of K = 16 tokens into one TMEM
// accumulator.
__global__ void __launch_bounds__(PJ_THREADS, 1)
    k_proj_dV(const __grid_constant__ CUtensorMap tmh, const __grid_constant__ CUtensorMap tmdz, const ProjArgs a,
              int nchunks) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t sraw = tc::smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - sraw);
    const int RP = a.RP, kz = (int)(a.R / 8);
    const uint32_t abytes = TC_M * TC_M * 2, bbytes = (uint32_t)(TC_M * RP * 2), sbytes = abytes + bbytes;
    const uint32_t bars = PV_NST * sbytes;  // full[NST] empty[NST] done
    auto full = [&](int s) { return sbase + bars + 8u * s; };
    auto empty = [&](int s) { return sbase + bars + 8u * (PV_NST + s); };
    const uint32_t done = sbase + bars + 8u * (2 * PV_NST);
    const uint32_t tslot = bars + 8u * (2 * PV_NST + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chunk = (int)(blockIdx.x % nchunks);
    const int64_t range = blockIdx.x / nchunks;
    const int64_t t_lo = range * a.tilesPerRange;
    const int ntl = (int)max((int64_t)0, min(a.tilesPerRange, a.ntiles - t_lo));
    const uint32_t ncols = pow2_cols(RP);

    if (tid == 0) {
        for (int s = 0; s < PV_NST; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), 1);
        }
        tc::mbar_init(done, 1);
        tc::fence_mbar_init();
    }
    for (int i = tid; i < PV_NST * (RP / 8 - kz) * TC_M; i += PJ_THREADS) {
        const int s = i / ((RP / 8 - kz) * TC_M), rem = i % ((RP / 8 - kz) * TC_M);
        *reinterpret_cast<uint4 *>(smem + s * sbytes + abytes + (uint32_t)(kz + rem / TC_M) * (TC_M * 16) +
                                   (uint32_t)(rem % TC_M) * 16) = make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async();
    if (warp == 5) tc::tmem_alloc(sbase + tslot, ncols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + tslot);
    bool timed_out = false;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (!timed_out && !tc::mbar_wait(bar, parity, TC_WAIT_LIMIT)) timed_out = true;
    };
    pdl_wait();
    pdl_trigger();

    if (warp == 4) {
        if (lane == 0 && ntl > 0) {
            tc::tma_prefetch_desc(&tmh);
            tc::tma_prefetch_desc(&tmdz);
            int s = 0;
            uint32_t ph = 0;
            for (int tl = 0; tl < ntl; ++tl) {
                if (tl >= PV_NST) wait(empty(s), ph ^ 1u);
                const uint32_t st = sbase + (uint32_t)s * sbytes;
                const int row = (int)((t_lo + tl) * TC_M);
                tc::mbar_expect_tx(full(s), abytes + (uint32_t)kz * (TC_M * 16));
                for (int j = 0; j < 2; ++j)
                    tc::tma_load_2d(st + (uint32_t)j * (TC_M * 128), &tmh, chunk * TC_M + 64 * j, row, full(s));
                for (int j = 0; j < kz; ++j)
                    tc::tma_load_2d(st + abytes + (uint32_t)j * (TC_M * 16), &tmdz, 8 * j, row, full(s));
                if (++s == PV_NST) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            for (int q = 0; q < PV_NST && q < ntl; ++q) {
                const int last = q + ((ntl - 1 - q) / PV_NST) * PV_NST;
                if (!tc::mbar_wait(full(q), (uint32_t)((last / PV_NST) & 1), TC_WAIT_LIMIT)) timed_out = true;
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t id = tc::idesc_bf16(TC_M, RP, 1, 1);
            int s = 0;
            uint32_t ph = 0;
            for (int tl = 0; tl < ntl; ++tl) {
                wait(full(s), ph);
                tc::fence_after_sync();
                const uint32_t st = sbase + (uint32_t)s * sbytes;
                for (int ks = 0; ks < TC_M / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc_sw128(st + (uint32_t)ks * 2048u, TC_M * 128, 1024);
                    const uint64_t bd = tc::smem_desc(st + abytes + (uint32_t)ks * 256u, 128, TC_M * 16);
                    tc::mma_bf16(tmem, ad, bd, id, (tl > 0 || ks > 0) ? 1u : 0u);
                }
                tc::mma_commit(empty(s));
                if (++s == PV_NST) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            tc::mma_commit(done);  // also completes when the range is empty
        }
    } else {
        wait(done, 0);
        tc::fence_after_sync();
        const int64_t row = (int64_t)chunk * TC_M + warp * 32 + lane;  // model row i of this thread's TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c = 0; c < kz; ++c) {
            float v[8];
            tc::tmem_ld8(tl + (uint32_t)(8 * c), v);
            tc::tmem_wait_ld();
            if (row < a.d) {
                float *p = a.part + (range * a.d + row) * a.R + 8 * c;
                if (ntl == 0)
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = 0.f;
                *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
    }
    if (timed_out) record_timeout();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 5) tc::tmem_dealloc(tmem, ncols);
}

// dV[i] = sum over ranges q (in order) of part[q][i].
__global__ void k_proj_dV_sum(const float *__restrict__ part, int64_t nranges, int64_t n, float *__restrict__ dV) {
    pdl_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int64_t q = 0; q < nranges; ++q) s += part[q * n + i];
        dV[i] = s;
    }
}

uint32_t z_smem(int RP) { return PJ_NST * (TC_M * PJ_KC * 2 + PJ_KC * RP * 2) + 8 * (2 * PJ_NST + 4) + 16 + 1024; }
uint32_t dh_smem(int RP) { return DhSmem(RP).total; }
uint32_t dV_smem(int RP) { return PV_NST * (TC_M * TC_M * 2 + TC_M * RP * 2) + 8 * (2 * PV_NST + 1) + 16 + 1024; }

bool map2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_in, uint32_t box_out,
           CUtensorMapSwizzle sw) {
    const uint64_t dims[2] = {inner, outer};
    const uint64_t strides[1] = {inner * 2};
    const uint32_t box[2] = {box_in, box_out};
    return make_map(m, base, 2, dims, strides, box, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

}  // namespace

// d a multiple of 128: every TMA box of h, V and dh starts inside its tensor
// (only the last token tile reaches past the end, filled with zeros).
bool proj_tc_ok(const dsc_problem &p, int64_t d) {
    return p.dtype == DSC_BF16 && p.R >= 8 && p.R <= 64 && p.R % 8 == 0 && d >= 128 && d % 128 == 0 &&
           d <= ((int64_t)1 << 30);
}

int64_t proj_ranges(const dsc_problem &p, int64_t d, int sms) {
    const int64_t ntiles = (p.B * p.T + TC_M - 1) / TC_M;
    const int64_t nchunks = (d + TC_M - 1) / TC_M;
    int64_t nr = sms / nchunks;
    if (nr < 1) nr = 1;
    if (nr > ntiles) nr = ntiles;
    const int64_t per = (ntiles + nr - 1) / nr;
    return (ntiles + per - 1) / per;
}

size_t proj_dV_part_bytes(const dsc_problem &p, int64_t d, int sms) {
    return proj_tc_ok(p, d) ? (size_t)proj_ranges(p, d, sms) * (size_t)d * (size_t)p.R * sizeof(float) : 0;
}

static ProjArgs proj_args(const dsc_problem &p, int64_t d) {
    ProjArgs a{};
    a.N = p.B * p.T;
    a.d = d;
    a.R = p.R;
    a.RP = (int)((p.R + 15) / 16) * 16;
    a.ntiles = (a.N + TC_M - 1) / TC_M;
    return a;
}

// z [N, R] = h [N, d] . V [d, R]
cudaError_t launch_proj_z(const Ctx &c, const dsc_problem &p, int64_t d, const void *h, const void *V, void *z) {
    const int64_t N = p.B * p.T;
    const bool bf = p.dtype == DSC_BF16;
    if (!proj_tc_ok(p, d))
        return launch_gemm(c, (int)N, (int)p.R, (int)d, h, !bf, d, 1, V, !bf, 1, p.R, z, !bf, p.R, bf);
    ProjArgs a = proj_args(p, d);
    a.z = static_cast<bf16 *>(z);
    CUtensorMap th, tv;
    if (!map2d(&th, h, (uint64_t)d, (uint64_t)N, 64, TC_M, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map2d(&tv, V, (uint64_t)p.R, (uint64_t)d, 8, PJ_KC, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorNotSupported;
    const uint32_t smem = z_smem(a.RP);
    static const cudaError_t attr = cudaFuncSetAttribute(k_proj_z, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                         z_smem(64));
    if (attr != cudaSuccess) return attr;
    const int64_t grid = a.ntiles < c.sms ? a.ntiles : c.sms;
    const cudaError_t e = launch_pdl(k_proj_z, dim3((unsigned)grid), dim3(PJ_THREADS), smem, c.stream, th, tv, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// dh [N, d] = dz [N, R] . V^T ; dV [d, R] = h^T . dz (part: per-range partials)
cudaError_t launch_proj_bwd(const Ctx &c, const dsc_problem &p, int64_t d, const void *h, const void *V, const void *dz,
                            void *dh, float *dV, float *part) {
    const int64_t N = p.B * p.T;
    const bool bf = p.dtype == DSC_BF16;
    if (!proj_tc_ok(p, d)) {
        cudaError_t e = launch_gemm(c, (int)N, (int)d, (int)p.R, dz, !bf, p.R, 1, V, !bf, p.R, 1, dh, !bf, d, bf);
        if (e != cudaSuccess) return e;
        return launch_gemm(c, (int)d, (int)p.R, (int)N, h, !bf, 1, d, dz, !bf, 1, p.R, dV, true, p.R, bf);
    }
    ProjArgs a = proj_args(p, d);
    a.dh = static_cast<bf16 *>(dh);
    a.part = part;
    CUtensorMap tdz, tvt, tdh, th;
    if (!map2d(&tdz, dz, (uint64_t)p.R, (uint64_t)N, 8, TC_M, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map2d(&tvt, V, (uint64_t)p.R, (uint64_t)d, 8, PH_NC, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map2d(&th, h, (uint64_t)d, (uint64_t)N, 64, TC_M, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorNotSupported;
    {
        const uint64_t dims[3] = {(uint64_t)d, (uint64_t)N, 1};
        const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)N * d * 2};
        const uint32_t box[3] = {64, TC_M, 1};
        if (!make_map(&tdh, dh, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE))
            return cudaErrorNotSupported;
    }
    static const cudaError_t attr1 = cudaFuncSetAttribute(k_proj_dh, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                          dh_smem(64));
    static const cudaError_t attr2 = cudaFuncSetAttribute(k_proj_dV, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                          dV_smem(64));
    if (attr1 != cudaSuccess) return attr1;
    if (attr2 != cudaSuccess) return attr2;
    const int nch = (int)((d + PH_NC - 1) / PH_NC);
    const int64_t nitems = a.ntiles * nch;
    cudaError_t e = launch_pdl(k_proj_dh, dim3((unsigned)(nitems < c.sms ? nitems : c.sms)), dim3(PH_THREADS), dh_smem(a.RP), c.stream, tdz,
                               tvt, tdh, a, nch);
    if (e != cudaSuccess) return e;
    const int nchV = (int)((d + TC_M - 1) / TC_M);
    const int64_t nr = proj_ranges(p, d, c.sms);
    a.tilesPerRange = (a.ntiles + nr - 1) / nr;
    e = launch_pdl(k_proj_dV, dim3((unsigned)(nchV * nr)), dim3(PJ_THREADS), dV_smem(a.RP), c.stream, th, tdz, a, nchV);
    if (e != cudaSuccess) return e;
    const int64_t n = d * p.R;
    e = launch_pdl(k_proj_dV_sum, dim3((unsigned)min((int64_t)1024, (n + 255) / 256)), dim3(256), 0, c.stream,
                   (const float *)part, nr, n, dV);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace dsc
