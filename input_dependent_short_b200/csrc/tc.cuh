// Blackwell (sm_100a) tensor-core helpers: tcgen05 MMA with operands in shared
// memory and the accumulator in tensor memory (TMEM), mbarriers with bounded
// waits, and the shared-memory matrix descriptors.
//
// Operand layout.  Every bf16 operand tile of P rows x Q columns (Q contiguous
// in the source) is stored in shared memory as 8-row x 16-byte "core
// matrices": element (p, q) lives at byte
//     ((p / 8) * (Q / 8) + q / 8) * 128 + (p % 8) * 16 + (q % 8) * 2.
// The same bytes serve as a K-major operand when the rows run along M (or N)
// and the columns along K, and as an MN-major operand when the rows run along
// K and the columns along M (or N); only the two descriptor strides differ:
//     K-major : leading (K) byte offset 128,        stride (M/N) byte offset Q/8*128
//     MN-major: leading (K) byte offset Q/8*128,    stride (M/N) byte offset 128
// (no swizzle; descriptor version 1).
#pragma once

#include <stdint.h>

namespace dsc {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of element (p, q) in a P x Q core-matrix tile.
__host__ __device__ constexpr uint32_t core_off(int p, int q, int Q) {
    return (uint32_t)(((p >> 3) * (Q >> 3) + (q >> 3)) * 128 + (p & 7) * 16 + (q & 7) * 2);
}

// Shared-memory matrix descriptor (no swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version (sm_100)
    return d;             // base offset 0, absolute LBO mode, layout type 0 (no swizzle)
}

// Shared-memory descriptor of a K-major operand written by TMA with a 32-,
// 64- or 128-byte swizzle (`swz` bytes per row): 8-row atoms of `swz`-byte
// rows, sbo = 8 * swz (the next 8 rows), lbo unused; a K step of 16 bf16
// inside a row moves `addr` by 32 bytes.  Layout-type field (bits 61-63):
// 2 = 128-byte, 4 = 64-byte, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_swz(uint32_t addr, uint32_t lbo, uint32_t sbo, int swz) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version (sm_100)
    d |= (uint64_t)(swz == 128 ? 2 : (swz == 64 ? 4 : 6)) << 61;
    return d;
}

// Shared-memory matrix descriptor of a tile written by TMA with 128-byte
// swizzling (rows of 128 bytes, 8-row atoms of 1024 bytes, atom base aligned
// to 1024 bytes; layout type 2).  K-major: the rows run along M/N, sbo = 1024
// (the next 8 rows), lbo unused, and a K step of 16 bf16 inside the 128-byte
// row moves `addr` by 32 bytes.  MN-major: the rows run along K, sbo = 1024
// (the next 8 K rows), lbo = the byte offset of the next 64 M/N elements.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return smem_desc_swz(addr, lbo, sbo, 128);
}

// Instruction descriptor of kind::f16 with bf16 A/B and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4)                        // D format: f32
           | (1u << 7)                      // A format: bf16
           | (1u << 10)                     // B format: bf16
           | ((uint32_t)a_mn_major << 15)   // A major-ness (0 = K-major)
           | ((uint32_t)b_mn_major << 16)   // B major-ness
           | ((uint32_t)(N >> 3) << 17)     // N / 8
           | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier at `bar` completes one arrival when all MMAs this thread issued so far are done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// TMEM allocation (one full warp executes these).
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns: thread i of the warp gets lane
// (warp's quarter base + i), columns [col, col + 8).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the tensor core.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity);

// Wait for phase `parity` of the mbarrier to complete, giving up after about
// `limit` clock cycles; returns false on time-out.  A phase that has already
// completed is found by the non-blocking test (measured: ~13 cycles, against
// ~200 for a suspending try that succeeds at once); otherwise each try
// suspends the thread until the phase completes or about 20 us pass, so a
// waiting warp takes no issue slots.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit) {
    if (mbar_test(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(bar), "r"(parity), "r"(20000)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// One try with a short suspend hint (in ns): true once phase `parity` has
// completed; returns false after at most about `hint_ns`.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// Non-blocking test of phase `parity`.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Prefetch `bytes` (a multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing `bytes` of the mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// One arrival on the mbarrier.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// One arrival that also raises the phase's expected transaction count by `bytes`.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Tensor-memory-access (TMA) tile loads into this CTA's shared memory; the
// mbarrier's transaction count drops by the box's bytes when they land.
// Coordinates are element indices, innermost first; boxes that reach outside
// the tensor are filled with zeros.  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *tmap, int c0, int c1, int c2, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
// TMA tile store from this CTA's shared memory (bulk-group completion; the
// parts of the box outside the tensor are not written).
__device__ __forceinline__ void tma_store_3d(const void *tmap, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// This thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// Byte offset of the 16-byte chunk `chunk` of row `row` in a tile that a TMA
// load wrote with 32-, 64- or 128-byte swizzling (rows of RB = 32, 64 or 128
// bytes, tile base aligned to 1024 bytes): address bits [4, 4+b) are XORed
// with bits [7, 7+b), b = log2(RB / 16).
template <int RB> __device__ __forceinline__ uint32_t swz(int row, int chunk) {
    static_assert(RB == 32 || RB == 64 || RB == 128, "32-, 64- or 128-byte rows");
    const uint32_t off = (uint32_t)row * RB;
    return off + ((((uint32_t)chunk) ^ ((off >> 7) & (RB / 16 - 1))) << 4);
}

}  // namespace tc
}  // namespace dsc
