// Thin wrappers over the sm_100a tensor-core (tcgen05) and mbarrier PTX used
// by the dense kernels: shared-memory matrix descriptors for K-major tiles
// with the 128-byte swizzle, the instruction descriptor of a bf16 x bf16 ->
// fp32 MMA, TMEM allocation, MMA issue / commit, and TMEM loads.
//
// Tile layout expected by make_kmajor_sw128_desc: rows of 64 bf16 (128 B)
// at a 128-byte pitch, 16-byte chunk c of row r stored at chunk (c ^ (r % 8)),
// 8-row groups 1024 bytes apart, the tile 1024-byte aligned.  Consecutive
// MMAs along K advance the start address by 32 bytes (16 bf16).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace rosa {
namespace umma {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (row, k) (k < 64) inside a K-major SW128 tile.
__device__ __forceinline__ uint32_t sw128_offset(int row, int k) {
    const int chunk = (k >> 3) ^ (row & 7);
    return (uint32_t)(row * 128 + chunk * 16 + (k & 7) * 2);
}

// Shared-memory matrix descriptor: start address, leading byte offset 16 B
// (unused by swizzled K-major tiles), stride byte offset 1024 B between
// 8-row groups, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t make_kmajor_sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);          // bits  0-13: start address >> 4
    d |= (uint64_t)1 << 16;                            // bits 16-29: leading byte offset >> 4
    d |= (uint64_t)(1024 >> 4) << 32;                  // bits 32-45: stride byte offset >> 4
    d |= (uint64_t)1 << 46;                            // bits 46-47: version
    d |= (uint64_t)2 << 61;                            // bits 61-63: 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: A and B bf16, D fp32, both K-major.
__host__ __device__ constexpr uint32_t make_idesc_bf16_f32(int M, int N) {
    return (1u << 4)                          // D format: fp32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// A waiting thread is suspended until the phase completes or this many
// nanoseconds pass, instead of re-polling the barrier word: the barrier stays
// free for the TMA engine's and the tensor cores' arrivals.
constexpr uint32_t kSuspendNs = 1000000;
// Polls of a bounded wait: about two seconds.
constexpr uint32_t kWaitPolls = 2000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete, at most `limit`
// polls (each suspends the thread for up to kSuspendNs).  Returns false when
// the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t limit = kWaitPolls) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Generic-proxy shared-memory writes -> visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Whole warp: allocate `ncols` TMEM columns (power of two >= 32); the base
// address is written to *slot (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Whole warp.
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// One thread: D[tmem] (+)= A[smem] * B[smem]^T, M x N x 16.
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One thread: arrive on `bar` once every MMA issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Whole warp: 32 consecutive fp32 columns of the warp's 32 TMEM lanes (lane
// i of the warp gets row 32*(warp % 4) + i).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace umma
}  // namespace rosa

// ---------------------------------------------------------------------------
// Tensor Memory Accelerator (TMA) loads, local GPU only (no cluster multicast).
// ---------------------------------------------------------------------------
namespace rosa {
namespace umma {

// One thread: expect `bytes` more transaction bytes on `bar`, then arrive.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One thread: 2-D tiled load of the box at (x, y) (x innermost, in elements;
// x * element size must be a multiple of 16 bytes) into shared memory,
// completing `bar`'s transaction count.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace umma
}  // namespace rosa

namespace rosa {
namespace umma {

// One thread: 2-D tiled store of the box at (x, y) from shared memory (the
// tensor map clips what lies outside the tensor), as one bulk group.
__device__ __forceinline__ void tma_store_2d(const void *tmap, int x, int y, const void *src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(x), "r"(y), "r"(smem_u32(src))
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// One thread: wait until the shared memory of every committed bulk store has
// been read (it may then be overwritten).
__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// One thread: wait until every committed bulk store has completed.
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace umma
}  // namespace rosa
