// 5th-generation tensor-core helpers (sm_100a): tcgen05.mma with operands in
// shared memory and the fp32 accumulator in tensor memory (TMEM).
//
// Operand layout: K-major, 128-byte swizzle, as the TMA tensor copies of the
// expert kernels write it: a tile of 64 bf16 columns per 128-byte row, rows
// in groups of eight (one 1 KiB swizzle atom), consecutive groups 1 KiB
// apart.  An MMA of K = 16 reads a 32-byte column slice of every row: the
// k-th slice of a 64-column tile starts 32 k bytes after the tile.
//
// Accumulator layout for M = 64 (cta_group::1): row m of the tile lives in
// TMEM lane (m % 16) + 32 (m / 16), column n in TMEM column n; a warp w
// reads lanes 32 (w % 4) .. 32 (w % 4) + 31, so its lanes 0..15 get rows
// 16 (w % 4) .. 16 (w % 4) + 15 (checked on the device against a CPU
// product before use).
#pragma once

#include <cstdint>

namespace moe {

constexpr int UMMA_M = 64;  // weight rows per MMA

// Shared-memory matrix descriptor: start address, leading byte offset 16
// (unused by swizzled K-major layouts), stride byte offset 1024 (between
// 8-row groups), descriptor version 1 (sm_100), swizzle mode 128B.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(16 >> 4) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, both
// operands K-major, M = 64, N = n (a multiple of 8, 8..256).
__device__ __forceinline__ uint32_t umma_idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(UMMA_M >> 4) << 24);
}

// D[tmem] (+)= A[adesc] B[bdesc]^T; accumulate = 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on an mbarrier when every tcgen05 operation this thread
// issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar_saddr) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_saddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_saddr, int cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_saddr), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Eight consecutive fp32 columns of the warp's 32 TMEM lanes (lane i of the
// warp gets TMEM lane base + i), waited for in the same statement so that no
// use of the registers can be scheduled before the load has completed.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}

}  // namespace moe
