// dsa_tcgen05.cuh -- 5th-generation tensor core (tcgen05) helpers for sm_100a:
// tensor-memory allocation, shared-memory matrix descriptors, the int8 MMA,
// completion tracking and tensor-memory loads.
//
// Descriptor formats (fields of the 64-bit shared-memory matrix descriptor and
// the 32-bit instruction descriptor) follow the PTX ISA's tcgen05 chapter.
#pragma once

#include "dsa_tma.cuh"

namespace dsa {
namespace tc {

// ---- tensor memory
// allocate `ncols` columns (power of two >= 32) for the CTA; the base address
// is written to shared memory at `dst`.  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// order tcgen05 operations around a thread synchronisation (barrier, mbarrier)
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// generic-proxy shared-memory writes become visible to the tensor core's async proxy
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- descriptors
// K-major operand tile in shared memory with 64-byte rows and the 64-byte
// swizzle (16-byte chunk c of row r stored at chunk c ^ ((r / 2) % 4)); groups
// of 8 rows are 512 bytes apart.  The tile base must be 512-byte aligned; a
// K offset inside the 64-byte row is added to the start address.
__device__ __forceinline__ uint64_t smem_desc_k64_sw64(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);         // start address
    d |= (uint64_t)1 << 16;                         // leading byte offset (unused with swizzle; 16 B)
    d |= (uint64_t)(512 >> 4) << 32;                // stride byte offset: 8 rows x 64 B
    d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
    d |= (uint64_t)4 << 61;                         // layout: 64-byte swizzle
    return d;
}

// instruction descriptor: int8 x int8 -> int32, both operands K-major, M x N
__device__ __forceinline__ constexpr uint32_t idesc_i8(int M, int N) {
    return (2u << 4)                    // D format: s32
         | (1u << 7)                    // A format: signed 8-bit
         | (1u << 10)                   // B format: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, K = 32 bytes.  One thread issues.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// the mbarrier at `bar` receives one arrival once every tcgen05 operation the
// thread issued so far has completed
__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane (warp w may read
// lanes 32*(w%4) .. +31).  Asynchronous: call wait_ld() before using v.
__device__ __forceinline__ void ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- mbarrier odds and ends used with cp.async producers
// arrival on `bar` once all of this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival)
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

}  // namespace tc
}  // namespace dsa
