// tcgen05.cuh -- 5th-generation tensor core (tcgen05) and tensor memory wrappers, sm_100a.
//
// Used by the wide-tile grouped kernel (grouped_wide.cu): a single thread issues
// tcgen05.mma with B in shared memory (K-major, 128-byte swizzle), A in shared memory or in
// tensor memory (TMEM), and the fp32 accumulator in TMEM; tcgen05.commit signals an mbarrier
// when the issued MMAs are complete; tcgen05.st / tcgen05.ld move columns between registers
// and TMEM.
#pragma once

#include <stdint.h>

namespace moe {

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle layout: rows of
// 64 16-bit elements (128 bytes), atoms of 8 rows (1024 bytes) stacked along M/N.  Fields: start address
// >> 4 (bits 0-13), leading byte offset >> 4 (16-29; unused for this layout, 16 bytes), stride
// byte offset >> 4 (32-45: 1024 bytes between 8-row atoms), descriptor version 1 (46-47),
// layout 2 = 128-byte swizzle (61-63).  Advancing K by 16 elements inside the atom adds 32
// bytes to the start address.
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t smem_addr)
{
    uint64_t d = static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16 with bf16 operands: f32 accumulator (bits 4-5 = 1), A and
// B bf16 (bits 7-9 and 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22,
// M >> 4 in bits 24-28.
__host__ __device__ inline uint32_t umma_idesc_bf16(int m, int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// Byte offset of 16-bit element (row r, k) in a K-major 128-byte-swizzled tile of 64-element rows
// (the layout umma_sdesc_sw128 describes and a 128B-swizzled TMA box produces).
__host__ __device__ inline uint32_t sw128_offset(int r, int k)
{
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((((k * 2) >> 4) ^ (r & 7)) << 4) + ((k * 2) & 15));
}

// TMEM allocation: one whole warp; the base address lands in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_dst), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, one kind::f16 instruction (K = 16).  A sits in TMEM with
// lane i = row i and column c holding K elements 2c (low half) and 2c + 1 (high half), so one
// K=16 step spans 8 columns.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane (lane as in tmem_ld16) from registers.
// The store is asynchronous: tmem_wait_st() must follow before the columns are read by anything
// else (the registers themselves are free again as soon as the instruction has issued).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                 "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
                 "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
                 "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
                 : "memory");
}

// Waits until every tcgen05.st this thread issued has completed.
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The mbarrier receives one arrival when every tcgen05 operation this thread issued before
// is complete.
__device__ __forceinline__ void umma_commit(uint32_t mbar_smem)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar_smem)
                 : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane (lane = 32 * (warp % 4) + lane id,
// encoded in bits 16-31 of taddr), then wait for the load.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                   "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                   "=r"(v[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace moe
