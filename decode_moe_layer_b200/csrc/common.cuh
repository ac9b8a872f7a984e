// common.cuh -- device helpers shared by the MoE kernels (sm_100a).
//
// mbarrier / TMA / bulk-copy wrappers in inline PTX, the warp-level f16 MMA,
// the hardware E2M1 -> f16x2 decode, and the bounded wait used by every
// producer/consumer handshake (a wait that gives up records MOE_ERR_TIMEOUT in
// the call's status word and lets the kernel run to completion instead of
// spinning forever).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {

// ------------------------------------------------------------------ status

// ~2 s at 2 GHz: far above any legitimate wait inside one layer call.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Where a call's device status goes: the workspace word, and the caller's optional slot.
struct StatusPtrs {
    int *ws;
    int32_t *out;
};

__device__ __forceinline__ void record_timeout(const StatusPtrs &st)
{
    if (st.ws) atomicExch(st.ws, kStatusTimeout);
    if (st.out) atomicExch(st.out, kStatusTimeout);
}

// ------------------------------------------------------------------ programmatic dependent launch

// Block until the grids this one depends on have completed and their writes are visible
// (returns at once when the kernel was launched without a programmatic dependency).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel in the stream to begin launching; it still waits in pdl_wait().
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ shared-memory addressing

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Once a wait
// has timed out (`aborted` set) later waits return at once, so every thread
// still reaches every CTA barrier and the kernel ends.  kLimit is in SM clock
// cycles (the kernels use kWaitLimitCycles; the wait self-test a short limit).
template <long long kLimit = kWaitLimitCycles>
__device__ __forceinline__ void mbar_wait(uint64_t *bar, uint32_t parity, bool &aborted, const StatusPtrs &st)
{
    if (aborted) return;
    if (mbar_try_wait(bar, parity)) return;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kLimit) {
            aborted = true;
            record_timeout(st);
            return;
        }
    }
}

// Bounded wait for copies already issued to land before a CTA exits.  It runs even after an
// earlier wait gave up: shared memory must not be released with copies still in flight.
__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity, const StatusPtrs &st)
{
    bool gave_up = false;
    mbar_wait(bar, parity, gave_up, st);
}

// ------------------------------------------------------------------ bulk copies (TMA engine)

// 2-D tiled tensor copy global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ------------------------------------------------------------------ MMA + decode

// D = A(16x16, row) * B(16x8, col) + C, f16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                              const float (&c)[4])
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// Four packed E2M1 pairs (one 32-bit word, byte i = K elements 2i, 2i+1, low
// nibble first) -> four f16x2 registers holding the exact element values.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                                uint32_t &r3)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
        : "r"(w));
}

// E8M0 byte e -> 2^(e-126) as fp32 (twice the block scale; valid for e <= 253).
// The factor 2 is removed once per output, keeping e = 0 (2^-127) exact.
__device__ __forceinline__ float e8m0_times2(uint32_t e)
{
    return __int_as_float(static_cast<int>((e + 1u) << 23));
}

}  // namespace moe
