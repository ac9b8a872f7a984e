// common.cuh -- device helpers shared by the MoE kernels (sm_100a).
//
// mbarrier / TMA / bulk-copy wrappers in inline PTX, the warp-level bf16 MMA,
// the exact E2M1 -> bf16 decode, and the bounded wait used by every
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

// One lane of the (converged) warp, chosen by the hardware.  Single-thread issue of tcgen05 and TMA
// instructions goes through it, with the operands computed by the whole warp before: issued from
// a lane-0 branch instead, the issue slowed about tenfold (measured) whenever the SM's other warps
// kept the integer pipes busy.
__device__ __forceinline__ bool elect_one()
{
    uint32_t p;
    asm volatile("{\n\t.reg .pred q;\n\telect.sync _|q, 0xffffffff;\n\tselp.u32 %0, 1, 0, q;\n\t}" : "=r"(p));
    return p != 0;
}

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

// D = A(16x16, row) * B(16x8, col) + C, bf16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                               const float (&c)[4])
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Interleaved K order of the activation operands ("P4" order).  Inside every group of 8
// consecutive K elements the bf16 values are stored as (0,4, 1,5, 2,6, 3,7): the 32-bit word i
// of the group holds elements i (low half) and i + 4 (high half), the pairing the E2M1 decode
// below produces for the weights.  Storage position of element n of a row:
__host__ __device__ __forceinline__ int p4_pos(int n) { return (n & ~7) | ((n & 3) << 1) | ((n >> 2) & 1); }

// Natural-order 8-element group (four bf16x2 words) -> its P4 words, and back.
__device__ __forceinline__ uint4 p4_from_natural(uint4 v)
{
    return make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                      prmt(v.y, v.w, 0x7632u));
}
__device__ __forceinline__ uint4 natural_from_p4(uint4 v)
{
    return make_uint4(prmt(v.x, v.y, 0x5410u), prmt(v.z, v.w, 0x5410u), prmt(v.x, v.y, 0x7632u),
                      prmt(v.z, v.w, 0x7632u));
}

constexpr uint32_t kBf16x2Pow126 = 0x7E807E80u;   // 2^126 in both bf16 halves

// Eight packed E2M1 codes (one 32-bit word; byte i = K elements 2i, 2i+1, low nibble first) ->
// four bf16x2 registers in P4 pairing, register i = (element i, element i + 4), each holding the
// code value times 2^-126.  E2M1 (OCP MX v1.0: sign, 2 exponent bits with bias 1, 1 mantissa bit)
// and bf16 share the sign / exponent / mantissa layout: the code's three magnitude bits placed on
// bf16 bits 6..8 (mantissa MSB and the two exponent LSBs) and its sign on bit 15 read as the code
// value times 2^-126, the subnormal code 0.5 landing on a bf16 subnormal.  One AND isolates the two
// codes 16 bits apart, one multiply by 2^6 + 2^12 moves both fields at once (the copies do not
// overlap) and one AND drops the stray copies.  A bf16 multiply by a power of two then gives the
// exact scaled weight (bf16x2_mxfp4_factor below).
__device__ __forceinline__ void e2m1x8_raw_p4(uint32_t w, uint32_t (&r)[4])
{
    constexpr uint32_t kKeep = 0x81C081C0u;   // bf16 sign + bits 6..8 in both halves
    const uint32_t w8 = w >> 8;
    r[0] = ((w & 0x000F000Fu) * 0x1040u) & kKeep;
    r[1] = ((w & 0x00F000F0u) * 0x104u) & kKeep;
    r[2] = ((w8 & 0x000F000Fu) * 0x1040u) & kKeep;
    r[3] = ((w8 & 0x00F000F0u) * 0x104u) & kKeep;
}

// The code values themselves: e2m1x8_raw_p4 times 2^126 (one exact bf16 multiply per register).
__device__ __forceinline__ void e2m1x8_to_bf16x2_p4(uint32_t w, uint32_t (&r)[4])
{
    e2m1x8_raw_p4(w, r);
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = bf16x2_mul(r[i], kBf16x2Pow126);
}

// bf16x2 factor 2^126 * 2^(e-127) = 2^(e-1) that turns e2m1x8_raw_p4's registers into the weights
// E2M1 * 2^(e-127) with one multiply: a bf16 power of two for E8M0 bytes e <= 128.
__device__ __forceinline__ uint32_t bf16x2_mxfp4_factor(uint32_t e) { return (e + 126u) * 0x00800080u; }

// The block scale 2^(e-127) itself as bf16x2, for every e <= 254 (e = 0: the subnormal 2^-127);
// with a multiply by 2^126 first it scales the raw registers for any e.
__device__ __forceinline__ uint32_t bf16x2_e8m0(uint32_t e)
{
    const uint32_t s = max(e << 7, 0x40u);
    return s | (s << 16);
}

// Exact weights of one word of codes with block scale byte e: r[i] = bf16(E2M1 * 2^(e-127)) in
// both halves whenever that value is a bf16 value (every e <= 252; above, codes of magnitude >= 2
// overflow as the real values would).  `any_large` (warp-uniform: some lane's byte exceeds 128)
// selects the two-multiply form, which is exact for every e.
__device__ __forceinline__ void mxfp4x8_to_bf16x2_p4(uint32_t w, uint32_t e, bool any_large, uint32_t (&r)[4])
{
    e2m1x8_raw_p4(w, r);
    if (!any_large) {
        const uint32_t f = bf16x2_mxfp4_factor(e);
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = bf16x2_mul(r[i], f);
    } else {
        const uint32_t f = bf16x2_e8m0(e);
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = bf16x2_mul(bf16x2_mul(r[i], kBf16x2Pow126), f);
    }
}

// E8M0 byte e -> 2^(e-127) as fp32, exact for every e <= 254 (e = 0 is the fp32 subnormal 2^-127).
__device__ __forceinline__ float e8m0_scale(uint32_t e)
{
    return __int_as_float(max(static_cast<int>(e << 23), 0x00400000));
}

}  // namespace moe
