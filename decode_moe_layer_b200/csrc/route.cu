// route.cu -- router select/normalize ("Native router select/normalize" row of
// "Post-Portfolio Device Attribution", "MTP1 Post-Portfolio Eager-Cycle Profile").
//
// Two kernels:
//  1. route_logits: fp32 partial logits x.W_r^T over H chunks of kRouteChunkH.
//     Grid (E/8, H chunks, M/32).  A CTA stages its 32 tokens' x chunk in shared
//     memory once; each warp owns one expert, keeps that expert's W_r chunk in
//     registers (read from HBM exactly once per token tile) and reduces with a
//     fixed xor-butterfly.  The CTAs of expert group 0 also write the binary16 copy
//     of x that the grouped GEMM consumes.
//  2. route_topk: one warp per token.  Sums the chunk partials in chunk order,
//     adds the bias, selects the top k by k rounds of a warp argmax over
//     (value desc, expert id asc), and renormalises with a softmax over the k
//     selected logits (equal to softmax-over-E followed by renormalisation).
// Every reduction has a fixed order, so ids and weights are bitwise reproducible.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "common.cuh"

namespace moe {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v)
{
    __half2 h = __floats2half2_rn(bf16_lo(v), bf16_hi(v));
    return *reinterpret_cast<uint32_t *>(&h);
}

__global__ void __launch_bounds__(256) route_logits_kernel(const uint16_t *__restrict__ x,
                                                           const float *__restrict__ wr, float *__restrict__ partial,
                                                           __half *__restrict__ x16, int *status, int M, int H, int E)
{
    extern __shared__ __align__(16) uint16_t xs[];   // [kRouteTokens][kRouteChunkH] bf16 bits
    const int split = blockIdx.y;
    const int h0 = split * kRouteChunkH;
    const int len = min(H - h0, kRouteChunkH);        // multiple of 32
    const int t0 = blockIdx.z * kRouteTokens;
    const int nt = min(kRouteTokens, M - t0);
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && status) *status = kStatusOk;

    const int vec_per_row = len / 8;
    const bool write_x16 = (blockIdx.x == 0) && (x16 != nullptr);
    for (int i = threadIdx.x; i < nt * vec_per_row; i += blockDim.x) {
        const int r = i / vec_per_row, c = i - r * vec_per_row;
        const size_t g = static_cast<size_t>(t0 + r) * H + h0 + 8 * c;
        uint4 v = *reinterpret_cast<const uint4 *>(x + g);
        *reinterpret_cast<uint4 *>(xs + r * kRouteChunkH + 8 * c) = v;
        if (write_x16) {
            uint4 o;
            o.x = bf16x2_to_f16x2(v.x);
            o.y = bf16x2_to_f16x2(v.y);
            o.z = bf16x2_to_f16x2(v.z);
            o.w = bf16x2_to_f16x2(v.w);
            *reinterpret_cast<uint4 *>(x16 + g) = o;
        }
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    if (e >= E) return;

    constexpr int kVec = kRouteChunkH / 128;   // float4 per lane
    float4 w[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
        const int c = 128 * i + 4 * lane;
        w[i] = (c < len) ? *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(e) * H + h0 + c)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int tg = 0; tg < nt; tg += 8) {
        float acc[8];
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) acc[tt] = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int c = 128 * i + 4 * lane;
            if (128 * i >= len) break;
            if (c < len) {
#pragma unroll
                for (int tt = 0; tt < 8; ++tt) {
                    if (tg + tt < nt) {
                        const uint2 xv = *reinterpret_cast<const uint2 *>(xs + (tg + tt) * kRouteChunkH + c);
                        float a = acc[tt];
                        a = fmaf(bf16_lo(xv.x), w[i].x, a);
                        a = fmaf(bf16_hi(xv.x), w[i].y, a);
                        a = fmaf(bf16_lo(xv.y), w[i].z, a);
                        a = fmaf(bf16_hi(xv.y), w[i].w, a);
                        acc[tt] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], off);
        }
        float mine = 0.f;
#pragma unroll
        for (int tt = 0; tt < 8; ++tt)
            if (tt == lane) mine = acc[tt];
        if (lane < 8 && tg + lane < nt)
            partial[(static_cast<size_t>(split) * M + t0 + tg + lane) * E + e] = mine;
    }
}

template <int kPerLane>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ partial,
                                                         const float *__restrict__ bias, int32_t *__restrict__ ids,
                                                         float *__restrict__ wout, int M, int E, int k, int splits)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= M) return;
    float v[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
        const int e = lane + 32 * j;
        float s = -CUDART_INF_F;
        if (e < E) {
            s = 0.f;
            for (int sp = 0; sp < splits; ++sp) s += partial[(static_cast<size_t>(sp) * M + t) * E + e];
            if (bias) s += bias[e];
        }
        v[j] = s;
    }
    uint32_t taken = 0;
    float sel_v = 0.f, vmax = 0.f;
    int sel_e = 0;
    for (int r = 0; r < k; ++r) {
        float bv = -CUDART_INF_F;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < kPerLane; ++j) {
            const int e = lane + 32 * j;
            if (!((taken >> j) & 1u) && e < E && (v[j] > bv || (v[j] == bv && e < be))) {
                bv = v[j];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == r) {
            sel_v = bv;
            sel_e = be;
        }
        if (r == 0) vmax = bv;
    }
    float ex = (lane < k) ? expf(sel_v - vmax) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
        ids[static_cast<size_t>(t) * k + lane] = sel_e;
        wout[static_cast<size_t>(t) * k + lane] = ex / sum;
    }
}

__global__ void convert_x_kernel(const uint16_t *__restrict__ x, __half *__restrict__ x16, int *status, size_t n8)
{
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i == 0 && status) *status = kStatusOk;
    if (i >= n8) return;
    uint4 v = reinterpret_cast<const uint4 *>(x)[i];
    uint4 o;
    o.x = bf16x2_to_f16x2(v.x);
    o.y = bf16x2_to_f16x2(v.y);
    o.z = bf16x2_to_f16x2(v.z);
    o.w = bf16x2_to_f16x2(v.w);
    reinterpret_cast<uint4 *>(x16)[i] = o;
}

cudaError_t launch_route_logits(const void *x, const float *router_w, float *partial, __half *x16, int *status,
                                int M, int H, int E, int splits, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>(kRouteTokens) * kRouteChunkH * sizeof(uint16_t);
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(route_logits_kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid((E + 7) / 8, splits, (M + kRouteTokens - 1) / kRouteTokens);
    route_logits_kernel<<<grid, 256, smem, s>>>(static_cast<const uint16_t *>(x), router_w, partial, x16, status, M,
                                                H, E);
    return cudaGetLastError();
}

cudaError_t launch_route_topk(const float *partial, const float *bias, int32_t *ids, float *w, int M, int E, int k,
                              int splits, cudaStream_t s)
{
    dim3 grid((M + 7) / 8);
    if (E <= 32) route_topk_kernel<1><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    else if (E <= 64) route_topk_kernel<2><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    else if (E <= 128) route_topk_kernel<4><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    else if (E <= 256) route_topk_kernel<8><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    else if (E <= 512) route_topk_kernel<16><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    else route_topk_kernel<32><<<grid, 256, 0, s>>>(partial, bias, ids, w, M, E, k, splits);
    return cudaGetLastError();
}

cudaError_t launch_convert_x(const void *x, __half *x16, int *status, int M, int H, cudaStream_t s)
{
    const size_t n8 = static_cast<size_t>(M) * H / 8;
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((n8 + threads - 1) / threads);
    convert_x_kernel<<<blocks > 0 ? blocks : 1, threads, 0, s>>>(static_cast<const uint16_t *>(x), x16, status, n8);
    return cudaGetLastError();
}

}  // namespace moe
