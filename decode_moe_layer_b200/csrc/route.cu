// route.cu -- router select/normalize ("Native router select/normalize" row of
// "Post-Portfolio Device Attribution", "MTP1 Post-Portfolio Eager-Cycle Profile").
//
//  1. route_logits: fp32 logits x.W_r^T on the tensor cores.  x is bf16 (exact in
//     a bf16 MMA); each fp32 W_r value is split exactly into three bf16 terms
//     hi + mid + lo (each residual of an fp32 value after rounding to 8 significant
//     bits is exact in fp32, and the last one has at most 8 significant bits), so
//     three bf16 m16n8k16 MMAs with fp32 accumulation form the fp32 dot product up
//     to accumulation rounding.  A CTA = 16 experts x one token block x the K ranges
//     of its 8 warps (route_plan); each warp splits its W_r slice once per pass and
//     runs it against every token tile.  The 8 warp partials are summed in warp
//     order in shared memory and the CTA writes its slice of partial logits
//     [split][M][E]; the top-k adds the slices in split order.  The CTAs of expert
//     group 0 also write x in the P4 K order (common.cuh) that the grouped GEMMs read;
//     the first CTA resets the call's status words.
//  2. top-k per token, one warp per token: sum the slices, add the bias, select the
//     top k by k rounds of a warp arg-max (warp max of order-preserving logit keys,
//     then warp min of the ids holding it: value desc, expert id asc), and
//     renormalise with a softmax over the k selected logits (equal to
//     softmax-over-E followed by renormalisation).  Either its own kernel
//     (route_topk), or, for small M (fused_select), fused with the route remap into
//     one single-CTA kernel (route_select_permute) that first sums the slices into
//     shared memory with all its threads.
// Every reduction has a fixed order, so ids and weights are bitwise reproducible.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "permute_impl.cuh"

namespace moe {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);   // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&b);
}

// (a, b) -> three bf16x2 registers with hi + mid + lo == (a, b) exactly.
__device__ __forceinline__ void split3_bf16x2(float a, float b, uint32_t &hi, uint32_t &mid, uint32_t &lo)
{
    hi = pack_bf16x2(a, b);
    const float ra = a - bf16_lo(hi), rb = b - bf16_hi(hi);
    mid = pack_bf16x2(ra, rb);
    lo = pack_bf16x2(ra - bf16_lo(mid), rb - bf16_hi(mid));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Fragment K order: inside each 16-K step, thread q (= lane & 3) holds the 4 consecutive K
// elements 4q..4q+3 as MMA k-slots (2q, 2q+1, 2q+8, 2q+9) of both operands, so W_r rows load
// as float4 and x rows as 8-byte words; the MMA sums over the same K either way.
template <int kSteps, int kTiles>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_logits_kernel(const uint16_t *__restrict__ x, const float *__restrict__ wr, float *__restrict__ partial,
                    uint16_t *__restrict__ x_p4, uint32_t *__restrict__ xmax, int *status, int32_t *status_out, int M,
                    int H, int E, int passes)
{
    constexpr int kPassK = 16 * kSteps;
    constexpr int kTokens = 8 * kTiles;
    constexpr int kPitch = kTokens + 8;                 // padded row of the warp partials
    __shared__ __align__(16) float red[kRouteWarps][kRouteExperts][kPitch];
    __shared__ uint32_t xm[kRouteWarps][kTokens];   // per warp and token: largest |x| bits seen
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int e0 = blockIdx.x * kRouteExperts;
    const int split = blockIdx.y;
    const int t0 = blockIdx.z * kTokens;
    const bool write_p4 = (blockIdx.x == 0) && (x_p4 != nullptr);
    pdl_trigger();
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
        if (status) {
            status[0] = kStatusOk;
            status[kQueueGateUp] = 0;
            status[kQueueDown] = 0;
            status[kQueueGateUpWide] = 0;
            status[kQueueDownWide] = 0;
            status[kQueueGateUpWideL] = 0;
            status[kQueueDownWideL] = 0;
        }
        if (status_out) *status_out = kStatusOk;
    }
    const int wg = split * kRouteWarps + warp;              // this warp's index along H
    const int ea = e0 + g, eb = e0 + g + 8;                 // its two W_r rows
    float acc[kTiles][4];
    uint32_t amax[kTiles];   // largest |x| bits of token t0 + 8j + g among this lane's elements
#pragma unroll
    for (int j = 0; j < kTiles; ++j) {
        amax[j] = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[j][r] = 0.f;
    }
    for (int pass = 0; pass < passes; ++pass) {
        const int kw = (wg * passes + pass) * kPassK;       // first K of this pass
        // issue every load of the pass before any use: W_r rows and the token tiles' x words
        float4 wa[kSteps], wb[kSteps];
        uint2 xv[kTiles][kSteps];
#pragma unroll
        for (int s = 0; s < kSteps; ++s) {
            const int kk = kw + 16 * s + 4 * q;
            const bool kin = kk < H;   // H % 32 == 0: a 4-element group is wholly in or out
            wa[s] = (kin && ea < E) ? *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(ea) * H + kk)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            wb[s] = (kin && eb < E) ? *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(eb) * H + kk)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kTiles; ++j) {
                const int t = t0 + 8 * j + g;
                xv[j][s] = (kin && t < M) ? *reinterpret_cast<const uint2 *>(x + static_cast<size_t>(t) * H + kk)
                                          : make_uint2(0u, 0u);
            }
        }
#pragma unroll
        for (int s = 0; s < kSteps; ++s) {
            uint32_t hi[4], mid[4], lo[4];
            split3_bf16x2(wa[s].x, wa[s].y, hi[0], mid[0], lo[0]);   // row g,   K 4q, 4q+1
            split3_bf16x2(wb[s].x, wb[s].y, hi[1], mid[1], lo[1]);   // row g+8, K 4q, 4q+1
            split3_bf16x2(wa[s].z, wa[s].w, hi[2], mid[2], lo[2]);   // row g,   K 4q+2, 4q+3
            split3_bf16x2(wb[s].z, wb[s].w, hi[3], mid[3], lo[3]);   // row g+8, K 4q+2, 4q+3
#pragma unroll
            for (int j = 0; j < kTiles; ++j) {
                if (t0 + 8 * j >= M) continue;   // warp-uniform
                mma_bf16_16816(acc[j], hi, xv[j][s].x, xv[j][s].y);
                mma_bf16_16816(acc[j], mid, xv[j][s].x, xv[j][s].y);
                mma_bf16_16816(acc[j], lo, xv[j][s].x, xv[j][s].y);
            }
        }
        if (write_p4) {
            // lanes q and q ^ 1 hold elements 0..3 and 4..7 of an 8-element group: the even lane
            // writes the group's P4 words 0, 1 = (x0,x4), (x1,x5), the odd one words 2, 3
#pragma unroll
            for (int s = 0; s < kSteps; ++s) {
                const int kk = kw + 16 * s + 4 * q;
#pragma unroll
                for (int j = 0; j < kTiles; ++j) {
                    const uint2 mine = xv[j][s];
                    amax[j] = max(amax[j], max(max(mine.x & 0x7FFFu, (mine.x >> 16) & 0x7FFFu),
                                               max(mine.y & 0x7FFFu, (mine.y >> 16) & 0x7FFFu)));
                    const uint2 other = make_uint2(__shfl_xor_sync(0xffffffffu, mine.x, 1),
                                                   __shfl_xor_sync(0xffffffffu, mine.y, 1));
                    const bool odd = (q & 1) != 0;
                    const uint32_t lo = odd ? other.y : mine.x, hi = odd ? mine.y : other.x;
                    const int t = t0 + 8 * j + g;
                    if (kk < H && t < M)
                        *reinterpret_cast<uint2 *>(x_p4 + static_cast<size_t>(t) * H + (kk & ~7) + (odd ? 4 : 0)) =
                            make_uint2(prmt(lo, hi, 0x5410u), prmt(lo, hi, 0x7632u));
                }
            }
        }
    }
    // warp partials: accumulator rows g, g+8 (experts), columns 2q, 2q+1 of tile j (tokens)
#pragma unroll
    for (int j = 0; j < kTiles; ++j) {
        *reinterpret_cast<float2 *>(&red[warp][g][8 * j + 2 * q]) = make_float2(acc[j][0], acc[j][1]);
        *reinterpret_cast<float2 *>(&red[warp][g + 8][8 * j + 2 * q]) = make_float2(acc[j][2], acc[j][3]);
        if (write_p4) {   // the four lanes of token g hold its 4-element groups of the warp's K
            uint32_t m = amax[j];
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (q == 0) xm[warp][8 * j + g] = m;
        }
    }
    __syncthreads();
    if (write_p4 && xmax != nullptr && threadIdx.x < kTokens) {
        const int t = t0 + threadIdx.x;
        uint32_t m = 0;
#pragma unroll
        for (int w = 0; w < kRouteWarps; ++w) m = max(m, xm[w][threadIdx.x]);
        if (t < M) xmax[static_cast<size_t>(split) * M + t] = m;
    }
    for (int i = threadIdx.x; i < kRouteExperts * kTokens; i += blockDim.x) {
        const int tl = i / kRouteExperts, el = i % kRouteExperts;   // consecutive threads: consecutive experts
        const int e = e0 + el, t = t0 + tl;
        if (e < E && t < M) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kRouteWarps; ++w) v += red[w][el][tl];
            partial[(static_cast<size_t>(split) * M + t) * E + e] = v;
        }
    }
}

// Order-preserving map of fp32 to uint32 (larger float -> larger integer; -inf -> 0x007FFFFF).
__device__ __forceinline__ uint32_t ordered_key(float v)
{
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_ordered_key(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp selects a token's top k from its E logits, lane-strided in v (v[j] = expert
// lane + 32 j, -inf past E).  Lane j < k ends with (sel_e, sel_w) of slot j.  Each round:
// every lane offers its best untaken (logit, id); a warp max over the ordered logit keys and a
// warp min over the ids of the lanes holding that max pick the winner (value desc, ties ->
// lower id).
template <int kPerLane>
__device__ __forceinline__ void topk_from_values(const float (&v)[kPerLane], int E, int k, int &sel_e, float &sel_w)
{
    const int lane = threadIdx.x & 31;
    uint32_t taken = 0;
    float sel_v = 0.f, vmax = 0.f;
    sel_e = 0;
    for (int r = 0; r < k; ++r) {
        float bv = -CUDART_INF_F;
        int be = 0x7fffffff;
        bool any = false;
#pragma unroll
        for (int j = 0; j < kPerLane; ++j) {
            const int e = lane + 32 * j;
            if (!((taken >> j) & 1u) && e < E && (!any || v[j] > bv)) {
                bv = v[j];
                be = e;
                any = true;
            }
        }
        const uint32_t key = any ? ordered_key(bv) : 0u;
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const int win = static_cast<int>(__reduce_min_sync(0xffffffffu, (any && key == kmax) ? static_cast<uint32_t>(be)
                                                                                              : 0xffffffffu));
        if ((win & 31) == lane) taken |= 1u << (win >> 5);
        const float wv = from_ordered_key(kmax);
        if (lane == r) {
            sel_v = wv;
            sel_e = win;
        }
        if (r == 0) vmax = wv;
    }
    const float ex = (lane < k) ? expf(sel_v - vmax) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    sel_w = ex / sum;
}

template <int kPerLane>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ partial, int splits,
                                                         const float *__restrict__ bias, int32_t *__restrict__ ids,
                                                         float *__restrict__ wout, const uint32_t *__restrict__ xmax,
                                                         int *__restrict__ xshift, int M, int E, int k)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= M) return;
    if (xmax != nullptr) {   // the token's activation shift, from its slices' largest |x|
        uint32_t m = 0;
        for (int sp = lane; sp < splits; sp += 32) m = max(m, xmax[static_cast<size_t>(sp) * M + t]);
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) xshift[t] = x_shift_from_max(m);
    }
    float v[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) v[j] = 0.f;
    for (int sp = 0; sp < splits; ++sp) {   // slices in split order; each round's loads are independent
#pragma unroll
        for (int j = 0; j < kPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e < E) v[j] += partial[(static_cast<size_t>(sp) * M + t) * E + e];
        }
    }
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < E ? (bias ? v[j] + bias[e] : v[j]) : -CUDART_INF_F;
    }
    int sel_e;
    float sel_w;
    topk_from_values<kPerLane>(v, E, k, sel_e, sel_w);
    if (lane < k) {
        ids[static_cast<size_t>(t) * k + lane] = sel_e;
        wout[static_cast<size_t>(t) * k + lane] = sel_w;
    }
}

// Sums of the partial-logit slices in split order (+ bias) into dst[0..n_log), by all threads.
// A thread keeps kBatch logits x kChunk slices of loads in flight before adding them.
template <int kBatch, int kChunk>
__device__ __forceinline__ void stage_logits(const float *__restrict__ partial, int splits, const float *__restrict__ bias,
                                             int n_log, int E, float *dst)
{
    for (int i0 = threadIdx.x; i0 < n_log; i0 += kBatch * blockDim.x) {
        float acc[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) acc[b] = 0.f;
        for (int sp0 = 0; sp0 < splits; sp0 += kChunk) {
            float v[kBatch][kChunk];
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
#pragma unroll
                for (int u = 0; u < kChunk; ++u) {
                    const int i = i0 + b * blockDim.x;
                    v[b][u] = (i < n_log && sp0 + u < splits) ? partial[static_cast<size_t>(sp0 + u) * n_log + i] : 0.f;
                }
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
#pragma unroll
                for (int u = 0; u < kChunk; ++u) acc[b] += v[b][u];
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * blockDim.x;
            if (i < n_log) dst[i] = bias ? acc[b] + bias[i % E] : acc[b];
        }
    }
}

// Top-k of every token and the route remap, in one CTA of kPermuteThreads threads, when
// fused_select(M, E, k) (M <= 64): all threads sum the partial-logit slices into shared memory,
// warps take the tokens' top-k and mark each chosen expert's token mask, warp 0 scans the
// experts' counts into offsets and tile bases, then every thread places assignments (stable rank
// = earlier tokens in the expert's mask).
template <int kPerLane>
__global__ void __launch_bounds__(kPermuteThreads, 1)
route_select_permute_kernel(const float *__restrict__ partial, int splits, const float *__restrict__ bias,
                            int32_t *__restrict__ ids, float *__restrict__ wout, int32_t *__restrict__ offsets,
                            int32_t *__restrict__ sorted_ids, int32_t *__restrict__ inv_pos, TileOut to,
                            const uint32_t *__restrict__ xmax, int M, int E, int k)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_e[kPermuteThreads];                    // expert of assignment f
    __shared__ unsigned long long s_mask[kMaxE];            // bit t: token t chose the expert
    __shared__ int s_off[kMaxE], s_tb[kMaxE];                // first position, first mma.sync tile
    __shared__ int s_wb[kMaxE], s_wbl[kMaxE];                // first small / large tensor-core tile
    __shared__ int s_shift[kFusedSelectMaxM];                // per token: activation shift of the mma.sync tiles
    float *s_log = reinterpret_cast<float *>(smem);         // [M][E]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_mask[e] = 0ull;
    if (xmax != nullptr) {
        for (int t = threadIdx.x; t < M; t += blockDim.x) {
            uint32_t m = 0;
            for (int sp = 0; sp < splits; ++sp) m = max(m, xmax[static_cast<size_t>(sp) * M + t]);
            s_shift[t] = x_shift_from_max(m);
        }
        to.shift = s_shift;
    }
    const int n_log = M * E;
    if (n_log <= kPermuteThreads)
        stage_logits<1, 32>(partial, splits, bias, n_log, E, s_log);
    else
        stage_logits<4, 8>(partial, splits, bias, n_log, E, s_log);
    __syncthreads();
    for (int t = warp; t < M; t += kPermuteThreads / 32) {
        float v[kPerLane];
#pragma unroll
        for (int j = 0; j < kPerLane; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? s_log[t * E + e] : -CUDART_INF_F;
        }
        int sel_e;
        float sel_w;
        topk_from_values<kPerLane>(v, E, k, sel_e, sel_w);
        if (lane < k) {
            const int f = t * k + lane;
            ids[f] = sel_e;
            wout[f] = sel_w;
            s_e[f] = sel_e;
            atomicOr(&s_mask[sel_e], 1ull << t);
        }
    }
    __syncthreads();
    if (warp == 0) warp_scan_experts(s_mask, E, to, s_off, s_tb, s_wb, s_wbl, offsets);
    __syncthreads();
    const int n = M * k;
    for (int f = threadIdx.x; f < n; f += blockDim.x) {
        const int e = s_e[f], t = f / k;
        const unsigned long long mk = s_mask[e];
        scatter_assignment(f, e, __popcll(mk & ((1ull << t) - 1ull)), __popcll(mk), s_off, s_tb, s_wb, s_wbl,
                           sorted_ids, inv_pos, to);
    }
}

template <int kSteps, int kTiles>
static cudaError_t logits_launch(const void *x, const float *router_w, float *partial, void *x_p4, uint32_t *xmax,
                                 int *status, int32_t *status_out, int M, int H, int E, const RoutePlan &plan,
                                 cudaStream_t s)
{
    const dim3 grid((E + kRouteExperts - 1) / kRouteExperts, plan.splits, plan.blocks_t);
    // first kernel of a call: fully ordered after whatever precedes it in the stream
    route_logits_kernel<kSteps, kTiles><<<grid, kRouteWarps * 32, 0, s>>>(
        static_cast<const uint16_t *>(x), router_w, partial, static_cast<uint16_t *>(x_p4), xmax, status, status_out,
        M, H, E, plan.passes);
    return cudaGetLastError();
}

cudaError_t launch_route_logits(const void *x, const float *router_w, float *partial, void *x_p4, uint32_t *xmax,
                                int *status, int32_t *status_out, int M, int H, int E, cudaStream_t s)
{
    const RoutePlan plan = route_plan(M, H, E);
    if (plan.tiles == 1 && plan.steps == 2)
        return logits_launch<2, 1>(x, router_w, partial, x_p4, xmax, status, status_out, M, H, E, plan, s);
    if (plan.tiles == 4 && plan.steps == 4)
        return logits_launch<4, 4>(x, router_w, partial, x_p4, xmax, status, status_out, M, H, E, plan, s);
    return cudaErrorInvalidConfiguration;   // route_plan yields only the two shapes above
}

template <int P>
static cudaError_t topk_p(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                          const uint32_t *xmax, int *xshift, int M, int E, int k, cudaStream_t s, bool pdl)
{
    return launch_ex(route_topk_kernel<P>, dim3((M + 7) / 8), dim3(256), 0, s, pdl, partial, splits, bias, ids, w,
                     xmax, xshift, M, E, k);
}

cudaError_t launch_route_topk(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                              const uint32_t *xmax, int *xshift, int M, int E, int k, cudaStream_t s, bool pdl)
{
    if (E <= 32) return topk_p<1>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
    if (E <= 64) return topk_p<2>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
    if (E <= 128) return topk_p<4>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
    if (E <= 256) return topk_p<8>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
    if (E <= 512) return topk_p<16>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
    return topk_p<32>(partial, splits, bias, ids, w, xmax, xshift, M, E, k, s, pdl);
}

template <int P>
static cudaError_t select_permute_p(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                                    int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, TileOut to,
                                    const uint32_t *xmax, int M, int E, int k, cudaStream_t s, bool pdl)
{
    const int smem = M * E * static_cast<int>(sizeof(float));
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(route_select_permute_kernel<P>), smem);
    if (e != cudaSuccess) return e;
    return launch_ex(route_select_permute_kernel<P>, dim3(1), dim3(kPermuteThreads), smem, s, pdl, partial, splits,
                     bias, ids, w, offsets, sorted_ids, inv_pos, to, xmax, M, E, k);
}

cudaError_t launch_route_select_permute(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                                        int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, TileOut to,
                                        const uint32_t *xmax, int M, int E, int k, cudaStream_t s, bool pdl)
{
#define MOE_SEL(P) select_permute_p<P>(partial, splits, bias, ids, w, offsets, sorted_ids, inv_pos, to, xmax, M, E, k, s, pdl)
    if (E <= 32) return MOE_SEL(1);
    if (E <= 64) return MOE_SEL(2);
    if (E <= 128) return MOE_SEL(4);
    if (E <= 256) return MOE_SEL(8);
    if (E <= 512) return MOE_SEL(16);
    return MOE_SEL(32);
#undef MOE_SEL
}

}  // namespace moe
