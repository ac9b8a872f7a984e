// route.cu -- router select/normalize ("Native router select/normalize" row of
// "Post-Portfolio Device Attribution", "MTP1 Post-Portfolio Eager-Cycle Profile").
//
//  1. route_logits: fp32 partial logits x.W_r^T over H chunks of 512 (H < 4096) or
//     1024 elements.
//     Grid (E/8, H chunks, M/32).  A CTA stages its 32 tokens' x chunk in shared
//     memory once; each warp owns one expert, keeps that expert's W_r chunk in
//     registers (read from HBM once per token tile) and reduces with a fixed
//     xor-butterfly.  The CTAs of expert group 0 also write the binary16 copy of
//     x that the grouped GEMM consumes and reset the call's status words.
//  2. top-k per token, one warp per token: sum the chunk partials in chunk order,
//     add the bias, select the top k by k rounds of a warp arg-max (warp max of
//     order-preserving logit keys, then warp min of the ids holding it: value
//     desc, expert id asc), and renormalise with a softmax over the k selected
//     logits (equal to softmax-over-E followed by renormalisation).
//     Either its own kernel (route_topk), or, for M*k <= kFusedSelectMaxN and
//     E <= kFusedSelectMaxE, fused with the route remap into one single-CTA kernel
//     (route_select_permute).
// Every reduction has a fixed order, so ids and weights are bitwise reproducible.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "permute_impl.cuh"

namespace moe {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v)
{
    __half2 h = __floats2half2_rn(bf16_lo(v), bf16_hi(v));
    return *reinterpret_cast<uint32_t *>(&h);
}

template <int kChunk>
__global__ void __launch_bounds__(256) route_logits_kernel(const uint16_t *__restrict__ x,
                                                           const float *__restrict__ wr, float *__restrict__ partial,
                                                           __half *__restrict__ x16, int *status, int32_t *status_out,
                                                           int M, int H, int E)
{
    extern __shared__ __align__(16) uint16_t xs[];   // [kRouteTokens][kChunk] bf16 bits
    pdl_trigger();
    const int split = blockIdx.y;
    const int h0 = split * kChunk;
    const int len = min(H - h0, kChunk);              // multiple of 32
    const int t0 = blockIdx.z * kRouteTokens;
    const int nt = min(kRouteTokens, M - t0);
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
        if (status) *status = kStatusOk;
        if (status_out) *status_out = kStatusOk;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;

    // this warp's expert chunk of W_r, requested before the x staging so both loads overlap
    constexpr int kVec = kChunk / 128;   // float4 per lane
    float4 w[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
        const int c = 128 * i + 4 * lane;
        w[i] = (e < E && c < len) ? *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(e) * H + h0 + c)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    const int vec_per_row = len / 8;
    const int n_vec = nt * vec_per_row;
    const bool write_x16 = (blockIdx.x == 0) && (x16 != nullptr);
    // a thread's x loads are issued in batches before any is stored, so they overlap
    constexpr int kBatch = 8;
    for (int i0 = threadIdx.x; i0 < n_vec; i0 += kBatch * blockDim.x) {
        uint4 v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * blockDim.x;
            if (i < n_vec) {
                const int r = i / vec_per_row, c = i - r * vec_per_row;
                v[b] = *reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t0 + r) * H + h0 + 8 * c);
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * blockDim.x;
            if (i < n_vec) {
                const int r = i / vec_per_row, c = i - r * vec_per_row;
                *reinterpret_cast<uint4 *>(xs + r * kChunk + 8 * c) = v[b];
                if (write_x16) {
                    uint4 o;
                    o.x = bf16x2_to_f16x2(v[b].x);
                    o.y = bf16x2_to_f16x2(v[b].y);
                    o.z = bf16x2_to_f16x2(v[b].z);
                    o.w = bf16x2_to_f16x2(v[b].w);
                    *reinterpret_cast<uint4 *>(x16 + static_cast<size_t>(t0 + r) * H + h0 + 8 * c) = o;
                }
            }
        }
    }
    __syncthreads();

    if (e >= E) return;

    for (int tg = 0; tg < nt; tg += 8) {
        float acc[8];
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) acc[tt] = 0.f;
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
            const int c = 128 * i + 4 * lane;
            if (c < len) {
#pragma unroll
                for (int tt = 0; tt < 8; ++tt) {
                    if (tg + tt < nt) {
                        const uint2 xv = *reinterpret_cast<const uint2 *>(xs + (tg + tt) * kChunk + c);
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
        // transpose-reduce: 3 halving exchanges leave each lane one token's sum over 8 lanes
        // (token index = lane bits 4,3,2), 2 more levels finish the 32-lane sum; 9 shuffles
        const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
        float r1[4], r2[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float keep = b4 ? acc[i + 4] : acc[i], send = b4 ? acc[i] : acc[i + 4];
            r1[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float keep = b3 ? r1[i + 2] : r1[i], send = b3 ? r1[i] : r1[i + 2];
            r2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        float mine = (b2 ? r2[1] : r2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? r2[0] : r2[1], 4);
        mine += __shfl_xor_sync(0xffffffffu, mine, 2);
        mine += __shfl_xor_sync(0xffffffffu, mine, 1);
        const int tt = 4 * b4 + 2 * b3 + b2;
        if ((lane & 3) == 0 && tg + tt < nt)
            partial[(static_cast<size_t>(split) * M + t0 + tg + tt) * E + e] = mine;
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

// One warp selects token t's top k.  Lane j < k ends with (sel_e, sel_w) of slot j.
// Each round: every lane offers its best untaken (logit, id); a warp max over the
// ordered logit keys and a warp min over the ids of the lanes holding that max pick
// the winner (value desc, ties -> lower id).
template <int kPerLane>
__device__ __forceinline__ void select_topk(const float *__restrict__ partial, const float *__restrict__ bias, int t,
                                            int M, int E, int k, int splits, int &sel_e, float &sel_w)
{
    const int lane = threadIdx.x & 31;
    float v[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
        const int e = lane + 32 * j;
        float s = -CUDART_INF_F;
        if (e < E) {
            // the splits' loads are independent: issue them together, then add in split order
            float part[kMaxRouteSplits];
#pragma unroll
            for (int sp = 0; sp < kMaxRouteSplits; ++sp)
                part[sp] = sp < splits ? partial[(static_cast<size_t>(sp) * M + t) * E + e] : 0.f;
            s = 0.f;
#pragma unroll
            for (int sp = 0; sp < kMaxRouteSplits; ++sp) s += part[sp];
            if (bias) s += bias[e];
        }
        v[j] = s;
    }
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
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ partial,
                                                         const float *__restrict__ bias, int32_t *__restrict__ ids,
                                                         float *__restrict__ wout, int M, int E, int k, int splits)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= M) return;
    int sel_e;
    float sel_w;
    select_topk<kPerLane>(partial, bias, t, M, E, k, splits, sel_e, sel_w);
    if (lane < k) {
        ids[static_cast<size_t>(t) * k + lane] = sel_e;
        wout[static_cast<size_t>(t) * k + lane] = sel_w;
    }
}

// Top-k of every token (warps loop over the tokens) and the route remap, in one CTA of
// kFusedSelectThreads threads, for n = M*k <= kFusedSelectMaxN assignments and E <= kFusedSelectMaxE.
// Thread f owns assignment f.  Its stable rank inside its expert (the number of earlier
// assignments routed to the same expert) is its rank among the matching lanes of its warp
// (__match_any_sync) plus the counts of that expert in the earlier warps, kept in a
// [warp][expert] table that one pass per expert turns into prefix counts.  One block scan
// of (tiles, count) per expert gives every expert offset and tile base; thread f then writes
// its sorted position, inverse position and tile slot directly.  Four block barriers, no sort.
template <int kPerLane>
__global__ void __launch_bounds__(kFusedSelectThreads, 1)
route_select_permute_kernel(const float *__restrict__ partial, const float *__restrict__ bias,
                            int32_t *__restrict__ ids, float *__restrict__ wout, int32_t *__restrict__ offsets,
                            int32_t *__restrict__ sorted_ids, int32_t *__restrict__ inv_pos,
                            ExpertTile *__restrict__ tiles, int *__restrict__ n_tiles, int M, int E, int k, int splits)
{
    constexpr int kWarps = kFusedSelectThreads / 32;
    static_assert(kFusedSelectMaxN <= kFusedSelectThreads, "one thread per assignment");
    __shared__ int s_e[kFusedSelectMaxN];                        // expert of assignment f
    __shared__ uint16_t s_wc[kWarps][kFusedSelectMaxE];          // per-warp counts, then prefix counts
    __shared__ int s_off[kFusedSelectMaxE], s_cnt[kFusedSelectMaxE], s_tb[kFusedSelectMaxE];
    __shared__ int scan_buf[33];
    const int n = M * k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the count table is cleared while the previous kernel may still run
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) s_wc[i / E][i % E] = 0;
    pdl_wait();
    pdl_trigger();
    for (int t = warp; t < M; t += kWarps) {
        int sel_e;
        float sel_w;
        select_topk<kPerLane>(partial, bias, t, M, E, k, splits, sel_e, sel_w);
        if (lane < k) {
            const int f = t * k + lane;
            ids[f] = sel_e;
            wout[f] = sel_w;
            s_e[f] = sel_e;
        }
    }
    __syncthreads();
    // rank among the lanes of this warp routed to the same expert (lanes past n carry -1)
    const int f = threadIdx.x;
    const int e = f < n ? s_e[f] : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(same & ((1u << lane) - 1u));
    if (e >= 0 && rank_w == 0) s_wc[warp][e] = static_cast<uint16_t>(__popc(same));
    __syncthreads();
    // per expert: prefix counts over the warps, the expert's total and its tile count
    int packed = 0;                       // (tiles << 16) | count
    if (threadIdx.x < E) {
        int run = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int c = s_wc[w][threadIdx.x];
            s_wc[w][threadIdx.x] = static_cast<uint16_t>(run);
            run += c;
        }
        packed = (((run + kTileTokens - 1) / kTileTokens) << 16) | run;
        s_cnt[threadIdx.x] = run;
    }
    int total = 0;
    const int base = block_exclusive_scan(packed, scan_buf, total);   // ends with a block barrier
    if (threadIdx.x < E) {
        s_off[threadIdx.x] = base & 0xFFFF;
        s_tb[threadIdx.x] = base >> 16;
        offsets[threadIdx.x] = base & 0xFFFF;
    }
    if (threadIdx.x == 0) {
        offsets[E] = n;
        *n_tiles = total >> 16;
    }
    __syncthreads();
    if (e >= 0) {
        const int rank = s_wc[warp][e] + rank_w;
        const int pos = s_off[e] + rank;
        sorted_ids[pos] = f;
        inv_pos[f] = pos;
        const int cnt = s_cnt[e];
        const int slot = rank % kTileTokens, tile_first = rank - slot;
        ExpertTile *tp = tiles + s_tb[e] + rank / kTileTokens;
        const int t = f / k;
        tp->tok[slot] = t;
        if (slot == 0) {
            tp->expert = e;
            tp->p0 = s_off[e] + tile_first;
            tp->count = min(kTileTokens, cnt - tile_first);
            tp->pad = 0;
        }
        if (rank == cnt - 1)   // the tile's last assignment repeats its token into the unused slots
            for (int j = slot + 1; j < kTileTokens; ++j) tp->tok[j] = t;
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
                                int32_t *status_out, int M, int H, int E, int splits, cudaStream_t s)
{
    const int chunk = route_chunk(H);
    const size_t smem = static_cast<size_t>(kRouteTokens) * chunk * sizeof(uint16_t);
    auto kern = chunk == 1024 ? route_logits_kernel<1024> : route_logits_kernel<512>;
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid((E + 7) / 8, splits, (M + kRouteTokens - 1) / kRouteTokens);
    // first kernel of a call: fully ordered after whatever precedes it in the stream
    kern<<<grid, 256, smem, s>>>(static_cast<const uint16_t *>(x), router_w, partial, x16, status, status_out, M, H, E);
    return cudaGetLastError();
}

template <int P>
static cudaError_t topk_p(const float *partial, const float *bias, int32_t *ids, float *w, int M, int E, int k,
                          int splits, cudaStream_t s, bool pdl)
{
    return launch_ex(route_topk_kernel<P>, dim3((M + 7) / 8), dim3(256), 0, s, pdl, partial, bias, ids, w, M, E, k,
                     splits);
}

cudaError_t launch_route_topk(const float *partial, const float *bias, int32_t *ids, float *w, int M, int E, int k,
                              int splits, cudaStream_t s, bool pdl)
{
    if (E <= 32) return topk_p<1>(partial, bias, ids, w, M, E, k, splits, s, pdl);
    if (E <= 64) return topk_p<2>(partial, bias, ids, w, M, E, k, splits, s, pdl);
    if (E <= 128) return topk_p<4>(partial, bias, ids, w, M, E, k, splits, s, pdl);
    if (E <= 256) return topk_p<8>(partial, bias, ids, w, M, E, k, splits, s, pdl);
    if (E <= 512) return topk_p<16>(partial, bias, ids, w, M, E, k, splits, s, pdl);
    return topk_p<32>(partial, bias, ids, w, M, E, k, splits, s, pdl);
}

template <int P>
static cudaError_t select_permute_p(const float *partial, const float *bias, int32_t *ids, float *w, int32_t *offsets,
                                    int32_t *sorted_ids, int32_t *inv_pos, ExpertTile *tiles, int *n_tiles, int M,
                                    int E, int k, int splits, cudaStream_t s, bool pdl)
{
    return launch_ex(route_select_permute_kernel<P>, dim3(1), dim3(kFusedSelectThreads), 0, s, pdl, partial, bias,
                     ids, w, offsets, sorted_ids, inv_pos, tiles, n_tiles, M, E, k, splits);
}

cudaError_t launch_route_select_permute(const float *partial, const float *bias, int32_t *ids, float *w,
                                        int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, ExpertTile *tiles,
                                        int *n_tiles, int M, int E, int k, int splits, cudaStream_t s, bool pdl)
{
#define MOE_SEL(P) select_permute_p<P>(partial, bias, ids, w, offsets, sorted_ids, inv_pos, tiles, n_tiles, M, E, k, \
                                       splits, s, pdl)
    if (E <= 32) return MOE_SEL(1);
    if (E <= 64) return MOE_SEL(2);
    if (E <= 128) return MOE_SEL(4);
    if (E <= 256) return MOE_SEL(8);
    if (E <= 512) return MOE_SEL(16);
    return MOE_SEL(32);
#undef MOE_SEL
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
