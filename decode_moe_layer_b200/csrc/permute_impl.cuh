// permute_impl.cuh -- route remap device code shared by the stand-alone
// permutation kernel and the fused router-select + permutation kernel.
//
// "Direct M=2 route remap" row of "Post-Portfolio Device Attribution" ("MTP1
// Post-Portfolio Eager-Cycle Profile").  Each assignment f = t*k + j is the
// unique key (expert << 16) | f; a shared-memory bitonic sort of the keys gives
// the stable expert-grouped order directly (keys are unique, so every sort
// yields the same bytes).  Expert offsets are lower bounds found by binary
// search in the sorted keys, and the expert tiles that drive the grouped GEMMs
// come from a block-wide exclusive scan of ceil(count_e / kTileTokens).  No
// atomics.  All functions are called by every thread of the CTA (a multiple of 32 threads).
#pragma once

#include "common.cuh"

namespace moe {

// Exclusive scan of one value per thread over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        if (lane < nwarps) warp_tot[lane] = wi - w;      // exclusive prefix of the warp totals
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    total = warp_tot[32];
    return warp_tot[warp] + incl - v;
}

// sorted_flat(p) returns the flat assignment id at position p of the expert-grouped order.
// Each thread owns a contiguous run of ceil(E / blockDim) experts.
template <typename SortedFlat>
__device__ inline void emit_tiles(const int *off, int E, int k, ExpertTile *tiles, int *n_tiles, int *scan_buf,
                                  SortedFlat sorted_flat)
{
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = threadIdx.x * per, e1 = min(E, e0 + per);
    int mine = 0;
    for (int e = e0; e < e1; ++e) mine += (off[e + 1] - off[e] + kTileTokens - 1) / kTileTokens;
    int total = 0;
    int base = block_exclusive_scan(mine, scan_buf, total);
    for (int e = e0; e < e1; ++e) {
        const int cnt = off[e + 1] - off[e];
        for (int i = 0; i * kTileTokens < cnt; ++i) {
            ExpertTile tl;
            tl.expert = e;
            tl.p0 = off[e] + i * kTileTokens;
            tl.count = min(kTileTokens, cnt - i * kTileTokens);
            tl.pad = 0;
#pragma unroll
            for (int j = 0; j < kTileTokens; ++j) tl.tok[j] = sorted_flat(tl.p0 + min(j, tl.count - 1)) / k;
            tiles[base++] = tl;
        }
    }
    if (threadIdx.x == 0) *n_tiles = total;
}

// keys[0..n2) hold the n assignment keys followed by 0xFFFFFFFF padding (n2 a power of two).
// Sorts them, then writes expert_offsets [E+1], sorted_ids [n], inv_pos [n] and (when
// tiles != nullptr) the expert tiles.  s_off must hold E+1 ints, scan_buf 33.
__device__ inline void sort_and_emit(uint32_t *keys, int n, int n2, int E, int k, int32_t *__restrict__ offsets,
                              int32_t *__restrict__ sorted_ids, int32_t *__restrict__ inv_pos,
                              ExpertTile *__restrict__ tiles, int *__restrict__ n_tiles, int *s_off, int *scan_buf)
{
    const int tid = threadIdx.x;
    for (int size = 2; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < (n2 >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const uint32_t a = keys[lo], b = keys[hi];
                if ((a > b) == up) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }
    for (int e = tid; e <= E; e += blockDim.x) {
        const uint32_t target = static_cast<uint32_t>(e) << 16;
        int lo = 0, hi = n;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (keys[mid] < target) lo = mid + 1;
            else hi = mid;
        }
        s_off[e] = lo;
        offsets[e] = lo;
    }
    for (int p = tid; p < n; p += blockDim.x) {
        const int f = static_cast<int>(keys[p] & 0xFFFFu);
        sorted_ids[p] = f;
        inv_pos[f] = p;
    }
    if (tiles == nullptr) return;
    __syncthreads();
    emit_tiles(s_off, E, k, tiles, n_tiles, scan_buf, [&](int p) { return static_cast<int>(keys[p] & 0xFFFFu); });
}

__host__ __device__ inline int pow2_at_least(int n)
{
    int n2 = 2;
    while (n2 < n) n2 <<= 1;
    return n2;
}

}  // namespace moe
