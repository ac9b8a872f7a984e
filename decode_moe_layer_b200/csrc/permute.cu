// permute.cu -- route remap ("Direct M=2 route remap" row of "Post-Portfolio
// Device Attribution", "MTP1 Post-Portfolio Eager-Cycle Profile").
//
// One CTA of 1024 threads.  Each assignment f = t*k + j becomes the unique key
// (expert << 16) | f; a shared-memory bitonic sort of the keys gives the stable
// expert-grouped order directly (keys are unique, so every sort yields the same
// bytes).  Expert offsets are lower bounds found by binary search in the sorted
// keys, and the expert tiles that drive the grouped GEMMs come from a block-wide
// exclusive scan of ceil(count_e / kTileTokens).  No atomics anywhere.
#include "common.cuh"

namespace moe {

// Exclusive scan of one value per thread over a 1024-thread block.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        warp_tot[lane] = wi - w;        // exclusive prefix of the warp totals
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    total = warp_tot[32];
    return warp_tot[warp] + incl - v;
}

__device__ void emit_tiles(const int *off, int E, ExpertTile *tiles, int *n_tiles, int *scan_buf)
{
    const int e = threadIdx.x;
    int cnt = 0;
    if (e < E) cnt = off[e + 1] - off[e];
    const int nt = (cnt + kTileTokens - 1) / kTileTokens;
    int total = 0;
    const int base = block_exclusive_scan(nt, scan_buf, total);
    for (int i = 0; i < nt; ++i) {
        ExpertTile tl;
        tl.expert = e;
        tl.p0 = off[e] + i * kTileTokens;
        tl.count = min(kTileTokens, cnt - i * kTileTokens);
        tl.pad = 0;
        tiles[base + i] = tl;
    }
    if (threadIdx.x == 0) *n_tiles = total;
}

__global__ void __launch_bounds__(1024, 1) permute_kernel(const int32_t *__restrict__ ids, int32_t *__restrict__ offsets,
                                                          int32_t *__restrict__ sorted_ids,
                                                          int32_t *__restrict__ inv_pos, ExpertTile *__restrict__ tiles,
                                                          int *__restrict__ n_tiles, int n, int E, int n2)
{
    extern __shared__ uint32_t keys[];   // n2 (power of two >= n) entries
    __shared__ int s_off[kMaxE + 1];
    __shared__ int scan_buf[33];
    const int tid = threadIdx.x;
    for (int i = tid; i < n2; i += blockDim.x) {
        uint32_t key = 0xFFFFFFFFu;
        if (i < n) {
            int e = ids[i];
            if (e < 0 || e >= E) e = E;          // out-of-range ids sort after every expert
            key = (static_cast<uint32_t>(e) << 16) | static_cast<uint32_t>(i);
        }
        keys[i] = key;
    }
    __syncthreads();
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
    emit_tiles(s_off, E, tiles, n_tiles, scan_buf);
}

__global__ void __launch_bounds__(1024, 1) build_tiles_kernel(const int32_t *__restrict__ offsets,
                                                              ExpertTile *__restrict__ tiles, int *__restrict__ n_tiles,
                                                              int *status, int E)
{
    __shared__ int s_off[kMaxE + 1];
    __shared__ int scan_buf[33];
    if (threadIdx.x == 0 && status) *status = kStatusOk;
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    emit_tiles(s_off, E, tiles, n_tiles, scan_buf);
}

cudaError_t launch_permute(const int32_t *ids, int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos,
                           ExpertTile *tiles, int *n_tiles, int M, int E, int k, cudaStream_t s)
{
    const int n = M * k;
    int n2 = 1;
    while (n2 < n) n2 <<= 1;
    if (n2 < 2) n2 = 2;
    const size_t smem = static_cast<size_t>(n2) * sizeof(uint32_t);
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(permute_kernel),
                                    static_cast<int>(kMaxAssignments * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    permute_kernel<<<1, 1024, smem, s>>>(ids, offsets, sorted_ids, inv_pos, tiles, n_tiles, n, E, n2);
    return cudaGetLastError();
}

cudaError_t launch_build_tiles(const int32_t *offsets, ExpertTile *tiles, int *n_tiles, int *status, int E,
                               cudaStream_t s)
{
    build_tiles_kernel<<<1, 1024, 0, s>>>(offsets, tiles, n_tiles, status, E);
    return cudaGetLastError();
}

}  // namespace moe
