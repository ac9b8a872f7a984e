// permute.cu -- stand-alone route remap kernel and the expert-tile builder used
// by the step-level entry points (see permute_impl.cuh for the algorithm).
#include "permute_impl.cuh"

namespace moe {

__global__ void __launch_bounds__(1024, 1) permute_kernel(const int32_t *__restrict__ ids, int32_t *__restrict__ offsets,
                                                          int32_t *__restrict__ sorted_ids,
                                                          int32_t *__restrict__ inv_pos, ExpertTile *__restrict__ tiles,
                                                          int *__restrict__ n_tiles, int n, int E, int k, int n2)
{
    extern __shared__ uint32_t keys[];   // n2 (power of two >= n) entries
    __shared__ int s_off[kMaxE + 1];
    __shared__ int scan_buf[33];
    pdl_wait();                          // topk_ids come from the previous kernel
    pdl_trigger();
    for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        uint32_t key = 0xFFFFFFFFu;
        if (i < n) {
            int e = ids[i];
            if (e < 0 || e >= E) e = E;          // out-of-range ids sort after every expert
            key = (static_cast<uint32_t>(e) << 16) | static_cast<uint32_t>(i);
        }
        keys[i] = key;
    }
    __syncthreads();
    sort_and_emit(keys, n, n2, E, k, offsets, sorted_ids, inv_pos, tiles, n_tiles, s_off, scan_buf);
}

// Expert tiles from given offsets / sorted ids; also resets the call's status word.
__global__ void __launch_bounds__(1024, 1) build_tiles_kernel(const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ sorted_ids,
                                                              ExpertTile *__restrict__ tiles, int *__restrict__ n_tiles,
                                                              int *status, int E, int k)
{
    __shared__ int s_off[kMaxE + 1];
    __shared__ int scan_buf[33];
    if (threadIdx.x == 0 && status) *status = kStatusOk;
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    emit_tiles(s_off, E, k, tiles, n_tiles, scan_buf, [&](int p) { return static_cast<int>(sorted_ids[p]); });
}

cudaError_t launch_permute(const int32_t *ids, int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos,
                           ExpertTile *tiles, int *n_tiles, int M, int E, int k, cudaStream_t s, bool pdl)
{
    const int n = M * k;
    const int n2 = pow2_at_least(n);
    const size_t smem = static_cast<size_t>(n2) * sizeof(uint32_t);
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(permute_kernel),
                                    static_cast<int>(kMaxAssignments * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    return launch_ex(permute_kernel, dim3(1), dim3(1024), smem, s, pdl, ids, offsets, sorted_ids, inv_pos, tiles,
                     n_tiles, n, E, k, n2);
}

cudaError_t launch_build_tiles(const int32_t *offsets, const int32_t *sorted_ids, ExpertTile *tiles, int *n_tiles,
                               int *status, int E, int k, cudaStream_t s)
{
    build_tiles_kernel<<<1, 1024, 0, s>>>(offsets, sorted_ids, tiles, n_tiles, status, E, k);
    return cudaGetLastError();
}

}  // namespace moe
