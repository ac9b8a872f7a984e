// permute.cu -- stand-alone route remap kernel (rank_and_scatter of permute_impl.cuh
// over given topk_ids), and the expert-tile builder and h reordering used by the step-level
// entry points.
#include "permute_impl.cuh"

namespace moe {

// Route remap of given topk_ids (rank_and_scatter in rounds of kPermuteThreads assignments).
__global__ void __launch_bounds__(kPermuteThreads, 1)
permute_kernel(const int32_t *__restrict__ topk_ids, int32_t *__restrict__ offsets, int32_t *__restrict__ sorted_ids,
               int32_t *__restrict__ inv_pos, TileOut to, int n, int E, int k)
{
    extern __shared__ __align__(16) uint8_t smem[];
    int *s_e = reinterpret_cast<int *>(smem + permute_smem_bytes(E));   // [n]
    pdl_wait();                          // topk_ids come from the previous kernel
    pdl_trigger();
    // stage the ids with each thread's loads issued in batches before any is stored
    constexpr int kBatch = 8;
    for (int i0 = threadIdx.x; i0 < n; i0 += kBatch * kPermuteThreads) {
        int v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * kPermuteThreads;
            v[b] = i < n ? topk_ids[i] : -1;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * kPermuteThreads;
            if (i < n) s_e[i] = v[b];
        }
    }
    __syncthreads();
    rank_and_scatter(s_e, n, E, k, rank_smem(smem, E), offsets, sorted_ids, inv_pos, to);
}

// Expert tiles (both kinds) from given offsets / sorted ids; also resets the call's status words.
__global__ void __launch_bounds__(1024, 1) build_tiles_kernel(const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ sorted_ids, TileOut to,
                                                              int *status, int E)
{
    __shared__ int s_off[kMaxE + 1];
    __shared__ int scan_buf[33];
    if (threadIdx.x == 0 && status) {
        status[0] = kStatusOk;
        status[kQueueGateUp] = 0;
        status[kQueueDown] = 0;
        status[kQueueGateUpWide] = 0;
        status[kQueueDownWide] = 0;
        status[kQueueGateUpWideL] = 0;
        status[kQueueDownWideL] = 0;
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    emit_tiles(s_off, E, to, scan_buf, [&](int p) { return static_cast<int>(sorted_ids[p]); });
}

// dst[r] = src[r] with every 8-element group moved from natural to P4 K order (common.cuh).
__global__ void __launch_bounds__(256) rows_to_p4_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                         size_t n_groups)
{
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n_groups) dst[i] = p4_from_natural(src[i]);
}

// xshift[t] = the activation shift of row t of x (x_shift_from_max of its largest |x| bits), one
// warp per row.
__global__ void __launch_bounds__(256) row_shift_kernel(const uint4 *__restrict__ x, int *__restrict__ xshift, int M,
                                                        int H)
{
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= M) return;
    const uint4 *row = x + static_cast<size_t>(t) * (H / 8);
    uint32_t m = 0;
    for (int i = lane; i < H / 8; i += 32) {
        const uint4 v = row[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) m = max(m, max(w[c] & 0x7FFFu, (w[c] >> 16) & 0x7FFFu));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0) xshift[t] = x_shift_from_max(m);
}

cudaError_t launch_row_shift(const __nv_bfloat16 *x, int *xshift, int M, int H, cudaStream_t s)
{
    row_shift_kernel<<<(M + 7) / 8 > 0 ? (M + 7) / 8 : 1, 256, 0, s>>>(reinterpret_cast<const uint4 *>(x), xshift, M, H);
    return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t *ids, int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, TileOut to,
                           int M, int E, int k, cudaStream_t s, bool pdl)
{
    const int n = M * k;
    const int smem = permute_smem_bytes(E) + n * static_cast<int>(sizeof(int));
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(permute_kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_ex(permute_kernel, dim3(1), dim3(kPermuteThreads), smem, s, pdl, ids, offsets, sorted_ids, inv_pos, to,
                     n, E, k);
}

cudaError_t launch_build_tiles(const int32_t *offsets, const int32_t *sorted_ids, TileOut to, int *status, int E,
                               cudaStream_t s)
{
    build_tiles_kernel<<<1, 1024, 0, s>>>(offsets, sorted_ids, to, status, E);
    return cudaGetLastError();
}

cudaError_t launch_rows_to_p4(const __nv_bfloat16 *src, __nv_bfloat16 *dst, size_t n_rows, int cols, cudaStream_t s)
{
    const size_t n_groups = n_rows * static_cast<size_t>(cols) / 8;
    const unsigned blocks = static_cast<unsigned>((n_groups + 255) / 256);
    rows_to_p4_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(reinterpret_cast<const uint4 *>(src),
                                                               reinterpret_cast<uint4 *>(dst), n_groups);
    return cudaGetLastError();
}

}  // namespace moe
