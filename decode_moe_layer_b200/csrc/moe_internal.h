// moe_internal.h -- declarations shared by the library's translation units
// (constants, workspace layout, kernel launchers).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -5;

// Grouped GEMM tiling (both projections).
constexpr int kTileTokens = 8;       // assignments per expert tile (one MMA n-tile)
constexpr int kItemMTiles = 4;       // MMA m-tiles (16 weight rows each) per work item
constexpr int kItemRows = 16 * kItemMTiles;
constexpr int kChunkK = 1024;        // K elements per pipeline stage (512 bytes of E2M1 per row)
constexpr int kBoxCols = kChunkK / 256;              // 128-byte TMA box columns per stage
constexpr int kStageBytes = kItemRows * kChunkK / 2; // packed weights of one stage (32 KB)
constexpr int kStageScaleBytes = kItemRows * kChunkK / 32;   // E8M0 bytes of one stage (per-stage mode)
constexpr int kActPitch = kChunkK * 2 + 64;         // one token's binary16 chunk, padded against bank conflicts
constexpr int kActStageBytes = kTileTokens * kActPitch;
constexpr int kStages = 3;
constexpr int kComputeWarps = 16;    // 2 m-tile pairs x 8 K slots
constexpr int kKSlots = kComputeWarps / 2;
constexpr int kEpilogueWarps = 2;
constexpr float kHScale = 1024.0f;   // h is stored as binary16(h * 2^10): exact for |h| >= 2^-27

// E8M0 scales travel with each stage (a TMA box of the scale matrix) when a scale row is a
// multiple of 16 bytes; otherwise the item's scale rows are copied once per item.
__host__ __device__ inline bool per_stage_scales(int K) { return (K / 32) % 16 == 0; }

// Router.
constexpr int kRouteChunkH = 512;    // H elements per partial-logit chunk (H < 4096)
constexpr int kMaxRouteSplits = 16;  // partial-logit chunks at most (H <= 16384)
// Router chunk: 512 elements for H < 4096 (more CTAs), 1024 above (fewer partial sums).
__host__ __device__ inline int route_chunk(int H) { return H >= 4096 ? 1024 : 512; }
__host__ __device__ inline int route_splits(int H) { return (H + route_chunk(H) - 1) / route_chunk(H); }
constexpr int kRouteTokens = 32;     // tokens per router CTA

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kMaxAssignments = 16384;

struct ExpertTile {   // one expert's run of <= kTileTokens consecutive assignments
    int expert;
    int p0;           // first position in the expert-grouped order
    int count;
    int pad;
    int tok[kTileTokens];   // token of each assignment (sorted_ids[p0+i] / k); entries >= count repeat the last
};

// Byte offsets of every buffer inside one call's workspace (256-byte aligned).
struct Layout {
    size_t status, partial, x16, topk_ids, topk_w, offsets, sorted_ids, inv_pos, tiles, n_tiles, h, y, total;
    int route_splits;   // number of H chunks of the router
    int max_tiles;
};

Layout make_layout(int M, int H, int I, int E, int k);

// Shared argument checks of the C entry points (api.cu): the MOE_* status of a shape, and
// recording a failed CUDA call (returns MOE_ERR_CUDA).
int check_dims(int M, int H, int I, int E, int k, bool need_hi);
int cuda_fail(cudaError_t e);

// Launch with an optional programmatic dependency on the previous kernel in the stream
// (the kernel must call pdl_wait() before touching what that kernel writes).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                      Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Router top-k and the permutation run as one single-CTA kernel when M*k <= kFusedSelectMaxN
// and E <= kFusedSelectMaxE; otherwise as route_topk followed by the permutation kernel.
constexpr int kFusedSelectThreads = 1024;
constexpr int kFusedSelectMaxN = 1024;
constexpr int kFusedSelectMaxE = 512;
__host__ __device__ inline bool fused_select(int M, int E, int k)
{
    return static_cast<long long>(M) * k <= kFusedSelectMaxN && E <= kFusedSelectMaxE;
}

// Kernel launchers (return cudaError_t of the launch).
cudaError_t launch_route_logits(const void *x, const float *router_w, float *partial, __half *x16, int *status,
                                int32_t *status_out, int M, int H, int E, int splits, cudaStream_t s);
cudaError_t launch_route_topk(const float *partial, const float *bias, int32_t *ids, float *w, int M, int E, int k,
                              int splits, cudaStream_t s, bool pdl);
cudaError_t launch_route_select_permute(const float *partial, const float *bias, int32_t *ids, float *w,
                                        int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, ExpertTile *tiles,
                                        int *n_tiles, int M, int E, int k, int splits, cudaStream_t s, bool pdl);
cudaError_t launch_permute(const int32_t *ids, int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos,
                           ExpertTile *tiles, int *n_tiles, int M, int E, int k, cudaStream_t s, bool pdl);
cudaError_t launch_build_tiles(const int32_t *offsets, const int32_t *sorted_ids, ExpertTile *tiles, int *n_tiles,
                               int *status, int E, int k, cudaStream_t s);
cudaError_t launch_convert_x(const void *x, __half *x16, int *status, int M, int H, cudaStream_t s);
cudaError_t launch_gate_up(const CUtensorMap &w13_map, const CUtensorMap &s13_map, const uint8_t *w13_s,
                           const __half *x16, const ExpertTile *tiles, const int *n_tiles, __half *h, int *status,
                           int32_t *status_out, int H, int I, int max_tiles, cudaStream_t s, bool pdl);
cudaError_t launch_down(const CUtensorMap &w2_map, const CUtensorMap &s2_map, const uint8_t *w2_s, const __half *h,
                        const int32_t *sorted_ids, const float *topk_w, const ExpertTile *tiles, const int *n_tiles,
                        float *y, int *status, int32_t *status_out, int H, int I, int max_tiles, cudaStream_t s,
                        bool pdl);
cudaError_t launch_combine(const float *y, void *out, int M, int H, int k, cudaStream_t s, bool pdl);

// Row blocks of the down projection per token (one arrival counter each).
__host__ __device__ inline int down_row_blocks(int H) { return (H + kItemRows - 1) / kItemRows; }

int num_sms();

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_max_smem(const void *kernel, int bytes);

}  // namespace moe
