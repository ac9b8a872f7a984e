// down_slab.h -- plan and launcher of the down projection fused with the weighted top-k combine
// at decode token counts (down_slab.cu).  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "moe_internal.h"

namespace moe {

constexpr int kSlabRows = 16;                    // output rows of H per CTA: one MMA m-tile
constexpr int kSlabComputeWarps = 8;             // tile i goes to compute warp i mod 8
constexpr int kSlabThreads = (kSlabComputeWarps + 2) * 32;   // + the copy producer and the landing watcher
constexpr int kSlabMaxM = 8;
constexpr int kSlabMaxI = 1024;                  // an expert's slab rows fit one 1024-K stage
constexpr int kSlabTileRows = 8;                 // activation rows of a stage: tiles of width 8
constexpr int kSlabMaxStages = 16;
constexpr int kSlabBoxBytes = kSlabRows * 128;   // one TMA box: 16 rows x 128 bytes of packed E2M1
constexpr int kSlabSmemLimit = 227 * 1024;

// Shared-memory plan of one CTA.  A stage holds one expert tile: the slab's packed weight rows
// (box columns of 16 rows x 128 bytes, 128-byte swizzle), their E8M0 rows (16 x I/32 bytes) and
// up to kSlabTileRows h rows at a pitch that keeps the 16-byte fragment loads of two rows on
// different banks; stages are 1024-byte aligned (the swizzle atom).  After the stages: the fp32
// down rows of every assignment ([M*k][16]), a copy of the call's tile list (kSlabTileInts ints
// per tile, at most M*k tiles), then the ring's barriers and two counters.
constexpr int kSlabTileInts = 12;   // expert, p0, count, pad, flat[0..7]: the head of an ExpertTile
struct SlabPlan {
    int wbytes, sbytes, hpitch, stage_bytes, stages, ys_bytes, tl_off, bars_off, total;
};

__host__ __device__ inline SlabPlan slab_plan(int M, int I, int k)
{
    SlabPlan p;
    const int cols = (I / 2 + 127) / 128;
    p.wbytes = cols * kSlabBoxBytes;
    p.sbytes = cols * 128;
    p.hpitch = 2 * I + ((I / 2) % 32 == 0 ? 64 : 0);
    p.stage_bytes = (p.wbytes + p.sbytes + kSlabTileRows * p.hpitch + 1023) / 1024 * 1024;
    p.ys_bytes = M * k * kSlabRows * 4;
    const int tl_bytes = M * k * kSlabTileInts * 4;
    const int tail = 2 * kSlabMaxStages * 8 + 16;   // barriers, landed count, abort flag
    const int s = (kSlabSmemLimit - 1024 - p.ys_bytes - tl_bytes - tail) / p.stage_bytes;   // 1024: base alignment slack
    p.stages = s > kSlabMaxStages ? kSlabMaxStages : s;
    p.tl_off = p.stages * p.stage_bytes + p.ys_bytes;
    p.bars_off = p.tl_off + tl_bytes;
    p.total = p.bars_off + tail + 1024;
    return p;
}

// The fused kernel serves calls of 1..8 tokens whose experts stream one 1024-K stage per slab
// (I <= 1024) and whose tiles hold at most 8 assignments (tile width 8, no tensor-core tiles), with
// at least two ring stages; every touched expert then has exactly one tile.  Each CTA walks all
// of the call's tiles, so its time grows with their number faster than the unfused pair's, whose
// items spread over every SM.  Measured on the decode-width layer (H 2048, I 768, E 128, top-8):
// at M = 1 (8 tiles) the call takes 32.8 us fused against 36.1 us unfused, at M = 8 (about 51
// tiles) 80.1 against 72.4; the tiny layer (H 1024, I 512, E 16, top-4) at M = 2 (8 tiles) 24.9
// against 28.9.  So it runs where a call can have at most kSlabMaxTiles tiles (min(M*k, E)).
constexpr int kSlabMaxTiles = 8;
__host__ __device__ inline bool slab_enabled(int M, int I, int E, int k, int width, bool wide)
{
    const long long tiles_max = static_cast<long long>(M) * k < E ? static_cast<long long>(M) * k : E;
    return M >= 1 && M <= kSlabMaxM && I <= kSlabMaxI && width == 8 && !wide && tiles_max <= kSlabMaxTiles &&
           slab_plan(M, I, k).stages >= 2;
}

// out[t][r] = sum_j w[t*k + j] * (W2_e h_(t,j))[r] for the tiles' assignments, j ascending, rounded
// to bf16 (or kept in fp32 for an I-sharded share).  wmap: the packed W2 [E*H][I/2] bytes with
// boxes of 16 rows x 128 bytes, 128-byte swizzle.
cudaError_t launch_down_slab(const CUtensorMap &wmap, const uint8_t *w2_s, const __nv_bfloat16 *h_p4,
                             const ExpertTile *tiles, const int *n_tiles, const float *topk_w, void *out,
                             bool f32_out, int *status, int32_t *status_out, int M, int H, int I, int k,
                             cudaStream_t s, bool pdl);

}  // namespace moe
