// moe_internal.h -- declarations shared by the library's translation units
// (constants, workspace layout, kernel launchers).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -5;
// The call's 256-byte status block: word 0 is the status; words kQueueGateUp and kQueueDown
// are the grouped kernels' work-queue counters, zeroed by the first kernel of the call.
constexpr int kQueueGateUp = 8;
constexpr int kQueueDown = 16;
constexpr int kQueueGateUpWide = 24;    // tensor-core launches: small tiles
constexpr int kQueueDownWide = 32;
constexpr int kQueueGateUpWideL = 40;   // and large tiles
constexpr int kQueueDownWideL = 48;

// Grouped GEMM tiling (both projections).
// An expert tile holds up to 8 or 16 assignments (tile_width): one or two MMA n-tiles of 8.
constexpr int kTileTokensMax = 16;
constexpr int kItemMTiles = 4;       // MMA m-tiles (16 weight rows each) per work item
constexpr int kItemRows = 16 * kItemMTiles;
constexpr int kChunkK = 1024;        // K elements per pipeline stage (512 bytes of E2M1 per row)
constexpr int kBoxCols = kChunkK / 256;              // 128-byte TMA box columns per stage
constexpr int kStageBytes = kItemRows * kChunkK / 2; // packed weights of one stage (32 KB)
constexpr int kStageScaleBytes = kItemRows * kChunkK / 32;   // E8M0 bytes of one stage (per-stage mode)
constexpr int kActPitch = kChunkK * 2 + 64;         // one token's bf16 chunk, padded against bank conflicts
constexpr int kStages = 3;
constexpr int kComputeWarps = 16;    // 2 m-tile pairs x 8 K slots
constexpr int kWarpMTiles = 2;       // m-tiles per compute warp (the activation fragment serves both)
constexpr int kKSlots = kComputeWarps * kWarpMTiles / kItemMTiles;
constexpr int kEpilogueWarps = 2;

// E8M0 scales travel with each stage (a TMA box of the scale matrix) when a scale row is a
// multiple of 16 bytes; otherwise the item's scale rows are copied once per item.
__host__ __device__ inline bool per_stage_scales(int K) { return (K / 32) % 16 == 0; }

// Router logits on the tensor cores (route_plan picks the launch).  A CTA covers 16 experts,
// one token block (8 tokens per MMA n-tile, `tiles` n-tiles) and `passes` K ranges of
// 8 warps x 16 * steps elements; the `splits` CTAs of one expert group and token block cover H
// between them and each writes its partial logits [split][M][E], summed in split order by
// the top-k.  Small M: one n-tile and short K ranges, so hundreds of light CTAs share the
// W_r read; large M: full-H CTAs (splits = 1) looping over their K ranges.  The plan uses a
// fixed SM count so that workspace sizes do not depend on the device.
constexpr int kRouteExperts = 16;
constexpr int kRouteWarps = 8;
constexpr int kPlanSMs = 148;
struct RoutePlan {
    int tiles;    // MMA n-tiles (8 tokens) per token block: 1 or 4
    int steps;    // 16-K MMA steps per pass: 2 or 4
    int splits;   // CTAs per (expert group, token block), each a partial-logit slice
    int passes;   // K ranges per warp
    int blocks_t; // token blocks
};
__host__ __device__ inline RoutePlan route_plan(int M, int H, int E)
{
    RoutePlan p;
    p.tiles = M <= 8 ? 1 : 4;
    p.steps = M <= 8 ? 2 : 4;   // 4: two CTAs' registers fit one SM
    p.blocks_t = (M + 8 * p.tiles - 1) / (8 * p.tiles);
    const int gx = (E + kRouteExperts - 1) / kRouteExperts;
    const int units = (H + kRouteWarps * 16 * p.steps - 1) / (kRouteWarps * 16 * p.steps);
    const long long base = static_cast<long long>(gx) * p.blocks_t;
    const int cap = (p.tiles == 1 ? 4 : 2) * kPlanSMs;   // resident CTAs per SM: 4 light ones, 2 heavy ones
    if (base * units <= cap) {
        p.splits = units;
    } else {
        const long long sp = cap / base;
        p.splits = sp < 1 ? 1 : static_cast<int>(sp);
    }
    p.passes = (units + p.splits - 1) / p.splits;
    return p;
}

constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kMaxAssignments = 16384;

// Activation shift of the mma.sync kernels (grouped_gemm.cu): they multiply each token's bf16
// activations by 2^s, s = clamp(120 - (exponent of the token's largest |x|), -7, 127), so that the
// weights can enter the MMA undecoded-scale (E2M1 value x 2^-126) and every product stays inside
// fp32's normal range; the epilogue multiplies the sums back by 2^(126 - s).  Both scalings are
// powers of two, so the fp32 sums are the same numbers times 2^(s - 126).  m: the largest bf16
// magnitude bits (|x| bits, 0 .. 0x7F7F) of the token's row.
__host__ __device__ inline int x_shift_from_max(uint32_t m)
{
    const int s = 247 - static_cast<int>(m >> 7);   // 120 - (biased exponent - 127)
    return s < -7 ? -7 : (s > 127 ? 127 : s);
}
constexpr int kHShift = 120;   // the same for h (|h| <= 49 < 2^6): a fixed shift

__device__ __forceinline__ int tile_flat_id(int packed) { return packed & 0xFFFFFF; }
__device__ __forceinline__ int tile_shift(int packed) { return packed >> 24; }   // arithmetic: signed

struct ExpertTile {   // one expert's run of <= tile_width consecutive assignments
    int expert;
    int p0;           // first position in the expert-grouped order
    int count;
    int pad;
    int flat[kTileTokensMax];   // flat assignment id t*k + j of each slot (sorted_ids[p0+i]) with its token's
                                // activation shift in the top byte (pack_flat); slots count..width-1
                                // repeat the last, slots past the width are not written
};

// Tile width of a call: 16 assignments (two n-tiles per decoded weight fragment) once the
// experts average at least 6 assignments, else 8.  Wider tiles stream each expert's weights
// once for up to 16 assignments at the price of twice the MMAs per decoded fragment, larger
// per-item buffers and a single partial-sum buffer, which only pays when many experts hold
// more than 8.
__host__ __device__ inline int tile_width(int M, int E, int k)
{
    return static_cast<long long>(M) * k >= 6LL * E ? 16 : 8;
}

// Experts with at least kWideMinTokens assignments go to the tensor-core path (grouped_wide.cu),
// when the call enables it: one small tile if they have at most kWideSmallMax, else large tiles
// of up to kWideTokens consecutive assignments.  The path is enabled
// (wide_enabled): H and I multiples of its 512-element packed stage, M >= kWideMinTokens (no
// expert can exceed M assignments), and on average at least kWideMinTokens / 2 assignments per
// expert, so that decode-size calls, whose experts hold one or two assignments, skip its three
// launches.  Every other expert streams its weights as mma.sync tiles of 8 or 16 assignments
// (grouped_gemm.cu).
constexpr int kWideTokens = 192;   // the large-tile kernel's MMA N: two 192-column accumulators + A units fill TMEM
constexpr int kWideSmallMax = 64;  // an expert with up to this many assignments is one small tile
constexpr int kWideStageK = 512;
// Measured (DeepSeek-class layer): 5 beats 9 by 10% at M=256 and 3% at M=512, and the path stays off
// at M <= 32 (average below 2.5), where mma.sync wins; 13 and 17 are slower.
constexpr int kWideMinTokens = 5;
struct WideTile {
    int expert;
    int p0;      // first position in the expert-grouped order
    int count;   // assignments, 1 .. kWideTokens
    int pad;
};
// The two tensor-core tile lists of a call (small: one tile per expert with kWideMinTokens ..
// kWideSmallMax assignments; large: tiles of up to kWideTokens of the experts with more).
struct WideLists {
    WideTile *small;
    int *n_small;
    WideTile *large;
    int *n_large;
    int max_small, max_large;
};
__host__ __device__ inline bool wide_small_expert(int c) { return c >= kWideMinTokens && c <= kWideSmallMax; }
__host__ __device__ inline bool wide_large_expert(int c) { return c > kWideSmallMax; }
__host__ __device__ inline int wide_large_tiles(int c) { return (c + kWideTokens - 1) / kWideTokens; }
__host__ __device__ inline bool wide_enabled(int M, int H, int I, int E, int k)
{
    return M >= kWideMinTokens && H % kWideStageK == 0 && I % kWideStageK == 0 &&
           2LL * M * k >= static_cast<long long>(kWideMinTokens) * E;
}

// Byte offsets of every buffer inside one call's workspace (256-byte aligned).
struct Layout {
    size_t status, partial, x_p4, xmax, xshift, topk_ids, topk_w, offsets, sorted_ids, inv_pos, tiles, n_tiles, h, y;
    size_t wide_small, n_wide_small, wide_large, n_wide_large, x_perm, total;
    int splits;   // router partial-logit slices (route_plan)
    int width;    // tile_width
    int max_tiles, max_small, max_large;
    bool wide;    // wide_enabled for this shape
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

// Router top-k and the permutation run as one single-CTA kernel when M <= kFusedSelectMaxM,
// M*k <= kPermuteThreads (one ranking round) and the M*E logits fit in shared memory; otherwise as route_topk (one warp per token
// across the grid) followed by the permutation kernel (one ranking round per kPermuteThreads
// assignments).  Both use kPermuteThreads threads.
constexpr int kPermuteThreads = 1024;
constexpr int kFusedSelectMaxM = 64;
constexpr int kFusedSelectMaxLogits = 16384;   // M * E logits staged in shared memory (64 KB)
__host__ __device__ inline bool fused_select(int M, int E, int k)
{
    return M <= kFusedSelectMaxM && static_cast<long long>(M) * k <= kPermuteThreads &&
           static_cast<long long>(M) * E <= kFusedSelectMaxLogits;
}
// Dynamic shared memory of the ranking (rank_smem): two [warp][expert] u16 tables (counts and
// prefix counts), six int arrays over E and a 33-int scan buffer.
__host__ __device__ inline int permute_smem_bytes(int E)
{
    return 2 * (kPermuteThreads / 32) * E * 2 + 6 * E * 4 + 64 * 4;
}

// Kernel launchers (return cudaError_t of the launch).
// x_p4 (nullable): x [M, H] rewritten in P4 K order for the grouped GEMMs.
// xmax (when x_p4 is written): per H slice and token, the largest bf16 magnitude bits of x's row
// in the slice, uint32 [splits][M]; the top-k kernels turn them into the per-token shifts.
cudaError_t launch_route_logits(const void *x, const float *router_w, float *partial, void *x_p4, uint32_t *xmax,
                                int *status, int32_t *status_out, int M, int H, int E, cudaStream_t s);
cudaError_t launch_route_topk(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                              const uint32_t *xmax, int *xshift, int M, int E, int k, cudaStream_t s, bool pdl);
// Per-token shifts straight from x rows (the step-level gate_up entry point, which has no router).
cudaError_t launch_row_shift(const __nv_bfloat16 *x, int *xshift, int M, int H, cudaStream_t s);
// Tile outputs of the route remap: tiles of `width` (8 or 16) assignments for the mma.sync
// kernels and, when wide_tiles is set, wide tiles (experts with at least kWideMinTokens
// assignments) for the tensor-core kernels; such experts then get no mma.sync tiles.
struct TileOut {
    ExpertTile *tiles;
    int *n_tiles;
    WideTile *wide_tiles;   // small tensor-core tiles; nullptr: every expert gets mma.sync tiles
    int *n_wide;
    WideTile *wide_large;   // large tensor-core tiles (set whenever wide_tiles is)
    int *n_wide_large;
    int width;
    const int *shift;       // per-token activation shifts packed into the tiles' flat ids (nullptr: 0)
    int k;                  // top-k, to find a flat id's token
};

// A tile slot's flat id with its token's activation shift in the top byte (tile_flat_id and
// tile_shift below take them apart; flat ids stay below 2^24).
__device__ __forceinline__ int pack_flat(int f, const TileOut &to)
{
    const int sh = to.shift != nullptr ? to.shift[f / to.k] : 0;
    return f | static_cast<int>(static_cast<uint32_t>(sh & 0xFF) << 24);
}
cudaError_t launch_route_select_permute(const float *partial, int splits, const float *bias, int32_t *ids, float *w,
                                        int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, TileOut to,
                                        const uint32_t *xmax, int M, int E, int k, cudaStream_t s, bool pdl);
cudaError_t launch_permute(const int32_t *ids, int32_t *offsets, int32_t *sorted_ids, int32_t *inv_pos, TileOut to,
                           int M, int E, int k, cudaStream_t s, bool pdl);
// Tiles of both kinds from given expert offsets and sorted ids (the step-level entry points);
// also resets the call's status words.
cudaError_t launch_build_tiles(const int32_t *offsets, const int32_t *sorted_ids, TileOut to, int *status, int E,
                               cudaStream_t s);
// Rows [n_rows, cols] in natural K order -> P4 order (the grouped GEMMs' activation layout).
cudaError_t launch_rows_to_p4(const __nv_bfloat16 *src, __nv_bfloat16 *dst, size_t n_rows, int cols, cudaStream_t s);
cudaError_t launch_gate_up(const CUtensorMap &w13_map, const CUtensorMap &s13_map, const uint8_t *w13_s,
                           const __nv_bfloat16 *x, const ExpertTile *tiles, const int *n_tiles, __nv_bfloat16 *h,
                           bool h_p4, int *status, int32_t *status_out, int H, int I, int k, int width, int max_tiles,
                           cudaStream_t s, bool pdl);
cudaError_t launch_down(const CUtensorMap &w2_map, const CUtensorMap &s2_map, const uint8_t *w2_s,
                        const __nv_bfloat16 *h_p4, const int32_t *sorted_ids, const ExpertTile *tiles,
                        const int *n_tiles, float *y, int *status, int32_t *status_out, int H, int I, int width,
                        int max_tiles, cudaStream_t s, bool pdl);
cudaError_t launch_combine(const float *y, const float *topk_w, void *out, bool f32_out, int M, int H, int k,
                           cudaStream_t s, bool pdl);
cudaError_t launch_reduce_partials(const float *partials, int G, void *out, int M, int H, cudaStream_t s);
cudaError_t launch_gather_wide_rows(const __nv_bfloat16 *x_p4, const int32_t *sorted_ids, const WideLists &wl,
                                    __nv_bfloat16 *x_perm, int H, int k, cudaStream_t s, bool pdl);
cudaError_t launch_wide(bool gate_up, bool small, const CUtensorMap &wmap, const CUtensorMap &smap,
                        const CUtensorMap &bmap, const WideTile *tiles, const int *n_tiles, int max_tiles,
                        const int32_t *sorted_ids, __nv_bfloat16 *h, bool h_p4, float *y, int *status,
                        int32_t *status_out, int H, int I, cudaStream_t s, bool pdl);
int wide_smem_bytes();
cudaError_t launch_wait_timeout_selftest(int32_t *status_out, cudaStream_t s);

// Row blocks of the down projection per token (one arrival counter each).
__host__ __device__ inline int down_row_blocks(int H) { return (H + kItemRows - 1) / kItemRows; }

int num_sms();

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_max_smem(const void *kernel, int bytes);

}  // namespace moe
