// grouped_gemm.cu -- grouped MXFP4 expert GEMMs for small per-expert token counts.
//
// "Compact routed MXFP4 GEMM" (gate_up and down), "Routed MoE gather" and
// "Routed clamp-SwiGLU" rows of "Post-Portfolio Device Attribution" ("MTP1
// Post-Portfolio Eager-Cycle Profile"); the page's "Decision" section plans a
// fused gate/up producer with a bf16-rounded exchange, and
// "row/QUANT-CT-MXFP4-C8-DIFF" measures the unfused gate_up (more grouped GEMM
// launches and CTAs per layer) as the dominant decode cost.  At decode token
// counts these GEMMs stream each touched expert's weights once and are bound by
// HBM bandwidth ("The Systematic Optimization Campaign", chunk 8.0).
//
// Design (one persistent CTA per SM, warp specialised):
//  * Work item = (expert tile of <= 8 or <= 16 assignments -- the call's tile
//    width -- and 64 weight rows).  gate_up: gate rows n0..n0+31 and the
//    matching up rows I+n0..; down: W2 rows r0..r0+63.  The item is 4 MMA
//    m-tiles of 16 rows; for gate_up an m-tile
//    holds 8 gate rows (fragment rows 0-7) and the same 8 up rows (fragment rows
//    8-15), so every thread ends with g and u of one output row and applies
//    clamp-SwiGLU and the bf16 rounding in registers.  Items are numbered in
//    (tile, row block) order; with few items per CTA each CTA first takes a
//    contiguous run of them (adjacent 32 KB weight regions of one expert back
//    to back, for DRAM page locality), then single items or small groups from
//    the call's work queue, so faster SMs take more.
//  * Producer warp: per 1024-K stage, TMA 2-D tiled copies of the item's packed
//    E2M1 bytes -- 4 column boxes of 32 or 64 rows x 128 bytes per row block,
//    issued together so that each row's 512 contiguous bytes are read at once --
//    with a 128-byte swizzle into a 3-stage ring of 32 KB; in the same stage a TMA
//    box of the matching E8M0 scales (when scale rows are 16-byte multiples, else
//    the item's scale rows once per item), and one 1-D bulk copy per tile token of
//    its bf16 activation chunk (the routed gather: x rows for gate_up, h rows
//    for down).
//  * 16 compute warps = 2 m-tile pairs x 8 K slots.  Per stage a warp takes 4 of
//    the 32 blocks of 32 K for its 2 m-tiles: a thread reads the 32-bit word q of
//    its rows' 16-byte block (conflict-free thanks to the swizzle), decodes it
//    exactly to the codes' values times 2^-126 (e2m1x8_raw_p4: the E2M1 subnormal 0.5
//    becomes a bf16 subnormal, which the MMA takes exactly) straight into MMA
//    A-fragment registers, and runs two m16n8k16 bf16 MMAs per block.  The 2^126
//    rides on the activations instead: each token's bf16 activations are multiplied by
//    2^s (s: the token's activation shift, x_shift_from_max; a fixed kHShift for h)
//    as the thread loads them, which keeps every product inside fp32's normal range,
//    and the epilogue multiplies the sums by 2^(126 - s).  Both are powers of two, so
//    the fp32 sums are the unshifted sums times 2^(s - 126), rounding for rounding;
//    the shift costs one multiply per 8 activations against one per 2 weights.  Inside a block the K order is
//    permuted identically for A and for the activation fragment: thread q's word
//    covers K 8q..8q+7, its registers pair K 8q+i with 8q+i+4, and the activation
//    rows are stored in that same P4 order (x by the router, h by gate_up).  So
//    each MMA pair spans exactly one scale block, and the E8M0 scale multiplies the
//    block's fp32 partial once (exact: a power of two).  With 16-assignment tiles
//    each decoded fragment feeds two MMA n-tiles.  At the end of an item a warp
//    parks its partial sums in a reduction area (two buffers for 8-wide tiles; one
//    for 16-wide, where the K slots first add up in pairs) and moves on.
//  * 2 epilogue warps (4 for 16-wide tiles) sum the K-slot partials in slot
//    order, then gate_up applies clamp-SwiGLU and stores h; down stores the
//    unweighted fp32 row of each
//    assignment (at its flat id, from the expert-grouped order) -- off the compute
//    path.  The item's position range reaches them from the producer through shared
//    memory.  The weighted top-k combine that follows is its own small kernel
//    (combine_kernel).
// Both MMA operands are bf16: x as the caller gives it and h as gate_up rounds it (both
// stored in the P4 K order of common.cuh, both times an exact power of two), and the
// weights decoded exactly (every E2M1 value times 2^-126 is a bf16 value); products
// accumulate in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {

constexpr int kProducerWarp = kComputeWarps;
constexpr int kFirstEpilogueWarp = kComputeWarps + 1;
constexpr int kBlocksPerStage = kChunkK / 32;
constexpr int kBlocksPerWarp = kBlocksPerStage / kKSlots;
constexpr int kItemQ = 8;   // item ids in flight between the producer and the compute warps (> kStages)
static_assert(kBlocksPerWarp * kKSlots == kBlocksPerStage, "stage blocks split evenly over K slots");
static_assert(8 % kBlocksPerWarp == 0, "a warp's blocks stay inside one 128-byte box column");
static_assert(kKSlots % 2 == 0, "K slots pair up");

// Per tile width kN (8 or 16 assignments): kN / 8 MMA n-tiles share every decoded weight
// fragment.  With 16, the K-slot partial sums are pre-reduced in pairs of warps (odd K slot into
// its even neighbour) so that one buffer of them fits next to the 16-row activation stages.
template <int kN>
struct Tiling {
    static constexpr int kHalves = kN / 8;
    static constexpr bool kPairRed = kN == 16;
    static constexpr int kRedSets = kPairRed ? kKSlots / 2 : kKSlots;   // partial sets per buffer
    static constexpr int kRedBufs = kPairRed ? 1 : 2;
    static constexpr int kRedFloats = kRedSets * kItemMTiles * 32 * 4 * kHalves;   // [set][m-tile][lane][4 kHalves]
    static constexpr int kEpiWarps = kN == 16 ? 4 : 2;
    static constexpr int kThreads = (kComputeWarps + 1 + kEpiWarps) * 32;
    static constexpr int kActStageBytes = kN * kActPitch;
    static constexpr int kRedArrivals = kPairRed ? kComputeWarps / 2 : kComputeWarps;   // warps that post partials
    static_assert(kItemMTiles % kEpiWarps == 0, "m-tiles split evenly over the epilogue warps");
};

struct SmemPlan {
    int wst_off, act_off, sst_off, sbuf_off, sbuf_bytes, red_off, bars_off, total;
};

constexpr int kNumBars = 2 * kStages + 8 + kComputeWarps / 2;   // ring, scale buffers, partials, K-slot pairs
constexpr int kMetaInts = (3 + kTileTokensMax) * (kItemQ + 2);   // item ids, positions, counts, token shifts

template <int kN>
__host__ __device__ inline SmemPlan smem_plan(int K)
{
    using T = Tiling<kN>;
    SmemPlan p;
    p.wst_off = 0;
    p.act_off = kStages * kStageBytes;
    p.sst_off = p.act_off + kStages * T::kActStageBytes;
    p.sbuf_off = p.sst_off + kStages * kStageScaleBytes;
    p.sbuf_bytes = per_stage_scales(K) ? 0 : (kItemRows * (K / 32) + 127) / 128 * 128;
    p.red_off = p.sbuf_off + 2 * p.sbuf_bytes;
    p.bars_off = p.red_off + T::kRedBufs * T::kRedFloats * 4;
    p.total = p.bars_off + kNumBars * 8 + kMetaInts * 4 + 1024;   // + alignment slack
    return p;
}

// v * 2^(126 - s) for an activation shift s in [-7, 127], in two exact power-of-two steps (the
// factor alone can exceed fp32's range).
__device__ __forceinline__ float unshift(float v, int s)
{
    return (v * 0x1p63f) * __int_as_float((190 - s) << 23);   // 2^63, then 2^(63 - s)
}

__device__ __forceinline__ float clamp_swiglu(float g, float u)
{
    const float a = fminf(g, 7.0f);
    const float c = fminf(fmaxf(u, -7.0f), 7.0f);
    return a / (1.0f + expf(-a)) * c;
}

template <bool kGateUp, int kN>
__global__ void __launch_bounds__(Tiling<kN>::kThreads, 1)
grouped_mxfp4_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                     const uint8_t *__restrict__ wscale, const __nv_bfloat16 *__restrict__ act,
                     const int32_t *__restrict__ sorted_ids, const ExpertTile *__restrict__ tiles, const int *__restrict__ n_tiles_ptr,
                     __nv_bfloat16 *__restrict__ hout, float *__restrict__ yout, int *status_ws, int32_t *status_out,
                     int *queue, int K, int I, int H, int k, int h_p4)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    using T = Tiling<kN>;
    constexpr int kRedBufs = T::kRedBufs;
    constexpr int kActStageBytes = T::kActStageBytes;
    const SmemPlan plan = smem_plan<kN>(K);
    uint8_t *wst = smem + plan.wst_off;
    uint8_t *ast = smem + plan.act_off;
    uint8_t *sst = smem + plan.sst_off;
    uint8_t *sbuf = smem + plan.sbuf_off;
    float *red = reinterpret_cast<float *>(smem + plan.red_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + plan.bars_off);
    uint64_t *full = bars, *empty = bars + kStages;
    uint64_t *sfull = bars + 2 * kStages, *sempty = sfull + 2, *rfull = sfull + 4, *rempty = sfull + 6;
    uint64_t *pair = sfull + 8;   // [kComputeWarps / 2]: odd K slot's partials posted (pair reduction)
    // per item in flight: id, first expert-grouped position and assignment count (producer ->
    // compute warps -> epilogue warps), so that no consumer reads the tile list itself
    volatile int *item_q = reinterpret_cast<volatile int *>(bars + kNumBars);         // [kItemQ]
    volatile int *item_p0 = item_q + kItemQ;                                          // [kItemQ]
    volatile int *item_cnt = item_p0 + kItemQ;                                        // [kItemQ]
    volatile int *red_item = item_cnt + kItemQ;                                       // [kRedBufs]
    volatile int *red_p0 = red_item + 2;                                              // [kRedBufs]
    volatile int *red_cnt = red_p0 + 2;                                               // [kRedBufs]
    // the activation shift of each tile slot (item_sh: per item in flight; red_sh: per partial buffer)
    volatile int *item_sh = red_cnt + 2;                                              // [kItemQ][16]
    volatile int *red_sh = item_sh + kItemQ * kTileTokensMax;                         // [kRedBufs][16]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const StatusPtrs status{status_ws, status_out};
    const int rows_total = kGateUp ? I : H;                 // output rows of this projection
    const int row_blocks = kGateUp ? I / 32 : down_row_blocks(H);
    const int kblocks = K / 32;                             // scale bytes per row
    const bool stage_scales = per_stage_scales(K);
    const int n_chunks = (K + kChunkK - 1) / kChunkK;
    const int kbytes = K / 2;                               // packed bytes per row
    constexpr int kBoxRows = kGateUp ? 32 : 64;
    constexpr int kBoxBytes = kBoxRows * 128;               // one weight box: rows x 128 bytes
    constexpr int kScaleBoxBytes = kBoxRows * (kChunkK / 32);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kComputeWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sfull[b], 1);
            mbar_init(&sempty[b], kComputeWarps);
        }
        for (int b = 0; b < kRedBufs; ++b) {
            mbar_init(&rfull[b], T::kRedArrivals);
            mbar_init(&rempty[b], T::kEpiWarps);
        }
        for (int i = 0; i < kComputeWarps / 2; ++i) mbar_init(&pair[i], 1);
        fence_barrier_init();
    }
    __syncthreads();
    // gate_up reads the tile list its predecessor (the permutation) writes, so it waits here.
    // The down kernel's predecessor is gate_up, which lets dependents launch only after its own
    // wait, so the tile list, sorted ids and routing weights (written before gate_up) are complete
    // when any down CTA runs.  Only h comes from gate_up: the down producer waits before its first
    // h copy, and the W2 weights and scales of its first stages stream in during gate_up's tail.
    // The producer's early reads of the tile list bypass L1 (ld.global.cg).
    if (kGateUp) pdl_wait();
    pdl_trigger();
    const int n_tiles = __ldcg(n_tiles_ptr);
    const int n_items = n_tiles * row_blocks;

    bool aborted = false;

    if (warp == kProducerWarp) {
        // ---------------------------------------------------------------- producer warp
        if (lane == 0) {
            prefetch_tensormap(&wmap);
            if (stage_scales) prefetch_tensormap(&smap);
        }
        int stage_ctr = 0, item_ctr = 0;
        int stages_issued = 0, scales_issued = 0;   // copies in flight must land before exit
        // the next item's descriptor, loaded one item ahead so that no copy waits on it
        int nx_e = 0, nx_p0 = 0, nx_cnt = 1, nx_flat = 0;
        auto fetch = [&](int it) {
            if (it < n_items) {
                const ExpertTile *tp = tiles + it / row_blocks;
                nx_e = __ldcg(&tp->expert);
                nx_p0 = __ldcg(&tp->p0);
                nx_cnt = __ldcg(&tp->count);
                nx_flat = __ldcg(&tp->flat[lane & (kTileTokensMax - 1)]);
            }
        };
        // down: h copies of the first stages, held back until gate_up has completed (the rows of
        // a down tile are consecutive in h, so a stage's copies are its first row, row count,
        // K offset and bytes per row)
        bool h_ready = kGateUp;
        int pend_p0[kStages], pend_cnt[kStages], pend_kc[kStages];
        uint32_t pend_bytes[kStages];
#pragma unroll
        for (int i = 0; i < kStages; ++i) pend_p0[i] = pend_cnt[i] = pend_kc[i] = 0, pend_bytes[i] = 0;
        auto release_h = [&]() {
            pdl_wait();
            if (elect_one()) {
#pragma unroll
                for (int i = 0; i < kStages; ++i)
                    for (int j = 0; j < pend_cnt[i]; ++j)
                        bulk_load(ast + i * kActStageBytes + j * kActPitch,
                                  act + static_cast<size_t>(pend_p0[i] + j) * K + pend_kc[i], pend_bytes[i], &full[i]);
            }
            __syncwarp();
            h_ready = true;
        };
        // Items come from the call's work queue (an atomic counter, zeroed by the first kernel of
        // the call) in tile-major order, so faster SMs take more of them and all SMs sweep the
        // weight matrices together.  With few items per CTA (coarse items, decode sizes) a CTA
        // first takes a contiguous run of 3/4 of its even share and then single items; with many,
        // it takes 2 or 4 consecutive items per grab (fewer atomics on the counter).  Two grabs
        // are always in flight, issued long before their ids are needed; the descriptor of the
        // next item loads one item ahead.
        const int per_cta = n_items / static_cast<int>(gridDim.x);
        const int grab_items = per_cta < 16 ? 1 : (per_cta < 48 ? 2 : 4);
        const int share = per_cta < 16 ? static_cast<int>((3LL * n_items) / (4LL * gridDim.x)) : 0;
        const int static_total = share * static_cast<int>(gridDim.x);
        int run = static_cast<int>(blockIdx.x) * share;
        int run_end = run + share;
        auto grab = [&]() { return lane == 0 ? atomicAdd(queue, 1) : 0; };
        int g0 = grab(), g1 = grab();
        auto take = [&]() -> int {
            if (run >= run_end) {
                run = static_total + grab_items * __shfl_sync(0xffffffffu, g0, 0);
                run_end = run + grab_items;
                g0 = g1;
                g1 = grab();
            }
            return run++;
        };
        int next_id = take();
        fetch(next_id);
        for (;; ++item_ctr) {
            const int item = next_id;
            if (item >= n_items) break;
            const int e = nx_e, p0 = nx_p0, cnt = nx_cnt, flat = tile_flat_id(nx_flat);
            next_id = take();
            fetch(next_id);
            if (lane == 0) {   // published by the first stage's arrival
                item_q[item_ctr % kItemQ] = item;
                item_p0[item_ctr % kItemQ] = p0;
                item_cnt[item_ctr % kItemQ] = cnt;
            }
            // the slots' activation shifts: x by its token's shift (packed with the flat id), h by
            // the fixed one
            if (lane < kTileTokensMax) item_sh[(item_ctr % kItemQ) * kTileTokensMax + lane] = kGateUp ? tile_shift(nx_flat) : kHShift;
            __syncwarp();   // orders these stores before the arrival of whichever lane issues it
            const int rb = item % row_blocks;
            // weight rows: gate_up = gate block a and up block b (32 rows each); down = one block of 64
            const int row_a = kGateUp ? e * 2 * I + rb * 32 : e * H + rb * kItemRows;
            const int row_b = row_a + I;                               // gate_up only
            const int valid_rows = kGateUp ? kItemRows : min(kItemRows, H - rb * kItemRows);
            // gate_up: lane j < cnt holds the element offset of the x row of the tile's token j
            // (down reads h rows p0 .. p0 + cnt - 1)
            const long long xrow = kGateUp ? static_cast<long long>(flat / k) * K : 0;
            if (!stage_scales) {
                const int b = item_ctr & 1;
                // the scale buffer frees only when compute has finished item_ctr - 2, which may
                // need the held-back h copies
                if (!h_ready && item_ctr >= 2) release_h();
                mbar_wait(&sempty[b], ((item_ctr >> 1) & 1) ^ 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);   // keep the warp's control flow uniform
                if (!aborted && elect_one()) {
                    uint8_t *dst = sbuf + b * plan.sbuf_bytes;
                    mbar_arrive_expect_tx(&sfull[b], static_cast<uint32_t>(valid_rows * kblocks));
                    if (kGateUp) {
                        bulk_load(dst, wscale + static_cast<size_t>(row_a) * kblocks, 32u * kblocks, &sfull[b]);
                        bulk_load(dst + 32 * kblocks, wscale + static_cast<size_t>(row_b) * kblocks, 32u * kblocks,
                                  &sfull[b]);
                    } else {
                        bulk_load(dst, wscale + static_cast<size_t>(row_a) * kblocks,
                                  static_cast<uint32_t>(valid_rows * kblocks), &sfull[b]);
                    }
                }
                if (!aborted) ++scales_issued;
            }
            for (int c = 0; c < n_chunks; ++c, ++stage_ctr) {
                const int s = stage_ctr % kStages;
                if (!h_ready && stage_ctr >= kStages) release_h();
                mbar_wait(&empty[s], ((stage_ctr / kStages) & 1) ^ 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) continue;
                const int kb = c * (kChunkK / 2);
                const int kc = c * kChunkK;
                const uint32_t act_bytes = 2u * static_cast<uint32_t>(min(kChunkK, K - kc));
                const int ncols = min(kBoxCols, (kbytes - kb + 127) / 128);   // skip columns wholly past K
                const int halves = kGateUp ? 2 : 1;
                const uint32_t bytes = halves * (ncols * kBoxBytes + (stage_scales ? kScaleBoxBytes : 0)) +
                                       cnt * act_bytes;
                // One elected lane issues every copy of the stage: copies issued from several lanes
                // of a divergent branch are serialised anyway, and slowly while the compute warps
                // keep the SM's issue slots busy.  Gate_up boxes: columns of the gate rows, then
                // columns of the up rows; down: columns.
                uint8_t *st = wst + s * kStageBytes;
                uint8_t *sa = ast + s * kActStageBytes;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[s], bytes);
                    for (int col = 0; col < ncols; ++col) {
                        tma_load_2d(st + col * kBoxBytes, &wmap, kb + 128 * col, row_a, &full[s]);
                        if (kGateUp) tma_load_2d(st + (kBoxCols + col) * kBoxBytes, &wmap, kb + 128 * col, row_b, &full[s]);
                    }
                    if (stage_scales) {
                        uint8_t *ss = sst + s * kStageScaleBytes;
                        tma_load_2d(ss, &smap, kc / 32, row_a, &full[s]);
                        if (kGateUp) tma_load_2d(ss + kScaleBoxBytes, &smap, kc / 32, row_b, &full[s]);
                    }
                    if (!kGateUp && h_ready)
                        for (int j = 0; j < cnt; ++j)
                            bulk_load(sa + j * kActPitch, act + static_cast<size_t>(p0 + j) * K + kc, act_bytes, &full[s]);
                }
                if (kGateUp) {
                    for (int j = 0; j < cnt; ++j) {
                        const long long row = __shfl_sync(0xffffffffu, xrow, j);
                        if (elect_one()) bulk_load(sa + j * kActPitch, act + row + kc, act_bytes, &full[s]);
                    }
                } else if (!h_ready) {
#pragma unroll
                    for (int i = 0; i < kStages; ++i)   // stage_ctr < kStages here, so s == stage_ctr
                        if (i == s) {
                            pend_p0[i] = p0;
                            pend_cnt[i] = cnt;
                            pend_kc[i] = kc;
                            pend_bytes[i] = act_bytes;
                        }
                }
                __syncwarp();
                ++stages_issued;
            }
        }
        if (!h_ready) release_h();
        // let every copy this CTA issued land before the CTA can exit (stages and per-item scale
        // rows are issued in order until a wait gives up, so the issued ones are a prefix).  This
        // comes before the end marker, whose arrival reuses the ring slot of stage
        // stages_issued - kStages and would make that stage's phase look pending again.
        for (int i = 0; i < kStages && i < stages_issued; ++i) {
            const int sc = stages_issued - 1 - i;
            mbar_wait_drain(&full[sc % kStages], (sc / kStages) & 1, status);
        }
        for (int i = 0; i < 2 && i < scales_issued; ++i) {
            const int j = scales_issued - 1 - i;
            mbar_wait_drain(&sfull[j & 1], (j >> 1) & 1, status);
        }
        {
            // end marker: one more ring slot whose arrival carries item -1 and no copies
            const int s = stage_ctr % kStages;
            mbar_wait(&empty[s], ((stage_ctr / kStages) & 1) ^ 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (!aborted && lane == 0) {
                item_q[item_ctr % kItemQ] = -1;
                mbar_arrive(&full[s]);
            }
        }
        return;
    }

    if (warp >= kFirstEpilogueWarp) {
        // ---------------------------------------------------------------- epilogue warps
        const int ep = warp - kFirstEpilogueWarp;
        const int g = lane >> 2, q = lane & 3;
        // nothing for the epilogue before the first item's partial sums; the down kernel's
        // epilogue waits for gate_up here so that its plain loads see the current call's data
        if (!kGateUp) pdl_wait();
        constexpr int kEpiMTiles = kItemMTiles / T::kEpiWarps;   // m-tiles ep, ep + kEpiWarps, ..
        constexpr int kVals = 4 * T::kHalves;                    // partial floats per lane and m-tile
        for (int item_ctr = 0;; ++item_ctr) {
            const int b = item_ctr % kRedBufs;
            const float *rbuf = red + b * T::kRedFloats;
            mbar_wait(&rfull[b], (item_ctr / kRedBufs) & 1, aborted, status);
            if (aborted) break;
            const int item = red_item[b];   // -1: no further item
            if (item < 0) break;
            const int rb = item % row_blocks;
            const int cnt = red_cnt[b], p0 = red_p0[b];
            // sums over the partial sets in set order (K slots, or K-slot pairs), per n-half
            float4 sums[kEpiMTiles][T::kHalves];
#pragma unroll
            for (int m = 0; m < kEpiMTiles; ++m) {
                const int j = ep + T::kEpiWarps * m;
#pragma unroll
                for (int hf = 0; hf < T::kHalves; ++hf) {
                    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int ks = 0; ks < T::kRedSets; ++ks) {
                        const float4 v =
                            *reinterpret_cast<const float4 *>(rbuf + ((ks * kItemMTiles + j) * 32 + lane) * kVals + 4 * hf);
                        sum.x += v.x;
                        sum.y += v.y;
                        sum.z += v.z;
                        sum.w += v.w;
                    }
                    sums[m][hf] = sum;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[b]);
#pragma unroll
            for (int m = 0; m < kEpiMTiles; ++m) {
                const int j = ep + T::kEpiWarps * m;
#pragma unroll
                for (int hf = 0; hf < T::kHalves; ++hf) {
                    float4 sum = sums[m][hf];
                    const int li0 = 8 * hf + 2 * q, li1 = li0 + 1;   // the fragment's two tile slots
                    // back to the true scale: the sums carry 2^(shift - 126) (exact powers of two)
                    if (kGateUp) {
                        const int s0 = red_sh[b * kTileTokensMax + li0], s1 = red_sh[b * kTileTokensMax + li1];
                        sum = make_float4(unshift(sum.x, s0), unshift(sum.y, s1), unshift(sum.z, s0), unshift(sum.w, s1));
                    } else {
                        constexpr float kBack = static_cast<float>(1u << (126 - kHShift));
                        sum = make_float4(sum.x * kBack, sum.y * kBack, sum.z * kBack, sum.w * kBack);
                    }
                    if (kGateUp) {
                        // h rounded to bf16 once, at column n (P4 storage order for the down kernels)
                        const int n = rb * 32 + 8 * j + g;
                        const int col = h_p4 ? p4_pos(n) : n;
                        if (li0 < cnt)
                            hout[static_cast<size_t>(p0 + li0) * I + col] = __float2bfloat16_rn(clamp_swiglu(sum.x, sum.z));
                        if (li1 < cnt)
                            hout[static_cast<size_t>(p0 + li1) * I + col] = __float2bfloat16_rn(clamp_swiglu(sum.y, sum.w));
                    } else {
                        // the unweighted row; the routing weight is applied by the combine
                        const int ra = rb * kItemRows + 16 * j + g, rbw = ra + 8;
                        if (li0 < cnt) {
                            float *yr = yout + static_cast<size_t>(sorted_ids[p0 + li0]) * H;
                            if (ra < rows_total) yr[ra] = sum.x;
                            if (rbw < rows_total) yr[rbw] = sum.z;
                        }
                        if (li1 < cnt) {
                            float *yr = yout + static_cast<size_t>(sorted_ids[p0 + li1]) * H;
                            if (ra < rows_total) yr[ra] = sum.y;
                            if (rbw < rows_total) yr[rbw] = sum.w;
                        }
                    }
                }
            }
        }
        return;
    }

    // -------------------------------------------------------------------- compute warps
    const int g = lane >> 2, q = lane & 3;
    constexpr int kGroups = kItemMTiles / kWarpMTiles;
    const int mgrp = warp % kGroups;        // m-tiles mgrp*kWarpMTiles ..
    const int kslot = warp / kGroups;       // blocks kslot*kBlocksPerWarp .. of every stage
    const int col = (kslot * kBlocksPerWarp) >> 3;
    const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
    const int bb0 = (kslot * kBlocksPerWarp) & 7;

    // per m-tile: smem byte offsets (inside a stage) of the top/bottom rows' 16-byte blocks,
    // and scale-row indices (rows of the item's 64 weight rows)
    int top_off[kWarpMTiles], bot_off[kWarpMTiles], top_sr[kWarpMTiles], bot_sr[kWarpMTiles];
#pragma unroll
    for (int m = 0; m < kWarpMTiles; ++m) {
        const int j = mgrp * kWarpMTiles + m;
        if (kGateUp) {
            top_off[m] = col * kBoxBytes + (8 * j + g) * 128;
            bot_off[m] = (kBoxCols + col) * kBoxBytes + (8 * j + g) * 128;
            top_sr[m] = 8 * j + g;
            bot_sr[m] = 32 + 8 * j + g;
        } else {
            top_off[m] = col * kBoxBytes + (16 * j + g) * 128;
            bot_off[m] = col * kBoxBytes + (16 * j + 8 + g) * 128;
            top_sr[m] = 16 * j + g;
            bot_sr[m] = 16 * j + 8 + g;
        }
    }
    // scale addressing: per stage, row pitch kChunkK/32 bytes and block index within the stage;
    // per item, row pitch kblocks and the global block index
    const int s_pitch = stage_scales ? kChunkK / 32 : kblocks;
    // pair reduction (kN == 16): the odd K slot posts its partials, the even one adds its own
    const bool odd_slot = (kslot & 1) != 0;
    const int pair_id = mgrp * (kKSlots / 2) + (kslot >> 1);
    constexpr int kVals = 4 * T::kHalves;   // partial floats per lane and m-tile

    int stage_ctr = 0, item_ctr = 0;
    for (;; ++item_ctr) {
        const int b = item_ctr & 1;
        // the item's first stage (or the end marker) names the item
        mbar_wait(&full[stage_ctr % kStages], (stage_ctr / kStages) & 1, aborted, status);
        if (aborted) break;
        if (item_q[item_ctr % kItemQ] < 0) break;
        // the second n-tile of a 16-wide tile only when it holds assignments (warp-uniform)
        const bool two = kN == 16 && item_cnt[item_ctr % kItemQ] > 8;
        const uint8_t *sbi = sbuf + b * plan.sbuf_bytes;
        if (!stage_scales) mbar_wait(&sfull[b], (item_ctr >> 1) & 1, aborted, status);
        // bf16x2 2^s of this thread's B-fragment tokens g and g + 8 (the activation shifts)
        const uint32_t fac_g = static_cast<uint32_t>(item_sh[(item_ctr % kItemQ) * kTileTokensMax + g] + 127) * 0x00800080u;
        const uint32_t fac_g8 =
            static_cast<uint32_t>(item_sh[(item_ctr % kItemQ) * kTileTokensMax + g + 8] + 127) * 0x00800080u;

        float acc[kWarpMTiles][kVals];
#pragma unroll
        for (int m = 0; m < kWarpMTiles; ++m)
#pragma unroll
            for (int r = 0; r < kVals; ++r) acc[m][r] = 0.f;

        for (int c = 0; c < n_chunks; ++c, ++stage_ctr) {
            const int s = stage_ctr % kStages;
            if (c > 0) mbar_wait(&full[s], (stage_ctr / kStages) & 1, aborted, status);
            const uint8_t *st = wst + s * kStageBytes;
            const uint8_t *xa = ast + s * kActStageBytes + g * kActPitch;   // token g of the tile
            const uint8_t *sc_base = stage_scales ? sst + s * kStageScaleBytes : sbi;
            const int blk_base = kslot * kBlocksPerWarp;                      // block index within the stage
            const int sc_col0 = stage_scales ? blk_base : c * kBlocksPerStage + blk_base;
#pragma unroll
            for (int bi = 0; bi < kBlocksPerWarp; ++bi) {
                if (c * kBlocksPerStage + blk_base + bi >= kblocks) continue;
                // K 8q..8q+7 of token g (and g + 8), stored in P4 order like the decoded weights, times
                // 2^(token's shift) (exact)
                uint4 xb = *reinterpret_cast<const uint4 *>(xa + (32 * (blk_base + bi) + 8 * q) * 2);
                xb = make_uint4(bf16x2_mul(xb.x, fac_g), bf16x2_mul(xb.y, fac_g), bf16x2_mul(xb.z, fac_g),
                                bf16x2_mul(xb.w, fac_g));
                uint4 xc = make_uint4(0u, 0u, 0u, 0u);   // token g + 8 (second n-tile)
                if (kN == 16 && two) {
                    xc = *reinterpret_cast<const uint4 *>(xa + 8 * kActPitch + (32 * (blk_base + bi) + 8 * q) * 2);
                    xc = make_uint4(bf16x2_mul(xc.x, fac_g8), bf16x2_mul(xc.y, fac_g8), bf16x2_mul(xc.z, fac_g8),
                                    bf16x2_mul(xc.w, fac_g8));
                }
                const int sw = (((bb0 + bi) ^ g) << 4) + 4 * q;   // 128-byte swizzle: chunk ^ (row & 7)
#pragma unroll
                for (int m = 0; m < kWarpMTiles; ++m) {
                    const uint32_t wt = *reinterpret_cast<const uint32_t *>(st + top_off[m] + sw);
                    const uint32_t wb = *reinterpret_cast<const uint32_t *>(st + bot_off[m] + sw);
                    const float st_scale = e8m0_scale(sc_base[top_sr[m] * s_pitch + sc_col0 + bi]);
                    const float sb_scale = e8m0_scale(sc_base[bot_sr[m] * s_pitch + sc_col0 + bi]);
                    // the codes' values times 2^-126 (the shifted activations carry the 2^126)
                    uint32_t t[4], u[4];
                    e2m1x8_raw_p4(wt, t);
                    e2m1x8_raw_p4(wb, u);
                    // registers i = K (8q+i, 8q+i+4): the first MMA takes i = 0, 1, the second 2, 3.
                    // Each block's MMA pair starts from zero (no dependence on the previous block's
                    // MMAs) and its fp32 partial times the block scale (exact) joins the K slot's sums.
                    const uint32_t a0[4] = {t[0], u[0], t[1], u[1]};
                    const uint32_t a1[4] = {t[2], u[2], t[3], u[3]};
                    float tmp[4];
                    mma_bf16_16816(tmp, a0, xb.x, xb.y, zero4);
                    mma_bf16_16816(tmp, a1, xb.z, xb.w, tmp);
                    acc[m][0] = fmaf(tmp[0], st_scale, acc[m][0]);
                    acc[m][1] = fmaf(tmp[1], st_scale, acc[m][1]);
                    acc[m][2] = fmaf(tmp[2], sb_scale, acc[m][2]);
                    acc[m][3] = fmaf(tmp[3], sb_scale, acc[m][3]);
                    if (kN == 16 && two) {
                        float tmq[4];
                        mma_bf16_16816(tmq, a0, xc.x, xc.y, zero4);
                        mma_bf16_16816(tmq, a1, xc.z, xc.w, tmq);
                        acc[m][kVals - 4] = fmaf(tmq[0], st_scale, acc[m][kVals - 4]);
                        acc[m][kVals - 3] = fmaf(tmq[1], st_scale, acc[m][kVals - 3]);
                        acc[m][kVals - 2] = fmaf(tmq[2], sb_scale, acc[m][kVals - 2]);
                        acc[m][kVals - 1] = fmaf(tmq[3], sb_scale, acc[m][kVals - 1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        __syncwarp();
        if (!stage_scales && lane == 0) mbar_arrive(&sempty[b]);

        // park the K-slot partial sums (and the item's ids) for the epilogue warps
        const int rb = item_ctr % kRedBufs;
        float *rbuf = red + rb * T::kRedFloats;
        const int set = T::kPairRed ? kslot >> 1 : kslot;
        if (T::kPairRed && odd_slot) {
            // post this slot's partials into the pair's set; the even neighbour adds to them
            mbar_wait(&rempty[rb], ((item_ctr / kRedBufs) & 1) ^ 1, aborted, status);
            if (aborted) break;
#pragma unroll
            for (int m = 0; m < kWarpMTiles; ++m)
#pragma unroll
                for (int v = 0; v < kVals; v += 4)
                    *reinterpret_cast<float4 *>(rbuf + ((set * kItemMTiles + mgrp * kWarpMTiles + m) * 32 + lane) * kVals + v) =
                        make_float4(acc[m][v], acc[m][v + 1], acc[m][v + 2], acc[m][v + 3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pair[pair_id]);
            continue;
        }
        if (T::kPairRed) {
            // the odd neighbour's partials are posted (it waited for the buffer); even + odd
            mbar_wait(&pair[pair_id], item_ctr & 1, aborted, status);
        } else {
            mbar_wait(&rempty[rb], ((item_ctr / kRedBufs) & 1) ^ 1, aborted, status);
        }
        if (aborted) break;
#pragma unroll
        for (int m = 0; m < kWarpMTiles; ++m)
#pragma unroll
            for (int v = 0; v < kVals; v += 4) {
                float4 *dst =
                    reinterpret_cast<float4 *>(rbuf + ((set * kItemMTiles + mgrp * kWarpMTiles + m) * 32 + lane) * kVals + v);
                float4 o = make_float4(acc[m][v], acc[m][v + 1], acc[m][v + 2], acc[m][v + 3]);
                if (T::kPairRed) {
                    const float4 p = *dst;
                    o.x += p.x;
                    o.y += p.y;
                    o.z += p.z;
                    o.w += p.w;
                }
                *dst = o;
            }
        if (warp == 0) {
            if (lane == 0) {
                red_item[rb] = item_q[item_ctr % kItemQ];
                red_p0[rb] = item_p0[item_ctr % kItemQ];
                red_cnt[rb] = item_cnt[item_ctr % kItemQ];
            }
            if (lane < kTileTokensMax) red_sh[rb * kTileTokensMax + lane] = item_sh[(item_ctr % kItemQ) * kTileTokensMax + lane];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[rb]);
    }
    // end marker for the epilogue warps (from the warps that post partials)
    if (T::kPairRed && odd_slot) return;
    const int rb = item_ctr % kRedBufs;
    mbar_wait(&rempty[rb], ((item_ctr / kRedBufs) & 1) ^ 1, aborted, status);
    if (!aborted) {
        if (warp == 0 && lane == 0) red_item[rb] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[rb]);
    }
}

// out[t] = bf16( sum_j w[t*k + j] * y[t*k + j] ), slots j ascending (a fixed order, no atomics);
// y holds the unweighted down-projection row of every assignment.  Four outputs per thread.
// kF32: the same sum stored unrounded in fp32 (one rank's share of an I-sharded layer).
template <bool kF32>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y, const float *__restrict__ topk_w,
                                                      void *__restrict__ out, int M, int H, int k)
{
    pdl_wait();
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int per_row = H / 4;
    if (idx >= static_cast<size_t>(M) * per_row) return;
    const int t = static_cast<int>(idx / per_row);
    const int c = static_cast<int>(idx - static_cast<size_t>(t) * per_row) * 4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const int f = t * k + j;
        const float w = topk_w[f];
        const float4 v = *reinterpret_cast<const float4 *>(y + static_cast<size_t>(f) * H + c);
        a.x = fmaf(w, v.x, a.x);
        a.y = fmaf(w, v.y, a.y);
        a.z = fmaf(w, v.z, a.z);
        a.w = fmaf(w, v.w, a.w);
    }
    const size_t o = static_cast<size_t>(t) * H + c;
    if (kF32) {
        *reinterpret_cast<float4 *>(static_cast<float *>(out) + o) = a;
    } else {
        __nv_bfloat162 b[2] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w)};
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + o) = *reinterpret_cast<uint2 *>(b);
    }
}

// out[i] = bf16( sum_g partials[g][i] ), g = 0 .. G-1 ascending: the fixed-order reduction of the
// ranks' fp32 shares of an I-sharded layer (the same bits on every rank and in every run).  Four
// outputs per thread; n4 = M * H / 4.
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float *__restrict__ partials, int G, size_t n4,
                                                              __nv_bfloat16 *__restrict__ out)
{
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 *p = reinterpret_cast<const float4 *>(partials);
    float4 a = __ldg(p + i);
    for (int g = 1; g < G; ++g) {
        const float4 v = __ldg(p + static_cast<size_t>(g) * n4 + i);
        a.x += v.x;
        a.y += v.y;
        a.z += v.z;
        a.w += v.w;
    }
    __nv_bfloat162 b[2] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w)};
    reinterpret_cast<uint2 *>(out)[i] = *reinterpret_cast<uint2 *>(b);
}

template <bool kGateUp, int kN>
static cudaError_t launch_grouped(const CUtensorMap &map, const CUtensorMap &smap, const uint8_t *scales,
                                  const __nv_bfloat16 *act, const int32_t *sorted_ids, const ExpertTile *tiles,
                                  const int *n_tiles, __nv_bfloat16 *h, float *y, int *status, int32_t *status_out,
                                  int K, int I, int H, int k, int h_p4, int max_tiles, cudaStream_t s, bool pdl)
{
    const SmemPlan plan = smem_plan<kN>(K);
    auto kern = grouped_mxfp4_kernel<kGateUp, kN>;
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(kern), plan.total);
    if (e != cudaSuccess) return e;
    const long long row_blocks = kGateUp ? I / 32 : down_row_blocks(H);
    const long long max_items = static_cast<long long>(max_tiles) * row_blocks;
    int grid = static_cast<int>(max_items < num_sms() ? max_items : num_sms());
    if (grid < 1) grid = 1;
    int *queue = status + (kGateUp ? kQueueGateUp : kQueueDown);
    return launch_ex(kern, dim3(grid), dim3(Tiling<kN>::kThreads), plan.total, s, pdl, map, smap, scales, act,
                     sorted_ids, tiles, n_tiles, h, y, status, status_out, queue, K, I, H, k, h_p4);
}

int grouped_smem_bytes(int K, int width) { return width == 16 ? smem_plan<16>(K).total : smem_plan<8>(K).total; }

cudaError_t launch_gate_up(const CUtensorMap &w13_map, const CUtensorMap &s13_map, const uint8_t *w13_s,
                           const __nv_bfloat16 *x, const ExpertTile *tiles, const int *n_tiles, __nv_bfloat16 *h,
                           bool h_p4, int *status, int32_t *status_out, int H, int I, int k, int width, int max_tiles,
                           cudaStream_t s, bool pdl)
{
    if (width == 16)
        return launch_grouped<true, 16>(w13_map, s13_map, w13_s, x, nullptr, tiles, n_tiles, h, nullptr, status,
                                        status_out, H, I, H, k, h_p4 ? 1 : 0, max_tiles, s, pdl);
    return launch_grouped<true, 8>(w13_map, s13_map, w13_s, x, nullptr, tiles, n_tiles, h, nullptr, status,
                                   status_out, H, I, H, k, h_p4 ? 1 : 0, max_tiles, s, pdl);
}

cudaError_t launch_down(const CUtensorMap &w2_map, const CUtensorMap &s2_map, const uint8_t *w2_s,
                        const __nv_bfloat16 *h_p4, const int32_t *sorted_ids, const ExpertTile *tiles,
                        const int *n_tiles, float *y, int *status, int32_t *status_out, int H, int I, int width,
                        int max_tiles, cudaStream_t s, bool pdl)
{
    if (width == 16)
        return launch_grouped<false, 16>(w2_map, s2_map, w2_s, h_p4, sorted_ids, tiles, n_tiles, nullptr, y, status,
                                         status_out, I, I, H, 1, 1, max_tiles, s, pdl);
    return launch_grouped<false, 8>(w2_map, s2_map, w2_s, h_p4, sorted_ids, tiles, n_tiles, nullptr, y, status,
                                    status_out, I, I, H, 1, 1, max_tiles, s, pdl);
}

cudaError_t launch_combine(const float *y, const float *topk_w, void *out, bool f32_out, int M, int H, int k,
                           cudaStream_t s, bool pdl)
{
    const size_t n = static_cast<size_t>(M) * H / 4;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    if (f32_out)
        return launch_ex(combine_kernel<true>, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s, pdl, y, topk_w, out, M,
                         H, k);
    return launch_ex(combine_kernel<false>, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s, pdl, y, topk_w, out, M, H,
                     k);
}

cudaError_t launch_reduce_partials(const float *partials, int G, void *out, int M, int H, cudaStream_t s)
{
    const size_t n4 = static_cast<size_t>(M) * H / 4;
    const unsigned blocks = static_cast<unsigned>((n4 + 255) / 256);
    reduce_partials_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(partials, G, n4, static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError();
}

}  // namespace moe
