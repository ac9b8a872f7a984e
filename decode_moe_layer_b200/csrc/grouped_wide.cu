// grouped_wide.cu -- grouped MXFP4 expert GEMMs on the 5th-generation tensor cores, for the
// experts that receive kWideMinTokens or more routed assignments ("wide" tiles of up to
// kWideTokens assignments of one expert).
//
// "Compact routed MXFP4 GEMM" and "Routed clamp-SwiGLU" rows of "Post-Portfolio Device
// Attribution" ("MTP1 Post-Portfolio Eager-Cycle Profile"), with the fused gate/up producer of
// the page's "Decision" section.  At large token counts the expert GEMMs become real dense
// contractions: an expert with many assignments is streamed once for all of them (the narrow
// kernel in grouped_gemm.cu re-streams it for every 8 or 16 assignments), and the MMA runs on
// tcgen05 with the fp32 accumulator in tensor memory.  The kernel keeps a kWideTokens-wide tile of
// one expert's assignments against 128 weight rows per item, and the wider the tile the more
// work each MMA instruction does (their issue cost hardly depends on N).
//
// One persistent CTA per SM, 16 warps:
//  * warp 0 (weights producer): per 512-K stage, TMA copies of the item's packed E2M1 rows
//    (128 rows x 256 bytes, 128-byte swizzle) and their E8M0 scales into a 3-stage ring;
//    items come from the call's work queue, the ids reach the other warps through shared
//    memory with the stage arrivals.
//  * warp 2 (activations producer): per 64-K sub-tile, TMA copies of the item's activation
//    rows (x gathered into expert-grouped order for gate_up, h for down), 16 rows per box,
//    128-byte swizzle, into a 4-slot ring.  Rows past the tile are read and ignored.
//  * warps 4..11 (dequant): per 64-K sub-tile, 256 threads each decode 32 weights of one row
//    (hardware E2M1 -> f16x2), apply the row's E8M0 block scale in f16 (exact for scale bytes
//    104..140: every scaled E2M1 value is then an f16 normal or subnormal; other bytes are
//    flagged), and store them with tcgen05.st into an A buffer in tensor memory (TMEM lane =
//    A row; a warp reaches the 32 lanes of its warp index mod 4, and warps 4..7 / 8..11 take
//    the low / high 32 K of the sub-tile).  gate_up interleaves gate row i and up row i as A
//    rows 2i, 2i+1, so one TMEM lane pair holds g and u.  A never passes through shared
//    memory, which leaves shared-memory bandwidth to the TMA copies and the B operand.
//  * warp 1 (MMA): one thread issues 4 tcgen05.mma kind::f16 (A from TMEM, B from shared
//    memory; M 128, N = the tile's tokens rounded up to 16, K 16) per sub-tile into one of two
//    TMEM accumulators and commits the consumed A and B buffers and, per item, the
//    accumulator.
//  * warps 12..15 (epilogue): tcgen05.ld of the accumulator (warp w reads TMEM lanes
//    32 (w % 4) ..); gate_up pairs g and u with one shuffle, applies clamp-SwiGLU and the bf16
//    rounding and stores h; down stores the assignment's fp32 row of y (the combine applies
//    the routing weight).
// Every wait is bounded; after a timeout the kernel records MOE_ERR_TIMEOUT, drains the
// copies it issued and frees its tensor memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace wide {
constexpr int kRows = 128;                               // weight rows per item (MMA M)
constexpr int kStageK = kWideStageK;                     // 512 K per packed stage
constexpr int kPStages = 3;                              // packed weight stages
constexpr int kSubK = 64;                                // K per A/B sub-tile (one swizzle atom of f16)
constexpr int kSubs = kStageK / kSubK;                   // 8
// A tcgen05.mma costs about the same issue time for any N, so N is as large as TMEM allows:
// two accumulators of kWideTokens columns plus the A buffers.
constexpr int kABufs = 2, kBBufs = 4, kDBufs = 2;
constexpr int kItemQ = 8;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kWProd = 0, kMma = 1, kBProd = 2, kDeq0 = 4, kDeqWarps = 8, kEpi0 = 12, kEpiWarps = 4;
constexpr int kPackedStage = kRows * kStageK / 2;        // 32 KB: 2 box columns x 128 rows x 128 B
constexpr int kPackedCol = kRows * 128;                  // one box column (two 64-row boxes)
constexpr int kScaleStage = kRows * kStageK / 32;        // 2 KB: 128 rows x 16 B
constexpr int kBTile = kWideTokens * kSubK * 2;          // 28 KB
constexpr int kBBox = 16 * kSubK * 2;                    // one 16-row activation box
constexpr int kACols = kSubK / 2;                        // TMEM columns of one A buffer (2 f16 per column)
constexpr int kACol0 = kDBufs * kWideTokens;             // accumulators first, then the A buffers
constexpr int kTmemCols = 512;                           // power of two >= kACol0 + kABufs * kACols
constexpr int kOffPacked = 0;
constexpr int kOffScale = kOffPacked + kPStages * kPackedStage;
constexpr int kOffB = kOffScale + kPStages * kScaleStage;
constexpr int kOffIds = kOffB + kBBufs * kBTile;         // down: each epilogue warp's copy of the tile's flat ids
constexpr int kOffBars = kOffIds + kEpiWarps * kWideTokens * 4;
constexpr int kSmemBytes = kOffBars + 512 + 1024;        // barriers and slots, + alignment slack
static_assert(kOffB % 1024 == 0 && kBTile % 1024 == 0, "swizzled tiles sit on 1024-byte boundaries");
static_assert(kACol0 + kABufs * kACols <= kTmemCols && kTmemCols <= 512, "TMEM budget");
static_assert(kSmemBytes <= 227 * 1024, "fits one SM");
}  // namespace wide

struct WideArgs {
    const WideTile *tiles;
    const int *n_tiles;
    const int32_t *sorted_ids;   // down: flat ids of the expert-grouped positions
    __half *h;                   // gate_up output [M*k][I] (binary16, h * 2^10), expert-grouped rows
    float *y;                    // down output [M*k][H] by flat id, before the routing weight
    int *status_ws;
    int32_t *status_out;
    int *queue;
    int H, I;
};

__device__ __forceinline__ float wide_clamp_swiglu(float g, float u)
{
    const float a = fminf(g, 7.0f);
    const float c = fminf(fmaxf(u, -7.0f), 7.0f);
    return a / (1.0f + expf(-a)) * c;
}

__device__ __forceinline__ void record_status(const StatusPtrs &st, int code)
{
    if (st.ws) atomicExch(st.ws, code);
    if (st.out) atomicExch(st.out, code);
}

template <bool kGateUp>
__global__ void __launch_bounds__(wide::kThreads, 1)
grouped_wide_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                    const __grid_constant__ CUtensorMap bmap, const __grid_constant__ WideArgs a)
{
    using namespace wide;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
    uint64_t *full_p = bars, *empty_p = bars + kPStages;                       // packed stages
    uint64_t *a_full = bars + 2 * kPStages, *a_empty = a_full + kABufs;        // A tiles
    uint64_t *b_full = a_empty + kABufs, *b_empty = b_full + kBBufs;          // B tiles
    uint64_t *d_full = b_empty + kBBufs, *d_empty = d_full + kDBufs;          // accumulators
    uint64_t *pub = d_empty + kDBufs;                                         // [kItemQ] item ids published
    uint64_t *mma_done = pub + kItemQ;                                        // final drain of the MMAs
    volatile int *item_q = reinterpret_cast<volatile int *>(mma_done + 1);   // [kItemQ]
    volatile int *a_item = item_q + kItemQ;                                   // [kABufs]
    volatile int *d_item = a_item + kABufs;                                   // [kDBufs]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(const_cast<int *>(d_item + kDBufs));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const StatusPtrs status{a.status_ws, a.status_out};
    const int H = a.H, I = a.I;
    const int K = kGateUp ? H : I;
    const int n_stages = K / kStageK;
    const int row_blocks = kGateUp ? I / 64 : H / kRows;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full_p[s], 1);
            mbar_init(&empty_p[s], kDeqWarps);
        }
        for (int b = 0; b < kABufs; ++b) {
            mbar_init(&a_full[b], kDeqWarps);
            mbar_init(&a_empty[b], 1);
        }
        for (int b = 0; b < kBBufs; ++b) {
            mbar_init(&b_full[b], 1);
            mbar_init(&b_empty[b], 1);
        }
        for (int b = 0; b < kDBufs; ++b) {
            mbar_init(&d_full[b], 1);
            mbar_init(&d_empty[b], kEpiWarps);
        }
        for (int i = 0; i < kItemQ; ++i) mbar_init(&pub[i], 1);
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == kMma) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the tile list comes from the permutation, the activations from the kernels before this one
    pdl_wait();
    pdl_trigger();
    const int n_tiles = __ldcg(a.n_tiles);
    const int n_items = n_tiles * row_blocks;
    bool aborted = false;

    if (warp == kWProd) {
        // ------------------------------------------------------------ weights producer
        if (lane == 0) {
            prefetch_tensormap(&wmap);
            prefetch_tensormap(&smap);
        }
        int stage_ctr = 0, item_ctr = 0, issued = 0;
        auto grab = [&]() { return lane == 0 ? atomicAdd(a.queue, 1) : 0; };
        int g0 = grab();
        for (;; ++item_ctr) {
            const int item = __shfl_sync(0xffffffffu, g0, 0);
            if (item >= n_items) break;
            g0 = grab();
            const WideTile *tp = a.tiles + item / row_blocks;
            const int e = __ldcg(&tp->expert);
            const int rb = item % row_blocks;
            // the 128 rows: gate rows rb*64.. then up rows I + rb*64.. (gate_up); rows rb*128.. (down)
            const int row_a = kGateUp ? e * 2 * I + rb * 64 : e * H + rb * kRows;
            const int row_b = kGateUp ? row_a + I : row_a + 64;
            if (lane == 0) {
                item_q[item_ctr % kItemQ] = item;
                mbar_arrive(&pub[item_ctr % kItemQ]);   // for the activations producer
            }
            for (int st = 0; st < n_stages; ++st, ++stage_ctr) {
                const int s = stage_ctr % kPStages;
                mbar_wait(&empty_p[s], ((stage_ctr / kPStages) & 1) ^ 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_p[s], kPackedStage + kScaleStage);
                    uint8_t *pk = smem + kOffPacked + s * kPackedStage;
                    uint8_t *sc = smem + kOffScale + s * kScaleStage;
                    const int kb = st * (kStageK / 2);
                    for (int c = 0; c < 2; ++c) {
                        tma_load_2d(pk + c * kPackedCol, &wmap, kb + 128 * c, row_a, &full_p[s]);
                        tma_load_2d(pk + c * kPackedCol + 64 * 128, &wmap, kb + 128 * c, row_b, &full_p[s]);
                    }
                    tma_load_2d(sc, &smap, st * (kStageK / 32), row_a, &full_p[s]);
                    tma_load_2d(sc + 64 * 16, &smap, st * (kStageK / 32), row_b, &full_p[s]);
                }
                __syncwarp();
                ++issued;
            }
            if (aborted) break;
        }
        // let the issued copies land (before the end marker reuses a ring slot), then the marker
        for (int i = 0; i < kPStages && i < issued; ++i) {
            const int sc = issued - 1 - i;
            mbar_wait_drain(&full_p[sc % kPStages], (sc / kPStages) & 1, status);
        }
        if (!aborted) {
            const int s = stage_ctr % kPStages;
            mbar_wait(&empty_p[s], ((stage_ctr / kPStages) & 1) ^ 1, aborted, status);
            if (!aborted && lane == 0) {
                item_q[item_ctr % kItemQ] = -1;
                mbar_arrive(&pub[item_ctr % kItemQ]);
                mbar_arrive(&full_p[s]);
            }
        }
    } else if (warp == kBProd) {
        // ------------------------------------------------------------ activations producer
        if (lane == 0) prefetch_tensormap(&bmap);
        int sub_ctr = 0, issued = 0;
        for (int item_ctr = 0;; ++item_ctr) {
            mbar_wait(&pub[item_ctr % kItemQ], (item_ctr / kItemQ) & 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (aborted) break;
            const int item = item_q[item_ctr % kItemQ];
            if (item < 0) break;
            const WideTile *tp = a.tiles + item / row_blocks;
            const int p0 = __ldcg(&tp->p0), cnt = __ldcg(&tp->count);
            const int nbox = (cnt + 15) / 16;
            for (int j = 0; j < n_stages * kSubs; ++j, ++sub_ctr) {
                const int bb = sub_ctr % kBBufs;
                mbar_wait(&b_empty[bb], ((sub_ctr / kBBufs) & 1) ^ 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) break;
                if (lane == 0) mbar_arrive_expect_tx(&b_full[bb], static_cast<uint32_t>(nbox * kBBox));
                __syncwarp();
                if (lane < nbox)
                    tma_load_2d(smem + kOffB + bb * kBTile + lane * kBBox, &bmap, j * kSubK, p0 + 16 * lane, &b_full[bb]);
                ++issued;
            }
            if (aborted) break;
        }
        for (int i = 0; i < kBBufs && i < issued; ++i) {
            const int sc = issued - 1 - i;
            mbar_wait_drain(&b_full[sc % kBBufs], (sc / kBBufs) & 1, status);
        }
    }
    else if (warp >= kDeq0 && warp < kDeq0 + kDeqWarps) {
        // ------------------------------------------------------------ dequant warps
        // a warp stores TMEM lanes 32 (warp % 4) ..; its thread owns A row ar = that lane and the
        // K half h (warps 4..7: low 32 K, 8..11: high 32 K) of each 64-K sub-tile
        const int dw = warp - kDeq0;
        const int quarter = warp & 3, h = dw >> 2;
        const int ar = 32 * quarter + lane;
        // packed row of A row ar: A rows 2i, 2i + 1 = gate row i (box rows 0..63), up row i (box
        // rows 64..127) for gate_up; row ar for down
        const int r = kGateUp ? (ar >> 1) + (ar & 1) * 64 : ar;
        const uint32_t a_lane = static_cast<uint32_t>(32 * quarter) << 16;
        bool bad_scale = false;
        int stage_ctr = 0, sub_ctr = 0;
        for (int item_ctr = 0;; ++item_ctr) {
            // the item's first stage (or the end marker) names the item
            mbar_wait(&full_p[stage_ctr % kPStages], (stage_ctr / kPStages) & 1, aborted, status);
            if (aborted) break;
            const int item = item_q[item_ctr % kItemQ];
            for (int st = 0; st < (item < 0 ? 1 : n_stages); ++st) {
                const int s = stage_ctr % kPStages;
                if (st > 0) {
                    mbar_wait(&full_p[s], (stage_ctr / kPStages) & 1, aborted, status);
                    if (aborted) break;
                }
                const uint8_t *pk = smem + kOffPacked + s * kPackedStage;
                const uint8_t *sc = smem + kOffScale + s * kScaleStage;
                for (int j = 0; j < (item < 0 ? 1 : kSubs); ++j, ++sub_ctr) {
                    const int ab = sub_ctr % kABufs;
                    mbar_wait(&a_empty[ab], ((sub_ctr / kABufs) & 1) ^ 1, aborted, status);
                    if (aborted) break;
                    tc_fence_after();   // the MMAs that read this A buffer are complete
                    if (item >= 0) {
                        // 16 packed bytes: box column j / 4, 16-byte chunk (j % 4) * 2 + h of row r
                        const int ch = (j & 3) * 2 + h;
                        const uint4 w = *reinterpret_cast<const uint4 *>(pk + (j >> 2) * kPackedCol + r * 128 +
                                                                         ((ch ^ (r & 7)) << 4));
                        const uint32_t sbyte = sc[r * 16 + 2 * j + h];
                        bad_scale |= (sbyte < 104u) | (sbyte > 140u);
                        // 2^(sbyte - 127) as f16 (exact for 103 <= sbyte <= 142), in both halves
                        const __half s16 = __float2half_rn(__int_as_float(static_cast<int>(sbyte << 23)));
                        const __half2 s2 = __halves2half2(s16, s16);
                        uint32_t f[16];
                        e2m1x8_to_f16x2(w.x, f[0], f[1], f[2], f[3]);
                        e2m1x8_to_f16x2(w.y, f[4], f[5], f[6], f[7]);
                        e2m1x8_to_f16x2(w.z, f[8], f[9], f[10], f[11]);
                        e2m1x8_to_f16x2(w.w, f[12], f[13], f[14], f[15]);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            __half2 v = *reinterpret_cast<__half2 *>(&f[i]);
                            v = __hmul2(v, s2);
                            f[i] = *reinterpret_cast<uint32_t *>(&v);
                        }
                        // columns 16h .. 16h + 15 of the buffer: K 32h + 2i, 32h + 2i + 1 in column 16h + i
                        tmem_st16(tmem + a_lane + static_cast<uint32_t>(kACol0 + ab * kACols + 16 * h), f);
                    }
                    if (dw == 0 && lane == 0) a_item[ab] = item;
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a_full[ab]);
                }
                if (aborted) break;
                if (item < 0) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_p[s]);
                ++stage_ctr;
            }
            if (aborted || item < 0) break;
        }
        if (__any_sync(0xffffffffu, bad_scale) && lane == 0) record_status(status, kStatusUnsupported);
    } else if (warp == kMma) {
        // ------------------------------------------------------------ MMA issuer
        int sub_ctr = 0, bsub = 0;
        for (int item_ctr = 0;; ++item_ctr) {
            const int db = item_ctr % kDBufs;
            int ab = sub_ctr % kABufs;
            mbar_wait(&a_full[ab], (sub_ctr / kABufs) & 1, aborted, status);
            if (aborted) break;
            const int item = a_item[ab];
            // the accumulator's previous item must have left the epilogue (also before the end
            // marker, whose arrival would otherwise make that item's phase look pending again)
            mbar_wait(&d_empty[db], ((item_ctr / kDBufs) & 1) ^ 1, aborted, status);
            if (aborted) break;
            if (item < 0) {
                if (lane == 0) {
                    d_item[db] = -1;
                    mbar_arrive(&d_full[db]);
                }
                break;
            }
            if (lane == 0) d_item[db] = item;
            const WideTile *tp = a.tiles + item / row_blocks;
            const int n_mma = ((__ldcg(&tp->count) + 15) / 16) * 16;
            const uint32_t idesc = umma_idesc_f16(kRows, n_mma);
            const uint32_t d_tmem = tmem + static_cast<uint32_t>(db * kWideTokens);
            for (int j = 0; j < n_stages * kSubs; ++j, ++sub_ctr, ++bsub) {
                ab = sub_ctr % kABufs;
                const int bb = bsub % kBBufs;
                if (j > 0) mbar_wait(&a_full[ab], (sub_ctr / kABufs) & 1, aborted, status);
                mbar_wait(&b_full[bb], (bsub / kBBufs) & 1, aborted, status);
                if (aborted) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_tmem = tmem + static_cast<uint32_t>(kACol0 + ab * kACols);
                    const uint32_t b_addr = smem_u32(smem + kOffB + bb * kBTile);
#pragma unroll
                    for (int ks = 0; ks < kSubK / 16; ++ks)
                        umma_f16_tmem_a(d_tmem, a_tmem + 8 * ks, umma_sdesc_sw128(b_addr + 32 * ks), idesc,
                                        (j > 0 || ks > 0) ? 1u : 0u);
                    umma_commit(smem_u32(&a_empty[ab]));
                    umma_commit(smem_u32(&b_empty[bb]));
                }
                __syncwarp();
            }
            if (aborted) break;
            if (lane == 0) umma_commit(smem_u32(&d_full[db]));
            __syncwarp();
        }
        // every MMA this thread issued is complete before the tensor memory can be freed
        if (lane == 0) umma_commit(smem_u32(mma_done));
        __syncwarp();
        bool gave_up = false;
        mbar_wait(mma_done, 0, gave_up, status);
    }
    else if (warp >= kEpi0) {
        // ------------------------------------------------------------ epilogue warps
        const int quarter = warp & 3;                    // TMEM lanes 32 * quarter .. + 31
        const int row = 32 * quarter + lane;             // accumulator row (A row)
        for (int item_ctr = 0;; ++item_ctr) {
            const int db = item_ctr % kDBufs;
            mbar_wait(&d_full[db], (item_ctr / kDBufs) & 1, aborted, status);
            if (aborted) break;
            tc_fence_after();
            const int item = d_item[db];
            if (item < 0) break;
            const WideTile *tp = a.tiles + item / row_blocks;
            const int rb = item % row_blocks;
            const int p0 = __ldcg(&tp->p0), cnt = __ldcg(&tp->count);
            const uint32_t taddr = tmem + static_cast<uint32_t>(db * kWideTokens) + (static_cast<uint32_t>(32 * quarter) << 16);
            // down: the tile's flat ids, loaded once per item (independent loads) into this warp's copy
            int *ids = reinterpret_cast<int *>(smem + kOffIds) + (warp - kEpi0) * kWideTokens;
            if (!kGateUp) {
                for (int i = lane; i < cnt; i += 32) ids[i] = __ldcg(&a.sorted_ids[p0 + i]);
                __syncwarp();
            }
            for (int c = 0; c < cnt; c += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + c, v);
                if (kGateUp) {
                    // even rows hold g, odd rows u of output column n
                    const int n = rb * 64 + (row >> 1);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float mine = __uint_as_float(v[j]);
                        const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
                        if (!(lane & 1) && c + j < cnt) {
                            const float hv = wide_clamp_swiglu(mine, other);
                            a.h[static_cast<size_t>(p0 + c + j) * I + n] =
                                __float2half_rn(__bfloat162float(__float2bfloat16_rn(hv)) * kHScale);
                        }
                    }
                } else {
                    // h carries the 2^10 storage scale; the routing weight is applied by the combine
                    const int r = rb * kRows + row;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c + j < cnt) a.y[static_cast<size_t>(ids[c + j]) * H + r] = __uint_as_float(v[j]) * (1.0f / kHScale);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
        }
    }
    // every role is done: the allocating warp frees the tensor memory
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMma) tmem_dealloc(tmem, kTmemCols);
}

// x_perm[p] = x16[sorted_ids[p] / k]: the activation rows in expert-grouped order, so that the
// wide kernel's activation boxes are plain TMA tiles.  One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __half *__restrict__ x16,
                                                          const int32_t *__restrict__ sorted_ids,
                                                          __half *__restrict__ x_perm, int n, int H, int k)
{
    pdl_wait();
    pdl_trigger();
    const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (p >= n) return;
    const int t = sorted_ids[p] / k;
    const uint4 *src = reinterpret_cast<const uint4 *>(x16 + static_cast<size_t>(t) * H);
    uint4 *dst = reinterpret_cast<uint4 *>(x_perm + static_cast<size_t>(p) * H);
    for (int i = threadIdx.x & 31; i < H / 8; i += 32) dst[i] = src[i];
}

int wide_smem_bytes() { return wide::kSmemBytes; }

cudaError_t launch_gather_rows(const __half *x16, const int32_t *sorted_ids, __half *x_perm, int n, int H, int k,
                               cudaStream_t s, bool pdl)
{
    return launch_ex(gather_rows_kernel, dim3((n + 7) / 8), dim3(256), 0, s, pdl, x16, sorted_ids, x_perm, n, H, k);
}

cudaError_t launch_wide(bool gate_up, const CUtensorMap &wmap, const CUtensorMap &smap, const CUtensorMap &bmap,
                        const WideTile *tiles, const int *n_tiles, int max_tiles, const int32_t *sorted_ids,
                        __half *h, float *y, int *status, int32_t *status_out, int H, int I,
                        cudaStream_t s, bool pdl)
{
    WideArgs a;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.sorted_ids = sorted_ids;
    a.h = h;
    a.y = y;
    a.status_ws = status;
    a.status_out = status_out;
    a.queue = status + (gate_up ? kQueueGateUpWide : kQueueDownWide);
    a.H = H;
    a.I = I;
    auto kern = gate_up ? grouped_wide_kernel<true> : grouped_wide_kernel<false>;
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(kern), wide::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long row_blocks = gate_up ? I / 64 : H / wide::kRows;
    const long long max_items = static_cast<long long>(max_tiles) * row_blocks;
    int grid = static_cast<int>(max_items < num_sms() ? max_items : num_sms());
    if (grid < 1) grid = 1;
    return launch_ex(kern, dim3(grid), dim3(wide::kThreads), wide::kSmemBytes, s, pdl, wmap, smap, bmap, a);
}

}  // namespace moe
