// grouped_wide.cu -- grouped MXFP4 expert GEMMs on the 5th-generation tensor cores, for the
// experts that receive kWideMinTokens or more routed assignments ("wide" tiles of up to
// kWideTokens assignments of one expert).
//
// "Compact routed MXFP4 GEMM" and "Routed clamp-SwiGLU" rows of "Post-Portfolio Device
// Attribution" ("MTP1 Post-Portfolio Eager-Cycle Profile"), with the fused gate/up producer of
// the page's "Decision" section.  At large token counts the expert GEMMs become real dense
// contractions: an expert with many assignments is streamed once for all of them (the narrow
// kernel in grouped_gemm.cu re-streams it for every 8 or 16 assignments), and the MMA runs on
// tcgen05 with the fp32 accumulator in tensor memory.  An item is one tile of an expert's
// assignments against 128 weight rows.
//
// Measured on this part (one CTA per SM issuing back to back): a kind::f16 MMA of 128 x N x 16
// with A in tensor memory takes about 40-50 cycles for N <= 64 and N / 2 above; every
// tcgen05.commit costs the issuing thread about 80 cycles and a check of an mbarrier phase about
// 100-130, even a completed one.  Inside this kernel the MMA warp shares its scheduler with
// ALU-heavy dequant warps and gets a small share of the issue slots (a clock64 timeline of one
// CTA: about 1500 cycles per 16-MMA unit, of which about 550 were its wait on the activation
// slot), so everything that can leave the MMA warp does: the dequant warps hand it large A units
// (one wait and one commit per 8 or 16 MMAs) only once their activations have landed, and its
// loop keeps the arithmetic between MMAs minimal.  The tensor memory is split by tile size (two
// kernels):
//  * small tiles (kWideMinTokens .. kWideSmallMax assignments): two 64-column accumulators and
//    three A units of 256 K (128 columns each);
//  * large tiles (up to kWideTokens): two 192-column accumulators and two A units of 128 K.
//
// One persistent CTA per SM, 16 warps:
//  * warp 0 (weights producer): per 512-K stage, TMA copies of the item's packed E2M1 rows
//    (128 rows x 256 bytes, 128-byte swizzle) and their E8M0 scales into a 3-stage ring;
//    items come from the call's work queue, the ids reach the other warps through shared
//    memory with the stage arrivals.
//  * warp 2 (activations producer): TMA copies of the item's activation rows (x gathered into
//    expert-grouped order for gate_up, h for down), 16 rows x 64 K per box, 128-byte swizzle,
//    into a 4-slot ring; a slot takes 1 to 8 consecutive 64-K sub-tiles, as many as fit, so
//    that narrow tiles keep many sub-tiles in flight against the copies' latency.  Rows past
//    the tile are read and ignored.
//  * warp 3 (activations watcher): waits on every slot load in load order and publishes the
//    count that has landed (a release store the dequant groups read with acquire loads).
//  * warps 4..11 (dequant, two groups of four): a group decodes a whole A unit, each thread
//    the weights of one row, to bf16 with the row's E8M0 block scales folded in
//    (mxfp4x8_to_bf16x2_p4: exact for every scale byte whose scaled values are bf16 values),
//    and stores them with tcgen05.st into the unit's A buffer in tensor memory (TMEM lane = A
//    row; a warp reaches the 32 lanes of its warp index mod 4).  The groups take units in turn
//    (group g always unit g), so one group's decoding overlaps the other's hand-over.  The
//    decode pairs K 8j+i with 8j+i+4 in a TMEM column, so the activation rows are stored in the
//    matching P4 K order (common.cuh): x by the router (gathered into x_perm by
//    gather_wide_rows_kernel), h by the gate_up epilogues.  gate_up interleaves gate row i and
//    up row i as A rows 2i, 2i+1, so one TMEM lane pair holds g and u.  A never passes through
//    shared memory, which leaves shared-memory bandwidth to the TMA copies and the B operand.
//  * warp 1 (MMA): one thread issues the unit's tcgen05.mma kind::f16 with bf16 operands (A
//    from TMEM, B from shared memory; M 128, N = the tile's tokens rounded up to 16, K 16) into
//    one of two TMEM accumulators, commits the consumed A unit and B slots and, per item, the
//    accumulator.
//  * warps 12..15 (epilogue): tcgen05.ld of the accumulator (warp w reads TMEM lanes
//    32 (w % 4) ..); gate_up pairs g and u with one shuffle, applies clamp-SwiGLU and the bf16
//    rounding and stores h (bf16); down stores the assignment's fp32 row of y (the combine
//    applies the routing weight).
// Every wait is bounded; after a timeout the kernel records MOE_ERR_TIMEOUT, drains the
// copies it issued and frees its tensor memory.
#include <cuda_bf16.h>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace wide {
constexpr int kRows = 128;                               // weight rows per item (MMA M)
constexpr int kStageK = kWideStageK;                     // 512 K per packed stage
constexpr int kPStages = 3;                              // packed weight stages
constexpr int kSubK = 64;                                // K per B sub-tile (one 128-byte swizzle atom of bf16)
constexpr int kSubs = kStageK / kSubK;                   // 8
constexpr int kBBufs = 4, kDBufs = 2;
constexpr int kItemQ = 8;
// Warps: 0 weights producer, 1 MMA issuer, 2 activations producer, 3 activations watcher, 4..11
// dequant (two groups of four: a group covers the 128 TMEM lanes and decodes whole A units, the
// groups taking units in turn), 12..15 epilogue.
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kWProd = 0, kMma = 1, kBProd = 2, kBWatch = 3, kDeq0 = 4, kDeqGroups = 2, kDeqWarps = 4 * kDeqGroups;
constexpr int kEpi0 = kDeq0 + kDeqWarps, kEpiWarps = 4;
static_assert(kDeq0 % 4 == 0 && kEpi0 % 4 == 0, "a group of four warps reaches all 128 TMEM lanes");
constexpr int kPackedStage = kRows * kStageK / 2;        // 32 KB: 2 box columns x 128 rows x 128 B
constexpr int kPackedCol = kRows * 128;                  // one box column (two 64-row boxes)
constexpr int kScaleStage = kRows * kStageK / 32;        // 2 KB: 128 rows x 16 B
constexpr int kBTile = kWideTokens * kSubK * 2;          // one activation slot: 24 KB
constexpr int kBBox = 16 * kSubK * 2;                    // one 16-row activation box (2 KB)
constexpr int kBoxesPerSlot = kBTile / kBBox;            // 12
// A slot holds `spb` consecutive sub-tiles of a tile with nbox 16-row boxes each: as many as fit,
// a power of two up to 8 (so that the sub-tiles of an item, a multiple of 8, split into whole
// slots).  Narrow tiles thus keep up to 32 sub-tiles of activations in flight, wide ones 4.
__host__ __device__ constexpr int subs_per_slot(int nbox)
{
    return 8 * nbox <= kBoxesPerSlot ? 8 : (4 * nbox <= kBoxesPerSlot ? 4 : (2 * nbox <= kBoxesPerSlot ? 2 : 1));
}
// Tensor-memory partition of a tile class (512 columns): accumulators first, then the A units.
template <bool kSmall>
struct Part {
    static constexpr int kAccCols = kSmall ? kWideSmallMax : kWideTokens;   // max N of the class
    static constexpr int kUnitK = kSmall ? 256 : 128;                       // K per A unit
    static constexpr int kUnitSubs = kUnitK / kSubK;
    static constexpr int kACols = kUnitK / 2;                               // 2 bf16 per column
    static constexpr int kABufs = kSmall ? 3 : 2;
    // Units rotate over the dequant groups and over the A buffers.  A group that waits for unit
    // u's buffer (the release of unit u - kABufs) must know the phase before it (unit
    // u - 2 kABufs) has completed, since a parity wait cannot tell a phase from the one two
    // before it: its own previous unit u - kGroups waited for unit u - kGroups - kABufs, and
    // units complete in order, so kGroups <= kABufs suffices.
    static constexpr int kGroups = kDeqGroups;
    static_assert(kGroups <= kABufs, "a group's waits see the phases in order");
    static constexpr int kACol0 = kDBufs * kAccCols;
    static_assert(kACol0 + kABufs * kACols <= 512, "TMEM budget");
    static_assert(kGroups <= kDeqGroups, "enough dequant groups");
    static_assert(kStageK % kUnitK == 0, "units tile a stage");
};
constexpr int kTmemCols = 512;
constexpr int kMaxABufs = 3;
constexpr int kOffPacked = 0;
constexpr int kOffScale = kOffPacked + kPStages * kPackedStage;
constexpr int kOffB = kOffScale + kPStages * kScaleStage;
constexpr int kOffIds = kOffB + kBBufs * kBTile;         // down: each epilogue warp's copy of the tile's flat ids
constexpr int kOffBars = kOffIds + kEpiWarps * kWideTokens * 4;
constexpr int kSmemBytes = kOffBars + 512 + 1024;        // barriers and slots, + alignment slack
static_assert(kOffB % 1024 == 0 && kBTile % 1024 == 0 && kBBox % 1024 == 0,
              "swizzled tiles sit on 1024-byte boundaries");
static_assert(kWideTokens % 16 == 0 && kWideTokens / 16 <= kBoxesPerSlot, "a sub-tile of the widest tile fits a slot");
static_assert(kSmemBytes <= 227 * 1024, "fits one SM");
}  // namespace wide

struct WideArgs {
    const WideTile *tiles;
    const int *n_tiles;
    const int32_t *sorted_ids;   // down: flat ids of the expert-grouped positions
    __nv_bfloat16 *h;            // gate_up output [M*k][I] bf16, expert-grouped rows (P4 K order if h_p4)
    float *y;                    // down output [M*k][H] by flat id, before the routing weight
    int *status_ws;
    int32_t *status_out;
    int *queue;
    int H, I;
    int h_p4;                    // gate_up: store h in P4 K order (the down kernels' operand layout)
};

__device__ __forceinline__ float wide_clamp_swiglu(float g, float u)
{
    const float a = fminf(g, 7.0f);
    const float c = fminf(fmaxf(u, -7.0f), 7.0f);
    return a / (1.0f + expf(-a)) * c;
}

// One dequant thread's share of an A unit: packed row r of the stage (128-byte swizzled box
// columns), sub-tiles j0 .. j0 + kSubsN - 1 (64 K each), E8M0 bytes eb (byte b of the unit's block
// b, two blocks per sub-tile).  Each sub-tile's 64 weights become 32 TMEM columns of this thread's
// lane, K 64c + 32h + 8u + i in the low half of column 32c + 16h + 4u + i and + 4 in its high half
// (the P4 pairing).  kLarge: some byte of the warp exceeds 128, so the two-multiply decode.
// The stores are left in flight; the caller waits for them.
__device__ __forceinline__ void st_release_shared(int *p, int v)
{
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire_shared(const int *p)
{
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Bounded poll (whole warp) until the count at p reaches `target` (acquire: what the publisher
// observed before its release store is visible after).  Gives up like mbar_wait.
__device__ __forceinline__ void poll_count(const int *p, int target, bool &aborted, const StatusPtrs &st)
{
    if (aborted) return;
    if (__all_sync(0xffffffffu, ld_acquire_shared(p) >= target)) return;
    const long long t0 = clock64();
    while (!__all_sync(0xffffffffu, ld_acquire_shared(p) >= target)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            aborted = true;
            record_timeout(st);
            return;
        }
    }
}

template <int kSubsN, bool kLarge>
__device__ __forceinline__ void dequant_unit(const uint8_t *pk, int r, int j0, const uint32_t (&eb)[2], uint32_t a_unit)
{
    using namespace wide;
#pragma unroll
    for (int c = 0; c < kSubsN; ++c) {
        const int j = j0 + c;
        uint32_t f[32];
        uint4 w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int ch = (j & 3) * 2 + h;
            w[h] = *reinterpret_cast<const uint4 *>(pk + (j >> 2) * kPackedCol + r * 128 + ((ch ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int b = 2 * c + h;
            const uint32_t e = (eb[b >> 2] >> (8 * (b & 3))) & 0xFFu;
            uint32_t(&fo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&f[16 * h]);
            mxfp4x8_to_bf16x2_p4(w[h].x, e, kLarge, *reinterpret_cast<uint32_t(*)[4]>(&fo[0]));
            mxfp4x8_to_bf16x2_p4(w[h].y, e, kLarge, *reinterpret_cast<uint32_t(*)[4]>(&fo[4]));
            mxfp4x8_to_bf16x2_p4(w[h].z, e, kLarge, *reinterpret_cast<uint32_t(*)[4]>(&fo[8]));
            mxfp4x8_to_bf16x2_p4(w[h].w, e, kLarge, *reinterpret_cast<uint32_t(*)[4]>(&fo[12]));
        }
        tmem_st32(a_unit + static_cast<uint32_t>(32 * c), f);
    }
}

template <bool kGateUp, bool kSmall>
__global__ void __launch_bounds__(wide::kThreads, 1)
grouped_wide_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                    const __grid_constant__ CUtensorMap bmap, const __grid_constant__ WideArgs a)
{
    using namespace wide;
    using P = Part<kSmall>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
    uint64_t *full_p = bars, *empty_p = bars + kPStages;                       // packed stages
    uint64_t *a_full = bars + 2 * kPStages, *a_empty = a_full + kMaxABufs;     // A units
    uint64_t *b_full = a_empty + kMaxABufs, *b_empty = b_full + kBBufs;       // B slots
    uint64_t *d_full = b_empty + kBBufs, *d_empty = d_full + kDBufs;          // accumulators
    uint64_t *pub = d_empty + kDBufs;                                         // [kItemQ] item ids published
    uint64_t *mma_done = pub + kItemQ;                                        // final drain of the MMAs
    volatile int *item_q = reinterpret_cast<volatile int *>(mma_done + 1);   // [kItemQ]
    volatile int *a_item = item_q + kItemQ;                                   // [kMaxABufs]
    volatile int *d_item = a_item + kMaxABufs;                                // [kDBufs]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(const_cast<int *>(d_item + kDBufs));
    int *b_seq = reinterpret_cast<int *>(tmem_slot + 4);   // B slot loads known to have landed, in load order

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const StatusPtrs status{a.status_ws, a.status_out};
    const int H = a.H, I = a.I;
    const int K = kGateUp ? H : I;
    const int n_stages = K / kStageK;
    const int n_units = K / P::kUnitK;
    constexpr int kUnitsPerStage = kStageK / P::kUnitK;
    const int row_blocks = kGateUp ? I / 64 : H / kRows;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full_p[s], 1);
            mbar_init(&empty_p[s], kDeqWarps);
        }
        for (int b = 0; b < P::kABufs; ++b) {
            mbar_init(&a_full[b], 4);   // the four warps of the group that decoded the unit
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
        *b_seq = 0;
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
                uint8_t *pk = smem + kOffPacked + s * kPackedStage;
                uint8_t *sc = smem + kOffScale + s * kScaleStage;
                const int kb = st * (kStageK / 2);
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full_p[s], kPackedStage + kScaleStage);
#pragma unroll
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
        int bload = 0, issued = 0;   // slot loads so far / issued (a prefix of them)
        for (int item_ctr = 0;; ++item_ctr) {
            mbar_wait(&pub[item_ctr % kItemQ], (item_ctr / kItemQ) & 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (aborted) break;
            const int item = item_q[item_ctr % kItemQ];
            if (item < 0) break;
            const WideTile *tp = a.tiles + item / row_blocks;
            const int p0 = __ldcg(&tp->p0), cnt = __ldcg(&tp->count);
            const int nbox = (cnt + 15) / 16;
            const int spb = subs_per_slot(nbox);
            for (int j0 = 0; j0 < n_stages * kSubs; j0 += spb, ++bload) {
                const int bb = bload % kBBufs;
                mbar_wait(&b_empty[bb], ((bload / kBBufs) & 1) ^ 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) break;
                // box (sub-tile u, rows 16 b..) -> slot offset (u * nbox + b) boxes
                uint8_t *slot = smem + kOffB + bb * kBTile;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&b_full[bb], static_cast<uint32_t>(spb * nbox * kBBox));
                    for (int u = 0; u < spb; ++u)
                        for (int bx = 0; bx < nbox; ++bx)
                            tma_load_2d(slot + (u * nbox + bx) * kBBox, &bmap, (j0 + u) * kSubK, p0 + 16 * bx,
                                        &b_full[bb]);
                }
                __syncwarp();
                ++issued;
            }
            if (aborted) break;
        }
        for (int i = 0; i < kBBufs && i < issued; ++i) {
            const int sc = issued - 1 - i;
            mbar_wait_drain(&b_full[sc % kBBufs], (sc / kBBufs) & 1, status);
        }
    } else if (warp == kBWatch) {
        // ------------------------------------------------------------ B landing watcher
        // Waits on every activation slot load in load order (an in-order waiter always sees the
        // load's own barrier phase) and publishes how many have landed.  The dequant group of a
        // unit checks that count before it hands the unit to the MMA warp, so the MMA warp's only
        // wait per unit is the unit's own.
        int bload = 0;
        for (int item_ctr = 0;; ++item_ctr) {
            mbar_wait(&pub[item_ctr % kItemQ], (item_ctr / kItemQ) & 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (aborted) break;
            const int item = item_q[item_ctr % kItemQ];
            if (item < 0) break;
            const WideTile *tp = a.tiles + item / row_blocks;
            const int spb = subs_per_slot((__ldcg(&tp->count) + 15) / 16);
            for (int j0 = 0; j0 < n_stages * kSubs; j0 += spb, ++bload) {
                mbar_wait(&b_full[bload % kBBufs], (bload / kBBufs) & 1, aborted, status);
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) break;
                if (lane == 0) st_release_shared(b_seq, bload + 1);
            }
            if (aborted) break;
        }
    } else if (warp >= kDeq0 && warp < kDeq0 + kDeqWarps) {
        // ------------------------------------------------------------ dequant warps
        // group grp takes the units whose running index u is grp mod P::kGroups, into A buffer
        // u mod P::kABufs; a warp stores TMEM lanes 32 (warp % 4) ..; its thread owns A row
        // ar = that lane, all K of the unit.  Every group releases every stage.
        const int grp = (warp - kDeq0) >> 2;
        const int quarter = warp & 3;
        const int ar = 32 * quarter + lane;
        // packed row of A row ar: A rows 2i, 2i + 1 = gate row i (box rows 0..63), up row i (box
        // rows 64..127) for gate_up; row ar for down
        const int r = kGateUp ? (ar >> 1) + (ar & 1) * 64 : ar;
        const uint32_t a_lane = static_cast<uint32_t>(32 * quarter) << 16;
        int stage_ctr = 0, unit_ctr = 0;   // every group counts every stage and unit
        int bload_base = 0;                // activation slot loads of the items before this one
        for (int item_ctr = 0;; ++item_ctr) {
            // the item's first stage (or the end marker) names the item
            mbar_wait(&full_p[stage_ctr % kPStages], (stage_ctr / kPStages) & 1, aborted, status);
            if (aborted) break;
            const int item = item_q[item_ctr % kItemQ];
            if (item < 0) {
                // the end marker reaches the MMA warp as one more unit, from the group whose turn it is
                if (unit_ctr % P::kGroups == grp) {
                    const int ab = unit_ctr % P::kABufs;
                    mbar_wait(&a_empty[ab], ((unit_ctr / P::kABufs) & 1) ^ 1, aborted, status);
                    if (!aborted) {
                        if (quarter == 0 && lane == 0) a_item[ab] = -1;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&a_full[ab]);
                    }
                }
                break;
            }
            // the item's activation slots (the loads the B producer issues for it, in order)
            const WideTile *tp = a.tiles + item / row_blocks;
            const int spb_shift = __ffs(subs_per_slot((__ldcg(&tp->count) + 15) / 16)) - 1;
            for (int st = 0; st < n_stages; ++st) {
                const int s = stage_ctr % kPStages;
                if (st > 0) {
                    mbar_wait(&full_p[s], (stage_ctr / kPStages) & 1, aborted, status);
                    if (aborted) break;
                }
                const uint8_t *pk = smem + kOffPacked + s * kPackedStage;
                const uint8_t *sc = smem + kOffScale + s * kScaleStage;
                for (int uu = 0; uu < kUnitsPerStage; ++uu, ++unit_ctr) {
                    if (unit_ctr % P::kGroups != grp) continue;
                    const int ab = unit_ctr % P::kABufs;
                    mbar_wait(&a_empty[ab], ((unit_ctr / P::kABufs) & 1) ^ 1, aborted, status);
                    if (aborted) break;
                    tc_fence_after();   // the MMAs that read this A unit are complete
                    // the unit's E8M0 bytes of row r (2 per 64-K sub-tile), one load; the scale
                    // folds into the decode's multiply unless some byte of the warp exceeds 128
                    uint32_t eb[2];
                    if (P::kUnitSubs == 4) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(sc + r * 16 + uu * 8);
                        eb[0] = v.x;
                        eb[1] = v.y;
                    } else {
                        eb[0] = *reinterpret_cast<const uint32_t *>(sc + r * 16 + uu * 4);
                        eb[1] = 0;
                    }
                    const bool large = __any_sync(0xffffffffu, __vcmpgtu4(eb[0], 0x80808080u) | __vcmpgtu4(eb[1], 0x80808080u));
                    const uint32_t a_unit = tmem + a_lane + static_cast<uint32_t>(P::kACol0 + ab * P::kACols);
                    if (!large)
                        dequant_unit<P::kUnitSubs, false>(pk, r, uu * P::kUnitSubs, eb, a_unit);
                    else
                        dequant_unit<P::kUnitSubs, true>(pk, r, uu * P::kUnitSubs, eb, a_unit);
                    tmem_wait_st();
                    if (quarter == 0) {
                        // the unit's activations have landed: the last slot load its sub-tiles use
                        const int last_sub = (st * kUnitsPerStage + uu + 1) * P::kUnitSubs - 1;
                        poll_count(b_seq, bload_base + (last_sub >> spb_shift) + 1, aborted, status);
                        if (lane == 0) a_item[ab] = item;
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a_full[ab]);
                }
                if (aborted) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_p[s]);
                ++stage_ctr;
            }
            if (aborted) break;
            bload_base += (n_stages * kSubs) >> spb_shift;
        }
    } else if (warp == kMma) {
        // ------------------------------------------------------------ MMA issuer
        // The warp shares its scheduler with ALU-heavy dequant warps and gets a small share of
        // its issue slots, so its loop keeps the arithmetic between MMAs minimal: ring indices
        // and phase bits advance incrementally, slot sizes are powers of two.
        int unit_ctr = 0;
        int bb = 0;               // slot of the current activation load (load count % kBBufs)
        int ab = 0;               // A buffer of unit unit_ctr (unit_ctr % kABufs)
        uint32_t a_par = 0;       // phase parity of that buffer ((unit_ctr / kABufs) & 1)
        for (int item_ctr = 0;; ++item_ctr) {
            const int db = item_ctr % kDBufs;
            mbar_wait(&a_full[ab], a_par, aborted, status);
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
            const int nbox = (__ldcg(&tp->count) + 15) / 16;
            const int spb = subs_per_slot(nbox);   // a power of two
            const uint32_t idesc = umma_idesc_bf16(kRows, 16 * nbox);
            const uint32_t d_tmem = tmem + static_cast<uint32_t>(db * P::kAccCols);
            // B descriptor units (16 bytes) between consecutive sub-tiles of a slot
            const uint32_t b_step = static_cast<uint32_t>(nbox * kBBox) >> 4;
            for (int u = 0; u < n_units; ++u, ++unit_ctr) {
                if (u > 0) mbar_wait(&a_full[ab], a_par, aborted, status);
                if (aborted) break;
                tc_fence_after();
                const uint32_t a_unit = tmem + static_cast<uint32_t>(P::kACol0 + ab * P::kACols);
                // the unit's sub-tiles, one B slot at a time (their activations have landed: the
                // dequant group checked before handing the unit over); one elected lane issues all of
                // the slot's MMAs of this unit back to back
                for (int c0 = 0; c0 < P::kUnitSubs;) {
                    const int j = u * P::kUnitSubs + c0;
                    const int uo = j & (spb - 1);
                    const int nsub = min(spb - uo, P::kUnitSubs - c0);
                    const bool slot_end = uo + nsub == spb;
                    const bool unit_end = c0 + nsub == P::kUnitSubs;
                    const uint64_t b0 = umma_sdesc_sw128(smem_u32(smem + kOffB + bb * kBTile + uo * nbox * kBBox));
                    if (elect_one()) {
#pragma unroll
                        for (int c = 0; c < P::kUnitSubs; ++c) {
                            if (c < nsub) {
                                // K steps of 16 advance A by 8 columns and B by 32 bytes (2 in the descriptor)
                                const uint32_t at = a_unit + static_cast<uint32_t>(32 * (c0 + c));
                                const uint64_t bd = b0 + static_cast<uint64_t>(c) * b_step;
                                umma_f16_tmem_a(d_tmem, at, bd, idesc, (j + c == 0) ? 0u : 1u);
                                umma_f16_tmem_a(d_tmem, at + 8, bd + 2, idesc, 1u);
                                umma_f16_tmem_a(d_tmem, at + 16, bd + 4, idesc, 1u);
                                umma_f16_tmem_a(d_tmem, at + 24, bd + 6, idesc, 1u);
                            }
                        }
                        if (slot_end) umma_commit(smem_u32(&b_empty[bb]));   // the slot's last sub-tile
                        if (unit_end) umma_commit(smem_u32(&a_empty[ab]));
                    }
                    __syncwarp();
                    if (slot_end && ++bb == kBBufs) bb = 0;
                    c0 += nsub;
                }
                if (aborted) break;
                if (++ab == P::kABufs) {
                    ab = 0;
                    a_par ^= 1u;
                }
            }
            if (aborted) break;
            if (elect_one()) umma_commit(smem_u32(&d_full[db]));
            __syncwarp();
        }
        // every MMA this warp issued is complete before the tensor memory can be freed
        if (elect_one()) umma_commit(smem_u32(mma_done));
        __syncwarp();
        bool gave_up = false;
        mbar_wait(mma_done, 0, gave_up, status);
    } else if (warp >= kEpi0) {
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
            const uint32_t taddr =
                tmem + static_cast<uint32_t>(db * P::kAccCols) + (static_cast<uint32_t>(32 * quarter) << 16);
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
                    const int col = a.h_p4 ? p4_pos(n) : n;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float mine = __uint_as_float(v[j]);
                        const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
                        if (!(lane & 1) && c + j < cnt)
                            a.h[static_cast<size_t>(p0 + c + j) * I + col] = __float2bfloat16_rn(wide_clamp_swiglu(mine, other));
                    }
                } else {
                    // the unweighted row; the routing weight is applied by the combine
                    const int r = rb * kRows + row;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c + j < cnt) a.y[static_cast<size_t>(ids[c + j]) * H + r] = __uint_as_float(v[j]);
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

// x_perm[p] = x_p4[sorted_ids[p] / k] (rows already in P4 K order), for the positions p of the
// wide tiles only (the rows the wide kernels' activation boxes read; the other rows of x_perm are
// never read).  CTA (w, c) copies rows 8c .. 8c + 7 of wide tile w -- tiles [0, max_small) of the
// small-tile list, then those of the large-tile list -- one warp per row, 16 bytes a lane.
__global__ void __launch_bounds__(256) gather_wide_rows_kernel(const __nv_bfloat16 *__restrict__ x_p4,
                                                               const int32_t *__restrict__ sorted_ids, WideLists wl,
                                                               __nv_bfloat16 *__restrict__ x_perm, int H, int k)
{
    pdl_wait();
    pdl_trigger();
    const bool small = static_cast<int>(blockIdx.x) < wl.max_small;
    const int w = small ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - wl.max_small;
    if (w >= __ldcg(small ? wl.n_small : wl.n_large)) return;
    const WideTile *tp = (small ? wl.small : wl.large) + w;
    const int p0 = __ldcg(&tp->p0), cnt = __ldcg(&tp->count);
    const int i = blockIdx.y * 8 + (threadIdx.x >> 5);
    if (i >= cnt) return;
    const int p = p0 + i;
    const int t = __ldcg(&sorted_ids[p]) / k;
    const uint4 *src = reinterpret_cast<const uint4 *>(x_p4 + static_cast<size_t>(t) * H);
    uint4 *dst = reinterpret_cast<uint4 *>(x_perm + static_cast<size_t>(p) * H);
    for (int g = threadIdx.x & 31; g < H / 8; g += 32) dst[g] = __ldcg(&src[g]);
}

int wide_smem_bytes() { return wide::kSmemBytes; }

cudaError_t launch_gather_wide_rows(const __nv_bfloat16 *x_p4, const int32_t *sorted_ids, const WideLists &wl,
                                    __nv_bfloat16 *x_perm, int H, int k, cudaStream_t s, bool pdl)
{
    const int n = wl.max_small + wl.max_large;
    const dim3 grid(n > 0 ? n : 1, (kWideTokens + 7) / 8);
    return launch_ex(gather_wide_rows_kernel, grid, dim3(256), 0, s, pdl, x_p4, sorted_ids, wl, x_perm, H, k);
}

template <bool kGateUp, bool kSmall>
static cudaError_t launch_wide_t(const CUtensorMap &wmap, const CUtensorMap &smap, const CUtensorMap &bmap,
                                 const WideArgs &a, int max_tiles, cudaStream_t s, bool pdl)
{
    auto kern = grouped_wide_kernel<kGateUp, kSmall>;
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(kern), wide::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long row_blocks = kGateUp ? a.I / 64 : a.H / wide::kRows;
    const long long max_items = static_cast<long long>(max_tiles) * row_blocks;
    int grid = static_cast<int>(max_items < num_sms() ? max_items : num_sms());
    if (grid < 1) grid = 1;
    return launch_ex(kern, dim3(grid), dim3(wide::kThreads), wide::kSmemBytes, s, pdl, wmap, smap, bmap, a);
}

cudaError_t launch_wide(bool gate_up, bool small, const CUtensorMap &wmap, const CUtensorMap &smap,
                        const CUtensorMap &bmap, const WideTile *tiles, const int *n_tiles, int max_tiles,
                        const int32_t *sorted_ids, __nv_bfloat16 *h, bool h_p4, float *y, int *status,
                        int32_t *status_out, int H, int I, cudaStream_t s, bool pdl)
{
    WideArgs a;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.sorted_ids = sorted_ids;
    a.h = h;
    a.y = y;
    a.status_ws = status;
    a.status_out = status_out;
    a.queue = status + (gate_up ? (small ? kQueueGateUpWide : kQueueGateUpWideL)
                                : (small ? kQueueDownWide : kQueueDownWideL));
    a.H = H;
    a.I = I;
    a.h_p4 = h_p4 ? 1 : 0;
    if (gate_up)
        return small ? launch_wide_t<true, true>(wmap, smap, bmap, a, max_tiles, s, pdl)
                     : launch_wide_t<true, false>(wmap, smap, bmap, a, max_tiles, s, pdl);
    return small ? launch_wide_t<false, true>(wmap, smap, bmap, a, max_tiles, s, pdl)
                 : launch_wide_t<false, false>(wmap, smap, bmap, a, max_tiles, s, pdl);
}

}  // namespace moe
