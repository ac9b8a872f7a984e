// Host-side check of the launch-planning helpers in moe_internal.h over a grid of shapes: the
// router plan covers every token and every K element and fills at most one wave of CTAs, the tile
// width and fused-select switches follow their stated rules, the per-shape shared-memory needs fit
// a B200 CTA, the mma.sync kernels' activation shift keeps every finite bf16 row in range, and the
// fused down + combine kernel's shared-memory accesses and copies stay inside its plan.
// Built and run by tests/test_host_plan.py (no GPU needed).
#include <cmath>
#include <cstdio>

#include "down_slab.h"
#include "moe_internal.h"

using namespace moe;

static int fails = 0;
#define CHECK(cond, M, H, E, k)                                                                  \
    do {                                                                                         \
        if (!(cond) && fails++ < 20)                                                             \
            std::printf("FAIL %s at M=%d H=%d E=%d k=%d\n", #cond, (M), (H), (E), (k));          \
    } while (0)

int main()
{
    const int Hs[] = {32, 96, 512, 1024, 2048, 4096, 7168, 16384};
    const int Es[] = {1, 4, 16, 100, 128, 256, 1000, 1024};
    const int Ks[] = {1, 2, 4, 8, 32};
    long long cases = 0;
    for (int M = 1; M <= 1024; ++M) {
        for (int H : Hs) {
            for (int E : Es) {
                const RoutePlan p = route_plan(M, H, E);
                CHECK(p.tiles == 1 || p.tiles == 4, M, H, E, 0);
                CHECK(p.steps == 2 || p.steps == 4, M, H, E, 0);
                // token blocks cover M exactly (no empty block)
                const int tb = 8 * p.tiles;
                CHECK(p.blocks_t * tb >= M && (p.blocks_t - 1) * tb < M, M, H, E, 0);
                // the H slices cover H (a slice past H reads zeros and writes zero partials)
                const long long per_unit = static_cast<long long>(kRouteWarps) * 16 * p.steps;
                CHECK(p.splits >= 1 && p.passes >= 1, M, H, E, 0);
                CHECK(static_cast<long long>(p.splits) * p.passes * per_unit >= H, M, H, E, 0);
                // at most one wave of the planned SM count, unless the plan is already unsplit
                const long long ctas = static_cast<long long>((E + kRouteExperts - 1) / kRouteExperts) * p.splits *
                                       p.blocks_t;
                const int cap = (p.tiles == 1 ? 4 : 2) * kPlanSMs;
                CHECK(p.splits == 1 || ctas <= cap, M, H, E, 0);
                for (int k : Ks) {
                    if (k > E || static_cast<long long>(M) * k > kMaxAssignments) continue;
                    ++cases;
                    const int w = tile_width(M, E, k);
                    CHECK(w == 8 || w == 16, M, H, E, k);
                    CHECK((w == 16) == (static_cast<long long>(M) * k >= 6LL * E), M, H, E, k);
                    CHECK(w <= kTileTokensMax, M, H, E, k);
                    // the fused select keeps one 64-bit token mask per expert, one thread per
                    // assignment and the M x E logits in shared memory
                    const bool fs = fused_select(M, E, k);
                    const bool fits = M <= 64 && M * k <= kPermuteThreads && M * E <= kFusedSelectMaxLogits;
                    CHECK(fs == fits, M, H, E, k);
                }
            }
        }
        for (int H : Hs)
            for (int I : Hs)
                for (int E : Es)
                    for (int k : Ks) {
                        if (k > E) continue;
                        // the tensor-core path needs whole 512-element stages, calls in which an
                        // expert can reach kWideMinTokens assignments, and experts averaging at
                        // least half that
                        if (wide_enabled(M, H, I, E, k))
                            CHECK(M >= kWideMinTokens && H % 512 == 0 && I % 512 == 0 &&
                                      2LL * M * k >= 1LL * kWideMinTokens * E,
                                  M, H, E, I);
                    }
    }
    for (int H = 32; H <= 16384; H += 32) {
        CHECK(down_row_blocks(H) * kItemRows >= H && (down_row_blocks(H) - 1) * kItemRows < H, 0, H, 0, 0);
        CHECK(per_stage_scales(H) == (H % 512 == 0), 0, H, 0, 0);
    }
    CHECK(permute_smem_bytes(kMaxE) <= 227 * 1024, 0, 0, kMaxE, 0);
    // the fused select's static arrays (token masks, offsets, tile bases, assignment experts)
    // plus its staged logits
    CHECK(kMaxE * (8 + 4 * 4) + kPermuteThreads * 4 + kFusedSelectMaxM * 4 + kFusedSelectMaxLogits * 4 <= 227 * 1024,
          0, 0, kMaxE, 0);
    // The mma.sync kernels' activation shift: for the largest |x| of a token (every finite bf16
    // magnitude m), x * 2^s must stay below 2^121 (bf16 and the products stay finite: the weights
    // enter as value * 2^-126 <= 6 * 2^-126), and reach 2^120 unless the shift is at its cap of 127
    // (tiny rows), so that products keep fp32's normal range.
    for (uint32_t m = 0; m <= 0x7F7Fu; ++m) {
        const int s = x_shift_from_max(m);
        const int e = static_cast<int>(m >> 7), mant = static_cast<int>(m & 0x7F);
        const double v = e == 0 ? std::ldexp(static_cast<double>(mant), -133)
                                : std::ldexp(1.0 + mant / 128.0, e - 127);
        const double shifted = std::ldexp(v, s);
        CHECK(s >= -7 && s <= 127, static_cast<int>(m), s, 0, 0);
        CHECK(shifted < std::ldexp(1.0, 121), static_cast<int>(m), s, 0, 0);
        CHECK(s == 127 || shifted >= std::ldexp(1.0, 120), static_cast<int>(m), s, 0, 0);
        CHECK(s == 127 || e >= 1, static_cast<int>(m), s, 0, 0);
    }
    // The fused down + combine kernel (down_slab.cu): for every shape it serves, its shared-memory
    // plan fits a CTA and every access the kernel makes stays inside its region -- the weight boxes
    // (16 rows x 128 bytes per box column, 1024-byte aligned for the 128-byte swizzle), the scale
    // rows, kSlabTileRows h rows, the fp32 rows of the M*k assignments, the tile list and the
    // barriers -- and every bulk copy has the 16-byte alignment and size it needs.
    for (int M = 1; M <= kSlabMaxM; ++M)
        for (int I = 32; I <= kSlabMaxI; I += 32)
            for (int k = 1; k <= kMaxK; ++k) {
                const SlabPlan p = slab_plan(M, I, k);
                const bool on = slab_enabled(M, I, 1024, k, 8, false);
                CHECK(on == (p.stages >= 2 && M * k <= kSlabMaxTiles), M, I, 0, k);
                // the plan itself is checked for every (M, I, k) the tile bound could admit (small E)
                if (p.stages < 2) continue;
                const int kblocks = I / 32, cols = (I / 2 + 127) / 128;
                CHECK(p.total <= 227 * 1024 && p.stages <= kSlabMaxStages, M, I, 0, k);
                CHECK(p.stage_bytes % 1024 == 0 && p.wbytes == cols * kSlabBoxBytes, M, I, 0, k);
                // compute reads: weight word q of rows g, g + 8 in box column blk / 8, swizzled chunk
                int wmax = 0, smax = 0, hmax = 0;
                for (int blk = 0; blk < kblocks; ++blk)
                    for (int g = 0; g < 8; ++g)
                        for (int q = 0; q < 4; ++q) {
                            const int off = (blk >> 3) * kSlabBoxBytes + (((blk & 7) ^ g) << 4) + (g + 8) * 128 + 4 * q;
                            wmax = off + 4 > wmax ? off + 4 : wmax;
                            const int so = (g + 8) * kblocks + blk;
                            smax = so + 1 > smax ? so + 1 : smax;
                            const int ho = g * p.hpitch + (32 * blk + 8 * q) * 2;
                            hmax = ho + 16 > hmax ? ho + 16 : hmax;
                            CHECK(ho % 16 == 0, M, I, g, k);
                        }
                CHECK(wmax <= p.wbytes, M, I, 0, k);
                CHECK(16 * kblocks == I / 2 && smax <= I / 2 && I / 2 <= p.sbytes, M, I, 0, k);
                // copies: h rows j < kSlabTileRows of 2I bytes at the pitch, after weights and scales
                CHECK(p.sbytes % 128 == 0 && p.hpitch % 16 == 0 && (2 * I) % 16 == 0 && (I / 2) % 16 == 0, M, I, 0, k);
                CHECK(hmax <= (kSlabTileRows - 1) * p.hpitch + 2 * I, M, I, 0, k);
                CHECK(p.wbytes + p.sbytes + kSlabTileRows * p.hpitch <= p.stage_bytes, M, I, 0, k);
                // two tile slots' 16-byte h loads (rows g and g + 1, words q) fall on disjoint banks
                CHECK((p.hpitch / 4) % 32 == 16, M, I, 0, k);
                // assignment rows, the tile list (at most M*k tiles), then 8-byte aligned barriers and the
                // two counters, then alignment slack
                CHECK(p.tl_off == p.stages * p.stage_bytes + M * k * kSlabRows * 4, M, I, 0, k);
                CHECK(p.bars_off == p.tl_off + M * k * kSlabTileInts * 4 && p.bars_off % 8 == 0, M, I, 0, k);
                CHECK(kSlabTileInts <= static_cast<int>(sizeof(ExpertTile) / sizeof(int)) &&
                          4 + kSlabTileRows <= kSlabTileInts, M, I, 0, k);
                CHECK(p.bars_off + 2 * kSlabMaxStages * 8 + 8 + 1024 <= p.total, M, I, 0, k);
            }
    // the decode-width layer (I = 768) keeps at least 11 tiles in flight at M = 8, top-8; the fused
    // path takes its M = 1 calls and the tiny layer's (I = 512, E = 16, top-4) calls up to M = 2
    CHECK(slab_plan(8, 768, 8).stages >= 11, 8, 768, 0, 8);
    CHECK(slab_enabled(1, 768, 128, 8, 8, false) && !slab_enabled(2, 768, 128, 8, 8, false), 1, 768, 128, 8);
    CHECK(slab_enabled(2, 512, 16, 4, 8, false) && !slab_enabled(3, 512, 16, 4, 8, false), 2, 512, 16, 4);
    CHECK(slab_enabled(8, 512, 8, 8, 8, false) && !slab_enabled(8, 512, 8, 8, 8, true), 8, 512, 8, 8);
    // h (|h| <= 49 from the clamps) with the fixed shift stays below 2^126
    CHECK(std::ldexp(49.0, kHShift) < std::ldexp(1.0, 126), 0, kHShift, 0, 0);
    if (fails) {
        std::printf("%d failures\n", fails);
        return 1;
    }
    std::printf("ok %lld cases\n", cases);
    return 0;
}
