// Host-side check of the launch-planning helpers in moe_internal.h over a grid of shapes: the
// router plan covers every token and every K element and fills at most one wave of CTAs, the tile
// width and fused-select switches follow their stated rules, the per-shape shared-memory needs fit
// a B200 CTA, and the mma.sync kernels' activation shift keeps every finite bf16 row in range.
// Built and run by tests/test_host_plan.py (no GPU needed).
#include <cmath>
#include <cstdio>

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
    // h (|h| <= 49 from the clamps) with the fixed shift stays below 2^126
    CHECK(std::ldexp(49.0, kHShift) < std::ldexp(1.0, 126), 0, kHShift, 0, 0);
    if (fails) {
        std::printf("%d failures\n", fails);
        return 1;
    }
    std::printf("ok %lld cases\n", cases);
    return 0;
}
