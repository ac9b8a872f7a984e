// down_slab.cu -- the down projection fused with the weighted top-k combine, for the smallest
// decode calls (M <= 8 tokens and at most 8 expert tiles; slab_enabled in down_slab.h gives the
// rule and the measurements behind it).
//
// "Compact routed MXFP4 GEMM" (down) row of "Post-Portfolio Device Attribution" ("MTP1
// Post-Portfolio Eager-Cycle Profile"), with the top-k combine folded into the same launch.  With
// at most 8 tokens each touched expert holds at most 8 assignments (top-k picks distinct experts),
// so the down GEMM is a stream of the touched experts' W2 with an N of a few columns.  Beside that
// stream the unfused form spends a round trip of fp32 rows y[M*k][H] through HBM and one more
// launch on the combine.  Here one CTA owns a slab of 16 output rows (H / 16 CTAs) and walks every
// expert tile of the call: per tile it streams the slab's 16 rows of that expert's W2 with their
// E8M0 scales and the tile's h rows, computes the 16 x (assignments) block of W2_e h on the
// tensor cores, and keeps the fp32 rows in shared memory under their flat assignment ids.  After
// the last tile it forms out[t][slab] = bf16(sum_j w_tj y_tj) with j = 0 .. k-1 in order: a
// fixed-order reduction, no atomics, no y workspace, no combine launch.
//
// The arithmetic is that of the narrow kernel (grouped_gemm.cu) for one 1024-K stage of a width-8
// tile: the weights decoded to code value x 2^-126 (e2m1x8_raw_p4), h multiplied by 2^kHShift as
// it is loaded, per 32-K block two m16n8k16 bf16 MMAs from zero whose fp32 partial times the
// block's E8M0 factor (exact) joins the block's K slot (4 blocks per slot, 8 slots), the slots
// summed in order and the sum multiplied by 2^(126 - kHShift); the combine is the combine
// kernel's.  So the output has the bits of the unfused pair on the same tiles.
//
// Warps: 0..7 compute (tile i goes to warp i mod 8: a thread holds rows g and g + 8 of the slab
// and tile slots 2q, 2q + 1, g = lane / 4, q = lane % 4), 8 producer (per tile one elected lane
// issues the weight boxes -- 16 rows x 128 bytes, 128-byte swizzle -- the scale rows and the h
// rows as bulk copies into a ring slot), 9 watcher.  A ring slot serves different compute warps in
// turn, and an mbarrier parity wait is only unambiguous for a waiter that sees every phase, so the
// watcher waits on every slot's copies in tile order and publishes how many tiles have landed
// (release store); compute warps poll that count (acquire load).  The weights and scales of the
// first ring slots stream in while gate_up finishes (they do not depend on it); h copies wait for
// it.  Every wait is bounded: after a timeout the kernel records MOE_ERR_TIMEOUT, lets the copies
// it issued land and leaves out unwritten.
#include <cuda_bf16.h>

#include "common.cuh"
#include "down_slab.h"

namespace moe {

namespace slab {
constexpr int kProducer = kSlabComputeWarps;
constexpr int kWatcher = kSlabComputeWarps + 1;
constexpr int kSlots = 8;             // K slots of a 1024-K stage, summed in order
constexpr int kBlocksPerSlot = 4;     // 32-K blocks per slot

__device__ __forceinline__ void st_release(int *p, int v)
{
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Bounded poll (whole warp) until the landed count reaches `target`; gives up like mbar_wait.
__device__ __forceinline__ void poll_landed(const int *p, int target, bool &aborted, const StatusPtrs &st)
{
    if (aborted) return;
    if (__all_sync(0xffffffffu, ld_acquire(p) >= target)) return;
    const long long t0 = clock64();
    while (!__all_sync(0xffffffffu, ld_acquire(p) >= target)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            aborted = true;
            record_timeout(st);
            return;
        }
    }
}
}  // namespace slab

__global__ void __launch_bounds__(kSlabThreads, 1)
down_slab_kernel(const __grid_constant__ CUtensorMap wmap, const uint8_t *__restrict__ w2_s,
                 const __nv_bfloat16 *__restrict__ h, const ExpertTile *__restrict__ tiles,
                 const int *__restrict__ n_tiles_ptr, const float *__restrict__ topk_w, void *__restrict__ out,
                 int f32_out, int *status_ws, int32_t *status_out, int M, int H, int I, int k)
{
    using namespace slab;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const SlabPlan plan = slab_plan(M, I, k);
    const int S = plan.stages;
    float *ys = reinterpret_cast<float *>(smem + S * plan.stage_bytes);   // [M*k][kSlabRows]
    int *tl = reinterpret_cast<int *>(smem + plan.tl_off);                  // [tile][kSlabTileInts]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + plan.bars_off);
    uint64_t *empty = full + kSlabMaxStages;
    int *landed = reinterpret_cast<int *>(empty + kSlabMaxStages);
    int *abort_flag = landed + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const StatusPtrs status{status_ws, status_out};
    const int h0 = static_cast<int>(blockIdx.x) * kSlabRows;
    const int kblocks = I / 32;
    const int n_assign = M * k;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *landed = 0;
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_trigger();
    // The tile list comes from the permutation, which completed before gate_up (this kernel's
    // predecessor) let dependents launch, so it is read before the wait; h is gate_up's output.
    // All threads copy it into shared memory at once (one round of independent loads): read tile
    // by tile, every descriptor would cost the producer a dependent L2 round trip.
    const int n_tiles = min(__ldcg(n_tiles_ptr), n_assign);   // a tile holds at least one assignment
    {
        const int *src = reinterpret_cast<const int *>(tiles);
        constexpr int kTileStride = static_cast<int>(sizeof(ExpertTile) / sizeof(int));
        for (int idx = threadIdx.x; idx < n_tiles * kSlabTileInts; idx += kSlabThreads) {
            const int t = idx / kSlabTileInts, f = idx - t * kSlabTileInts;
            tl[idx] = __ldcg(src + t * kTileStride + f);
        }
    }
    __syncthreads();
    bool aborted = false;

    if (warp == kProducer) {
        // ---------------------------------------------------------------- copy producer
        if (lane == 0) prefetch_tensormap(&wmap);
        const int cols = plan.wbytes / kSlabBoxBytes;
        auto rows_of = [&](int i) { return min(tl[i * kSlabTileInts + 2], kSlabTileRows); };
        auto issue_weights = [&](int i, int s) {
            const int row = tl[i * kSlabTileInts] * H + h0;
            const int c = rows_of(i);
            uint8_t *st = smem + s * plan.stage_bytes;
            if (elect_one()) {
                mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(plan.wbytes + I / 2 + c * 2 * I));
                for (int col = 0; col < cols; ++col) tma_load_2d(st + col * kSlabBoxBytes, &wmap, 128 * col, row, &full[s]);
                bulk_load(st + plan.wbytes, w2_s + static_cast<size_t>(row) * (I / 32), static_cast<uint32_t>(I / 2),
                          &full[s]);
            }
            __syncwarp();
        };
        auto issue_h = [&](int i, int s) {
            const int p0 = tl[i * kSlabTileInts + 1];
            const int c = rows_of(i);
            uint8_t *sh = smem + s * plan.stage_bytes + plan.wbytes + plan.sbytes;
            if (elect_one()) {
                for (int j = 0; j < c; ++j)
                    bulk_load(sh + j * plan.hpitch, h + static_cast<size_t>(p0 + j) * I, static_cast<uint32_t>(2 * I),
                              &full[s]);
            }
            __syncwarp();
        };
        const int first = min(n_tiles, S);
        for (int i = 0; i < first; ++i) issue_weights(i, i);
        pdl_wait();
        for (int i = 0; i < first; ++i) issue_h(i, i);
        int issued = first;
        for (int i = first; i < n_tiles; ++i) {
            const int s = i % S;
            mbar_wait(&empty[s], ((i / S) & 1) ^ 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (aborted) break;
            issue_weights(i, s);
            issue_h(i, s);
            ++issued;
        }
        // every copy issued must land before the CTA can exit (the issued fills are a prefix; a
        // slot's previous fill had landed before its next one was issued)
        for (int j = 0; j < S && j < issued; ++j) {
            const int i = issued - 1 - j;
            mbar_wait_drain(&full[i % S], (i / S) & 1, status);
        }
    } else if (warp == kWatcher) {
        // ---------------------------------------------------------------- landing watcher
        pdl_wait();
        for (int i = 0; i < n_tiles; ++i) {
            mbar_wait(&full[i % S], (i / S) & 1, aborted, status);
            aborted = __any_sync(0xffffffffu, aborted);
            if (aborted) break;
            if (lane == 0) st_release(landed, i + 1);
        }
    } else {
        // ---------------------------------------------------------------- compute warps
        pdl_wait();
        const int g = lane >> 2, q = lane & 3;
        const uint32_t fac = static_cast<uint32_t>(kHShift + 127) * 0x00800080u;   // bf16x2 2^kHShift
        constexpr float kBack = static_cast<float>(1u << (126 - kHShift));
        const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = warp; i < n_tiles; i += kSlabComputeWarps) {
            poll_landed(landed, i + 1, aborted, status);
            if (aborted) break;
            const int s = i % S;
            const uint8_t *st = smem + s * plan.stage_bytes;
            const uint8_t *sc = st + plan.wbytes;
            const uint8_t *xa = st + plan.wbytes + plan.sbytes + g * plan.hpitch;   // tile slot g's h row
            const uint8_t *wtop = st + g * 128 + 4 * q;          // slab row g in every box column
            const uint8_t *wbot = st + (g + 8) * 128 + 4 * q;    // slab row g + 8
            float tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int ks = 0; ks < kSlots; ++ks) {
                float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int bi = 0; bi < kBlocksPerSlot; ++bi) {
                    const int blk = ks * kBlocksPerSlot + bi;
                    if (blk >= kblocks) continue;
                    // K 8q..8q+7 of h (P4 order, like the decoded weights) times 2^kHShift (exact)
                    uint4 xb = *reinterpret_cast<const uint4 *>(xa + (32 * blk + 8 * q) * 2);
                    xb = make_uint4(bf16x2_mul(xb.x, fac), bf16x2_mul(xb.y, fac), bf16x2_mul(xb.z, fac),
                                    bf16x2_mul(xb.w, fac));
                    // word q of the rows' 16-byte block: box column blk / 8, chunk (blk % 8) ^ (row % 8)
                    const int off = (blk >> 3) * kSlabBoxBytes + (((blk & 7) ^ g) << 4);
                    const uint32_t wt = *reinterpret_cast<const uint32_t *>(wtop + off);
                    const uint32_t wb = *reinterpret_cast<const uint32_t *>(wbot + off);
                    const float st_scale = e8m0_scale(sc[g * kblocks + blk]);
                    const float sb_scale = e8m0_scale(sc[(g + 8) * kblocks + blk]);
                    uint32_t t[4], u[4];
                    e2m1x8_raw_p4(wt, t);
                    e2m1x8_raw_p4(wb, u);
                    const uint32_t a0[4] = {t[0], u[0], t[1], u[1]};
                    const uint32_t a1[4] = {t[2], u[2], t[3], u[3]};
                    float tmp[4];
                    mma_bf16_16816(tmp, a0, xb.x, xb.y, zero4);
                    mma_bf16_16816(tmp, a1, xb.z, xb.w, tmp);
                    part[0] = fmaf(tmp[0], st_scale, part[0]);
                    part[1] = fmaf(tmp[1], st_scale, part[1]);
                    part[2] = fmaf(tmp[2], sb_scale, part[2]);
                    part[3] = fmaf(tmp[3], sb_scale, part[3]);
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) tot[r] += part[r];
            }
            // the slot's shared memory has been read by every lane: release it
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // the unweighted down rows of tile slots 2q, 2q + 1 (rows g and g + 8 of the slab)
            // (flat ids outside the call, possible only with a caller's malformed routing, are dropped)
            const int c = min(tl[i * kSlabTileInts + 2], kSlabTileRows);
            const int l0 = 2 * q, l1 = l0 + 1;
            if (l0 < c) {
                const int f = tile_flat_id(tl[i * kSlabTileInts + 4 + l0]);
                if (f < n_assign) {
                    ys[f * kSlabRows + g] = tot[0] * kBack;
                    ys[f * kSlabRows + g + 8] = tot[2] * kBack;
                }
            }
            if (l1 < c) {
                const int f = tile_flat_id(tl[i * kSlabTileInts + 4 + l1]);
                if (f < n_assign) {
                    ys[f * kSlabRows + g] = tot[1] * kBack;
                    ys[f * kSlabRows + g + 8] = tot[3] * kBack;
                }
            }
        }
    }
    if (aborted) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag != 0) return;
    // ------------------------------------------------------------------ the weighted combine
    // out[t][h0 + r] = sum_j w[t*k + j] * y[t*k + j][r], j ascending (fmaf, like combine_kernel)
    for (int idx = threadIdx.x; idx < M * kSlabRows; idx += kSlabThreads) {
        const int t = idx / kSlabRows, r = idx % kSlabRows;
        float a = 0.f;
        for (int j = 0; j < k; ++j) {
            const int f = t * k + j;
            a = fmaf(__ldcg(&topk_w[f]), ys[f * kSlabRows + r], a);
        }
        const size_t o = static_cast<size_t>(t) * H + h0 + r;
        if (f32_out)
            static_cast<float *>(out)[o] = a;
        else
            static_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(a);
    }
}

cudaError_t launch_down_slab(const CUtensorMap &wmap, const uint8_t *w2_s, const __nv_bfloat16 *h_p4,
                             const ExpertTile *tiles, const int *n_tiles, const float *topk_w, void *out,
                             bool f32_out, int *status, int32_t *status_out, int M, int H, int I, int k,
                             cudaStream_t s, bool pdl)
{
    const SlabPlan plan = slab_plan(M, I, k);
    cudaError_t e = ensure_max_smem(reinterpret_cast<const void *>(down_slab_kernel), plan.total);
    if (e != cudaSuccess) return e;
    return launch_ex(down_slab_kernel, dim3(H / kSlabRows), dim3(kSlabThreads), plan.total, s, pdl, wmap, w2_s, h_p4,
                     tiles, n_tiles, topk_w, out, f32_out ? 1 : 0, status, status_out, M, H, I, k);
}

}  // namespace moe
