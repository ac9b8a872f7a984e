// permute_impl.cuh -- route remap device code shared by the stand-alone
// permutation kernel and the fused router-select + permutation kernel.
//
// "Direct M=2 route remap" row of "Post-Portfolio Device Attribution" ("MTP1
// Post-Portfolio Eager-Cycle Profile").  The expert-grouped order is the stable
// counting sort of the assignments f = t*k + j by expert: position(f) =
// offset[e_f] + rank(f), rank(f) = the number of earlier assignments on the same
// expert.  Two ways to rank:
//  * the fused router select (M <= 64) keeps one 64-bit token mask per expert (see
//    warp_scan_experts / scatter_assignment below);
//  * rank_and_scatter (the stand-alone permutation, any M) takes one thread per
//    assignment, in rounds of blockDim assignments:
//    - a warp's lanes that share an expert find each other with __match_any_sync
//      (rank inside the warp = matching lanes below it);
//    - the lowest of them records the warp's count of that expert in a
//      [warp][expert] table, one pass per expert turns the table into prefix counts
//      (plus the counts of earlier rounds) and the thread reads its rank back;
//    - counts per expert come first (shared-memory atomics: order-free), then one
//      block scan of (tiles << 16 | count) gives every expert offset and tile base
//      at once; two block barriers per round, no sort.
// Every result is unique, so the bytes do not depend on scheduling.
#pragma once

#include "common.cuh"

namespace moe {

// Exclusive scan of one value per thread over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        if (lane < nwarps) warp_tot[lane] = wi - w;      // exclusive prefix of the warp totals
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    total = warp_tot[32];
    return warp_tot[warp] + incl - v;
}

// Shared memory of the ranking, carved from one dynamic buffer of permute_smem_bytes(E) bytes:
// wc at 0, pref at 64 E, the six int arrays at 128 E, the scan buffer at 152 E (+132 bytes).
struct RankSmem {
    uint16_t *wc;     // [32][E] counts of the current round's warps
    uint16_t *pref;   // [32][E] their prefix counts (with earlier rounds)
    int *cnt, *off, *tb, *base, *wb, *wbl;   // [E] count, offset, first tile, ranked so far, small / large wide tile
    int *scan;        // 33
};

__device__ __forceinline__ RankSmem rank_smem(uint8_t *raw, int E)
{
    constexpr int kW = kPermuteThreads / 32;
    RankSmem r;
    r.wc = reinterpret_cast<uint16_t *>(raw);
    r.pref = r.wc + kW * E;
    int *ints = reinterpret_cast<int *>(raw + 2 * kW * E * 2);
    r.cnt = ints;
    r.off = ints + E;
    r.tb = ints + 2 * E;
    r.base = ints + 3 * E;
    r.wb = ints + 4 * E;
    r.wbl = ints + 5 * E;
    r.scan = ints + 6 * E;
    return r;
}

// Stable expert-grouped order of n assignments whose experts are s_e[0..n) (shared memory).
// Writes expert_offsets [E+1], sorted_ids [n], inv_pos [n] and, when tiles != nullptr, the
// expert tiles and their count.  Assignments with an expert outside [0, E) are out of
// contract: they are left out (inv_pos = -1, offsets[E] counts only the others) and never
// index past an array.  Called by every thread of a kPermuteThreads-thread CTA.
__device__ inline void rank_and_scatter(const int *s_e, int n, int E, int k, RankSmem sm,
                                        int32_t *__restrict__ offsets, int32_t *__restrict__ sorted_ids,
                                        int32_t *__restrict__ inv_pos, TileOut to)
{
    ExpertTile *__restrict__ tiles = to.tiles;
    constexpr int kW = kPermuteThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // only the warps that hold assignments in some round use table rows
    const int rows = min(kW, (n + 31) / 32);
    for (int i = tid; i < rows * E; i += kPermuteThreads) sm.wc[i] = 0;
    for (int e = tid; e < E; e += kPermuteThreads) {
        sm.cnt[e] = 0;
        sm.base[e] = 0;
    }
    __syncthreads();
    for (int f = tid; f < n; f += kPermuteThreads) {
        const int e = s_e[f];
        if (e >= 0 && e < E) atomicAdd(&sm.cnt[e], 1);
    }
    __syncthreads();
    // offsets and tile bases: (tiles << 16) | count per expert, one scan (counts <= 16384); an
    // expert with at least kWideMinTokens assignments takes tensor-core tiles instead, when enabled
    const int my_cnt = tid < E ? sm.cnt[tid] : 0;
    const bool wide_on = to.wide_tiles != nullptr;
    const bool my_small = wide_on && wide_small_expert(my_cnt);
    const bool my_large = wide_on && wide_large_expert(my_cnt);
    const int W = to.width, wsh = W == 16 ? 4 : 3;   // 8 or 16 assignments per tile
    const int mine = tid < E ? (((my_small || my_large) ? 0 : (my_cnt + W - 1) >> wsh) << 16) | my_cnt : 0;
    int total = 0;
    const int base = block_exclusive_scan(mine, sm.scan, total);   // ends with a block barrier
    if (tid < E) {
        sm.off[tid] = base & 0xFFFF;
        sm.tb[tid] = base >> 16;
        offsets[tid] = base & 0xFFFF;
    }
    if (tid == 0) {
        offsets[E] = total & 0xFFFF;
        if (tiles) *to.n_tiles = total >> 16;
    }
    if (wide_on) {
        __syncthreads();   // every thread has read the first scan's totals before the buffer is reused
        int wtotal = 0;
        const int wbase = block_exclusive_scan(my_small ? 1 : 0, sm.scan, wtotal);
        if (tid < E) sm.wb[tid] = wbase;
        if (tid == 0) *to.n_wide = wtotal;
        __syncthreads();
        int ltotal = 0;
        const int lbase = block_exclusive_scan(my_large ? wide_large_tiles(my_cnt) : 0, sm.scan, ltotal);
        if (tid < E) sm.wbl[tid] = lbase;
        if (tid == 0) *to.n_wide_large = ltotal;
    }
    for (int r0 = 0; r0 < n; r0 += kPermuteThreads) {
        const int f = r0 + tid;
        int e = f < n ? s_e[f] : -1;
        if (e >= E) e = -1;
        if (f < n && e < 0) inv_pos[f] = -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank_w = __popc(same & ((1u << lane) - 1u));
        if (e >= 0 && rank_w == 0) sm.wc[warp * E + e] = static_cast<uint16_t>(__popc(same));
        __syncthreads();
        if (tid < E) {
            const int active = min(kW, (n - r0 + 31) / 32);   // warps holding assignments this round
            int c[kW];
#pragma unroll
            for (int w = 0; w < kW; ++w) c[w] = w < active ? sm.wc[w * E + tid] : 0;   // all loads first
            int run = sm.base[tid];
#pragma unroll
            for (int w = 0; w < kW; ++w) {
                if (w < active) {
                    sm.wc[w * E + tid] = 0;
                    sm.pref[w * E + tid] = static_cast<uint16_t>(run);
                }
                run += c[w];
            }
            sm.base[tid] = run;
        }
        __syncthreads();
        if (e >= 0) {
            const int rank = sm.pref[warp * E + e] + rank_w;
            const int pos = sm.off[e] + rank;
            sorted_ids[pos] = f;
            inv_pos[f] = pos;
            const int cnt = sm.cnt[e];
            if (wide_on && wide_small_expert(cnt)) {
                if (rank == 0) {
                    WideTile *wp = to.wide_tiles + sm.wb[e];
                    wp->expert = e;
                    wp->p0 = pos;
                    wp->count = cnt;
                    wp->pad = 0;
                }
            } else if (wide_on && wide_large_expert(cnt)) {
                if (rank % kWideTokens == 0) {
                    WideTile *wp = to.wide_large + sm.wbl[e] + rank / kWideTokens;
                    wp->expert = e;
                    wp->p0 = pos;
                    wp->count = min(kWideTokens, cnt - rank);
                    wp->pad = 0;
                }
            } else if (tiles) {
                const int slot = rank & (W - 1), tile_first = rank - slot;
                ExpertTile *tp = tiles + sm.tb[e] + (rank >> wsh);
                tp->flat[slot] = pack_flat(f, to);
                if (slot == 0) {
                    tp->expert = e;
                    tp->p0 = sm.off[e] + tile_first;
                    tp->count = min(W, cnt - tile_first);
                    tp->pad = 0;
                }
                if (rank == cnt - 1)   // the last assignment repeats into the unused slots
                    for (int j = slot + 1; j < W; ++j) tp->flat[j] = pack_flat(f, to);
            }
        }
    }
}

// Route remap of the fused router select (M <= 64 tokens), in two helpers.  Every token picks
// each expert at most once, so the stable rank of assignment f = t*k + j on its expert e is the
// number of earlier tokens that chose e: with mask[e] = the set of tokens that chose e (one bit
// per token), rank = popc(mask[e] & (2^t - 1)) and count = popc(mask[e]).

// One warp (the calling warp): per expert, (mma.sync tiles << 16) | count and the small and large
// tensor-core tiles (when the wide path is on), one warp scan over the experts (lane l takes the
// contiguous experts [l * per, (l + 1) * per)); writes off, tb, wb, wbl (shared) and
// expert_offsets, the tile counts (global).
__device__ inline void warp_scan_experts(const unsigned long long *mask, int E, TileOut to, int *off, int *tb, int *wb,
                                         int *wbl, int32_t *__restrict__ offsets)
{
    const bool wide_on = to.wide_tiles != nullptr;
    const int lane = threadIdx.x & 31;
    const int W = to.width, wsh = W == 16 ? 4 : 3;   // 8 or 16 assignments per tile
    auto narrow = [&](int c) { return !wide_on || c < kWideMinTokens; };
    auto packed = [&](int c) { return ((narrow(c) ? (c + W - 1) >> wsh : 0) << 16) | c; };
    auto small_n = [&](int c) { return (wide_on && wide_small_expert(c)) ? 1 : 0; };
    auto large_n = [&](int c) { return (wide_on && wide_large_expert(c)) ? wide_large_tiles(c) : 0; };
    const int per = (E + 31) / 32;
    const int ea = min(E, lane * per), eb = min(E, ea + per);
    int local = 0, wlocal = 0, llocal = 0;
    for (int e = ea; e < eb; ++e) {
        const int c = __popcll(mask[e]);
        local += packed(c);
        wlocal += small_n(c);
        llocal += large_n(c);
    }
    int incl = local, wincl = wlocal, lincl = llocal;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        const int wo = __shfl_up_sync(0xffffffffu, wincl, d);
        const int lo = __shfl_up_sync(0xffffffffu, lincl, d);
        if (lane >= d) {
            incl += o;
            wincl += wo;
            lincl += lo;
        }
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int wtotal = __shfl_sync(0xffffffffu, wincl, 31);
    const int ltotal = __shfl_sync(0xffffffffu, lincl, 31);
    int run = incl - local, wrun = wincl - wlocal, lrun = lincl - llocal;
    for (int e = ea; e < eb; ++e) {
        const int c = __popcll(mask[e]);
        off[e] = run & 0xFFFF;
        tb[e] = run >> 16;
        wb[e] = wrun;
        wbl[e] = lrun;
        offsets[e] = run & 0xFFFF;
        run += packed(c);
        wrun += small_n(c);
        lrun += large_n(c);
    }
    if (lane == 0) {
        offsets[E] = total & 0xFFFF;
        *to.n_tiles = total >> 16;
        if (wide_on) {
            *to.n_wide = wtotal;
            *to.n_wide_large = ltotal;
        }
    }
}

// Assignment f (token t, expert e, rank r among the expert's c assignments): its position, the
// inverse map and its slot of an mma.sync tile or a tensor-core tile (off, tb, wb, wbl from
// warp_scan_experts).
__device__ inline void scatter_assignment(int f, int e, int r, int c, const int *off, const int *tb, const int *wb,
                                          const int *wbl, int32_t *__restrict__ sorted_ids,
                                          int32_t *__restrict__ inv_pos, TileOut to)
{
    const int pos = off[e] + r;
    sorted_ids[pos] = f;
    inv_pos[f] = pos;
    if (to.wide_tiles != nullptr && wide_small_expert(c)) {
        if (r == 0) {
            WideTile *wp = to.wide_tiles + wb[e];
            wp->expert = e;
            wp->p0 = pos;
            wp->count = c;
            wp->pad = 0;
        }
        return;
    }
    if (to.wide_tiles != nullptr && wide_large_expert(c)) {
        if (r % kWideTokens == 0) {
            WideTile *wp = to.wide_large + wbl[e] + r / kWideTokens;
            wp->expert = e;
            wp->p0 = pos;
            wp->count = min(kWideTokens, c - r);
            wp->pad = 0;
        }
        return;
    }
    const int W = to.width, wsh = W == 16 ? 4 : 3;
    const int slot = r & (W - 1), tile_first = r - slot;
    ExpertTile *tp = to.tiles + tb[e] + (r >> wsh);
    tp->flat[slot] = pack_flat(f, to);
    if (slot == 0) {
        tp->expert = e;
        tp->p0 = off[e] + tile_first;
        tp->count = min(W, c - tile_first);
        tp->pad = 0;
    }
    if (r == c - 1)   // the last assignment repeats into the unused slots
        for (int j = slot + 1; j < W; ++j) tp->flat[j] = pack_flat(f, to);
}

// Tiles from expert offsets (the step-level entry points, whose caller gives the permutation):
// mma.sync tiles of to.width assignments and, when to.wide_tiles is set, small and large
// tensor-core tiles (the same split as the route remap kernels make).  sorted_flat(p) returns the
// flat assignment id at position p of the expert-grouped order.  Each thread owns a contiguous run
// of ceil(E / blockDim) experts.
template <typename SortedFlat>
__device__ inline void emit_tiles(const int *off, int E, TileOut to, int *scan_buf, SortedFlat sorted_flat)
{
    const int W = to.width;
    const bool wide_on = to.wide_tiles != nullptr;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
    int mine = 0, smine = 0, lmine = 0;
    for (int e = e0; e < e1; ++e) {
        const int cnt = off[e + 1] - off[e];
        if (wide_on && wide_small_expert(cnt))
            ++smine;
        else if (wide_on && wide_large_expert(cnt))
            lmine += wide_large_tiles(cnt);
        else
            mine += (cnt + W - 1) / W;
    }
    int total = 0, stotal = 0, ltotal = 0;
    int base = block_exclusive_scan(mine, scan_buf, total);
    __syncthreads();   // every thread has read a scan's totals before the buffer is reused
    int sbase = block_exclusive_scan(smine, scan_buf, stotal);
    __syncthreads();
    int lbase = block_exclusive_scan(lmine, scan_buf, ltotal);
    for (int e = e0; e < e1; ++e) {
        const int cnt = off[e + 1] - off[e];
        if (wide_on && (wide_small_expert(cnt) || wide_large_expert(cnt))) {
            const bool small = wide_small_expert(cnt);
            const int step = small ? cnt : kWideTokens;
            for (int i = 0; i * step < cnt; ++i) {
                WideTile wt;
                wt.expert = e;
                wt.p0 = off[e] + i * step;
                wt.count = min(step, cnt - i * step);
                wt.pad = 0;
                if (small)
                    to.wide_tiles[sbase++] = wt;
                else
                    to.wide_large[lbase++] = wt;
            }
            continue;
        }
        for (int i = 0; i * W < cnt; ++i) {
            ExpertTile tl{};
            tl.expert = e;
            tl.p0 = off[e] + i * W;
            tl.count = min(W, cnt - i * W);
            tl.pad = 0;
            for (int j = 0; j < W; ++j) tl.flat[j] = pack_flat(sorted_flat(tl.p0 + min(j, tl.count - 1)), to);
            to.tiles[base++] = tl;
        }
    }
    if (threadIdx.x == 0) {
        *to.n_tiles = total;
        if (wide_on) {
            *to.n_wide = stotal;
            *to.n_wide_large = ltotal;
        }
    }
}

}  // namespace moe
