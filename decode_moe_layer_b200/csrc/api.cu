// api.cu -- the C ABI of libmoe.so (declared in include/moe.h): argument
// validation, workspace layout and ownership, TMA descriptor encoding, and the
// enqueue order of the layer's kernels on the caller's stream.
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "down_slab.h"
#include "moe.h"
#include "moe_internal.h"

namespace moe {

int grouped_smem_bytes(int K, int width);

static thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e)
{
    g_last_cuda_error = static_cast<int>(e);
    return MOE_ERR_CUDA;
}

int num_sms()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

cudaError_t ensure_max_smem(const void *kernel, int bytes)
{
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    int &have = done[std::make_pair(kernel, dev)];
    if (have >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) have = bytes;
    return e;
}

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

Layout make_layout(int M, int H, int I, int E, int k)
{
    Layout L;
    const size_t n = static_cast<size_t>(M) * k;
    // 16-wide tiles when the experts average 6 or more assignments (tile_width) and their larger stages fit
    L.width = tile_width(M, E, k);
    if (L.width == 16 && (grouped_smem_bytes(H, 16) > 227 * 1024 || grouped_smem_bytes(I, 16) > 227 * 1024))
        L.width = 8;
    L.max_tiles = static_cast<int>((n < static_cast<size_t>(E) ? n : static_cast<size_t>(E)) +
                                   (n + L.width - 1) / L.width);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += round_up(bytes > 0 ? bytes : 1, 256);
        return o;
    };
    L.status = take(256);
    L.splits = route_plan(M, H, E).splits;
    L.partial = take(static_cast<size_t>(L.splits) * M * E * sizeof(float));
    L.x_p4 = take(static_cast<size_t>(M) * H * 2);
    L.xmax = take(static_cast<size_t>(L.splits) * M * 4);
    L.xshift = take(static_cast<size_t>(M) * 4);
    L.topk_ids = take(n * 4);
    L.topk_w = take(n * 4);
    L.offsets = take(static_cast<size_t>(E + 1) * 4);
    L.sorted_ids = take(n * 4);
    L.inv_pos = take(n * 4);
    L.tiles = take(static_cast<size_t>(L.max_tiles) * sizeof(ExpertTile));
    L.n_tiles = take(4);
    L.h = take(n * I * 2);
    L.y = take(n * H * sizeof(float));
    L.wide = wide_enabled(M, H, I, E, k);
    // small tensor-core tiles: one per expert with kWideMinTokens .. kWideSmallMax assignments;
    // large: the experts with more, in tiles of up to kWideTokens
    const size_t ne = static_cast<size_t>(E);
    const size_t n_small = n / kWideMinTokens, n_big = n / (kWideSmallMax + 1);
    L.max_small = L.wide ? static_cast<int>(n_small < ne ? n_small : ne) : 0;
    L.max_large = L.wide ? static_cast<int>((n_big < ne ? n_big : ne) + n / kWideTokens + 1) : 0;
    L.wide_small = take(static_cast<size_t>(L.max_small) * sizeof(WideTile));
    L.n_wide_small = take(4);
    L.wide_large = take(static_cast<size_t>(L.max_large) * sizeof(WideTile));
    L.n_wide_large = take(4);
    L.x_perm = take(L.wide ? n * H * 2 : 0);
    L.total = off;
    return L;
}

// ------------------------------------------------------------------ validation

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_dims(int M, int H, int I, int E, int k, bool need_hi)
{
    if (M < 0 || E <= 0 || k <= 0 || H <= 0 || (need_hi && I <= 0)) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK || k > E) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (H % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (need_hi && (I % 32 != 0)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(M) * k > kMaxAssignments) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (need_hi) {
        if (static_cast<long long>(E) * 2 * I >= (1LL << 31) || static_cast<long long>(E) * H >= (1LL << 31))
            return MOE_ERR_UNSUPPORTED_SHAPE;
        if (grouped_smem_bytes(H, 8) > 227 * 1024 || grouped_smem_bytes(I, 8) > 227 * 1024)
            return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    return MOE_OK;
}

static bool overlaps(const void *a, size_t an, const void *b, size_t bn)
{
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + bn && pb < pa + an;
}

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Packed E2M1 matrix viewed as [rows][row_bytes] uint8; boxes of box_rows rows x 128 bytes, 128-byte swizzle.
static int make_weight_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return MOE_OK;
}

// E8M0 scale matrix viewed as [rows][row_bytes] uint8; boxes of box_rows rows x (kChunkK / 32) bytes,
// unswizzled.  Only used when row_bytes is a multiple of 16 (per_stage_scales).
static int make_scale_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, int box_rows,
                          int box_bytes = kChunkK / 32)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return MOE_OK;
}

// bf16 activation rows [rows][K] (expert-grouped x or h, P4 K order) for the wide kernel: boxes
// of 16 rows x 64 elements (128 bytes), 128-byte swizzle, the K-major operand layout of tcgen05.mma.
static int make_act_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t K)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return MOE_OK;
}

// ------------------------------------------------------------------ library-owned workspaces

static std::mutex g_pool_mu;
static std::map<std::pair<int, uintptr_t>, std::pair<void *, size_t>> g_pool;

// Workspace of (current device, stream), grown outside stream capture only.  A
// buffer replaced by a larger one stays allocated: work already queued may use it.
static int library_workspace(cudaStream_t s, size_t need, char **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    std::lock_guard<std::mutex> lock(g_pool_mu);
    auto &ent = g_pool[std::make_pair(dev, reinterpret_cast<uintptr_t>(s))];
    if (ent.second >= need) {
        *out = static_cast<char *>(ent.first);
        return MOE_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return cuda_fail(e);
    if (cs != cudaStreamCaptureStatusNone) return MOE_ERR_WORKSPACE;
    const size_t bytes = need > 2 * ent.second ? need : 2 * ent.second;
    void *p = nullptr;
    e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    ent = std::make_pair(p, bytes);
    *out = static_cast<char *>(p);
    return MOE_OK;
}

#define MOE_TRY(expr)                                   \
    do {                                                \
        cudaError_t _e = (expr);                        \
        if (_e != cudaSuccess) return cuda_fail(_e);    \
    } while (0)

// ------------------------------------------------------------------ step bodies (arguments already validated)

static int run_gate_up(const void *w13_q, const uint8_t *w13_s, const __nv_bfloat16 *x, const ExpertTile *tiles,
                       const int *n_tiles, __nv_bfloat16 *h, bool h_p4, int *status, int32_t *status_out, int H,
                       int I, int E, int k, int width, int max_tiles, cudaStream_t s, bool pdl)
{
    CUtensorMap map, smap;
    // gate rows and up rows of an item are two boxes of kItemRows / 2 rows
    int rc = make_weight_map(&map, w13_q, static_cast<uint64_t>(E) * 2 * I, static_cast<uint64_t>(H) / 2,
                             kItemRows / 2);
    if (rc != MOE_OK) return rc;
    memset(&smap, 0, sizeof(smap));
    if (per_stage_scales(H)) {
        rc = make_scale_map(&smap, w13_s, static_cast<uint64_t>(E) * 2 * I, static_cast<uint64_t>(H) / 32,
                            kItemRows / 2);
        if (rc != MOE_OK) return rc;
    }
    MOE_TRY(launch_gate_up(map, smap, w13_s, x, tiles, n_tiles, h, h_p4, status, status_out, H, I, k, width, max_tiles,
                           s, pdl));
    return MOE_OK;
}

// Optional per-launch event marks (profiling entry point only): an event before the first launch
// and one after every launch, each launch's slot (moe.h, moe_mxfp4_forward_profile) remembering
// the event that closes it.
struct Marks {
    cudaEvent_t ev[MOE_PROFILE_KERNELS + 1];
    int slot[MOE_PROFILE_KERNELS] = {};   // index of the event after the slot's launch; 0: not launched
    int n = 0;
    cudaError_t start(cudaStream_t s) { return cudaEventRecord(ev[n++], s); }
    cudaError_t after(cudaStream_t s, int k)
    {
        slot[k] = n;
        return cudaEventRecord(ev[n++], s);
    }
};

enum ProfileSlot {
    kProfLogits = 0, kProfSelect, kProfPermute, kProfGateUp, kProfGather, kProfGateUpTcSmall, kProfGateUpTcLarge,
    kProfDown, kProfDownTcSmall, kProfDownTcLarge, kProfCombine
};
static_assert(kProfCombine + 1 == MOE_PROFILE_KERNELS, "one slot per launch kind");

#define MOE_AFTER(m, s, k)                              \
    do {                                                \
        if (m) MOE_TRY((m)->after((s), (k)));           \
    } while (0)

static int run_down(const void *w2_q, const uint8_t *w2_s, const __nv_bfloat16 *h_p4, const int32_t *sorted_ids,
                    const ExpertTile *tiles, const int *n_tiles, float *y, int *status,
                    int32_t *status_out, int H, int I, int E, int width, int max_tiles, cudaStream_t s, bool pdl)
{
    CUtensorMap map, smap;
    int rc = make_weight_map(&map, w2_q, static_cast<uint64_t>(E) * H, static_cast<uint64_t>(I) / 2, kItemRows);
    if (rc != MOE_OK) return rc;
    memset(&smap, 0, sizeof(smap));
    if (per_stage_scales(I)) {
        rc = make_scale_map(&smap, w2_s, static_cast<uint64_t>(E) * H, static_cast<uint64_t>(I) / 32, kItemRows);
        if (rc != MOE_OK) return rc;
    }
    MOE_TRY(launch_down(map, smap, w2_s, h_p4, sorted_ids, tiles, n_tiles, y, status, status_out, H, I, width,
                        max_tiles, s, pdl));
    return MOE_OK;
}

// The smallest calls (slab_enabled): the down projection and the weighted top-k combine in one
// launch; weight boxes of 16 rows x 128 bytes (one slab).
static int run_down_slab(const void *w2_q, const uint8_t *w2_s, const __nv_bfloat16 *h_p4, const ExpertTile *tiles,
                         const int *n_tiles, const float *topk_w, void *out, bool f32_out, int *status,
                         int32_t *status_out, int M, int H, int I, int E, int k, cudaStream_t s, bool pdl)
{
    CUtensorMap map;
    int rc = make_weight_map(&map, w2_q, static_cast<uint64_t>(E) * H, static_cast<uint64_t>(I) / 2, kSlabRows);
    if (rc != MOE_OK) return rc;
    MOE_TRY(launch_down_slab(map, w2_s, h_p4, tiles, n_tiles, topk_w, out, f32_out, status, status_out, M, H, I, k, s,
                             pdl));
    return MOE_OK;
}

// The tensor-core path for the wide tiles of one projection (gate_up: x rows gathered into
// expert-grouped P4 order -> h; down: h (P4) -> y).  Weight boxes of 64 rows x 128 bytes, scale
// boxes of 64 rows x 16 bytes (one 512-element stage), activation boxes of 16 rows x 64 elements.
static int run_wide(bool gate_up, const void *wq, const uint8_t *ws_, const __nv_bfloat16 *act,
                    const WideLists &wl, const int32_t *sorted_ids, __nv_bfloat16 *h, bool h_p4, float *y,
                    int *status, int32_t *status_out, int M, int H, int I, int E, int k, cudaStream_t s, bool pdl,
                    Marks *marks = nullptr)
{
    CUtensorMap wmap, smap, bmap;
    const uint64_t rows = gate_up ? static_cast<uint64_t>(E) * 2 * I : static_cast<uint64_t>(E) * H;
    const uint64_t K = gate_up ? H : I;
    int rc = make_weight_map(&wmap, wq, rows, K / 2, 64);
    if (rc == MOE_OK) rc = make_scale_map(&smap, ws_, rows, K / 32, 64, kWideStageK / 32);
    if (rc == MOE_OK) rc = make_act_map(&bmap, act, static_cast<uint64_t>(M) * k, K);
    if (rc != MOE_OK) return rc;
    // small tiles, then large ones (two launches: each kernel splits tensor memory for its tile size)
    MOE_TRY(launch_wide(gate_up, true, wmap, smap, bmap, wl.small, wl.n_small, wl.max_small, sorted_ids, h, h_p4, y,
                        status, status_out, H, I, s, pdl));
    MOE_AFTER(marks, s, gate_up ? kProfGateUpTcSmall : kProfDownTcSmall);
    MOE_TRY(launch_wide(gate_up, false, wmap, smap, bmap, wl.large, wl.n_large, wl.max_large, sorted_ids, h, h_p4, y,
                        status, status_out, H, I, s, pdl));
    MOE_AFTER(marks, s, gate_up ? kProfGateUpTcLarge : kProfDownTcLarge);
    return MOE_OK;
}

static WideLists wide_lists(char *ws, const Layout &L)
{
    WideLists wl;
    wl.small = reinterpret_cast<WideTile *>(ws + L.wide_small);
    wl.n_small = reinterpret_cast<int *>(ws + L.n_wide_small);
    wl.large = reinterpret_cast<WideTile *>(ws + L.wide_large);
    wl.n_large = reinterpret_cast<int *>(ws + L.n_wide_large);
    wl.max_small = L.max_small;
    wl.max_large = L.max_large;
    return wl;
}

static int forward_impl(const void *x, const float *router_w, const float *router_bias, const uint8_t *w13_q,
                        const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s, void *out, int M, int H,
                        int I, int E, int k, int32_t *topk_ids_out, float *topk_w_out, int32_t *status_out,
                        char *ws, const Layout &L, cudaStream_t s, Marks *marks = nullptr, bool f32_out = false)
{
    int *status = reinterpret_cast<int *>(ws + L.status);
    float *partial = reinterpret_cast<float *>(ws + L.partial);
    __nv_bfloat16 *x_p4 = reinterpret_cast<__nv_bfloat16 *>(ws + L.x_p4);   // x in P4 K order (router)
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(ws + L.topk_ids);
    float *tw = topk_w_out ? topk_w_out : reinterpret_cast<float *>(ws + L.topk_w);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    int32_t *sorted_ids = reinterpret_cast<int32_t *>(ws + L.sorted_ids);
    int32_t *inv_pos = reinterpret_cast<int32_t *>(ws + L.inv_pos);
    ExpertTile *tiles = reinterpret_cast<ExpertTile *>(ws + L.tiles);
    int *n_tiles = reinterpret_cast<int *>(ws + L.n_tiles);
    __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);   // P4 K order
    float *y = reinterpret_cast<float *>(ws + L.y);
    const WideLists wl = wide_lists(ws, L);
    __nv_bfloat16 *x_perm = reinterpret_cast<__nv_bfloat16 *>(ws + L.x_perm);
    uint32_t *xmax = reinterpret_cast<uint32_t *>(ws + L.xmax);
    int *xshift = reinterpret_cast<int *>(ws + L.xshift);
    // the unfused path's remap reads the shifts route_topk writes; the fused one makes its own
    const TileOut to{tiles, n_tiles, L.wide ? wl.small : nullptr, wl.n_small, wl.large, wl.n_large, L.width,
                     xshift, k};
    // The first kernel is ordered after everything before it on the stream; each later
    // kernel of the call is launched early (programmatic dependent launch) and waits on
    // device for its predecessor.  Event marks (profiling) break that overlap, so the
    // profiling entry point launches without it.
    const bool pdl = (marks == nullptr);

    if (marks) MOE_TRY(marks->start(s));
    MOE_TRY(launch_route_logits(x, router_w, partial, x_p4, xmax, status, status_out, M, H, E, s));
    MOE_AFTER(marks, s, kProfLogits);
    if (fused_select(M, E, k)) {
        MOE_TRY(launch_route_select_permute(partial, L.splits, router_bias, ids, tw, offsets, sorted_ids, inv_pos, to,
                                            xmax, M, E, k, s, pdl));
        MOE_AFTER(marks, s, kProfSelect);
    } else {
        MOE_TRY(launch_route_topk(partial, L.splits, router_bias, ids, tw, xmax, xshift, M, E, k, s, pdl));
        MOE_AFTER(marks, s, kProfSelect);
        MOE_TRY(launch_permute(ids, offsets, sorted_ids, inv_pos, to, M, E, k, s, pdl));
        MOE_AFTER(marks, s, kProfPermute);
    }
    // gate_up: the 8/16-assignment tiles on mma.sync, then (large M) the tensor-core tiles
    int rc = run_gate_up(w13_q, w13_s, x_p4, tiles, n_tiles, h, true, status, status_out, H, I, E, k, L.width,
                         L.max_tiles, s, pdl);
    if (rc != MOE_OK) return rc;
    MOE_AFTER(marks, s, kProfGateUp);
    if (L.wide) {
        MOE_TRY(launch_gather_wide_rows(x_p4, sorted_ids, wl, x_perm, H, k, s, pdl));
        MOE_AFTER(marks, s, kProfGather);
        rc = run_wide(true, w13_q, w13_s, x_perm, wl, sorted_ids, h, true, y, status, status_out, M, H, I, E, k, s,
                      pdl, marks);
        if (rc != MOE_OK) return rc;
    }
    if (slab_enabled(M, I, E, k, L.width, L.wide)) {
        // the smallest calls: down and the weighted top-k combine in one launch, no y round trip
        rc = run_down_slab(w2_q, w2_s, h, tiles, n_tiles, tw, out, f32_out, status, status_out, M, H, I, E, k, s, pdl);
        if (rc != MOE_OK) return rc;
        MOE_AFTER(marks, s, kProfDown);
        return MOE_OK;
    }
    // down likewise, then the weighted top-k combine
    rc = run_down(w2_q, w2_s, h, sorted_ids, tiles, n_tiles, y, status, status_out, H, I, E, L.width, L.max_tiles, s,
                  pdl);
    if (rc != MOE_OK) return rc;
    MOE_AFTER(marks, s, kProfDown);
    if (L.wide) {
        rc = run_wide(false, w2_q, w2_s, h, wl, sorted_ids, nullptr, true, y, status, status_out, M, H, I, E, k, s,
                      pdl, marks);
        if (rc != MOE_OK) return rc;
    }
    MOE_TRY(launch_combine(y, tw, out, f32_out, M, H, k, s, pdl));
    MOE_AFTER(marks, s, kProfCombine);
    return MOE_OK;
}

static int check_forward_args(const void *x, const float *router_w, const float *router_bias, const uint8_t *w13_q,
                              const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s, void *out, int M,
                              int H, int I, int E, int k, const int32_t *topk_ids_out, const float *topk_w_out,
                              const int32_t *status_out, size_t out_elem_bytes = 2)
{
    int rc = check_dims(M, H, I, E, k, true);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;   // nothing is read or written
    if (!x || !router_w || !w13_q || !w13_s || !w2_q || !w2_s || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(w13_q, 16) || !aligned(w13_s, 16) ||
        !aligned(w2_q, 16) || !aligned(w2_s, 16) || !aligned(out, 16))
        return MOE_ERR_INVALID_ARG;
    if ((router_bias && !aligned(router_bias, 4)) || (topk_ids_out && !aligned(topk_ids_out, 4)) ||
        (topk_w_out && !aligned(topk_w_out, 4)) || (status_out && !aligned(status_out, 4)))
        return MOE_ERR_INVALID_ARG;
    const size_t xbytes = static_cast<size_t>(M) * H * 2;
    if (M > 0 && overlaps(x, xbytes, out, static_cast<size_t>(M) * H * out_elem_bytes)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

size_t moe_workspace_bytes(int M, int H, int I, int E, int k)
{
    if (check_dims(M, H, I, E, k, true) != MOE_OK) return 0;
    return make_layout(M, H, I, E, k).total;
}

int moe_selftest_wait_timeout(int32_t *status_out, cudaStream_t stream)
{
    if (!status_out || !aligned(status_out, 4)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(launch_wait_timeout_selftest(status_out, stream));
    return MOE_OK;
}

int moe_forward_launches(int M, int H, int I, int E, int k)
{
    const int rc = check_dims(M, H, I, E, k, true);
    if (rc != MOE_OK) return rc;
    if (M == 0) return 0;
    // route_logits, select (+ permute), gate_up, down, combine (down and combine one launch for the
    // smallest calls); gather + four tensor-core GEMMs
    const Layout L = make_layout(M, H, I, E, k);
    return (fused_select(M, E, k) ? 5 : 6) + (L.wide ? 5 : 0) - (slab_enabled(M, I, E, k, L.width, L.wide) ? 1 : 0);
}

int moe_route(const void *x_bf16, const float *router_w, const float *router_bias, int32_t *topk_ids, float *topk_w,
              int M, int H, int E, int k, cudaStream_t stream)
{
    int rc = check_dims(M, H, 32, E, k, false);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    if (!x_bf16 || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(router_w, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) ||
        (router_bias && !aligned(router_bias, 4)))
        return MOE_ERR_INVALID_ARG;
    if (M == 0) return MOE_OK;
    const Layout L = make_layout(M, H, 32, E, k);
    char *ws = nullptr;
    rc = library_workspace(stream, L.total, &ws);
    if (rc != MOE_OK) return rc;
    float *partial = reinterpret_cast<float *>(ws + L.partial);
    MOE_TRY(launch_route_logits(x_bf16, router_w, partial, nullptr, nullptr, reinterpret_cast<int *>(ws + L.status),
                                nullptr, M, H, E, stream));
    MOE_TRY(launch_route_topk(partial, L.splits, router_bias, topk_ids, topk_w, nullptr, nullptr, M, E, k, stream,
                              false));
    return MOE_OK;
}

int moe_permute(const int32_t *topk_ids, int32_t *expert_offsets, int32_t *sorted_ids, int32_t *inv_pos, int M, int E,
                int k, cudaStream_t stream)
{
    int rc = check_dims(M, 32, 32, E, k, false);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    if (!topk_ids || !expert_offsets || !sorted_ids || !inv_pos) return MOE_ERR_INVALID_ARG;
    if (!aligned(topk_ids, 4) || !aligned(expert_offsets, 4) || !aligned(sorted_ids, 4) || !aligned(inv_pos, 4))
        return MOE_ERR_INVALID_ARG;
    if (M == 0) return MOE_OK;
    const TileOut none{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 8, nullptr, k};
    MOE_TRY(launch_permute(topk_ids, expert_offsets, sorted_ids, inv_pos, none, M, E, k, stream, false));
    return MOE_OK;
}

int moe_gate_up_swiglu(const void *x_bf16, const uint8_t *w13_q, const uint8_t *w13_s, const int32_t *expert_offsets,
                       const int32_t *sorted_ids, void *h_bf16, int M, int H, int I, int E, int k, cudaStream_t stream)
{
    int rc = check_dims(M, H, I, E, k, true);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    if (!x_bf16 || !w13_q || !w13_s || !expert_offsets || !sorted_ids || !h_bf16) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(w13_q, 16) || !aligned(w13_s, 16) || !aligned(h_bf16, 16) ||
        !aligned(expert_offsets, 4) || !aligned(sorted_ids, 4))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(M, H, I, E, k);
    char *ws = nullptr;
    rc = library_workspace(stream, L.total, &ws);
    if (rc != MOE_OK) return rc;
    int *status = reinterpret_cast<int *>(ws + L.status);
    ExpertTile *tiles = reinterpret_cast<ExpertTile *>(ws + L.tiles);
    int *n_tiles = reinterpret_cast<int *>(ws + L.n_tiles);
    const WideLists wl = wide_lists(ws, L);
    __nv_bfloat16 *x_perm = reinterpret_cast<__nv_bfloat16 *>(ws + L.x_perm);
    __nv_bfloat16 *x_p4 = reinterpret_cast<__nv_bfloat16 *>(ws + L.x_p4);
    __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(h_bf16);
    int *xshift = reinterpret_cast<int *>(ws + L.xshift);
    // the tokens' activation shifts (the whole layer's router computes them), then the same tiles
    // as a whole-layer call (mma.sync tiles, and tensor-core tiles)
    MOE_TRY(launch_row_shift(static_cast<const __nv_bfloat16 *>(x_bf16), xshift, M, H, stream));
    const TileOut to{tiles, n_tiles, L.wide ? wl.small : nullptr, wl.n_small, wl.large, wl.n_large, L.width,
                     xshift, k};
    MOE_TRY(launch_build_tiles(expert_offsets, sorted_ids, to, status, E, stream));
    // x into the P4 K order the grouped GEMMs read (the whole layer's router writes it)
    MOE_TRY(launch_rows_to_p4(static_cast<const __nv_bfloat16 *>(x_bf16), x_p4, static_cast<size_t>(M), H, stream));
    rc = run_gate_up(w13_q, w13_s, x_p4, tiles, n_tiles, h, false, status, nullptr, H, I, E, k, L.width, L.max_tiles,
                     stream, false);
    if (rc != MOE_OK) return rc;
    if (L.wide) {
        MOE_TRY(launch_gather_wide_rows(x_p4, sorted_ids, wl, x_perm, H, k, stream, false));
        rc = run_wide(true, w13_q, w13_s, x_perm, wl, sorted_ids, h, false, nullptr, status, nullptr, M, H, I, E, k,
                      stream, false);
    }
    return rc;
}

int moe_down_combine(const void *h_bf16, const uint8_t *w2_q, const uint8_t *w2_s, const float *topk_w,
                     const int32_t *expert_offsets, const int32_t *sorted_ids, void *out_bf16, int M, int H, int I,
                     int E, int k, cudaStream_t stream)
{
    int rc = check_dims(M, H, I, E, k, true);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    if (!h_bf16 || !w2_q || !w2_s || !topk_w || !expert_offsets || !sorted_ids || !out_bf16) return MOE_ERR_INVALID_ARG;
    if (!aligned(h_bf16, 16) || !aligned(w2_q, 16) || !aligned(w2_s, 16) || !aligned(out_bf16, 16) ||
        !aligned(topk_w, 4) || !aligned(expert_offsets, 4) || !aligned(sorted_ids, 4))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(M, H, I, E, k);
    char *ws = nullptr;
    rc = library_workspace(stream, L.total, &ws);
    if (rc != MOE_OK) return rc;
    int *status = reinterpret_cast<int *>(ws + L.status);
    ExpertTile *tiles = reinterpret_cast<ExpertTile *>(ws + L.tiles);
    int *n_tiles = reinterpret_cast<int *>(ws + L.n_tiles);
    const WideLists wl = wide_lists(ws, L);
    __nv_bfloat16 *h_p4 = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);
    float *y = reinterpret_cast<float *>(ws + L.y);
    // (the down kernels scale h by a fixed power of two: no per-token shifts)
    const TileOut to{tiles, n_tiles, L.wide ? wl.small : nullptr, wl.n_small, wl.large, wl.n_large, L.width, nullptr,
                     k};
    MOE_TRY(launch_build_tiles(expert_offsets, sorted_ids, to, status, E, stream));
    // the caller's h rows (natural K order) into the P4 order the down kernels read
    MOE_TRY(launch_rows_to_p4(static_cast<const __nv_bfloat16 *>(h_bf16), h_p4, static_cast<size_t>(M) * k, I,
                              stream));
    if (slab_enabled(M, I, E, k, L.width, L.wide))   // the same launch plan as a whole-layer call
        return run_down_slab(w2_q, w2_s, h_p4, tiles, n_tiles, topk_w, out_bf16, false, status, nullptr, M, H, I, E, k,
                             stream, false);
    rc = run_down(w2_q, w2_s, h_p4, sorted_ids, tiles, n_tiles, y, status, nullptr, H, I, E, L.width, L.max_tiles,
                  stream, false);
    if (rc != MOE_OK) return rc;
    if (L.wide) {
        rc = run_wide(false, w2_q, w2_s, h_p4, wl, sorted_ids, nullptr, true, y, status, nullptr, M, H, I, E, k,
                      stream, false);
        if (rc != MOE_OK) return rc;
    }
    MOE_TRY(launch_combine(y, topk_w, out_bf16, false, M, H, k, stream, false));
    return MOE_OK;
}

int moe_mxfp4_forward_ex(const void *x, const float *router_w, const float *router_bias, const uint8_t *w13_q,
                         const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s, void *out, int M, int H,
                         int I, int E, int k, int32_t *topk_ids_out, float *topk_w_out, int32_t *status_out,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    int rc = check_forward_args(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, topk_ids_out,
                                topk_w_out, status_out);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    const Layout L = make_layout(M, H, I, E, k);
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    return forward_impl(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, topk_ids_out,
                        topk_w_out, status_out, static_cast<char *>(workspace), L, stream);
}

int moe_mxfp4_forward_partial(const void *x, const float *router_w, const float *router_bias,
                              const uint8_t *w13_q, const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s,
                              float *partial_out, int M, int H, int I_shard, int E, int k, int32_t *topk_ids_out,
                              float *topk_w_out, int32_t *status_out, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream)
{
    int rc = check_forward_args(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, partial_out, M, H, I_shard, E, k,
                                topk_ids_out, topk_w_out, status_out, 4);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    const Layout L = make_layout(M, H, I_shard, E, k);
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    return forward_impl(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, partial_out, M, H, I_shard, E, k,
                        topk_ids_out, topk_w_out, status_out, static_cast<char *>(workspace), L, stream, nullptr,
                        true);
}

int moe_reduce_partials(const float *partials, int G, void *out_bf16, int M, int H, cudaStream_t stream)
{
    if (G <= 0 || M < 0 || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 4 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (M == 0) return MOE_OK;
    if (!partials || !out_bf16 || !aligned(partials, 16) || !aligned(out_bf16, 16)) return MOE_ERR_INVALID_ARG;
    const size_t pbytes = static_cast<size_t>(G) * M * H * 4;
    if (overlaps(partials, pbytes, out_bf16, static_cast<size_t>(M) * H * 2)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(launch_reduce_partials(partials, G, out_bf16, M, H, stream));
    return MOE_OK;
}

int moe_mxfp4_forward_profile(const void *x, const float *router_w, const float *router_bias, const uint8_t *w13_q,
                              const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s, void *out, int M, int H,
                              int I, int E, int k, int32_t *topk_ids_out, float *topk_w_out, int32_t *status_out,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream, float *kernel_ms)
{
    int rc = check_forward_args(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, topk_ids_out,
                                topk_w_out, status_out);
    if (rc != MOE_OK) return rc;
    if (!kernel_ms) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < MOE_PROFILE_KERNELS; ++i) kernel_ms[i] = 0.f;
    if (M == 0) return MOE_OK;
    const Layout L = make_layout(M, H, I, E, k);
    if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    Marks marks;
    int created = 0;
    cudaError_t e = cudaSuccess;
    for (; created <= MOE_PROFILE_KERNELS && e == cudaSuccess; ++created) e = cudaEventCreate(&marks.ev[created]);
    if (e == cudaSuccess) {
        rc = forward_impl(x, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, topk_ids_out,
                          topk_w_out, status_out, static_cast<char *>(workspace), L, stream, &marks);
        if (rc == MOE_OK) {
            e = cudaEventSynchronize(marks.ev[marks.n - 1]);
            for (int i = 0; i < MOE_PROFILE_KERNELS && e == cudaSuccess; ++i)
                if (marks.slot[i] > 0)
                    e = cudaEventElapsedTime(&kernel_ms[i], marks.ev[marks.slot[i] - 1], marks.ev[marks.slot[i]]);
        }
    } else {
        --created;
    }
    for (int i = 0; i < created; ++i) cudaEventDestroy(marks.ev[i]);
    if (rc != MOE_OK) return rc;
    if (e != cudaSuccess) return cuda_fail(e);
    return MOE_OK;
}

int moe_mxfp4_forward(const void *x, const float *router_w, const uint8_t *w13_q, const uint8_t *w13_s,
                      const uint8_t *w2_q, const uint8_t *w2_s, void *out, int M, int H, int I, int E, int k,
                      cudaStream_t stream)
{
    int rc = check_forward_args(x, router_w, nullptr, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, nullptr, nullptr,
                                nullptr);
    if (rc != MOE_OK) return rc;
    if (M == 0) return MOE_OK;
    const Layout L = make_layout(M, H, I, E, k);
    char *ws = nullptr;
    rc = library_workspace(stream, L.total, &ws);
    if (rc != MOE_OK) return rc;
    return forward_impl(x, router_w, nullptr, w13_q, w13_s, w2_q, w2_s, out, M, H, I, E, k, nullptr, nullptr, nullptr,
                        ws, L, stream);
}

}  // extern "C"
