/*
 * moe.h -- C ABI of libmoe.so: one routed MXFP4 Mixture-of-Experts layer call
 * for LLM decode on NVIDIA B200 (sm_100a).
 *
 * The layer (the kernel family that "MTP1 Post-Portfolio Eager-Cycle Profile",
 * table "Post-Portfolio Device Attribution", lists as native router
 * select/normalize, direct route remap, routed MoE gather, compact routed MXFP4
 * GEMM and routed clamp-SwiGLU; the grouped MoE GEMM structure that
 * "row/QUANT-CT-MXFP4-C8-DIFF" (vllm.cpp PR #52) traces at c8 decode):
 *
 *   logits = x W_r^T (+ b)              fp32, one per expert            moe_route
 *   ids    = top-k(softmax(logits))     descending, ties -> lower id    moe_route
 *   w      = renormalised top-k probs   sum to 1 per token              moe_route
 *   order  = expert-grouped assignments stable in flat id t*k+j         moe_permute
 *   h      = bf16(silu(min(g,7)) * clamp(u,-7,7)),
 *            g,u = gate/up rows of expert ids[t,j] applied to x[t]    moe_gate_up_swiglu
 *   out[t] = bf16( sum_j w[t,j] * (W2_{ids[t,j]} h[t,j]) )            moe_down_combine
 *
 * Data formats (all tensors row-major, contiguous, in caller-owned DEVICE memory):
 *   x, out            bf16 [M, H]
 *   router_w          fp32 [E, H];   router_bias fp32 [E] (nullable)
 *   w13_q             uint8 [E, 2I, H/2]  packed FP4 E2M1 (OCP MX v1.0), low nibble = even K
 *                                         rows 0..I-1 are gate, rows I..2I-1 are up
 *   w13_s             uint8 [E, 2I, H/32] E8M0 scale per 32 consecutive K of a row
 *   w2_q              uint8 [E, H, I/2];  w2_s uint8 [E, H, I/32]
 *   weight value      E2M1(code) * 2^(scale - 127)
 *   topk_ids / topk_w int32 / fp32 [M, k], slot j in descending router probability
 *   expert_offsets    int32 [E+1];  sorted_ids, inv_pos int32 [M*k]
 *   h                 bf16 [M*k, I] in expert-grouped order (row p holds the
 *                     assignment sorted_ids[p])
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers the caller owns; the library keeps none after
 *     returning.  Bulk tensors (x, out, router_w, w13_*, w2_*, h) must be 16-byte
 *     aligned; int32/fp32 index and weight arrays 4-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).  They
 *     never synchronise the host, and allocate nothing while `stream` is being
 *     captured into a CUDA graph.
 *   - Arguments are validated before anything is enqueued; a call that returns an
 *     error status has enqueued nothing.  M == 0 returns MOE_OK after the shape checks,
 *     reads no pointer (they may be NULL) and enqueues nothing.
 *   - Supported shapes: H % 32 == 0, I % 32 == 0, H,I >= 32, H <= 16384,
 *     1 <= k <= min(E, 32), E <= 1024, M*k <= 16384.  Others return
 *     MOE_ERR_UNSUPPORTED_SHAPE.
 *   - Arithmetic: bf16 x and the exactly decoded bf16 weights multiply into fp32
 *     accumulators; h is rounded to bf16 once; out is rounded to bf16 once.
 *   - Out of contract (undefined output, no fault): NaN/Inf in x, E8M0 scale
 *     byte 255 (NaN), and values beyond the fp32 range: a weight value of 2^128 or
 *     more (scale byte 253 or 254 with a large code) or a dot product, logit or
 *     output that overflows fp32.  Products that fall below fp32's normal range
 *     (weights and activations both far below 1) lose relative precision.
 *   - Determinism: for a given device and inputs, every output is bitwise
 *     reproducible (no floating-point atomics; fixed reduction orders).
 *
 * Workspace: the forms without a workspace argument use a library-owned device
 * buffer per (device, stream).  It grows with cudaMalloc on first use and never
 * while the stream is capturing; a capture that needs a larger one fails with
 * MOE_ERR_WORKSPACE (warm up once outside capture).  Two calls on the same stream
 * share it safely (stream order); calls on different streams get different
 * buffers.  moe_mxfp4_forward_ex takes the caller's buffer instead.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *cudaStream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,        /* null/misaligned pointer, negative size, aliasing */
    MOE_ERR_UNSUPPORTED_SHAPE = -2,  /* shape outside the supported set above */
    MOE_ERR_WORKSPACE = -3,          /* workspace too small (or growth refused during capture) */
    MOE_ERR_CUDA = -4,               /* a CUDA runtime/driver call or launch failed */
    MOE_ERR_TIMEOUT = -5             /* a bounded device-side wait gave up (reported via status_out) */
} moe_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *moe_status_string(int status);

/* Last CUDA error code seen by the library on this host thread (0 if none). */
int moe_last_cuda_error(void);

/*
 * Router select/normalize.  Defined by the "Native router select/normalize" row
 * of "Post-Portfolio Device Attribution" ("MTP1 Post-Portfolio Eager-Cycle
 * Profile"): per token, fp32 logits x.W_r^T (+ router_bias), softmax over the E
 * experts, the k largest in descending order (ties -> lower expert id), and their
 * probabilities renormalised to sum to 1 (equal to a softmax over the k selected
 * logits).  Writes topk_ids [M,k] int32 and topk_w [M,k] fp32.
 * Uses the library-owned workspace of `stream` for per-chunk partial logits.
 */
int moe_route(const void *x_bf16, const float *router_w, const float *router_bias,
              int32_t *topk_ids, float *topk_w, int M, int H, int E, int k, cudaStream_t stream);

/*
 * Route remap: expert-grouped order of the M*k assignments.  Defined by the
 * "Direct M=2 route remap" row of the same table (route-direct compact routes):
 * a histogram of topk_ids, its exclusive prefix sum expert_offsets [E+1], and a
 * stable scatter of the flat ids f = t*k + j into sorted_ids [M*k] (ascending f
 * within an expert); inv_pos[f] is the position of f in sorted_ids.
 * topk_ids values must lie in [0, E).  No workspace.
 */
int moe_permute(const int32_t *topk_ids, int32_t *expert_offsets, int32_t *sorted_ids,
                int32_t *inv_pos, int M, int E, int k, cudaStream_t stream);

/*
 * Grouped MXFP4 gate_up GEMM with the routed gather and clamp-SwiGLU fused in.
 * Defined by the "Compact routed MXFP4 GEMM", "Routed MoE gather" and "Routed
 * clamp-SwiGLU" rows of the same table, with the gate and up producers fused and
 * the intermediate rounded to bf16 (the "Decision" section of the same page).
 * For each position p of the expert-grouped order, f = sorted_ids[p], t = f / k,
 * e = the expert whose offsets range holds p:
 *   g = W_gate,e x[t], u = W_up,e x[t] (bf16 products, fp32 accumulation),
 *   h[p] = bf16_rne(silu(min(g,7)) * clamp(u,-7,7))  (bf16 [M*k, I], h_bf16).
 * expert_offsets/sorted_ids are moe_permute's outputs.  The experts' assignments are
 * split into tiles exactly as in moe_mxfp4_forward.  Uses the library-owned
 * workspace of `stream`.
 */
int moe_gate_up_swiglu(const void *x_bf16, const uint8_t *w13_q, const uint8_t *w13_s,
                       const int32_t *expert_offsets, const int32_t *sorted_ids, void *h_bf16,
                       int M, int H, int I, int E, int k, cudaStream_t stream);

/*
 * Down GEMM with the weighted top-k combine fused behind it.  Defined by the
 * down half of the "Compact routed MXFP4 GEMM" row of the same table (h bf16
 * [M*k, I] in expert-grouped order, as moe_gate_up_swiglu writes it):
 *   y[f] = W2_e h[inv position of f] (fp32 accumulation),
 *   out[t] = bf16_rne( sum_{j=0..k-1} topk_w[t,j] * y[t*k+j] ), summed in slot
 *   order j with no atomics.
 * For the smallest calls (I <= 1024 and at most 8 expert tiles: min(M*k, E) <= 8, with M <= 8,
 * fewer than 6 assignments per expert on average and no expert tiles for the tensor cores) one
 * kernel does both: each CTA owns 16 rows of H, keeps those rows of y for every assignment in
 * shared memory and writes out.  Otherwise the fp32 rows of y go through the library-owned
 * workspace of `stream` and a combine kernel.  Same bits either way.
 */
int moe_down_combine(const void *h_bf16, const uint8_t *w2_q, const uint8_t *w2_s, const float *topk_w,
                     const int32_t *expert_offsets, const int32_t *sorted_ids, void *out_bf16,
                     int M, int H, int I, int E, int k, cudaStream_t stream);

/*
 * Whole layer: moe_route -> moe_permute -> moe_gate_up_swiglu -> moe_down_combine,
 * enqueued back to back on `stream` with the library-owned workspace and no router
 * bias.  `out` must not overlap `x`.
 */
int moe_mxfp4_forward(const void *x, const float *router_w, const uint8_t *w13_q, const uint8_t *w13_s,
                      const uint8_t *w2_q, const uint8_t *w2_s, void *out,
                      int M, int H, int I, int E, int k, cudaStream_t stream);

/*
 * moe_route without any device allocation, for callers that cannot allocate at the
 * point where they route (an allocator that owns all device memory, a decode loop
 * that must not allocate between steps).  The pages have no counterpart: this is
 * an interface choice of this library.  Same arguments, results and checks as
 * moe_route; the scratch (the router's fp32 partial logits and a status word)
 * lives in a 4 MiB device array compiled into the library instead of the
 * library-owned workspace.
 *   - Limit: 256 + S * M * E * 4 bytes must fit in 4 MiB, where S is the number of
 *     H slices the router splits each expert group into: ceil(H / 256) for M <= 8,
 *     ceil(H / 512) for larger M, reduced toward 1 as M * E grows (for example
 *     33 KB at M = 8, H = 2048, E = 128; 1 MB at M = 1024, H = 7168, E = 256).
 *     Larger shapes return MOE_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on a device looks the array's device address up (once per
 *     device); make that first call before any stream capture.
 *   - Calls no cudaMalloc/cudaFree.  Every call shares the one array, which keeps
 *     the last call's contents (nothing in it needs to start at zero): calls that
 *     overlap on the GPU (other streams, other host threads) race on it.
 */
int moe_route_noalloc(const void *x_bf16, const float *router_w, const float *router_bias,
                      int32_t *topk_ids, float *topk_w, int M, int H, int E, int k, cudaStream_t stream);

/* Bytes of device workspace moe_mxfp4_forward_ex needs for this shape (0 if unsupported). */
size_t moe_workspace_bytes(int M, int H, int I, int E, int k);

/*
 * Kernel launches one moe_mxfp4_forward / moe_mxfp4_forward_ex call enqueues for this shape
 * (router logits, top-k + permutation as one or two kernels, the grouped GEMMs, the gather and
 * tensor-core GEMMs when the call can give experts 5 or more assignments, the combine -- one launch
 * with the down GEMM for the smallest calls, see moe_down_combine); 0 for M == 0 and a
 * negative MOE_* status for an unsupported shape.  For sizing CUDA graphs and for accounting.
 */
int moe_forward_launches(int M, int H, int I, int E, int k);

/*
 * Self-test of the device-side failure path.  Every producer/consumer wait inside the layer's
 * kernels is bounded: when it runs out, the kernel records MOE_ERR_TIMEOUT in the call's status
 * (moe_mxfp4_forward_ex's status_out), skips its remaining waits and ends, so the CUDA context
 * stays usable.  This call launches one small kernel that waits, through the same bounded wait
 * with a limit of about 10 ms, on a barrier that nothing ever completes.  It writes
 * MOE_ERR_TIMEOUT (int32) to status_out, a 4-byte-aligned DEVICE pointer, which the caller reads
 * after synchronising `stream`.  Returns MOE_ERR_INVALID_ARG for a null or misaligned pointer,
 * MOE_ERR_CUDA if the launch fails, else MOE_OK.  It faults nothing and touches no other memory.
 */
int moe_selftest_wait_timeout(int32_t *status_out, cudaStream_t stream);

/*
 * Whole layer with a caller-owned workspace (>= moe_workspace_bytes, 256-byte
 * aligned; its contents need no initialisation and are overwritten), an optional
 * router bias, optional copies of the routing (topk_ids_out [M,k] int32,
 * topk_w_out [M,k] fp32) and an optional device int32 `status_out` that receives
 * MOE_OK or MOE_ERR_TIMEOUT once the enqueued work has run.
 * A workspace smaller than required returns MOE_ERR_WORKSPACE.
 */
int moe_mxfp4_forward_ex(const void *x, const float *router_w, const float *router_bias,
                         const uint8_t *w13_q, const uint8_t *w13_s, const uint8_t *w2_q,
                         const uint8_t *w2_s, void *out, int M, int H, int I, int E, int k,
                         int32_t *topk_ids_out, float *topk_w_out, int32_t *status_out,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * One rank's share of the layer split over G GPUs along the expert intermediate dimension
 * ("I-sharding"; the pages' multi-GPU data point, expert parallelism over 8 GPUs in "The
 * Systematic Optimization Campaign", chunk 8.0, ran slower than one GPU at low concurrency and
 * failed under load, so the split here keeps every expert on every rank instead).
 * Rank r of G holds, for every expert, gate rows [r*I_shard, (r+1)*I_shard) followed by the
 * same up rows, as w13_q [E, 2*I_shard, H/2] / w13_s [E, 2*I_shard, H/32], and the matching K
 * range of the down projection, w2_q [E, H, I_shard/2] / w2_s [E, H, I_shard/32]: exactly the
 * weights of a layer with intermediate size I_shard (I_shard a multiple of 32).  Routing runs in
 * full on every rank, so ids and weights are the same bits everywhere.  partial_out [M,H] fp32
 * (16-byte aligned) receives sum_j w[t,j] * (W2_slice h_slice)[t,j] in slot order, NOT rounded.
 * The ranks then exchange their partials (an all-gather into [G,M,H], rank order) and each calls
 * moe_reduce_partials.  Workspace: moe_workspace_bytes(M, H, I_shard, E, k).  Other arguments,
 * errors and status as moe_mxfp4_forward_ex.
 */
int moe_mxfp4_forward_partial(const void *x, const float *router_w, const float *router_bias,
                              const uint8_t *w13_q, const uint8_t *w13_s, const uint8_t *w2_q, const uint8_t *w2_s,
                              float *partial_out, int M, int H, int I_shard, int E, int k, int32_t *topk_ids_out,
                              float *topk_w_out, int32_t *status_out, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * out[t,c] = bf16( sum_{g = 0 .. G-1} partials[g][t][c] ) with g ascending: the fixed-order
 * reduction of G ranks' moe_mxfp4_forward_partial outputs, stacked as partials [G,M,H] fp32
 * (device, 16-byte aligned; out [M,H] bf16, 16-byte aligned, not overlapping it).  Every rank
 * that reduces the same stack gets the same bits.  With G = 1 it returns what
 * moe_mxfp4_forward_ex writes for the same layer.  H must be a multiple of 4.
 * Asynchronous on `stream`; MOE_ERR_INVALID_ARG for G <= 0, M < 0, H <= 0 or a bad pointer.
 */
int moe_reduce_partials(const float *partials, int G, void *out_bf16, int M, int H, cudaStream_t stream);

/* Entries of moe_mxfp4_forward_profile's output. */
#define MOE_PROFILE_KERNELS 11

/*
 * Per-launch device-time attribution of one layer call, in the manner of the per-kernel
 * buckets of "Post-Portfolio Device Attribution" ("MTP1 Post-Portfolio Eager-Cycle
 * Profile").  Same arguments and results as moe_mxfp4_forward_ex; additionally records a
 * CUDA event before the first launch and after every launch, WAITS for the stream to finish
 * (host synchronisation: not for use under stream capture) and writes into the HOST array
 * kernel_ms the milliseconds of each launch (0 for a launch this shape does not make):
 *   [0] router logits, [1] router top-k (fused with the route remap when M <= 64),
 *   [2] route remap (0 when fused), [3] gate_up + clamp-SwiGLU on mma.sync tiles,
 *   [4] gather of the tensor-core tiles' x rows, [5] / [6] gate_up + clamp-SwiGLU on small /
 *   large tensor-core tiles, [7] down on mma.sync tiles, [8] / [9] down on small / large
 *   tensor-core tiles, [10] the weighted top-k combine (for the smallest calls [7] is down and
 *   the combine in one launch and [10] is 0; see moe_down_combine).
 * Kernels run back to back here instead of overlapping their launches as in
 * moe_mxfp4_forward_ex, so the sum exceeds a normal call's time.
 */
int moe_mxfp4_forward_profile(const void *x, const float *router_w, const float *router_bias,
                              const uint8_t *w13_q, const uint8_t *w13_s, const uint8_t *w2_q,
                              const uint8_t *w2_s, void *out, int M, int H, int I, int E, int k,
                              int32_t *topk_ids_out, float *topk_w_out, int32_t *status_out,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream,
                              float *kernel_ms);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
