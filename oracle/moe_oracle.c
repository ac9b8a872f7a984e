/*
 * moe_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow fp64 CPU reference for one routed MXFP4 Mixture-of-Experts layer
 * call.  Only the test suite, the smoke check and the bench's CPU-baseline leg
 * load it.  It shares no code, header or table with the CUDA library.
 *
 * What the layer computes (the kernel family that the attribution table
 * "Post-Portfolio Device Attribution" of "MTP1 Post-Portfolio Eager-Cycle
 * Profile" lists as native router select/normalize, route remap, routed gather,
 * compact routed MXFP4 GEMM and routed clamp-SwiGLU):
 *
 *   l      = x . W_r^T (+ b)                    router logits, one per expert
 *   p      = softmax(l)                         over all E experts
 *   ids    = top-k of p, descending, ties -> lower expert id
 *   w_j    = p_{ids_j} / sum_j p_{ids_j}        renormalised routing weights
 *   g, u   = W_gate,e . x,  W_up,e . x          e = ids_j, MXFP4 weights
 *   h      = bf16_rne( silu(min(g,7)) * clamp(u,-7,7) )
 *   y_j    = W2_e . h
 *   out64  = sum_j w_j * y_j,   out = bf16_rne(out64)
 *
 * MXFP4 (OCP Microscaling Formats v1.0, FP4 E2M1 element + E8M0 block scale):
 * packed bytes hold two E2M1 codes, the low nibble being the even K index; one
 * E8M0 byte scales each 32 consecutive K elements of a row; value = E2M1(code)
 * * 2^(scale-127).  w13 holds the I gate rows, then the I up rows, of each expert.
 *
 * Readings this oracle takes where the pages say nothing (each is listed in the
 * design notes): the E2M1 table is the OCP one; bias is added to the logits before
 * the softmax; the intermediate h is rounded to bf16 once ("rounded BF16"
 * exchange of the "Decision" section of the same page), y is not rounded, out
 * is rounded once; the expert-grouped order is stable (ascending flat id t*k+j).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC moe_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ number formats */

/* FP4 E2M1: sign bit 3, two exponent bits (bias 1), one mantissa bit.  Exponent
 * field 0 is subnormal: 0.m * 2^0.  Written from the format's definition. */
double oracle_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E8M0: an unsigned biased exponent, 2^(byte-127); 0xFF is NaN. */
double oracle_e8m0_scale(int byte)
{
    if (byte == 255) return NAN;
    return ldexp(1.0, byte - 127);
}

/* Weight element (row, k) of an MXFP4 matrix with K columns. */
static double mx_weight(const uint8_t *q, const uint8_t *s, int K, long row, int k)
{
    uint8_t byte = q[row * (K / 2) + k / 2];
    int code = (k & 1) ? (byte >> 4) : (byte & 15);
    return oracle_e2m1_value(code) * oracle_e8m0_scale(s[row * (K / 32) + k / 32]);
}

double oracle_mxfp4_weight(const uint8_t *q, const uint8_t *s, int K, long row, int k)
{
    return mx_weight(q, s, K, row, k);
}

double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round an fp64 value to bf16 (8 significant bits), nearest, ties to even. */
uint16_t oracle_round_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    double r;
    double a = fabs(v);
    if (a == 0.0 || isinf(v)) {
        r = v;
    } else if (a < ldexp(1.0, -126)) {
        r = nearbyint(ldexp(v, 133)) * ldexp(1.0, -133);   /* bf16 subnormal spacing 2^-133 */
    } else {
        int e;
        double m = frexp(v, &e);                            /* v = m 2^e, 0.5 <= |m| < 1 */
        r = ldexp(nearbyint(m * 256.0), e - 8);
    }
    if (fabs(r) >= ldexp(1.0, 128)) r = v > 0 ? INFINITY : -INFINITY;
    float f = (float)r;                                     /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ router */

/* Router select/normalize for one token: fp64 logits, softmax over all E,
 * top-k by descending probability, i.e. descending logit (ties -> lower id),
 * renormalise over the k selected. */
static void route_token(const uint16_t *x, const float *wr, const float *bias, int H, int E, int k,
                        int32_t *ids, double *w, double *logits)
{
    double lmax = -INFINITY;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += oracle_bf16_to_double(x[h]) * (double)wr[(long)e * H + h];
        if (bias) acc += (double)bias[e];
        logits[e] = acc;
        if (acc > lmax) lmax = acc;
    }
    double *p = (double *)malloc(sizeof(double) * E);
    char *taken = (char *)calloc(E, 1);
    double z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = exp(logits[e] - lmax); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double sel = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || logits[e] > logits[best])) best = e;
        taken[best] = 1;
        ids[j] = best;
        sel += p[best];
    }
    for (int j = 0; j < k; ++j) w[j] = p[ids[j]] / sel;
    free(p);
    free(taken);
}

void oracle_route(const uint16_t *x, const float *router_w, const float *router_bias,
                  int M, int H, int E, int k, int32_t *topk_ids, double *topk_w, double *logits)
{
    #pragma omp parallel for schedule(dynamic)
    for (int t = 0; t < M; ++t)
        route_token(x + (long)t * H, router_w, router_bias, H, E, k,
                    topk_ids + (long)t * k, topk_w + (long)t * k, logits + (long)t * E);
}

/* ------------------------------------------------------------------ route remap */

/* Expert-grouped order: histogram of expert ids, exclusive prefix sum, stable
 * scatter of the flat assignment ids f = t*k + j (ascending f within an expert).
 * inv_pos[f] is the position of f in that order. */
void oracle_permute(const int32_t *topk_ids, int M, int E, int k,
                    int32_t *expert_offsets, int32_t *sorted_ids, int32_t *inv_pos)
{
    int n = M * k;
    int32_t *fill = (int32_t *)calloc(E + 1, sizeof(int32_t));
    for (int e = 0; e <= E; ++e) expert_offsets[e] = 0;
    for (int f = 0; f < n; ++f) expert_offsets[topk_ids[f] + 1] += 1;
    for (int e = 0; e < E; ++e) expert_offsets[e + 1] += expert_offsets[e];
    for (int f = 0; f < n; ++f) {
        int e = topk_ids[f];
        int pos = expert_offsets[e] + fill[e]++;
        sorted_ids[pos] = f;
        inv_pos[f] = pos;
    }
    free(fill);
}

/* ------------------------------------------------------------------ expert MLP */

/* gate_up GEMV of one token through one expert, then clamp-SwiGLU rounded to bf16.
 * w13q/w13s point at the expert's [2I, H/2] and [2I, H/32] blocks. */
void oracle_expert_swiglu(const uint16_t *x, const uint8_t *w13q, const uint8_t *w13s, int H, int I,
                          double *g_out, double *u_out, uint16_t *h_out)
{
    for (int n = 0; n < I; ++n) {
        double g = 0.0, u = 0.0;
        for (int kk = 0; kk < H; ++kk) {
            double xv = oracle_bf16_to_double(x[kk]);
            g += mx_weight(w13q, w13s, H, n, kk) * xv;
            u += mx_weight(w13q, w13s, H, (long)I + n, kk) * xv;
        }
        double a = g < 7.0 ? g : 7.0;
        double c = u < -7.0 ? -7.0 : (u > 7.0 ? 7.0 : u);
        double silu = a / (1.0 + exp(-a));
        if (g_out) g_out[n] = g;
        if (u_out) u_out[n] = u;
        h_out[n] = oracle_round_bf16(silu * c);
    }
}

/* down GEMV of one bf16 intermediate row through one expert's [H, I/2] / [H, I/32] w2. */
void oracle_expert_down(const uint16_t *h, const uint8_t *w2q, const uint8_t *w2s, int H, int I, double *y)
{
    for (int c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += mx_weight(w2q, w2s, I, c, i) * oracle_bf16_to_double(h[i]);
        y[c] = acc;
    }
}

/* ------------------------------------------------------------------ full layer */

/*
 * Layer forward for the tokens listed in `tokens` (all M tokens when tokens == NULL).
 * Expert weights are passed as per-expert pointer tables so that a caller may
 * supply only the experts a token touches.  Outputs for a listed token t:
 * topk_ids/topk_w rows t, h rows t*k+j (flat order, bf16 bits), out64/out_bf16 rows t.
 * Routing is computed for every token (the permutation needs all of them).
 */
void oracle_forward(const uint16_t *x, const float *router_w, const float *router_bias,
                    const uint8_t *const *w13q, const uint8_t *const *w13s,
                    const uint8_t *const *w2q, const uint8_t *const *w2s,
                    int M, int H, int I, int E, int k,
                    const int32_t *tokens, int n_tokens,
                    int32_t *topk_ids, double *topk_w, uint16_t *h, double *out64, uint16_t *out_bf16)
{
    double *logits = (double *)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * E);
    oracle_route(x, router_w, router_bias, M, H, E, k, topk_ids, topk_w, logits);
    free(logits);
    int nt = tokens ? n_tokens : M;
    /* one (token, slot) assignment per iteration */
    #pragma omp parallel for schedule(dynamic)
    for (long a = 0; a < (long)nt * k; ++a) {
        int t = tokens ? tokens[a / k] : (int)(a / k);
        int j = (int)(a % k);
        int e = topk_ids[(long)t * k + j];
        oracle_expert_swiglu(x + (long)t * H, w13q[e], w13s[e], H, I, NULL, NULL, h + ((long)t * k + j) * I);
    }
    #pragma omp parallel for schedule(dynamic)
    for (int ti = 0; ti < nt; ++ti) {
        int t = tokens ? tokens[ti] : ti;
        double *y = (double *)malloc(sizeof(double) * H);
        for (int c = 0; c < H; ++c) out64[(long)t * H + c] = 0.0;
        for (int j = 0; j < k; ++j) {
            int e = topk_ids[(long)t * k + j];
            oracle_expert_down(h + ((long)t * k + j) * I, w2q[e], w2s[e], H, I, y);
            for (int c = 0; c < H; ++c) out64[(long)t * H + c] += topk_w[(long)t * k + j] * y[c];
        }
        for (int c = 0; c < H; ++c) out_bf16[(long)t * H + c] = oracle_round_bf16(out64[(long)t * H + c]);
        free(y);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
