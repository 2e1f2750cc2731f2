/*
 * lhcal.h - C ABI of liblhcal.so: local-Hessian NVFP4 weight-scale calibration on B200 (sm_100a).
 *
 * The method (NVIDIA Model-Optimizer pull requests, cited by page title and section):
 *   - "add local hessian calibration" (PR #788), Overview: weight-scale candidates are
 *     weighed by a per-16-wide-input-block Hessian H_n = X_b^T X_b / B.
 *   - "Add activation-aware local Hessian scale calibration" (PR #1976), "What does this PR
 *     do?": H = X_q^T X_q / B, P = X_q^T (X_q - X) / B and the loss dW^T H dW + 2 dW^T (P W0),
 *     dW = quant(w) - w; the reviews: losses may be negative, best loss starts at +inf,
 *     kernels validate device placement and sizes.
 *   - "Add WMSE weight scale search calibration" (PR #2283), "What"/"How": Imp_i = ||X[:,i]||^2
 *     kept as [n_blocks, 16], loss sum_i Imp_i dW_i^2, 126 candidate E4M3 block scales.
 *   - "Add composable scale calibration to GPTQ" (PR #2004): 448-normalized NVFP4 scaling,
 *     g = amax / (6 * 448).
 *   - "[2/3] Speed up layerwise GPTQ on MoE models" (PR #2864), embedded #2840 description:
 *     per-expert Hessians over the tokens routed to each expert; an expert that no token
 *     reaches gets the plain search. Embedded #2877: launch on the tensors' own device.
 *
 * Conventions for every call:
 *   - All tensors are caller-owned device memory on the CURRENT device; the library keeps
 *     no state across calls, allocates nothing and never synchronises. Work is enqueued on
 *     `stream` (a cudaStream_t; NULL = legacy default stream) and runs asynchronously.
 *   - Sizes are element counts. Row-major, C order. cin must be a positive multiple of 16.
 *   - Status codes: LHCAL_ERR_INVALID_ARG for a null/misaligned pointer, a bad size or a
 *     host pointer where device memory is required; LHCAL_ERR_DEVICE_MISMATCH for memory of
 *     another device than the current one; LHCAL_ERR_UNSUPPORTED for an unknown mode/dtype;
 *     LHCAL_ERR_CUDA when a launch fails (the CUDA error string is kept). On any error
 *     nothing is enqueued, except for LHCAL_ERR_CUDA, where earlier launches of the same
 *     call may have been enqueued. lhcal_last_error_string() describes the last error of
 *     the calling thread.
 *   - Inputs must be finite; results for NaN/Inf inputs are unspecified.
 */
#ifndef LHCAL_H_
#define LHCAL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LHCAL_OK = 0,
  LHCAL_ERR_INVALID_ARG = 1,
  LHCAL_ERR_UNSUPPORTED = 2,
  LHCAL_ERR_DEVICE_MISMATCH = 3,
  LHCAL_ERR_CUDA = 4,
  LHCAL_ERR_TIMEOUT = 5 /* reserved for bounded device waits; no current kernel waits */
} lhcal_status;

typedef enum { LHCAL_F32 = 0, LHCAL_BF16 = 1 } lhcal_dtype;

typedef enum {
  LHCAL_FULL = 0,      /* H_n = X_b^T X_b / B                      (PR #788)  */
  LHCAL_ACT_AWARE = 1, /* H = X_q^T X_q / B, P = X_q^T (X_q - X) / B (PR #1976) */
  LHCAL_DIAG = 2,      /* Imp_i = ||X[:, i]||^2                      (PR #2283) */
  LHCAL_MSE = 3        /* plain block MSE, H = I: the "mse" method (PR #2283 fingerprint
                          control); lhcal_scale_sweep only, with h = p = NULL */
} lhcal_mode;

/* lhcal_accumulate flags. */
#define LHCAL_ACCUM_ADD 0       /* h (and p) += this call's sums                  */
#define LHCAL_ACCUM_OVERWRITE 1 /* h (and p) = this call's sums (no read of h / p) */

/* Number of 126 candidate block scales (E4M3 codes 0x01..0x7E), PR #2283 "How". */
#define LHCAL_N_CANDIDATES 126
#define LHCAL_BLOCK 16
/* Most multipliers lhcal_multiplier_search takes. */
#define LHCAL_MAX_MULTIPLIERS 1024

/*
 * Bytes of workspace lhcal_accumulate needs for these sizes (0 is possible). Host-only
 * computation; needs no GPU. groups > 1 (grouped) needs none.
 */
lhcal_status lhcal_accumulate_workspace(lhcal_mode mode, lhcal_dtype dtype, int64_t tokens,
                                        int64_t cin, int32_t groups, size_t* bytes);

/*
 * Hessian accumulation (raw sums, no 1/B), PR #788 Overview, PR #1976, PR #2283 "How".
 *   x, xq   : [tokens, cin] activations, row stride ldx elements (ldx >= cin, ldx * element
 *             size a multiple of 16 bytes, base 16-byte aligned). xq only for ACT_AWARE
 *             (the input quantizer's output), else NULL.
 *   groups  : 1 with group_offsets = token_ids = NULL sums over all rows of x. Grouped
 *             (fused-MoE experts, PR #2864 / #2840): group_offsets [groups + 1] (device,
 *             non-decreasing, offsets[0] = 0) and token_ids [offsets[groups]] (device,
 *             each in [0, tokens)); group e sums rows token_ids[offsets[e] .. offsets[e+1]).
 *   h       : FULL/ACT: [groups, cin/16, 16, 16] fp32, h[e][n][i][j] = sum x_{t,16n+i} x_{t,16n+j}
 *             (x = xq for ACT). DIAG: [groups, cin/16, 16] fp32 sum of squares per column.
 *   p       : ACT only: [groups, cin/16, 16, 16], p[e][n][i][j] = sum xq_{t,16n+i} (xq - x)_{t,16n+j};
 *             NULL otherwise.
 *   flags   : LHCAL_ACCUM_ADD or LHCAL_ACCUM_OVERWRITE.
 *   workspace: device scratch of at least lhcal_accumulate_workspace() bytes, 256-byte
 *             aligned; may be NULL when that size is 0. Its contents need no initialisation.
 * tokens = 0 with one group: x may be NULL (ACT_AWARE still takes a non-NULL xq, which is not
 * read); OVERWRITE writes zero sums, ADD leaves h and p as they are. A grouped call needs x,
 * group_offsets and token_ids as device pointers even when it routes no token, since the
 * offsets live on the device and the host cannot see that no row will be read; a NULL one is
 * LHCAL_ERR_INVALID_ARG. A caller with an empty grouped batch skips the call (ADD) or zeroes
 * h and p itself (OVERWRITE).
 * Results are deterministic for fixed sizes (fixed summation order). bf16 products are exact
 * in fp32; sums are fp32.
 */
lhcal_status lhcal_accumulate(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                              int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                              const int32_t* group_offsets, const int32_t* token_ids, int32_t flags,
                              float* h, float* p, void* workspace, size_t workspace_bytes, void* stream);

/*
 * NVFP4 fake quant of activations, the input quantizer whose output X_q the activation-aware
 * capture records (PR #1976, re-review: the input-quantizer hook captures X_q). Per token and
 * 16-wide block along cin:
 *   c = E4M3 code nearest to amax_blk / (6 * gx) (exact quotient, ties to the even code,
 *       saturating at 448; c = 0 gives a zero block);
 *   s = fp32(v_c * gx);
 *   xq = bf16(fp32(q * s)) with the sign of x, q = E2M1 of the exact |x| / s (nearest, ties
 *        to even, clamped at 6).
 *   dtype : LHCAL_BF16 only (LHCAL_ERR_UNSUPPORTED otherwise).
 *   x     : [tokens, cin] bf16, row stride ldx; xq: out [tokens, cin] bf16, row stride ldxq
 *           (both strides >= cin with stride * 2 a multiple of 16 bytes, bases 16-byte aligned;
 *           x and xq must not overlap).
 *   act_gx: device fp32 scalar, the per-tensor global scale gx (for example lhcal_global_scale
 *           of X viewed as [1, tokens, cin]: amax / (6 * 448)); finite and >= 0.
 * Bit-exact: every rounding decision is taken on the exact quotient.
 */
lhcal_status lhcal_act_fake_quant(lhcal_dtype dtype, const void* x, int64_t tokens, int64_t cin, int64_t ldx,
                                  const float* act_gx, void* xq, int64_t ldxq, void* stream);

/*
 * Bytes of workspace lhcal_accumulate_act_quant needs for these sizes (0 is possible).
 * Host-only computation; needs no GPU. dtype must be LHCAL_BF16 (LHCAL_ERR_UNSUPPORTED
 * otherwise); a bad cin, groups or tokens is LHCAL_ERR_INVALID_ARG, as for
 * lhcal_accumulate_workspace.
 */
lhcal_status lhcal_accumulate_act_quant_workspace(lhcal_dtype dtype, int64_t tokens, int64_t cin, int32_t groups,
                                                  size_t* bytes);

/*
 * Activation-aware accumulation (PR #1976, "What does this PR do?": H and P from the input
 * quantizer's output X_q; re-review: X_q is what that quantizer produces), i.e.
 * lhcal_accumulate with LHCAL_ACT_AWARE, with the input quantizer fused: X_q is not read from
 * memory but derived from x inside the kernel exactly as lhcal_act_fake_quant computes it, so
 * the activations are read once. The sums are those of
 * lhcal_act_fake_quant followed by lhcal_accumulate(LHCAL_ACT_AWARE, ...) with that X_q, up to
 * the fp32 summation order (the two may split the tokens differently; grouped sums and equal
 * splits give identical bits).
 *   dtype : LHCAL_BF16 only (LHCAL_ERR_UNSUPPORTED otherwise).
 *   act_gx: device fp32 scalar, the input quantizer's global scale (see lhcal_act_fake_quant);
 *           it is an input because the quantizer's amax is calibrated before the capture.
 *   other arguments as for lhcal_accumulate with mode LHCAL_ACT_AWARE; the workspace size is
 *   lhcal_accumulate_act_quant_workspace(LHCAL_BF16, tokens, cin, groups).
 * Errors as for lhcal_accumulate; a NULL act_gx is LHCAL_ERR_INVALID_ARG.
 */
lhcal_status lhcal_accumulate_act_quant(lhcal_dtype dtype, const void* x, int64_t tokens, int64_t cin,
                                        int64_t ldx, int32_t groups, const int32_t* group_offsets,
                                        const int32_t* token_ids, const float* act_gx, int32_t flags,
                                        float* h, float* p, void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * Token counts B per group, the B of "/B" (PR #1976) counted per expert over its routed tokens
 * (PR #2864 / #2840): counts[e] (+)= offsets[e+1] - offsets[e], or counts[0] (+)= tokens when
 * group_offsets is NULL. counts: device int64 [groups], 8-byte aligned. flags as for
 * lhcal_accumulate. Errors: groups outside [1, 65535], groups > 1 without group_offsets,
 * negative tokens or unknown flags are LHCAL_ERR_INVALID_ARG.
 */
lhcal_status lhcal_count_tokens(int32_t groups, int64_t tokens, const int32_t* group_offsets,
                                int32_t flags, int64_t* counts, void* stream);

/*
 * Finalisation in place (PR #1976: "/B"; PR #2864 / #2840: zero-token fallback).
 *   FULL/ACT: h /= counts[e], p /= counts[e] (IEEE fp32 division).
 *   DIAG: Imp is left as the raw sum (PR #2283).
 *   counts[e] == 0: h := I (DIAG: Imp := 1) and p := 0, i.e. the plain block-MSE search.
 *   counts: device int64 [groups]; h, p laid out as in lhcal_accumulate (p NULL unless ACT).
 */
lhcal_status lhcal_finalize(lhcal_mode mode, int32_t groups, int64_t cin, const int64_t* counts,
                            float* h, float* p, void* stream);

/*
 * Global scale per group (PR #2004: 448-normalized): g[e] = fp32(max |W_e| / 2688), the
 * maximum taken exactly and divided with IEEE round-to-nearest.
 *   w: [groups, rows, cin] (fp32 or bf16), 16-byte aligned. g: device fp32 [groups].
 */
lhcal_status lhcal_global_scale(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                int64_t cin, float* g, void* stream);

/*
 * lhcal_global_scale with the FP8 normalization as a parameter: g[e] = fp32(max |W_e| /
 * (6 * fp8_max)). fp8_max = 448 is lhcal_global_scale; 256 is the NVFP4 "4/6" variant, which
 * "Add composable scale calibration to GPTQ" (PR #2004) names as 256-normalized. fp8_max must
 * be finite and in (0, 448] with 6 * fp8_max exact in fp32 (any value with at most 21
 * significant bits); LHCAL_ERR_INVALID_ARG otherwise.
 */
lhcal_status lhcal_global_scale_ex(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                   int64_t cin, float fp8_max, float* g, void* stream);

/*
 * Exhaustive FP8 scale sweep (PR #2283 "How", PR #1976 reviews). For each unit (e, r, n):
 *   for code k = 1..126: s_k = fp32(v_k * g[e]) with v_k the E4M3 value of k;
 *     q_i = E2M1 round-to-nearest-even of the exact |w_i| / s_k, clamped at 6;
 *     wq_i = copysign(fp32(q_i * s_k), w_i); dW = wq - w;
 *     L_k = dW^T H_n dW (FULL), + 2 dW^T (P_n w) (ACT), or sum_i Imp_{n,i} dW_i^2 (DIAG);
 *     MSE: sum_i dW_i^2 (h = p = NULL);
 *   k* = the lowest k with the smallest L_k (losses may be negative).
 * Decisions on the quotient are exact for g >= 2^-90 or g == 0 (g == 0 gives wq = +-0 and
 * code 1). Losses are evaluated in fp32.
 *   w     : [groups, rows, cin] fp32 or bf16, 16-byte aligned.
 *   h     : FULL/ACT: [groups, cin/16, 16, 16] finalized H; DIAG: [groups, cin/16, 16] Imp.
 *   p     : ACT: [groups, cin/16, 16, 16] finalized P; else NULL.
 *   g     : device fp32 [groups].
 *   codes : out [groups, rows, cin/16] uint8, the E4M3 bit pattern of the chosen scale.
 *   wq    : out [groups, rows, cin] fp32 fake-quantized weights (16-byte aligned), or NULL.
 *   loss  : out [groups, rows, cin/16] fp32 winning loss, or NULL.
 * Sizes: rows <= 65535 * 128, cin / 16 <= 65535, groups <= 65535 (LHCAL_ERR_INVALID_ARG otherwise).
 */
lhcal_status lhcal_scale_sweep(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                               int64_t rows, int64_t cin, const float* h, const float* p,
                               const float* g, uint8_t* codes, float* wq, float* loss, void* stream);

/*
 * Amax-multiplier search: the block-scale search without the FP8 sweep that "add local hessian
 * calibration" (PR #788, Changes table: configurable step size and multipliers) runs with the
 * same Hessian-weighted losses. For each unit (e, r, n), amax_blk = max |w| of its 16 weights,
 * and for each multiplier m_i in the given order:
 *   a_i = fp32(m_i * amax_blk) (a negative or NaN value counts as 0);
 *   c_i = the E4M3 code nearest to a_i / (6 * g[e]) on the exact quotient (ties to the even code,
 *         saturating at 448; 0 is a zero scale; g[e] == 0 gives 0): the NVFP4 block scale
 *         the quantizer derives from that amax;
 *   L_i = the loss of lhcal_scale_sweep's mode at s = fp32(v_{c_i} * g[e]).
 * The first multiplier with the smallest L_i wins. Outputs as for lhcal_scale_sweep: codes (the
 * winner's c, which may be 0), wq (or NULL), loss (or NULL).
 *   mode        : LHCAL_FULL, LHCAL_ACT_AWARE, LHCAL_DIAG or LHCAL_MSE (h = p = NULL).
 *   multipliers : device fp32 [n_multipliers], 1 <= n_multipliers <= LHCAL_MAX_MULTIPLIERS;
 *                 finite and >= 0 (for example start + i * step).
 *   other arguments as for lhcal_scale_sweep.
 */
lhcal_status lhcal_multiplier_search(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                                     int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                                     const float* multipliers, int32_t n_multipliers, uint8_t* codes, float* wq,
                                     float* loss, void* stream);

/*
 * Outputs for chosen block-scale codes (for example the codes lhcal_scale_sweep wrote): for each
 * unit (e, r, n) with s = fp32(v_c * g[e]), v_c the E4M3 value of code c:
 *   wq   : out [groups, rows, cin] fp32, copysign(fp32(q_i * s), w_i), q_i the E2M1 rounding
 *          of the exact |w_i| / s as in lhcal_scale_sweep (bit-identical to its wq), or NULL;
 *   wq16 : out [groups, rows, cin] bf16, that fp32 value rounded to nearest even, or NULL;
 *   amax : out [groups, rows, cin/16] fp32, the block's amax fp32(6 * v_c * g[e]) (the value
 *          that maps to the chosen scale), or NULL.
 * Code 0 is a zero scale (wq = +-0, amax = 0); codes above 126 are taken as 126. w: fp32 or
 * bf16 [groups, rows, cin], 16-byte aligned; codes: device uint8 [groups, rows, cin/16].
 * The fake-quantized weights are what the quantizer state of "Add WMSE weight scale search
 * calibration" (PR #2283, refactor check) records next to amax and the per-block _amax.
 */
lhcal_status lhcal_apply_scales(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                const float* g, const uint8_t* codes, float* wq, void* wq16, float* amax,
                                void* stream);

/*
 * lhcal_accumulate for callers that cannot allocate device memory. The pages have no
 * counterpart to this call: it exists for deployment. Some callers cannot call cudaMalloc:
 * a plugin that a host framework hands only input and output pointers, a runtime whose
 * memory planner owns every device allocation up front, or code that must not trigger the
 * implicit device synchronisation an allocation can cause. They cannot provide the
 * workspace lhcal_accumulate asks for.
 *
 * Same arguments and results as lhcal_accumulate, without workspace. The split partials go
 * to a fixed scratch array of LHCAL_NOALLOC_SCRATCH_BYTES compiled into the library: every
 * GPU that loads the library holds it until the process exits. Sizes whose workspace
 * (lhcal_accumulate_workspace) exceeds it are rejected with LHCAL_ERR_INVALID_ARG before
 * anything is enqueued. The call allocates nothing and frees nothing.
 *   - The first call on each device looks up the scratch's device address (with that device
 *     current); make that first call before any stream capture on the device. The address is
 *     kept for the rest of the process, so destroying the device's primary context after that
 *     call (cudaDeviceReset) is not supported: the module would be reloaded at another address.
 *   - All calls on a device share the one scratch array, and it keeps the last call's
 *     contents. The kernels overwrite every partial before reading it, so no clearing is
 *     needed. Calls that can overlap on the GPU (on different streams, or from different
 *     threads without ordering) race on the scratch and give wrong results: order them.
 */
#define LHCAL_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
lhcal_status lhcal_accumulate_noalloc(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                                      int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                                      const int32_t* group_offsets, const int32_t* token_ids, int32_t flags,
                                      float* h, float* p, void* stream);

/*
 * Number of kernels this library enqueued from the calling thread since the last reset
 * (reset != 0 returns the count and sets it to zero). Host-side bookkeeping only.
 */
int64_t lhcal_launch_count(int32_t reset);

/* Message for the calling thread's last non-OK status ("" if none). */
const char* lhcal_last_error_string(void);

/* ABI version of this header (major * 100 + minor). */
int32_t lhcal_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LHCAL_H_ */
