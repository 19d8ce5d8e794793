/*
 * moe_mxfp4.h -- C ABI of the MoE feed-forward layer with MXFP4 experts on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (page "GPT-OSS-20B : Architecture MoE & Résumé du Model Card"):
 *   §3.1 Le Routeur: for each token h in R^d_model, scores = W_router . h
 *        (+ an optional per-expert bias), the top_k experts by score are
 *        selected, and a softmax over the selected scores gives weights that
 *        sum to 1;
 *   §3.2 Les Experts: each expert is a SwiGLU FFN
 *        (Swish(h . W_gate) (.) (h . W_up)) . W_down, Swish(z) = z sigma(z);
 *   §2.1: the layer output is the weighted sum of the top_k expert outputs;
 *   §4 Quantification MXFP4: the expert weights are stored at 4.25 bits per
 *        parameter -- FP4 E2M1 codes in blocks of 32 along the contraction
 *        axis, each block sharing one E8M0 power-of-two scale.
 *
 * Conventions for every call:
 *  - Pointers marked "device" are caller-owned CUDA device memory on the
 *    device that was current when the handle was created; "host" pointers are
 *    caller-owned host memory.  The library never frees caller memory.
 *  - Calls are asynchronous on the given stream unless stated otherwise.  The
 *    returned status reports host-detectable errors and CUDA launch errors;
 *    device-side failures (a pipeline wait that timed out) are reported by
 *    moe_mxfp4_get_status.
 *  - A handle may be used by one host thread at a time.  Calls on one handle
 *    that overlap on the GPU (different streams, no ordering) race on the
 *    handle's internal workspace.
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_mxfp4 moe_mxfp4_t; /* opaque: owns quantised weights and workspace */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but outside the supported envelope  */
    MOE_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed          */
    MOE_ERR_NOT_QUANTIZED = 4, /* forward before quantize_weights            */
    MOE_ERR_TIMEOUT = 5,       /* a device-side pipeline wait ran out        */
    MOE_ERR_BOUNDS = 6         /* debug build: an index check failed or a guard region changed */
} moe_status_t;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype_t;

/* Test-only flag: the expert-GEMM producer skips its first copy, so a
 * consumer wait runs out after config.wait_timeout_ms and the forward reports
 * MOE_ERR_TIMEOUT through moe_mxfp4_get_status. */
#define MOE_FLAG_TEST_SKIP_FIRST_COPY (1u << 30)

/* Token rows per expert-GEMM tile (BN).  0 (default): chosen per forward from
 * T, top_k and n_experts; v = 1..8 forces BN = 16 v (16 .. 128).  Every choice
 * computes the same layer; the tile only changes how work is cut. */
#define MOE_FLAG_TOKEN_TILE_SHIFT 8
#define MOE_FLAG_TOKEN_TILE_MASK (0xFu << MOE_FLAG_TOKEN_TILE_SHIFT)

/* Forwards of at most 16 tokens run as one cooperative launch (router, both
 * expert GEMMs and the combine in one persistent grid) when the layer's shape
 * allows it.  This flag (or a forced token tile) keeps every forward on the
 * multi-launch path instead; both compute the same layer. */
#define MOE_FLAG_UNFUSED_DECODE (1u << 12)

/* Activation operand format of the expert GEMMs.  Default: every activation
 * block (32 values along K: x for gate/up, the SwiGLU output H for down) is a
 * sum of three MXFP4 terms multiplied with the MXFP4 weights by the block-
 * scaled FP4 MMA (kind::mxf4).  With this flag it is a sum of two MXFP8 (E4M3)
 * terms multiplied with the same MXFP4 weights by kind::mxf8f6f4; the weights
 * are then stored in a padded layout (about 4.5 % more bytes for 2880 x 2880
 * experts) and forwards of at most 16 tokens take the multi-launch path.  Both
 * compute the layer of "GPT-OSS-20B : Architecture MoE & Résumé du Model
 * Card" §3.2/§4 within the same tolerance; export_weights returns the same
 * canonical codes and scales. */
#define MOE_FLAG_ACT_MXF8X2 (1u << 13)

/* Test-only: the n-th device allocation of moe_mxfp4_create (n = 1..255 in
 * this field; 0 = off) fails as if cudaMalloc had, so the failure path can be
 * exercised; create then returns MOE_ERR_CUDA having freed everything. */
#define MOE_FLAG_TEST_FAIL_ALLOC_SHIFT 16
#define MOE_FLAG_TEST_FAIL_ALLOC_MASK (0xFFu << MOE_FLAG_TEST_FAIL_ALLOC_SHIFT)

typedef struct {
    int32_t d_model;        /* model width; multiple of 32                    */
    int32_t d_ff;           /* expert hidden width; multiple of 32            */
    int32_t n_experts;      /* E, 1..256                                       */
    int32_t top_k;          /* k, 1..min(8, E)                                 */
    int32_t max_tokens;     /* largest T passed to forward, >= 1               */
    int32_t act_dtype;      /* moe_dtype_t of x, y and the router weight      */
    uint32_t flags;         /* 0, or MOE_FLAG_* test flags                     */
    int32_t wait_timeout_ms;/* device pipeline wait limit; <= 0 selects 2000   */
} moe_mxfp4_config_t;

/* Create a handle on the current device.  Allocates every buffer the layer
 * needs for up to cfg->max_tokens tokens, so forward allocates nothing.
 * Defines: the layer's shape -- d_model (the token width, 2880 for
 * gpt-oss-20b, §3.1), E experts and top_k selected per token (32 and 4, §2.1),
 * each expert a SwiGLU FFN of width d_ff (§3.2).
 * Errors: INVALID_ARG (null, non-positive sizes, bad dtype), UNSUPPORTED
 * (d_model or d_ff not a multiple of 32, E > 256, k > min(8, E),
 * d_model or d_ff above 16384), CUDA (allocation failed; nothing leaks). */
moe_status_t moe_mxfp4_create(const moe_mxfp4_config_t* cfg, moe_mxfp4_t** out);

/* Destroy a handle and free everything it owns.  NULL-safe.  Synchronises
 * the device work the handle issued. */
void moe_mxfp4_destroy(moe_mxfp4_t* h);

/* Quantise all expert weights to MXFP4 and store the router.
 * Defines: §4 Quantification MXFP4 (4.25 bits per parameter: blocks of 32 E2M1
 * codes sharing one E8M0 scale) applied to the three matrices of each §3.2
 * expert, and the §3.1 router weight W_router.
 *   w_gate, w_up: device fp32 [E][d_model][d_ff]   (expert e maps x -> x . W)
 *   w_down:       device fp32 [E][d_ff][d_model]
 *   w_router:     device [E][d_model] in act_dtype (scores = W_router . h)
 *   router_bias:  device fp32 [E], or NULL for no bias
 * Blocks of 32 run along the contraction axis (d_model for gate/up, d_ff for
 * down).  Block rule: scale exponent floor(log2(max|w|)) - 2 clamped to
 * [-127, 127]; elements round to the nearest E2M1 value, ties to the even
 * code, above 6 saturating, sign kept; an all-zero block gets scale 2^0.
 * Inputs must be finite; w_gate, w_up, w_down 4-byte aligned (else
 * INVALID_ARG).  May be called again to replace the weights. */
moe_status_t moe_mxfp4_quantize_weights(moe_mxfp4_t* h, const float* w_gate,
                                        const float* w_up, const float* w_down,
                                        const void* w_router, const float* router_bias,
                                        cudaStream_t stream);

/* Same quantisation for one expert e (lets callers stream very large expert
 * sets through a small fp32 staging buffer).  Defines: §4 on one §3.2 expert.
 * w_gate/w_up: device fp32 [d_model][d_ff]; w_down: device fp32
 * [d_ff][d_model]; all 4-byte aligned. */
moe_status_t moe_mxfp4_quantize_expert(moe_mxfp4_t* h, int32_t e, const float* w_gate,
                                       const float* w_up, const float* w_down,
                                       cudaStream_t stream);

/* Store the router weight (device [E][d_model], act_dtype) and optional bias
 * (device fp32 [E] or NULL).  Defines: W_router of §3.1 (scores =
 * W_router . h).  Copies; the caller may free its buffers after the stream
 * reaches this call. */
moe_status_t moe_mxfp4_set_router(moe_mxfp4_t* h, const void* w_router,
                                  const float* router_bias, cudaStream_t stream);

/* Steps adjacent to the MoE block, fused into its kernels (page "GPT-OSS vs
 * Qwen3 : comparaison détaillée", Adoption de RMSNorm: the block input is
 * normalised by its root mean square; and the skip connection around the
 * block).
 *   gamma:    device fp32 [d_model] (4-byte aligned), or NULL for no pre-norm.
 *             With it, the router and the experts see
 *             h = x / sqrt(mean(x^2) + eps) * gamma  (formed in fp32) instead of x.
 *   eps:      finite, >= 0 (else INVALID_ARG).
 *   residual: != 0 makes forward write y = x + (the MoE output).
 * Copies gamma (asynchronously on `stream`); applies to later forwards. */
moe_status_t moe_mxfp4_set_norm_residual(moe_mxfp4_t* h, const float* gamma, float eps,
                                         int32_t residual, cudaStream_t stream);

/* The layer for T tokens (0 <= T <= max_tokens; T == 0 launches nothing).
 * Defines: §3.1 (scores, top-k, softmax over the selected scores), §3.2 (each
 * selected expert's SwiGLU FFN) and §2.1 step 2 (the k outputs aggregated with
 * their routing weights).
 *   x:             device [T][d_model], act_dtype
 *   y:             device [T][d_model], act_dtype (written, not accumulated)
 *   topk_idx:      device int32 [T][k] or NULL -- selected experts, score-descending,
 *                  ties to the lower index
 *   topk_w:        device fp32 [T][k] or NULL -- softmax over the selected scores
 *   expert_counts: device int32 [E] or NULL -- rows routed to each expert
 * x and y must not overlap.  x and y must be 16-byte aligned and topk_idx,
 * topk_w, expert_counts 4-byte aligned; the device current at the call must be
 * the handle's; otherwise INVALID_ARG is returned before anything is
 * launched.  The expert matmuls are block-scaled MXFP4 x MXFP4 products with
 * fp32 accumulation: the weights enter as quantised, x and the SwiGLU output
 * H enter as sums of three MXFP4 terms (each block of 32 values and its
 * residuals, each term with its own E8M0 scale; H is formed in fp32).  The
 * layer output matches the double-precision definition within about 3e-3 of
 * max|y| on the 2880-wide workloads.  Asynchronous; allocates nothing. */
moe_status_t moe_mxfp4_forward(moe_mxfp4_t* h, const void* x, int32_t T, void* y,
                               int32_t* topk_idx, float* topk_w, int32_t* expert_counts,
                               cudaStream_t stream);

/* forward with HOST buffers (the same layer as moe_mxfp4_forward, §3.1, §3.2,
 * §2.1): copies x (host [T][d_model], act_dtype) in,
 * runs the layer, copies y (host [T][d_model]) and, if non-NULL, topk_idx
 * (host int32 [T][k]) and topk_w (host fp32 [T][k]) out, and synchronises
 * the stream before returning.  Uses handle-owned device staging buffers and
 * two handle-owned copy streams: a batch of T >= 8192 tokens runs as up to 8
 * chunks whose copies in and out overlap the forwards of their neighbours
 * (pinned host buffers make the copies asynchronous). */
moe_status_t moe_mxfp4_forward_host(moe_mxfp4_t* h, const void* x_host, int32_t T,
                                    void* y_host, int32_t* topk_idx_host,
                                    float* topk_w_host, cudaStream_t stream);

/* Export the quantised weights of one matrix in the canonical MXFP4 layout
 * (§4: E2M1 codes in blocks of 32 along the contraction axis, one E8M0 scale
 * per block); codes must be 16-byte aligned:
 * which = 0 gate, 1 up, 2 down.  For contraction length K and N outputs
 * (gate/up: K = d_model, N = d_ff; down: K = d_ff, N = d_model):
 *   codes:  device uint8 [E][N][K/2]   element k of row n in byte k/2,
 *                                      even k in the low nibble
 *   scales: device uint8 [E][N][K/32]  E8M0 (value 2^(s-127))  */
moe_status_t moe_mxfp4_export_weights(const moe_mxfp4_t* h, int32_t which, uint8_t* codes,
                                      uint8_t* scales, cudaStream_t stream);

/* Grouping produced by the last forward (for inspection and tests; the
 * tokens each §2.1 expert received):
 *   offsets:    device int32 [E+1]  rows of expert e are [offsets[e], offsets[e+1])
 *   row_token:  device int32 [T*k]  token of each grouped row (or NULL)
 *   row_weight: device fp32  [T*k]  routing weight of each grouped row (or NULL)
 * Rows of one expert appear in (token, slot) order.  After a forward that ran
 * the fused decode kernel (no grouping is built) this returns UNSUPPORTED. */
moe_status_t moe_mxfp4_get_grouping(const moe_mxfp4_t* h, int32_t* offsets, int32_t* row_token,
                                    float* row_weight, cudaStream_t stream);

/* Synchronise the handle's last stream and return (and clear) the device
 * status: MOE_OK, MOE_ERR_TIMEOUT if a pipeline wait ran out, or (debug
 * build) MOE_ERR_BOUNDS if an index check failed. */
moe_status_t moe_mxfp4_get_status(moe_mxfp4_t* h);

/* Debug build (the library compiled with MOE_DEBUG_CHECKS,
 * libmoe_mxfp4_debug.so): every device buffer a handle owns is followed by a
 * 4096-byte guard region of a fixed pattern, and the kernels check the
 * indices they scatter and gather through (grouped rows, token tiles, units,
 * tokens of the combine); a failed check skips the access and makes
 * moe_mxfp4_get_status return MOE_ERR_BOUNDS.  This call synchronises the
 * device and returns MOE_ERR_BOUNDS if any guard byte changed, else MOE_OK.
 * In the release library it returns MOE_ERR_UNSUPPORTED.  No counterpart on
 * the pages: a debugging aid. */
moe_status_t moe_mxfp4_check_guards(moe_mxfp4_t* h);

/* Test hook of the debug build: overwrite one byte of the i-th guard region
 * (from the host), so the detection of moe_mxfp4_check_guards can be tested
 * without any kernel writing out of bounds.  UNSUPPORTED in the release
 * library; INVALID_ARG for an i past the handle's guard regions. */
moe_status_t moe_mxfp4_test_write_guard(moe_mxfp4_t* h, int32_t i);

/* Static description of a status code. */
const char* moe_mxfp4_status_string(moe_status_t s);

/* Per-stage timing of later forwards (CUDA events on the forward's stream).
 * enable = 0 turns it off.  A forward captured into a CUDA graph while
 * profiling is on records its stage events as event-record nodes of the
 * graph, so moe_mxfp4_kernel_times then reports the last replay (also after
 * profiling is turned off again; a forward run eagerly with profiling off
 * ends the record). */
moe_status_t moe_mxfp4_set_profiling(moe_mxfp4_t* h, int32_t enable);

/* Stage names in the order moe_mxfp4_kernel_times reports them. */
#define MOE_NUM_STAGES 7
/* 0 router + top-k + softmax + grouping schedule, 1 gather into grouped rows,
 * 2 gate/up + SwiGLU, 3 H encoding (three MXFP4 terms), 4 down (weighted row
 * outputs), 5 combine of each token's k rows into y, 6 the fused decode kernel
 * (forwards of at most 16 tokens).  Synchronises;
 * writes the last profiled forward's durations in ms (0 for stages that did
 * not run) into ms[0..min(n, MOE_NUM_STAGES)). */
moe_status_t moe_mxfp4_kernel_times(moe_mxfp4_t* h, float* ms, int32_t n);
const char* moe_mxfp4_stage_name(int32_t stage);

/* Number of kernels this handle has launched since creation. */
uint64_t moe_mxfp4_launch_count(const moe_mxfp4_t* h);

/* Parameters of one expert: 3 * d_model * d_ff (three matrices, §3.2; the
 * page "OpenAI lance gpt-oss-20b" gives 3,145,728 for the GLU variant at
 * width 1024). */
int64_t moe_mxfp4_expert_param_count(const moe_mxfp4_config_t* cfg);

/* MXFP4 bytes of one expert: codes + scales = 17/32 byte per parameter
 * (4.25 bits, §4). */
int64_t moe_mxfp4_expert_weight_bytes(const moe_mxfp4_config_t* cfg);

/* Routing without any device allocation.  No counterpart on the pages: this
 * is an interface convenience, not part of the method.  Some callers cannot
 * call cudaMalloc -- code that must not synchronise the device (cudaMalloc
 * may), hosts whose device memory is owned by another allocator, or a
 * process that has no handle (moe_mxfp4_create allocates).  This call runs
 * the same router kernel as moe_mxfp4_forward (scores, top-k with ties to the
 * lower index, softmax over the selected scores, per-expert counts) with its
 * scratch in one fixed static device array inside the library
 * (MOE_ROUTE_NOALLOC_SCRATCH_BYTES on every device that loads the library,
 * held until exit).  Inputs and outputs are caller-owned device memory:
 *   x:             [T][d_model], act_dtype (MOE_DTYPE_F32 or MOE_DTYPE_BF16)
 *   w_router:      [E][d_model], act_dtype
 *   router_bias:   fp32 [E] or NULL
 *   topk_idx:      int32 [T][top_k]; topk_w: fp32 [T][top_k]
 *   expert_counts: int32 [E] or NULL
 * Limits: 1 <= T <= MOE_ROUTE_NOALLOC_MAX_TOKENS, E <= MOE_ROUTE_NOALLOC_MAX_EXPERTS,
 * 1 <= top_k <= min(8, E), d_model a positive multiple of 32 up to 16384;
 * anything larger returns MOE_ERR_UNSUPPORTED (nothing is launched).  x and
 * w_router must be 16-byte aligned, router_bias and the outputs 4-byte
 * aligned (else MOE_ERR_INVALID_ARG, checked before the device is touched).
 * The first call on a device looks up the array's device address (with that
 * device current) and sets the router kernel's shared-memory limit to the
 * value layer handles use (never lower): make that first call before any
 * stream capture.  Every call resets the counters it needs and
 * otherwise reuses the array, so calls that overlap on the GPU (different
 * streams without ordering, or several host threads) race on it.
 * Asynchronous on `stream`. */
#define MOE_ROUTE_NOALLOC_MAX_TOKENS 256
#define MOE_ROUTE_NOALLOC_MAX_EXPERTS 128
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (2304 * 1024)
moe_status_t moe_mxfp4_route_noalloc(const void* x, const void* w_router, const float* router_bias,
                                     int32_t T, int32_t d_model, int32_t n_experts, int32_t top_k,
                                     int32_t act_dtype, int32_t* topk_idx, float* topk_w,
                                     int32_t* expert_counts, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_MXFP4_H */
