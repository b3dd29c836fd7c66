/*
 * lmoe.h -- C ABI of the B200 (sm_100a) LatentMoE layer forward library.
 *
 * The library computes, for every token row x of width d (rows independent):
 *
 *   r   = sigmoid(W_r x)                       router scores at model width
 *   T_k = TopK(r + b, k)                       the bias changes selection only
 *   p_i = r_i / sum_{j in T_k} r_j             mixture weights from raw scores
 *   z   = W_down x                             latent width l = d / alpha
 *   u   = sum_{i in T_k} p_i D_i act(G_i z, U_i z)   routed experts l -> f -> l
 *   y   = S_1(x) + S_2(x) + W_up RMSNorm(u)    two shared experts at width d
 *
 * as defined by the "Stable LatentMoE" problem (TensorTonic, Kimi K3 set:
 * equations for r, T_k(x), p_i, u and y; Requirements and Constraints), with
 * the routed/shared split of the cooking-agi page "LatentMoE: must experts be
 * as wide as the backbone?" (section "Which part becomes narrower?") and the
 * variant arithmetic of the PyPI latent_moe README (section "Latent-MoE").
 * act is SwiGLU, silu(g) * v, or the capped SiTU-GLU gate
 * cg tanh(g/cg) sigmoid(g) * cu tanh(v/cu).
 *
 * Conventions for every entry point:
 *  - Every call returns an lmoe_status; nothing throws, nothing aborts.
 *    On failure lmoe_last_error() returns a message for the calling thread.
 *  - "device" pointers are CUDA global-memory addresses on the device that is
 *    current when lmoe_create was called; "host" pointers are CPU memory.
 *  - Matrices are dense row-major, "out x in" (W @ x): the layouts below.
 *  - Streams are passed as void* holding a cudaStream_t (NULL = legacy
 *    default stream).  Calls that take a stream only enqueue work on it and
 *    return without synchronising, unless stated otherwise.
 *  - Floating tensors use the configuration's dtype (fp32 or bf16, "the token
 *    dtype"), except W_r and b, which are always fp32.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LMOE_API __attribute__((visibility("default")))
#else
#define LMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LMOE_OK = 0,
    LMOE_ERR_INVALID_ARG = 1,     /* a pointer, size or configuration value is invalid */
    LMOE_ERR_UNSUPPORTED = 2,     /* valid, but outside what the kernels handle (alignment) */
    LMOE_ERR_OOM = 3,             /* cudaMalloc for handle-owned memory failed */
    LMOE_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
    LMOE_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait gave up (see lmoe_check_device) */
    LMOE_ERR_WORKSPACE = 6        /* the workspace passed in is too small */
} lmoe_status;

typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1 } lmoe_dtype;
typedef enum { LMOE_ACT_SWIGLU = 0, LMOE_ACT_SITU = 1 } lmoe_act;

/* Layer configuration.
 *  d         model width                  l      latent width (l <= d)
 *  f         routed expert intermediate   E      routed experts
 *  k         selected experts, 1 <= k <= E ("Selected count is positive and
 *            no larger than the routed expert count", Stable LatentMoE,
 *            Constraints)
 *  f_shared  shared expert intermediate   n_shared  must be 2 ("Exactly two
 *            shared experts are supplied", Stable LatentMoE, Constraints)
 *  eps       RMSNorm epsilon, inside the square root; the norm has unit gain
 *  dtype     lmoe_dtype of tokens, outputs and all weights except W_r and b
 *  act       lmoe_act; gate_cap / up_cap are the SiTU caps (ignored for SwiGLU)
 *  gemm      0 = tensor cores (tcgen05) for bf16, CUDA cores for fp32;
 *            1 = CUDA cores for every GEMM (a slower cross-check path)
 *  standard  0 = LatentMoE (above); 1 = the standard MoE it is compared with
 *            (cooking-agi LatentMoE page: a standard MoE routes and computes its
 *            experts at the model width; "Does the saving pay for more
 *            experts?" counts no projections when the latent width equals the
 *            width): requires l = d, skips W_down, RMSNorm and W_up, so
 *            y = S1(x) + S2(x) + u with u = sum_j p_j E_j(x) at width d.  The
 *            router, selection and shared experts are unchanged.
 */
typedef struct {
    int32_t d, l, f, E, k, f_shared, n_shared;
    float eps;
    int32_t dtype;
    int32_t act;
    float gate_cap, up_cap;
    int32_t gemm;
    int32_t standard;
} lmoe_config;

/* Weights, all device pointers, read only during lmoe_create:
 *  W_r    [E, d]  fp32       router projection
 *  b      [E]     fp32       selection bias
 *  W_down [l, d]             shared down-projection (unused, may be NULL, when standard)
 *  W_up   [d, l]             up-projection (unused, may be NULL, when standard)
 *  G, U   [E, f, l]          routed gate / up projections
 *  D      [E, l, f]          routed down projections
 *  Gs, Us [2, f_shared, d]   shared gate / up projections
 *  Ds     [2, d, f_shared]   shared down projections
 */
typedef struct {
    const float *W_r;
    const float *b;
    const void *W_down, *W_up;
    const void *G, *U, *D;
    const void *Gs, *Us, *Ds;
} lmoe_weights;

typedef struct lmoe_handle lmoe_handle;

/* Fill *out from the base-MoE description of the PyPI latent_moe README
 * (LatentMoEConfig: d, m, n_experts N, top_k K, alpha, n_shared, variant) and
 * its variant list: l = d / alpha, E = alpha * N routed experts; "eff" keeps
 * k = K, "acc" takes k = alpha * K; f = f_shared = m.  "std" is the base
 * standard MoE itself (l = d, E = N, k = K, standard = 1).  eps = 1e-6, bf16,
 * SwiGLU, tensor cores.  INVALID_ARG if a value is not positive, alpha does
 * not divide d, the variant is not "acc", "eff" or "std", or k > E. */
LMOE_API lmoe_status lmoe_config_from_base(int32_t d, int32_t m, int32_t N, int32_t K, int32_t alpha,
                                  int32_t n_shared, const char *variant, lmoe_config *out);

/* Validate cfg, allocate handle-owned device memory on the current device and
 * repack the weights into it (gate/up rows interleaved in blocks, the shared
 * down projections and W_up concatenated, the router split for the tensor
 * cores).  Work is enqueued on `stream`, which is synchronised before return,
 * so the caller may free its weight copies afterwards.
 * INVALID_ARG: null pointer, non-positive size, l > d, k < 1 or k > E,
 *              n_shared != 2, eps < 0, unknown dtype/act, standard not 0/1,
 *              standard with l != d.
 * UNSUPPORTED: d, l, f or f_shared not a multiple of 64, E > 1024, k > 64,
 *              l > 8192, or (bf16
 *              tensor-core path) f or f_shared not a multiple of 128.
 * OOM / CUDA on allocation or launch failure (nothing is leaked). */
LMOE_API lmoe_status lmoe_create(const lmoe_config *cfg, const lmoe_weights *w, void *stream, lmoe_handle **out);

/* Device workspace bytes that lmoe_forward needs for T tokens (0 for T = 0). */
LMOE_API lmoe_status lmoe_workspace_size(const lmoe_handle *h, int64_t T, size_t *bytes);

/* The layer forward ("Stable LatentMoE", equations for r, T_k, p_i, u, y, and
 * its return contract) for T tokens, enqueued on `stream`:
 *  x                        [T, d] device, token dtype (input)
 *  output                   [T, d] device, token dtype
 *  selected_experts         [T, k] device int32, per row in selection order
 *                           (biased score descending, equal scores to the
 *                           lower expert index)
 *  mixture_weights          [T, k] device, token dtype, aligned with
 *                           selected_experts; each row sums to one
 *  latent_routed_aggregate  [T, l] device, token dtype: u before RMSNorm
 *  workspace                device scratch of >= lmoe_workspace_size(T) bytes,
 *                           256-byte aligned; its contents on entry are
 *                           irrelevant and it is clobbered
 * Outputs must not overlap x, each other or the workspace.  T = 0 is a no-op.
 * Inputs must be finite.  Overlapping calls on one handle are allowed; calls
 * that share a workspace must be ordered on one stream.
 * On the tensor-core path, when no stage events are set, the down-projection
 * and the shared experts' gate/up GEMM run on a stream owned by the handle,
 * forked from `stream` at the start of the call; `stream` waits for z before
 * the permute and for the shared hidden before the routed gate/up GEMM.  The
 * call as a whole stays ordered on `stream` and can be captured into a CUDA
 * graph from it; while such a capture is open, the handle's other forwards
 * belong in that capture too.
 * INVALID_ARG for null pointers (T > 0) or T < 0; WORKSPACE if ws_bytes is too
 * small or misaligned; CUDA if a launch fails. */
LMOE_API lmoe_status lmoe_forward(lmoe_handle *h, const void *x, int64_t T, void *output, int32_t *selected_experts,
                         void *mixture_weights, void *latent_routed_aggregate, void *workspace,
                         size_t ws_bytes, void *stream);

/* Device workspace bytes for lmoe_forward_host with T tokens: staging for x
 * and the four outputs plus the lmoe_forward workspace. */
LMOE_API lmoe_status lmoe_host_workspace_size(const lmoe_handle *h, int64_t T, size_t *bytes);

/* lmoe_forward on HOST buffers (same shapes and dtypes as lmoe_forward; use
 * pinned memory for asynchronous copies): copies x to the device, runs the
 * forward, and copies the four outputs back.  The host outputs are valid once
 * `stream` has been synchronised.  From 2 x max(2048, 192 E / k) tokens on, the
 * call cuts the batch into up to 8 chunks of whole rows and pipelines them:
 * chunk j's input crosses on a copy stream the handle owns while chunk j - 1
 * computes on `stream`, and its outputs return on a second one while chunk
 * j + 1 computes; `stream` waits for the last copy.  Rows are independent, so
 * every row's result is that of lmoe_forward on the chunk that holds it.  The
 * device status word (lmoe_check_device) covers the whole call.
 * Errors as lmoe_forward. */
LMOE_API lmoe_status lmoe_forward_host(lmoe_handle *h, const void *x_host, int64_t T, void *output_host,
                              int32_t *selected_experts_host, void *mixture_weights_host,
                              void *latent_routed_aggregate_host, void *workspace, size_t ws_bytes,
                              void *stream);

/* Replace the selection bias with b [E] (device fp32), enqueued on `stream`.
 * The bias changes only which experts are selected ("Stable LatentMoE": "The
 * bias changes selection only"; the cooking-agi page, section "Quantile
 * Balancing", updates it between steps and freezes it for inference). */
LMOE_API lmoe_status lmoe_set_bias(lmoe_handle *h, const float *b, void *stream);

/* Quantile-Balancing statistics (cooking-agi LatentMoE page, section
 * "Quantile Balancing: measure now, use next step": the current (k+1)-th biased
 * score is the cutoff, expert-wise margins against it estimate the next bias,
 * which takes effect the next step; global quantiles come from histograms).
 *
 * lmoe_qb_histogram: after an lmoe_forward of T tokens with `workspace` on the
 * same stream, ADD the batch's margin histogram to hist [E, bins] (device
 * int32, row-major, zeroed by the caller before the first batch; several
 * batches, or an all-reduce over ranks, accumulate into it).  The margin of
 * token t for expert e is m = (r[t, e] + b[e]) - cutoff[t] with r the router
 * scores and cutoff[t] the token's (k+1)-th biased score (workspace region 11);
 * its bin is computed in fp32 as x = (m - lo) * (bins / (hi - lo)): bin 0 if
 * x < 0, bins - 1 if x >= bins, floor(x) otherwise.  Reads workspace regions 0
 * and 11, which the next forward on that workspace overwrites.  workspace
 * NULL reads the built-in area of lmoe_forward_noalloc (handle's device current).
 * INVALID_ARG: NULL handle or hist, T < 0, bins outside [1, 2^20], lo or hi not
 * finite, hi <= lo.  T = 0 adds nothing. */
LMOE_API lmoe_status lmoe_qb_histogram(const lmoe_handle *h, const void *workspace, int64_t T, int32_t bins,
                                       float lo, float hi, int32_t *hist, void *stream);

/* lmoe_qb_bias_update: the next step's bias from an accumulated histogram, into
 * bias_out [E] (device fp32; may not alias the handle's bias): per expert, the
 * target-th largest margin (0-based; the page's fixed-cutoff rule takes it from
 * sorted margins) is estimated from the histogram -- scanning bins from the
 * top with C the count above bin j, it lies in the bin with C <= target <
 * C + h_j, placed at that bin's upper edge minus (target - C + 1/2) / h_j of the
 * bin width -- and bias_out[e] = b[e] - q_e (lo when the expert has no more
 * than `target` margins).  Apply it with lmoe_set_bias before the next step.
 * target is normally the batch's slots per expert, T k / E.
 * INVALID_ARG: NULL pointer, bins outside [1, 2^20], lo or hi not finite,
 * hi <= lo, target < 0. */
LMOE_API lmoe_status lmoe_qb_bias_update(const lmoe_handle *h, const int32_t *hist, int32_t bins, float lo,
                                         float hi, int64_t target, float *bias_out, void *stream);

/* Stages of one forward, in launch order (for lmoe_set_stage_events):
 *  0 router GEMM, 1 top-k, 2 counting-sort scan, 3 dispatch, 4 down-projection
 *  GEMM, 5 copy of z to the expert-sorted slot rows, 6 routed gate/up GEMM,
 *  7 routed down GEMM + weighting, 8 combine + RMSNorm, 9 shared gate/up GEMM,
 *  10 final GEMM (shared down + up-projection). */
#define LMOE_NUM_STAGES 11

/* Ask subsequent lmoe_forward calls on this handle to record events[i] (each
 * a cudaEvent_t created by the caller) on the forward's stream right before
 * stage i, and events[LMOE_NUM_STAGES] after the last stage, so that the
 * caller can time every kernel with cudaEventElapsedTime.  n must be
 * LMOE_NUM_STAGES + 1, or 0 with events NULL to stop recording.  The array is
 * read at each forward, not copied: the caller keeps it alive.  While events
 * are set, every stage runs on the forward's stream in the order listed above
 * (no side stream), so that each interval times one stage. */
LMOE_API lmoe_status lmoe_set_stage_events(lmoe_handle *h, void *const *events, int32_t n);

/* Test hooks for failure detection (no counterpart in the pages):
 *  LMOE_INJECT_STALL_NEXT_GEMM  the next tensor-core GEMM this process launches
 *      makes its MMA warp wait on a barrier that nothing signals.  The wait is
 *      bounded (about 2 s of SM cycles): it gives up, the kernel records the
 *      failure in the forward's status word, drains and returns, and
 *      lmoe_check_device then reports LMOE_ERR_DEVICE_TIMEOUT.  Nothing faults
 *      or hangs; the context stays usable.  (arg ignored.)
 *  LMOE_INJECT_FAIL_ALLOC  the arg-th device allocation (1-based) of the next
 *      lmoe_create fails as if cudaMalloc had: lmoe_create returns LMOE_ERR_OOM
 *      and frees what it had allocated.
 * INVALID_ARG for an unknown `what` or arg < 1 with LMOE_INJECT_FAIL_ALLOC. */
#define LMOE_INJECT_STALL_NEXT_GEMM 1
#define LMOE_INJECT_FAIL_ALLOC 2
LMOE_API lmoe_status lmoe_debug_inject(int32_t what, int32_t arg);

/* Number of kernels one lmoe_forward of T tokens launches (its two memsets,
 * of the status word and of the per-block expert counts, are not counted). */
LMOE_API lmoe_status lmoe_launch_count(const lmoe_handle *h, int64_t T, int32_t *launches);

/* Byte offset and size of one intermediate inside the forward workspace, so
 * tests can read stage results after a forward on the same stream.
 * region: 0 router scores r [T, E] fp32; 1 mixture weights fp32 [T, k];
 * 2 per-expert counts [E] int32; 3 expert offsets [E+1] int32;
 * 4 slot index of (t, j) [T, k] int32; 5 token of each permuted slot [T*k]
 * int32; 6 latent rows z [T, l] (0 bytes in the standard form); 7 routed
 * hidden H [T*k, f] (slot order); 8 p-weighted expert outputs [T*k, l] (token
 * dtype); 9 [shared hidden | RMSNorm(u)] [T, 2 f_shared + l] (no RMSNorm
 * columns in the standard form); 10 device status word (int32); 11 Quantile-Balancing
 * cutoff [T] fp32 (each token's (k+1)-th biased score, -inf when k = E);
 * 12 slot rows [T*k, l] (z of each slot's token, expert-sorted; 0 bytes when
 * the routed GEMVs of a few tokens read z through the slot -> token map).
 * INVALID_ARG for an unknown region. */
LMOE_API lmoe_status lmoe_workspace_region(const lmoe_handle *h, int64_t T, int32_t region, size_t *offset,
                                  size_t *bytes);

/* Synchronise `stream`, then read and clear the device status word that the
 * kernels of the last forward on this workspace wrote: LMOE_OK, or
 * LMOE_ERR_DEVICE_TIMEOUT if a bounded wait gave up (its outputs are then
 * invalid).  `workspace` is the one passed to lmoe_forward, or NULL for the
 * built-in area of lmoe_forward_noalloc (the handle's device must then be
 * current; INVALID_ARG otherwise). */
LMOE_API lmoe_status lmoe_check_device(lmoe_handle *h, int64_t T, void *workspace, void *stream);

/* lmoe_check_device for the workspace of an lmoe_forward_host call of T
 * tokens (its status word covers every chunk of the call). */
LMOE_API lmoe_status lmoe_check_device_host(lmoe_handle *h, int64_t T, void *workspace, void *stream);

/* Size of the scratch area built into the library for lmoe_forward_noalloc. */
#define LMOE_NOALLOC_WORKSPACE_BYTES ((size_t)64 << 20)

/* lmoe_forward without a caller workspace, for callers that cannot allocate
 * device memory where they run the layer (inside a stream capture that must
 * not allocate, under an allocator owned by another runtime, or on a path
 * that must not take allocator locks).  There is no counterpart in the
 * LatentMoE pages: this is a deployment convenience of this library.
 * Arguments and outputs are those of lmoe_forward minus the workspace; the
 * scratch is a fixed 64 MiB device array inside the library
 * (LMOE_NOALLOC_WORKSPACE_BYTES), which every GPU that loads the library holds
 * until the process exits.  Nothing is allocated by the call.
 *  - If lmoe_workspace_size(h, T) exceeds the area, it returns
 *    LMOE_ERR_WORKSPACE and launches nothing (the area covers, for example,
 *    up to 132 tokens of a d = 7168, l = 1792, f = 2048, k = 32, E = 384
 *    layer on a 148-SM B200).
 *  - The first call on a device looks up the area's device address with that
 *    device current; make it before any stream capture.
 *  - All calls on a device share the area and find the previous call's data
 *    in it (the forward resets what must start at zero itself).  Calls that
 *    overlap on the GPU race on it: order them on one stream.
 *  - The device the handle was created on must be current: INVALID_ARG
 *    otherwise.
 *  - lmoe_check_device (and lmoe_qb_histogram) with workspace NULL read this
 *    area: the status word of the last call, LMOE_ERR_DEVICE_TIMEOUT if one of
 *    its bounded waits gave up.
 * Errors as lmoe_forward. */
LMOE_API lmoe_status lmoe_forward_noalloc(lmoe_handle *h, const void *x, int64_t T, void *output,
                                          int32_t *selected_experts, void *mixture_weights,
                                          void *latent_routed_aggregate, void *stream);

/* Message for the last failure on the calling thread ("" if none). */
LMOE_API const char *lmoe_last_error(void);

/* Free the handle and its device memory (after pending work on it is done).
 * NULL is ignored. */
LMOE_API void lmoe_destroy(lmoe_handle *h);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H */
