/*
 * moe.h - C ABI of the B200 (sm_100a) OLMoE mixture-of-experts FFN layer.
 *
 * The layer, per token x_t (row of x, width d):
 *   h_t = W_r x_t (+ b)                      router logits over E experts
 *   p_t = softmax(h_t)                       over all E experts, in fp32
 *   S_t = the k largest p_t (ties: lower expert index), slots in descending p
 *   w_tj = p_t,S_tj                          no renormalisation
 *   y_t = sum_j w_tj * W_down,e (SiLU(W_gate,e x_t) * W_up,e x_t),  e = S_tj
 *   L_lb = E * sum_i f_i P_i,  f_i = count_i / (T k),  P_i = mean_t p_t,i
 *   L_z  = mean_t (log sum_i exp h_t,i)^2
 * Sources: "Mixture-of-experts LLMs from scratch with OLMoE", section 2 "The
 * router and the experts" (softmax then top-k, grouped dispatch, the SwiGLU
 * experts stored as stacked gate_up [E, 2f, d] and down [E, d, f]) and section 3
 * "OLMoE in PyTorch" (norm_topk_prob False); "OLMoE Guide: 64-Expert
 * Fine-Grained Open MoE Architecture", section "Router Mechanics & Loss
 * Formulations" (the load-balancing loss and the router z-loss); "OLMoE: Open
 * Mixture-of-Experts Language Models", "Pretraining architecture" (dropless
 * token choice, alpha = 0.01, beta = 0.001).
 *
 * Conventions for every entry point:
 *   - Pointers marked [device] are CUDA device pointers on the current device;
 *     [host] are host pointers. The caller owns and allocates every buffer; the
 *     library allocates no device memory. Scratch lives in the caller's
 *     workspace `ws` (moe_workspace_bytes), which must be 256-byte aligned.
 *   - All matrices are row-major and contiguous. Activations and weights have the
 *     dtype of cfg->dtype (bf16 or fp32); router weights w [T,k], router bias and
 *     losses are fp32; indices are int32.
 *   - Calls are asynchronous on `stream` and never synchronise the host, except
 *     moe_forward_host and moe_get_device_status, which say so.
 *   - Argument and shape errors are returned synchronously, before anything is
 *     launched. A failed launch returns MOE_ERR_CUDA. Invariant violations the
 *     kernels detect (an expert index out of range, a wait that timed out) are
 *     recorded in the workspace and read with moe_get_device_status.
 *   - Expert-contiguous ("permuted") buffers have moe_padded_rows(cfg) rows.
 *     Expert e's rows start at group_start[e], a multiple of MOE_ROW_ALIGN, and
 *     its count_e valid rows are followed by zero rows up to group_start[e+1].
 *   - Results are deterministic: the same inputs give bitwise-equal outputs.
 */
#ifndef MOE_B200_MOE_H_
#define MOE_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* cudaStream_t;

#define MOE_ABI_VERSION 6
#define MOE_ROW_ALIGN 128

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, misaligned pointer, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the supported set (moe_check_config) */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moe_workspace_bytes(cfg, ...) */
  MOE_ERR_CUDA = 4,                /* a CUDA call or kernel launch failed */
  MOE_ERR_DEVICE_CHECK = 5,        /* a kernel recorded a failed invariant (moe_get_device_status) */
  MOE_ERR_NO_DEVICE = 6            /* no usable sm_100 device is current */
} moe_status;

typedef enum moe_dtype { MOE_BF16 = 0, MOE_FP32 = 1 } moe_dtype;

/* Router weights. MOE_ROUTER_SOFTMAX_TOPK (OLMoE, the default): softmax over
 * all experts, the k largest probabilities are both the choice and the weights,
 * not renormalised ("Mixture-of-experts LLMs from scratch with OLMoE", sections
 * 2 and 3, norm_topk_prob False). MOE_ROUTER_RENORM: the same choice, weights
 * divided by their sum, i.e. a softmax over the k largest logits ("OLMoE Guide",
 * "Top-8 Softmax Routing Formulation"). Losses are the same in both modes. */
typedef enum moe_router_mode { MOE_ROUTER_SOFTMAX_TOPK = 0, MOE_ROUTER_RENORM = 1 } moe_router_mode;

/* Shapes and loss weights of one layer. Supported: 1 <= T <= 2^24;
 * d_model a multiple of 128 in [128, 4096] (bf16) or [128, 2048] (fp32);
 * d_ff a multiple of 128 in [128, 4096]; 1 <= top_k <= min(16, E);
 * 1 <= n_experts <= 256. alpha_lb and beta_z weight L_lb and L_z in the backward
 * objective <dy, y> + alpha_lb * L_lb + beta_z * L_z (OLMoE: 0.01 and 0.001).
 * grad_dtype is the type moe_backward writes the three weight gradients in:
 * MOE_BF16 (0, the zero-initialised default: the same type as bf16 weights) or
 * MOE_FP32 (fp32 gradients for an fp32 optimizer state; the accumulation is fp32
 * either way, so the bf16 result is the fp32 one rounded once). Ignored by the
 * forward entry points; an fp32 cfg always gets fp32 gradients. */
typedef struct moe_config {
  int64_t T;
  int32_t d_model;
  int32_t n_experts;
  int32_t top_k;
  int32_t d_ff;
  int32_t dtype; /* moe_dtype */
  float alpha_lb;
  float beta_z;
  int32_t grad_dtype; /* moe_dtype of dw_router, dw_gate_up, dw_down */
  int32_t router_mode; /* moe_router_mode */
} moe_config;

/* Human-readable name of a status code. Never NULL. */
const char* moe_status_string(int32_t status);

/* MOE_ABI_VERSION of the built library. */
int32_t moe_abi_version(void);

/* Validates the shapes of cfg. MOE_OK or MOE_ERR_UNSUPPORTED_SHAPE / _INVALID_ARG. */
moe_status moe_check_config(const moe_config* cfg);

/* Row capacity of every expert-contiguous buffer: T*k + E*(MOE_ROW_ALIGN-1),
 * rounded up to MOE_ROW_ALIGN. Returns -1 for an invalid cfg. */
int64_t moe_padded_rows(const moe_config* cfg);

/* Bytes of workspace for moe_forward/moe_route/moe_dispatch/moe_expert_* and
 * moe_combine (for_backward = 0), or for moe_forward(save_for_backward=1)
 * followed by moe_backward (for_backward = 1). 0 for an invalid cfg. */
size_t moe_workspace_bytes(const moe_config* cfg, int32_t for_backward);

/* Clears the workspace's control words (status word and completion counters).
 * Call once on a freshly allocated workspace, before its first use; the
 * kernels keep the counters at zero afterwards. Asynchronous on `stream`. */
moe_status moe_workspace_init(void* ws, cudaStream_t stream);

/* Router: logits, softmax over all experts, top-k without renormalisation,
 * per-expert counts and both losses ("Mixture-of-experts LLMs from scratch with
 * OLMoE", section 2, softmax_topk; "OLMoE Guide", "Router Mechanics & Loss
 * Formulations").
 *   x          [device] [T, d]            tokens
 *   w_router   [device] [E, d]            router weight (one row per expert)
 *   router_bias[device] [E] fp32 or NULL  additive logit offset per expert
 *   topk_idx   [device] [T, k] int32 out  chosen experts, descending probability
 *   topk_w     [device] [T, k] fp32 out   their softmax probabilities
 *   counts     [device] [E] int32 out     assignments per expert (sum = T*k)
 *   losses     [device] [2] fp32 out      {L_lb, L_z}, unscaled
 * The softmax probabilities and log-normalisers are also kept in `ws` for
 * moe_backward. */
moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                     int32_t* topk_idx, float* topk_w, int32_t* counts, float* losses, void* ws,
                     size_t ws_bytes, cudaStream_t stream);

/* moe_route without a workspace: the same routing, outputs and output buffers,
 * but its scratch is a fixed MOE_ROUTE_STATIC_SCRATCH_BYTES array inside the
 * library, so the call allocates nothing and needs no `ws`. It always runs the
 * CUDA-core router (logits summed in fp64): the same experts as moe_route under
 * the exact-logit tie rule, weights and losses equal within the agreement
 * tolerances (not bit for bit), and a slower call than moe_route's tensor-core
 * router for bf16 layers. The pages have no
 * counterpart: this is for callers that cannot provide device memory of their
 * own, such as code whose device memory is planned and owned by a host
 * framework or serving runtime, or a loop that must not call cudaMalloc because
 * it synchronises the device.
 *   - Limit: the scratch holds T * (4.5 * E + 4.5) bytes plus under 2 KB of
 *     alignment, so at E = 64 up to 7,167 tokens (the 4,096-token OLMoE layer
 *     fits); larger calls return MOE_ERR_WORKSPACE_TOO_SMALL before
 *     launching anything.
 *   - The first call on a device looks up the array's device address on that
 *     device (it must be the current device); make that first call before any
 *     stream capture. The address is kept with the context it belongs to and
 *     looked up again after a device reset or in another context.
 *   - Every device that loads the library keeps the array until the process
 *     exits. All calls share it and find the last call's contents in it; the
 *     part that must start at zero is cleared on `stream` before each launch.
 *     Calls that overlap on the GPU (different streams or host threads) race on
 *     the array and must be serialised by the caller. */
#define MOE_ROUTE_STATIC_SCRATCH_BYTES (2u << 20)
moe_status moe_route_static(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                            int32_t* topk_idx, float* topk_w, int32_t* counts, float* losses, cudaStream_t stream);

/* Dispatch: group the T*k (token, slot) pairs by expert, dropless and stable in
 * token order, and gather the token rows into expert-contiguous order
 * ("Mixture-of-experts LLMs from scratch with OLMoE", section 2, `dispatch`:
 * argsort(stable) of the flattened choices, bincount, rows = order // k).
 *   topk_idx    [device] [T, k] int32     expert choices (entries in [0, E))
 *   x           [device] [T, d]           tokens
 *   offsets     [device] [E+1] int32 out  exclusive prefix sum of per-expert counts
 *   perm        [device] [T*k] int32 out  pair id t*k+j at each sorted position
 *   inv_perm    [device] [T*k] int32 out  padded row of pair t*k+j in x_perm
 *   group_start [device] [E+1] int32 out  first padded row of each expert
 *   x_perm      [device] [moe_padded_rows, d] out  gathered rows, pad rows zero
 * An out-of-range expert index is recorded as a device check failure. */
moe_status moe_dispatch(const moe_config* cfg, const int32_t* topk_idx, const void* x, int32_t* offsets,
                        int32_t* perm, int32_t* inv_perm, int32_t* group_start, void* x_perm, void* ws,
                        size_t ws_bytes, cudaStream_t stream);

/* Gate/up grouped GEMM with the SwiGLU epilogue, for every expert group:
 * h[r] = SiLU(W_gate,e x_perm[r]) * (W_up,e x_perm[r]) ("OLMoE Guide",
 * "Top-8 Softmax Routing Formulation", the SwiGLU expert).
 *   x_perm      [device] [P, d]   P = moe_padded_rows(cfg)
 *   group_start [device] [E+1]    from moe_dispatch
 *   offsets     [device] [E+1]    from moe_dispatch (valid rows per expert)
 *   w_gate_up   [device] [E, 2f, d]  gate rows then up rows per expert
 *   h           [device] [P, f] out, pad rows zero
 *   preact      [device] [P, 2f] fp32 out or NULL: the gate and up
 *                pre-activations, unrounded (moe_forward keeps them for the
 *                backward's SwiGLU derivative, which is no contraction, so they
 *                are not rounded to the layer dtype). */
moe_status moe_expert_gate_up(const moe_config* cfg, const void* x_perm, const int32_t* group_start,
                              const int32_t* offsets, const void* w_gate_up, void* h, void* preact,
                              void* ws, size_t ws_bytes, cudaStream_t stream);

/* Down-projection grouped GEMM: o_perm[r] = W_down,e h[r].
 *   h      [device] [P, f];  w_down [device] [E, d, f];  o_perm [device] [P, d] out. */
moe_status moe_expert_down(const moe_config* cfg, const void* h, const int32_t* group_start,
                           const int32_t* offsets, const void* w_down, void* o_perm, void* ws,
                           size_t ws_bytes, cudaStream_t stream);

/* Both expert GEMMs (moe_expert_gate_up then moe_expert_down); h is caller scratch. */
moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* group_start,
                          const int32_t* offsets, const void* w_gate_up, const void* w_down, void* h,
                          void* o_perm, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Combine: y_t = sum_{j=0..k-1} topk_w[t,j] * o_perm[inv_perm[t*k+j]], summed in
 * fp32 in slot order and rounded once ("OLMoE Guide", "Top-8 Softmax Routing
 * Formulation": y = sum_i P_i Expert_i(x)). A gather, so no atomics.
 *   o_perm [device] [P, d];  inv_perm [device] [T*k];  topk_w [device] [T, k] fp32;
 *   y [device] [T, d] out. */
moe_status moe_combine(const moe_config* cfg, const void* o_perm, const int32_t* inv_perm, const float* topk_w,
                       void* y, cudaStream_t stream);

/* The whole layer: moe_route, moe_dispatch, the two expert GEMMs, moe_combine.
 *   y        [device] [T, d] out
 *   losses   [device] [2] fp32 out {L_lb, L_z}
 *   topk_idx [device] [T, k] int32 out or NULL;  topk_w [device] [T, k] fp32 out or NULL
 *   save_for_backward: 1 keeps what moe_backward needs in ws (which must then be
 *   moe_workspace_bytes(cfg, 1) bytes and stay untouched until moe_backward);
 *   the expert outputs and the gate/up pre-activations are then kept in fp32
 *   (y is summed from the fp32 expert outputs), since no contraction reads
 *   them: only h, do = w dy and [da; db] enter the GEMMs in the layer dtype. */
moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                       const void* w_gate_up, const void* w_down, void* y, float* losses, int32_t* topk_idx,
                       float* topk_w, int32_t save_for_backward, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* moe_forward for a decode-sized batch as one kernel: routing, both expert
 * projections and the combine in a single persistent cooperative launch (one
 * CTA per SM, two grid-wide barriers), reading each touched expert's weights
 * once ("Mixture-of-experts LLMs from scratch with OLMoE", section 6: at a batch
 * of one token the layer reads only the chosen experts). The router logits are
 * summed in fp64 from exact products, so the choice is the exact one (equal
 * logits: the lower expert index). Same arguments and results as moe_forward
 * without save_for_backward (counts are not written). moe_forward takes this
 * path by itself for T <= 4 when nothing is saved for the backward (beyond
 * that the layered tensor-core path is faster), and moe_stack_forward(_trace)
 * runs each layer of such a batch as one launch of it with the RMSNorm and the
 * residual add fused.
 * Supported: bf16, T <= 8, E <= 64, d_ff <= 2 d_model, and
 * max(T*d, T*k*f)*2 + 8*d bytes at most 192 KiB (the staged rows and two
 * weight stages in shared memory); otherwise MOE_ERR_UNSUPPORTED_SHAPE. The
 * kernel does nothing when the workspace status word is already set (see
 * moe_get_device_status). */
moe_status moe_forward_decode(const moe_config* cfg, const void* x, const void* w_router, const float* router_bias,
                              const void* w_gate_up, const void* w_down, void* y, float* losses, int32_t* topk_idx,
                              float* topk_w, void* ws, size_t ws_bytes, cudaStream_t stream);

/* moe_forward on host buffers, for callers whose tokens live in host memory:
 * copies x_host [host] [T, d] to the device (inside ws), runs moe_forward with
 * the device-resident weights, copies y back to y_host [host] [T, d] and the two
 * losses to losses_host [host] [2], then synchronises `stream`. Pinned host
 * memory makes the copies asynchronous DMA; pageable memory also works. */
moe_status moe_forward_host(const moe_config* cfg, const void* x_host, const void* w_router,
                            const float* router_bias, const void* w_gate_up, const void* w_down, void* y_host,
                            float* losses_host, void* ws, size_t ws_bytes, cudaStream_t stream);

/* moe_forward_host without the final synchronisation: the copy of x_host in,
 * the layer and the copies of y and the losses out are queued on `stream` and
 * the call returns; y_host and losses_host hold the results once that work has
 * completed (synchronise the stream, or wait on an event recorded after the
 * call). x_host must stay unchanged and y_host unread until then. With pinned
 * host buffers the copies are asynchronous DMA, so a caller that keeps two
 * calls in flight on two streams, each with its own workspace and output
 * buffer, overlaps one call's host transfers with the other's kernels. */
moe_status moe_forward_host_async(const moe_config* cfg, const void* x_host, const void* w_router,
                                  const float* router_bias, const void* w_gate_up, const void* w_down, void* y_host,
                                  float* losses_host, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Backward of <dy, y> + alpha_lb * L_lb + beta_z * L_z for the forward saved in
 * ws (same cfg, inputs and weights). No gradient flows through the expert choice
 * or through the counts f_i.
 *   dy [device] [T, d];  dx [device] [T, d] out;  dw_router [device] [E, d] out;
 *   dw_gate_up [device] [E, 2f, d] out;  dw_down [device] [E, d, f] out.
 * dx has the input dtype; the weight gradients have cfg->grad_dtype.
 * Weight gradients are overwritten, not accumulated. bf16 only: an fp32 cfg
 * returns MOE_ERR_UNSUPPORTED_SHAPE (its GEMMs would need MN-major tf32 operands). */
moe_status moe_backward(const moe_config* cfg, const void* dy, const void* x, const void* w_router,
                        const void* w_gate_up, const void* w_down, void* dx, void* dw_router, void* dw_gate_up,
                        void* dw_down, void* ws, size_t ws_bytes, cudaStream_t stream);

/* RMSNorm of the fp32 residual stream into the layer input dtype:
 * out_t = resid_t / sqrt(mean(resid_t^2) + eps) * weight ("Mixture-of-experts
 * LLMs from scratch with OLMoE", section 3, RMSNorm; weight may be NULL = ones).
 *   resid [device] [T, d] fp32;  weight [device] [d] fp32 or NULL;  out [device] [T, d]. */
moe_status moe_rmsnorm(const moe_config* cfg, const float* resid, const float* weight, float eps, void* out,
                       cudaStream_t stream);

/* Combine added into an fp32 residual stream: resid_t += sum_j w_tj * o_perm[...]
 * (section 3's Block: x + mlp(norm(x)).float()). Same arguments as moe_combine. */
moe_status moe_combine_residual(const moe_config* cfg, const void* o_perm, const int32_t* inv_perm,
                                const float* topk_w, float* resid, cudaStream_t stream);

/* A stack of n_layers MoE blocks on an fp32 residual stream,
 * resid <- resid + MoE_l(RMSNorm(resid)) for l = 0..n_layers-1 (pre-norm with unit
 * weight, eps 1e-5). Weight arrays hold one device pointer per layer, [host]
 * arrays of [device] pointers; router_biases may be NULL or hold NULL entries.
 *   resid [device] [T, d] fp32 in/out. */
moe_status moe_stack_forward(const moe_config* cfg, int32_t n_layers, const void* const* w_router,
                             const float* const* router_biases, const void* const* w_gate_up,
                             const void* const* w_down, float* resid, void* ws, size_t ws_bytes,
                             cudaStream_t stream);

/* moe_stack_forward that also exports, per layer, what the router did ("Mixture-
 * of-experts LLMs from scratch with OLMoE", section 3 MoE.forward's routing
 * trace and section 6's per-layer expert usage). Each output may be NULL:
 *   counts    [device] [n_layers, E] int32: rows routed to each expert;
 *   losses    [device] [n_layers, 2] fp32: L_lb and L_z of each layer;
 *   topk_idx  [device] [n_layers, T, k] int32: the experts each token chose, in
 *             slot order (descending probability).
 * The residual stream is bit-identical to moe_stack_forward's. */
moe_status moe_stack_forward_trace(const moe_config* cfg, int32_t n_layers, const void* const* w_router,
                                   const float* const* router_biases, const void* const* w_gate_up,
                                   const void* const* w_down, float* resid, int32_t* counts, float* losses,
                                   int32_t* topk_idx, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Expert-choice routing ("OLMoE: Open Mixture-of-Experts Language Models",
 * section 4.1.4 "Expert Choice vs. Token Choice": the experts choose the tokens;
 * the pages give no formula, so this is its plain reading). The router
 * probabilities are token choice's, p = softmax over experts of W_r x (+ bias);
 * expert e takes the C tokens with the largest p[t, e] (equal values: the lower
 * token index) as its rows, in ascending token order, each weighted by p[t, e];
 * a token sums its experts' outputs in ascending expert order, in fp32, rounded
 * once, and is zero when no expert took it. There is no load-balancing loss
 * (losses[0] = 0); losses[1] is the z-loss, as in token choice.
 * Supported for bf16 layers with E <= 64 and router_mode 0; other configs return
 * MOE_ERR_UNSUPPORTED_SHAPE. `capacity` is C: 0 takes the default
 * moe_expert_choice_capacity(cfg); otherwise 1 <= C <= T and the E groups of C
 * rows, each padded to MOE_ROW_ALIGN, must fit in moe_padded_rows(cfg) rows
 * (always true for the default), else MOE_ERR_INVALID_ARG. The workspace is
 * moe_workspace_bytes(cfg, 0) bytes; forward only (no backward). */

/* The default capacity ceil(T * k / E), capped at T: the experts then process
 * about T * k rows, the expert work of top-k token choice. -1 for a bad cfg. */
int64_t moe_expert_choice_capacity(const moe_config* cfg);

/* Routing only.
 *   x, w_router, router_bias as in moe_route
 *   sel    [device] [E, C] int32 out   chosen tokens of each expert, ascending
 *   gates  [device] [E, C] fp32 out    their probabilities p[sel, e]
 *   probs  [device] [T, E] fp32 out or NULL: the softmax probabilities
 *   counts [device] [E] int32 out or NULL: rows per expert (all C)
 *   losses [device] [2] fp32 out or NULL: {0, L_z} */
moe_status moe_route_expert_choice(const moe_config* cfg, int64_t capacity, const void* x, const void* w_router,
                                   const float* router_bias, int32_t* sel, float* gates, float* probs,
                                   int32_t* counts, float* losses, void* ws, size_t ws_bytes, cudaStream_t stream);

/* The whole layer under expert choice: route, gather each expert's C rows, the
 * two grouped expert GEMMs (the token-choice kernels), and the combine.
 *   y      [device] [T, d] out
 *   losses [device] [2] fp32 out or NULL: {0, L_z}
 *   sel    [device] [E, C] int32 out or NULL;  gates [device] [E, C] fp32 out or NULL
 * moe_set_stage_events marks the same six points as for moe_forward. */
moe_status moe_forward_expert_choice(const moe_config* cfg, int64_t capacity, const void* x, const void* w_router,
                                     const float* router_bias, const void* w_gate_up, const void* w_down, void* y,
                                     float* losses, int32_t* sel, float* gates, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);

/* Stage timing for profiling. When `events` is non-NULL, the next call of
 * moe_forward records events[0] on its stream before the router and events[i]
 * after stage i (1 router, 2 dispatch, 3 gate/up GEMM, 4 down GEMM, 5 combine;
 * on the one-kernel decode path all five follow that kernel), then forgets them; `events` holds MOE_STAGE_EVENTS cudaEvent_t handles owned by
 * the caller. Per host thread. */
#define MOE_STAGE_EVENTS 6
moe_status moe_set_stage_events(void* const* events);

/* Reads the workspace status word (0 = no failure recorded) into *code and clears
 * it, together with the workspace's completion counters (so a workspace whose
 * kernel gave up part-way can be used again). Synchronises `stream`. Returns
 * MOE_ERR_DEVICE_CHECK when *code != 0. */
moe_status moe_get_device_status(void* ws, int32_t* code, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H_ */
