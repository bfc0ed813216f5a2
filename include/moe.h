/*
 * moe.h - C ABI of a single-GPU Mixture-of-Experts layer (forward and backward) for B200
 * (sm_100a).
 *
 * The layer is the expert-parallel MoE layer of the tutorial "第4章 分布式训练" (MoE distributed
 * training), section "专家并行", part 二 (the four-step workflow table): a replicated router
 * gates each token (step 1), tokens move to the experts they were routed to (step 2: here an
 * in-HBM permutation into expert-contiguous buffers, the payload an all-to-all would ship),
 * each expert runs its FFN on the tokens it received (step 3), and the results return to token
 * order (step 4).  The backward pass follows section "专家并行与数据并行的结合", part 三.3
 * (gradients routed back to the experts; expert weight gradients computed locally).  The
 * problem statement (tokens, experts, top-k, expert capacity) is that of section
 * "All-to-All 通信模式", part 二 and of the Piper digest's resource model ("方法论" 1).
 *
 * Notation: T tokens, d hidden size, E routed experts, k experts per token, F = d_ff expert
 * inner size, S = n_shared always-on shared experts, E_tot = E + S, C expert capacity.
 *
 * Conventions for every entry point
 *  - All pointers are DEVICE pointers on the current CUDA device unless stated otherwise, and
 *    must be 16-byte aligned (MOE_ERR_MISALIGNED otherwise).  The caller owns every buffer;
 *    the library never allocates, frees or synchronises (except moe_read_status).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and returns
 *    without waiting.  Arguments are validated on the host before anything is enqueued; a bad
 *    argument returns an error and enqueues nothing.  A failed launch returns MOE_ERR_CUDA.
 *  - Element types: dtype MOE_DTYPE_F32 -> every activation/weight buffer is float;
 *    MOE_DTYPE_BF16 -> activations and weights are bf16 (uint16 bit patterns).  Logits, gate
 *    weights, bias and weight gradients are always float.  Accumulation is always float.
 *  - Layouts are row-major:  x, y, dx, dy [T, d];  Wg [E, d];  bias [E];
 *    W1, W3 [E_tot, F, d];  W2 [E_tot, d, F] (experts 0..E-1 routed, E..E_tot-1 shared);
 *    logits [T, E];  topk_idx, topk_w, slot [T, k].
 *  - Dispatched rows: one row space of R rows (see moe_layout_t).  Rows [s*T_pad, s*T_pad + T)
 *    belong to shared expert s (T_pad = T rounded up to 128); routed expert e owns rows
 *    [offsets[e], offsets[e+1]), its kept assignments first (in token order), then zero rows
 *    up to a multiple of 128.  Buffers indexed by this row space: Xd, O [R, d]; Gu, Gv, H [R, F].
 *  - Grad outputs are overwritten, never accumulated.
 *  - Calls are stream-ordered; concurrent calls on different streams need different scratch.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, non-positive size, k > E, ... */
  MOE_ERR_UNSUPPORTED = 2,         /* valid but outside this build's limits (see moe_config_t) */
  MOE_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4, /* the library's fixed scratch is too small (moe_dispatch_noalloc) */
  MOE_ERR_CUDA = 5,                /* a CUDA launch or runtime call failed */
  MOE_ERR_DEVICE_TIMEOUT = 6       /* a bounded device-side wait gave up (moe_read_status) */
} moe_status;

#define MOE_DROPLESS 2147483647 /* capacity value meaning "no capacity limit" */
#define MOE_ACT_GELU 0          /* GELU, erf form: u * Phi(u) */
#define MOE_ACT_SWIGLU 1        /* silu(x W1^T) * (x W3^T) */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

/* Limits of this build: 1 <= k <= min(E, 8); 1 <= E <= 256; 0 <= S <= 8; d % 8 == 0 and
 * F % 8 == 0 (bf16) or d % 4 == 0 and F % 4 == 0 (fp32); T <= 2^24.  The bf16 path runs its
 * expert GEMMs on tcgen05 tensor cores when d % 64 == 0 and F % 64 == 0, else on CUDA cores. */
typedef struct {
  int32_t T, d, E, k, d_ff, n_shared;
  int32_t act;             /* MOE_ACT_GELU | MOE_ACT_SWIGLU */
  int32_t gate_norm;       /* 0: softmax over all E logits; 1: softmax over the k chosen logits */
  float capacity_factor;   /* used when capacity < 0 */
  int32_t capacity;        /* < 0: C = ceil(capacity_factor * k * T / E) in double precision;
                              MOE_DROPLESS: no limit;  otherwise C itself */
  int32_t dtype;           /* MOE_DTYPE_F32 | MOE_DTYPE_BF16 */
  int32_t has_bias;        /* bias[E] (a constant logit offset, no gradient) is read when 1 */
  float aux_loss_coef;     /* >= 0, finite: weight of the auxiliary load-balancing loss
                              coef * E * sum_e (counts[e] / (T k)) * mean_t softmax(logits_t)[e]
                              (Ch.4 "框架" DeepSpeed loss_coef; "实践" 四 aux_loss_factor; the
                              pages give no formula, this is the reading taken).  0: the forward
                              does not compute it and the backward adds no gradient for it. */
  int32_t drop_order;      /* capacity drop priority within an expert.  0: token order (position
                              priority, "drop by token order");  1: choice-major -- all first
                              choices in token order, then all second choices, ... (a routing
                              variant; the FSMoE summary names several routing functions) */
} moe_config_t;

/* Sizes and the layout of the forward context (state saved for the backward pass).
 * Every ctx_* field is a byte offset into the ctx buffer, 256-byte aligned. */
typedef struct {
  int64_t capacity;       /* resolved C, or MOE_DROPLESS */
  int64_t T_pad;          /* T rounded up to 128 */
  int64_t rows;           /* R: rows of the dispatched row space (upper bound for any routing) */
  int64_t routed_row0;    /* first routed row = S * T_pad */
  int64_t max_group_rows; /* largest row count any one expert can own (multiple of 128) */
  size_t ctx_logits, ctx_topk_idx, ctx_topk_w, ctx_counts, ctx_kept, ctx_offsets, ctx_slot,
      ctx_row_token, ctx_Xd, ctx_Gu, ctx_Gv, ctx_H, ctx_O;
  size_t ctx_bytes;       /* total ctx size */
  size_t scratch_bytes;   /* total scratch size (forward and backward) */
  size_t ctx_aux_loss;    /* one float: the load-balancing loss of the last forward (written
                             only when aux_loss_coef > 0) */
} moe_layout_t;

/* Validate a config and report the workspace sizes / ctx layout.  Host only, no CUDA calls. */
moe_status moe_get_layout(const moe_config_t* cfg, moe_layout_t* out);
moe_status moe_workspace_size(const moe_config_t* cfg, size_t* ctx_bytes, size_t* scratch_bytes);

/* Step 1, the router: logits = x Wg^T (+ bias), top-k and gate weights.
 * (Ch.4 "专家并行" 二 step 1; top-k gate: "框架" Tutel gate_type top-k.)
 * logits [T,E] float (written); topk_idx [T,k] int32, best first, equal logits -> lower expert
 * index; topk_w [T,k] float: gate_norm 0 -> softmax over all E read at the chosen experts,
 * gate_norm 1 -> softmax over the k chosen logits.  bias may be NULL when has_bias == 0. */
moe_status moe_route(const moe_config_t* cfg, const void* x, const void* Wg, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* The top-k / gate-weight half of moe_route, from given float logits [T,E]. */
moe_status moe_route_from_logits(const moe_config_t* cfg, const float* logits, int32_t* topk_idx,
                                 float* topk_w, moe_stream_t stream);

/* Step 2, capacity-limited dispatch.  For each expert its assignments are ranked by token
 * index (drop_order 0; drop_order 1: by choice index, then token index); rank < C is kept
 * (position priority, "drop by token order").
 * Outputs: counts[E] demand before the drop; kept[E] = min(counts, C); offsets[E+1] first row
 * of each routed segment (offsets[E] = end); slot[T,k] row of each assignment or -1 if
 * dropped; row_token[R] token of each row (-1 for padding and shared rows); Xd[R,d] rows of x
 * copied bit-exactly, padding rows zero.  scratch: moe_layout_t.scratch_bytes bytes. */
moe_status moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                        int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot,
                        int32_t* row_token, void* Xd, void* scratch, moe_stream_t stream);

/* moe_dispatch for callers that cannot allocate device memory.  The pages have no counterpart to
 * this entry point; it exists for deployments, not for the method.
 * Some callers cannot hand the library a scratch buffer: a host framework that owns all device
 * memory through its own fixed pool and does not expose it to plug-ins, a deployment whose memory
 * is budgeted once at start-up so a later allocation could fail, or a latency-critical loop that
 * cannot afford an allocation's cost.  This call takes the same arguments as moe_dispatch minus
 * `scratch`, produces identical outputs, and allocates nothing: the per-CTA expert histograms live
 * in a fixed 256 KB array inside the library, which every GPU that loads the library holds until
 * the process exits.
 * Limit: ceil(T / 256) * E * L <= 65536, with L = 1 for token-order drops (drop_order 0) and L = k
 * for choice-major drops (drop_order 1), which keep one histogram layer per choice index (for
 * example T = 65536 with E = 256 in token order, or T = 2^20 with E = 16); larger configs return
 * MOE_ERR_WORKSPACE_TOO_SMALL and enqueue nothing.
 * The first call on a device looks up the array's device address with that device current; make
 * that first call before any stream capture.  The address is remembered per device together with
 * the CUDA context it belongs to: after the caller resets the device (cudaDeviceReset), the next
 * call looks it up again in the new context.
 * All calls share the one array: calls that overlap on the GPU (for example on two streams) race
 * and corrupt each other's results, so serialise them.  The array keeps the last call's contents;
 * each call rewrites every entry it reads, so nothing needs clearing. */
moe_status moe_dispatch_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot,
                                int32_t* row_token, void* Xd, moe_stream_t stream);

/* Step 3, the expert FFNs as grouped GEMMs over the row space, with u = Xd W1_e^T, v = Xd W3_e^T:
 *   GELU:   H = gelu(u);            Gu = gelu'(u)
 *   SwiGLU: H = silu(u) * v;        Gu = v s (1 + u (1 - s)),  Gv = silu(u),  s = sigmoid(u)
 *   O = H W2_e^T.
 * Gu and Gv are the factors the backward pass needs (dU = dH * Gu, dV = dH * Gv): they are stored
 * instead of u and v.  Shared experts read x directly (all T tokens).  Gv may be NULL and W3 may
 * be NULL for GELU. */
moe_status moe_expert_ffn(const moe_config_t* cfg, const void* Xd, const void* x,
                          const int32_t* offsets, const void* W1, const void* W3, const void* W2,
                          void* Gu, void* Gv, void* H, void* O, void* scratch,
                          moe_stream_t stream);

/* Step 4, combine: y_t = sum over kept j of topk_w[t,j] * O[slot[t,j]] + sum_s O[s*T_pad + t].
 * A gather in a fixed order: deterministic, no atomics. */
moe_status moe_combine(const moe_config_t* cfg, const void* O, const int32_t* slot,
                       const float* topk_w, void* y, moe_stream_t stream);

/* The auxiliary load-balancing loss from float logits [T,E] and counts [E] (the demand per
 * expert before the capacity drop, as moe_dispatch reports it): loss[0] = aux_loss_coef * E *
 * sum_e (counts[e] / (T k)) * P_e, P_e the mean over tokens of softmax(logits_t)[e] over all E
 * (whatever gate_norm is).  Fixed-order reductions: bitwise reproducible.  Uses the scratch
 * buffer of moe_get_layout.  moe_layer_fwd computes the same into ctx when aux_loss_coef > 0,
 * and moe_layer_bwd then adds its gradient, aux_loss_coef * E / T * p_t * (f - <p_t, f>), to
 * the router's logit gradient. */
moe_status moe_aux_loss(const moe_config_t* cfg, const float* logits, const int32_t* counts,
                        float* loss, void* scratch, moe_stream_t stream);

/* Whole forward: steps 1-4.  ctx (moe_layout_t.ctx_bytes) receives the saved state; y [T,d]. */
moe_status moe_layer_fwd(const moe_config_t* cfg, const void* x, const void* Wg,
                         const float* bias, const void* W1, const void* W3, const void* W2,
                         void* y, void* ctx, void* scratch, moe_stream_t stream);

/* The whole forward of a small layer in one launch, for inference (Ch.4 "框架": Tutel's fused
 * MoE kernel; the four steps of "专家并行" 二).  Computes the same y [T,d] as moe_layer_fwd (routing,
 * capacity drops in the configured order, experts, combine) but keeps every intermediate on chip
 * and writes no ctx, so no backward can follow.  topk_idx [T,k], topk_w [T,k] and counts [E]
 * receive the routing when given (all three or none).  Takes layers with T*E*d <= 2^19 whose
 * routing state fits in shared memory, else returns MOE_ERR_UNSUPPORTED (use moe_layer_fwd);
 * aux_loss_coef is ignored. */
moe_status moe_layer_fwd_fused(const moe_config_t* cfg, const void* x, const void* Wg,
                               const float* bias, const void* W1, const void* W3, const void* W2,
                               void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                               moe_stream_t stream);

/* Whole backward for upstream gradient dy [T,d], from the ctx of the matching forward.
 * dx [T,d] (activation dtype); dWg [E,d], dW1/dW3 [E_tot,F,d], dW2 [E_tot,d,F] float.
 * dW3 may be NULL for GELU.  Gradients do not flow through the chosen indices or the drops;
 * bias receives none. */
moe_status moe_layer_bwd(const moe_config_t* cfg, const void* ctx, const void* dy, const void* x,
                         const void* Wg, const void* W1, const void* W3, const void* W2,
                         void* dx, float* dWg, float* dW1, float* dW3, float* dW2, void* scratch,
                         moe_stream_t stream);

/* One training step of the layer from and to HOST memory: copies x and dy (host, ideally pinned)
 * into the device buffers x_dev and dy_dev, runs moe_layer_fwd and moe_layer_bwd, and copies y and
 * dx back into y_host and dx_host, all enqueued on `stream` (plain cudaMemcpyAsync, one per
 * tensor).  Weights and weight gradients stay on the device.  Returns after enqueueing; the host
 * buffers must stay valid until the stream has passed the step.  Two calls on two streams with
 * separate buffers overlap one step's copies with the other's compute.  bias may be NULL when
 * has_bias == 0; W3 and dW3 may be NULL for GELU. */
moe_status moe_layer_step_host(const moe_config_t* cfg, const void* x_host, const void* dy_host,
                               void* y_host, void* dx_host, void* x_dev, void* dy_dev,
                               const void* Wg, const float* bias, const void* W1, const void* W3,
                               const void* W2, void* y_dev, void* dx_dev, float* dWg, float* dW1,
                               float* dW3, float* dW2, void* ctx, void* scratch,
                               moe_stream_t stream);

/* The backward pass in its three steps, for callers that run the expert step elsewhere (expert
 * parallelism: the experts' rows cross to the GPU that owns them and back, Ch.4 "All-to-All
 * 通信模式" 二 and "专家并行与数据并行的结合" 三.3).  moe_layer_bwd is exactly
 * moe_combine_bwd, then moe_expert_ffn_bwd on the ctx's row space, then moe_router_bwd, with
 * dO and dXd kept in scratch.
 *
 * Step 4 backward, from the ctx of the matching forward: dg [T,k] and dlogits [T,E] (with the
 * router's softmax backward and, when aux_loss_coef > 0, the load-balancing loss gradient) into
 * scratch (moe_scratch_grad_offsets); dO [R,d] (the row space of ctx) receives g * dy at every kept
 * row and zero at padding rows; shared experts' rows are not written (their dO is dy itself). */
moe_status moe_combine_bwd(const moe_config_t* cfg, const void* ctx, const void* dy, void* dO,
                           void* scratch, moe_stream_t stream);

/* Step 3 backward over a row space with the layout of moe_expert_ffn (offsets [E+1] on the
 * device, padding rows of dO and Xd zero): dXd [R,d] = the rows' input gradients, dW1, dW3
 * [E_tot,F,d] and dW2 [E_tot,d,F] float (overwritten), from the forward's saved Gu, Gv, H.  dy and
 * x (the shared experts' dO and input rows) may be NULL when n_shared == 0.  Uses scratch as
 * moe_layer_bwd does (dU, dV). */
moe_status moe_expert_ffn_bwd(const moe_config_t* cfg, const void* dO, const void* dy,
                              const void* Xd, const void* x, const int32_t* offsets,
                              const void* W1, const void* W3, const void* W2, const void* Gu,
                              const void* Gv, const void* H, void* dXd, float* dW1, float* dW3,
                              float* dW2, void* scratch, moe_stream_t stream);

/* Steps 1-2 backward on the token side, after moe_combine_bwd on the same scratch:
 * dWg [E,d] = dlogits^T x (float, overwritten) and dx [T,d] = dlogits Wg + the sum of each
 * token's kept rows of dXd and its shared experts' rows (fixed-order sums, no float atomics). */
moe_status moe_router_bwd(const moe_config_t* cfg, const void* ctx, const void* x, const void* Wg,
                          const void* dXd, void* dx, float* dWg, void* scratch,
                          moe_stream_t stream);

/* Byte offset, inside scratch, of dg [T,k] float (dL/dg of each assignment, 0 if dropped) and
 * of dlogits [T,E] float, both valid after moe_layer_bwd until the scratch is reused. */
moe_status moe_scratch_grad_offsets(const moe_config_t* cfg, size_t* dg_offset,
                                    size_t* dlogits_offset);

/* Synchronise `stream`, then report and clear the device status word kept in scratch:
 * MOE_ERR_DEVICE_TIMEOUT if a bounded device wait gave up since the last call, MOE_ERR_CUDA
 * if the stream reported an error, else MOE_OK.
 * Failure detection (the tutorial's debugging notes on deadlocked or mismatched collectives,
 * Ch.4 "分布式训练"): every wait of the tensor-core kernels on a barrier (a TMA copy, an MMA, the
 * accumulator hand-off) is bounded.  When one runs out, the CTA stops taking work, lets its own
 * copies and MMAs in flight finish, frees its tensor memory and sets MOE_STATUS_TIMEOUT in the
 * status word; the context stays usable.  Outputs of that launch are then undefined, but well
 * formed: the router writes the placeholder routing experts 0..k-1 with weight 0, so the kernels
 * after it in the same pass stay in bounds.  moe_route and moe_combine take no scratch and cannot
 * report a timeout. */
moe_status moe_read_status(moe_stream_t stream, void* scratch);

/* Time budget of every bounded device wait, in nanoseconds, for kernels launched after the call
 * (default 2e9 = 2 s; accepted range 1e3 .. 6e10, else MOE_ERR_INVALID_ARG).  Process-wide. */
moe_status moe_set_wait_budget_ns(uint64_t budget_ns);

/* Test hook of the failure path: with on = 1, every tensor-core kernel launched afterwards first
 * waits on a barrier that nothing arrives on, so that wait runs out after the budget and the
 * kernel takes the abort path above (no fault, no hang: the wait is bounded).  on = 0 restores
 * normal operation.  Process-wide; for tests only. */
moe_status moe_set_wait_stall(int32_t on);

/* Name and description of the CUDA error behind the most recent MOE_ERR_CUDA in this process
 * ("" if none).  Process-wide; the text stays valid until the next failure. */
const char* moe_last_cuda_error(void);

/* Static, human-readable name of a status code. */
const char* moe_status_string(moe_status s);

/* Which expert-GEMM engine a config runs on: 0 = CUDA-core (fp32 FMA), 1 = tcgen05. */
int32_t moe_gemm_engine(const moe_config_t* cfg);

/* Number of kernels this library has launched in this process so far (monotone counter). */
int64_t moe_kernel_launches(void);

/* Profiling hook.  fwd_events: NULL, or MOE_FWD_PHASES + 1 cudaEvent_t handles; bwd_events:
 * NULL, or MOE_BWD_PHASES + 1.  While set, moe_layer_fwd records events[0] on its stream before
 * its first launch and events[i] after the launches of phase i (1-based, order below), and
 * moe_layer_bwd does the same with bwd_events.  The caller owns the events and must keep them
 * alive while set.  A NULL entry is not recorded (so a caller can time one phase only: events
 * between kernels keep consecutive launches from overlapping).  Process-wide setting; not for
 * concurrent use from several threads.
 *   forward phases:  router, dispatch, expert_up, expert_down, combine
 *   backward phases: combine_bwd, router_bwd, dgrad_h, dgrad_x, wgrad_w1 (and w3), wgrad_w2,
 *                    undispatch */
#define MOE_FWD_PHASES 5
#define MOE_BWD_PHASES 7
moe_status moe_set_profile_events(void* const* fwd_events, void* const* bwd_events);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
