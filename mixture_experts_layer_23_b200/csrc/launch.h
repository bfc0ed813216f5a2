// Internal launch functions of the MoE kernels (host side).  Each enqueues work on `st` and
// returns MOE_ERR_CUDA if a launch fails.
#pragma once
#include "common.cuh"

namespace moe {

size_t router_smem_bytes(int E);
moe_status launch_router(const Dims& D, const void* x, const void* Wg, const float* bias,
                         float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st);
bool router_warp_supported(const Dims& D);
moe_status launch_router_warp(const Dims& D, const void* x, const void* Wg, const float* bias,
                              float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st);
moe_status launch_topk_from_logits(const Dims& D, const float* logits, int32_t* topk_idx,
                                   float* topk_w, cudaStream_t st);
// status: the scratch status word, or null (moe_dispatch_noalloc)
moe_status launch_dispatch(const Dims& D, const void* x, const int32_t* topk_idx, int32_t* counts,
                           int32_t* kept, int32_t* offsets, int32_t* slot, int32_t* row_token,
                           void* Xd, int32_t* blk_counts, uint32_t* status, cudaStream_t st);
moe_status launch_combine(const Dims& D, const void* O, const int32_t* slot, const float* topk_w,
                          void* y, cudaStream_t st);
moe_status launch_combine_bwd(const Dims& D, const void* dy, const void* O, const int32_t* slot,
                              const float* topk_w, const int32_t* topk_idx, const float* logits,
                              const int32_t* kept, const int32_t* offsets, const int32_t* counts,
                              float* dg, float* dlogits, __nv_bfloat16* dl16, void* dO,
                              cudaStream_t st);
// Router backward on the tensor cores (bf16, d a multiple of 64): dWg partials over token
// chunks and their fixed-order sum; dl Wg with the un-dispatch gather fused into its epilogue.
bool router_bwd_tc_supported(const Dims& D);
// One-launch forward of small layers (inference): routing recomputed per CTA, no ctx.
bool fused_small_supported(const Dims& D);
moe_status launch_fused_small_fwd(const Dims& D, const void* x, const void* Wg, const float* bias,
                                  const void* W1, const void* W3, const void* W2, void* y,
                                  int32_t* topk_idx, float* topk_w, int32_t* counts,
                                  cudaStream_t st);
// Load-balancing loss (forward): loss[0] from the logits and the pre-drop counts.
moe_status launch_aux_loss(const Dims& D, const float* logits, const int32_t* counts, float* part,
                           float* loss, cudaStream_t st);
moe_status launch_router_wgrad_tc(const Dims& D, const __nv_bfloat16* dl16, const void* x,
                                  float* part, int* n_chunks, uint32_t* status, cudaStream_t st);
moe_status launch_router_wgrad_reduce(const Dims& D, const float* part, int n_chunks, float* dWg,
                                      cudaStream_t st);
moe_status launch_undispatch_tc(const Dims& D, const __nv_bfloat16* dl16, const void* Wg,
                                const void* dXd, const int32_t* slot, void* dx, uint32_t* status,
                                cudaStream_t st);
moe_status launch_router_wgrad(const Dims& D, const float* dlogits, const void* x, float* part,
                               float* dWg, cudaStream_t st);
moe_status launch_undispatch(const Dims& D, const float* dlogits, const void* Wg, const void* dXd,
                             const int32_t* slot, void* dx, cudaStream_t st);
moe_status launch_expert_up_simt(const Dims& D, const void* Xd, const void* x,
                                 const int32_t* offsets, const void* W1, const void* W3, void* U,
                                 void* V, void* H, cudaStream_t st);
moe_status launch_expert_down_simt(const Dims& D, const void* H, const int32_t* offsets,
                                   const void* W2, void* O, cudaStream_t st);
moe_status launch_dgrad_h_simt(const Dims& D, const void* dO, const void* dy,
                               const int32_t* offsets, const void* W2, const void* U,
                               const void* V, void* dU, void* dV, cudaStream_t st);
moe_status launch_dgrad_x_simt(const Dims& D, const void* dU, const void* dV,
                               const int32_t* offsets, const void* W1, const void* W3, void* dXd,
                               cudaStream_t st);
moe_status launch_wgrad_w13_simt(const Dims& D, const void* dU, const void* dV, const void* Xd,
                                 const void* x, const int32_t* offsets, float* dW1, float* dW3,
                                 cudaStream_t st);
moe_status launch_wgrad_w2_simt(const Dims& D, const void* H, const void* dO, const void* dy,
                                const int32_t* offsets, float* dW2, cudaStream_t st);

// Column-major copies of bf16 activations for the weight gradients: dst[c][col0 + r] =
// src[row0 + r][c] for r < nrows, c < cols, with source rows r >= nvalid read as zeros (nvalid < 0:
// all nrows); cols a multiple of 64, rows and destinations 16-byte aligned, the destination holds
// round_up(nrows, 8) columns from col0.  Up to 8 jobs per launch.
struct TransposeSpec {
  const void* src;
  void* dst;
  long long src_ld, dst_ld, row0, col0, nrows, nvalid, cols;
};
moe_status launch_transpose_bf16(const TransposeSpec* specs, int n, cudaStream_t st);

// tcgen05 router (bf16, d a multiple of 64, E <= 256); status may be null
bool router_tc_supported(const Dims& D);
moe_status launch_router_tc(const Dims& D, const void* x, const void* Wg, const float* bias,
                            float* logits, int32_t* topk_idx, float* topk_w, uint32_t* status,
                            cudaStream_t st);

// tcgen05 engine (bf16, d and F multiples of 64)
bool tc_supported(const Dims& D);
moe_status launch_expert_up_tc(const Dims& D, const void* Xd, const void* x, const int32_t* offsets,
                               const void* W1, const void* W3, void* U, void* V, void* H,
                               uint32_t* status, cudaStream_t st);
moe_status launch_expert_down_tc(const Dims& D, const void* H, const int32_t* offsets,
                                 const void* W2, void* O, uint32_t* status, cudaStream_t st);
moe_status launch_dgrad_h_tc(const Dims& D, const void* dO, const void* dy, const int32_t* offsets,
                             const void* W2, const void* U, const void* V, void* dU, void* dV,
                             int* zero, int zero_n, uint32_t* status, cudaStream_t st);
// zero[0..zero_n): the weight gradients' tile counters, reset by the input gradient that runs
// before them
moe_status launch_dgrad_x_tc(const Dims& D, const void* dU, const void* dV, const int32_t* offsets,
                             const void* W1, const void* W3, void* dXd, int* zero, int zero_n,
                             uint32_t* status, cudaStream_t st);
// The weight gradients.  With wgrad_kmajor(D) they read one operand through a column-major copy
// (launch_transpose_bf16): X / xs are Xdt [d][R] (routed columns) / xt [d][T_pad] (shared experts)
// and G / gs are dOt [d][R] / dyt [d][T_pad], xs and gs null without shared experts; otherwise X,
// xs, G, gs are Xd, x, dO, dy themselves (all valid pointers).
bool wgrad_kmajor(const Dims& D);
// sched: zeroed tile counters, one per launch (w13: dW1 at [0], dW3 at [1]; w2: [0])
moe_status launch_wgrad_w13_tc(const Dims& D, const void* dU, const void* dV, const void* X,
                               const void* xs, const int32_t* offsets, float* dW1, float* dW3,
                               int* sched, uint32_t* status, cudaStream_t st);
moe_status launch_wgrad_w2_tc(const Dims& D, const void* H, const void* G, const void* gs,
                              const int32_t* offsets, float* dW2, int* sched, uint32_t* status,
                              cudaStream_t st);

}  // namespace moe
