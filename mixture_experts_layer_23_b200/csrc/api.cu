// The C ABI of the MoE layer: argument checks, workspace layout and the call sequences of the
// forward and backward passes.  Declarations and the contract are in include/moe.h.
#include <math.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include "launch.h"
#include "tc_host.h"

namespace moe {

unsigned long long g_kernel_launches = 0;

static char g_last_cuda_error[256] = "";

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_DISABLE_PDL");
    return !(v && v[0] == '1');
  }();
  return on;
}
void note_cuda_error(cudaError_t e) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
}

// Profiling hook (moe_set_profile_events): events recorded between the phases of a pass.
static cudaEvent_t g_fwd_events[MOE_FWD_PHASES + 1];
static cudaEvent_t g_bwd_events[MOE_BWD_PHASES + 1];
static bool g_fwd_prof = false, g_bwd_prof = false;

static inline moe_status mark_fwd(int i, cudaStream_t st) {
  if (g_fwd_prof && g_fwd_events[i] && cudaEventRecord(g_fwd_events[i], st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
static inline moe_status mark_bwd(int i, cudaStream_t st) {
  if (g_bwd_prof && g_bwd_events[i] && cudaEventRecord(g_bwd_events[i], st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

static inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

moe_status resolve_dims(const moe_config_t* cfg, Dims* out) {
  if (!cfg || !out) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  if (c.T < 1 || c.d < 1 || c.E < 1 || c.k < 1 || c.d_ff < 1 || c.n_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (c.k > c.E) return MOE_ERR_INVALID_ARG;
  if (c.act != MOE_ACT_GELU && c.act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c.gate_norm != 0 && c.gate_norm != 1) return MOE_ERR_INVALID_ARG;
  if (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (c.has_bias != 0 && c.has_bias != 1) return MOE_ERR_INVALID_ARG;
  if (!(c.aux_loss_coef >= 0.f) || !isfinite(c.aux_loss_coef)) return MOE_ERR_INVALID_ARG;
  if (c.drop_order != 0 && c.drop_order != 1) return MOE_ERR_INVALID_ARG;
  if (c.k > 8 || c.E > 256 || c.n_shared > 8 || c.T > (1 << 24)) return MOE_ERR_UNSUPPORTED;
  const int vec = (c.dtype == MOE_DTYPE_BF16) ? 8 : 4;
  if (c.d % vec != 0 || c.d_ff % vec != 0) return MOE_ERR_UNSUPPORTED;

  Dims D;
  D.T = c.T; D.d = c.d; D.E = c.E; D.k = c.k; D.F = c.d_ff; D.S = c.n_shared;
  D.E_tot = c.E + c.n_shared;
  D.act = c.act; D.gate_norm = c.gate_norm; D.dtype = c.dtype; D.has_bias = c.has_bias;
  D.elem = (c.dtype == MOE_DTYPE_BF16) ? 2 : 4;
  if (c.capacity == MOE_DROPLESS) {
    D.C = MOE_DROPLESS;
  } else if (c.capacity >= 0) {
    D.C = c.capacity;
  } else {
    if (!(c.capacity_factor > 0.f) || !isfinite(c.capacity_factor)) return MOE_ERR_INVALID_ARG;
    const double cap = ceil((double)c.capacity_factor * c.k * c.T / c.E);
    D.C = cap >= (double)MOE_DROPLESS ? (int64_t)MOE_DROPLESS : (int64_t)cap;
  }
  const int64_t kmax = D.C < D.T ? D.C : D.T;            // rows one expert can keep
  D.T_pad = round_up(D.T, MOE_ROW_ALIGN);
  D.routed_row0 = (int64_t)D.S * D.T_pad;
  int64_t n_assign = (int64_t)D.T * D.k;
  if ((int64_t)D.E * kmax < n_assign) n_assign = (int64_t)D.E * kmax;
  const int64_t routed = (n_assign + (int64_t)(MOE_ROW_ALIGN - 1) * D.E) / MOE_ROW_ALIGN * MOE_ROW_ALIGN;
  D.R = D.routed_row0 + routed;
  if (D.R < MOE_ROW_ALIGN) D.R = MOE_ROW_ALIGN;
  if (D.R >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  int64_t mg = round_up(kmax, MOE_ROW_ALIGN);
  if (D.S > 0 && D.T_pad > mg) mg = D.T_pad;
  D.max_group_rows = mg < MOE_ROW_ALIGN ? MOE_ROW_ALIGN : mg;
  D.n_blk = (D.T + kDispatchTokensPerBlock - 1) / kDispatchTokensPerBlock;
  // token chunks of the router-weight gradient: enough CTAs (chunks x 256-column slices) to fill
  // the GPU twice, chunks of at least 64 tokens
  {
    const int slices = (D.d + 255) / 256;
    int chunks = (2 * 148 + slices - 1) / slices;
    const int max_chunks = (D.T + 63) / 64;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    D.n_tchunk = chunks;
  }
  D.aux_coef = c.aux_loss_coef;
  D.choice_major = c.drop_order;
  D.n_layers = c.drop_order ? c.k : 1;
  D.n_aux = (D.T + kAuxTokensPerChunk - 1) / kAuxTokensPerChunk;
  if (D.n_aux > kAuxMaxChunks) D.n_aux = kAuxMaxChunks;
  *out = D;
  return MOE_OK;
}

ScratchLayout scratch_layout(const Dims& D) {
  ScratchLayout S;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align256(off + bytes); return o; };
  const size_t R = (size_t)D.R, T = (size_t)D.T;
  S.status = take(256);
  S.blk_counts = take((size_t)D.n_blk * D.n_layers * D.E * 4);
  S.local_rank = 0;  // the dispatch keeps local ranks in the slot array
  S.groups = take((size_t)D.E_tot * 16);
  S.dO = take(R * D.d * D.elem);
  S.dU = take(R * D.F * D.elem);
  S.dV = (D.act == MOE_ACT_SWIGLU) ? take(R * D.F * D.elem) : 0;
  S.dXd = take(R * D.d * D.elem);
  S.dg = take(T * D.k * 4);
  S.dlogits = take(T * D.E * 4);
  S.dWg_part = take((size_t)D.n_tchunk * D.E * D.d * 4);
  S.dl16 = 0;
  if (router_bwd_tc_supported(D)) S.dl16 = take(T * (size_t)round_up(D.E, 8) * 2);
  S.aux_part = take((size_t)D.n_aux * D.E * 4);
  S.wg_sched = take(16);
  S.Xdt = S.dOt = S.xt = S.dyt = 0;
  if (wgrad_kmajor(D)) {
    S.Xdt = take(R * D.d * 2);
    S.dOt = take(R * D.d * 2);
    if (D.S > 0) {
      S.xt = take((size_t)D.T_pad * D.d * 2);
      S.dyt = take((size_t)D.T_pad * D.d * 2);
    }
  }
  S.total = off;
  return S;
}

moe_status ctx_layout(const Dims& D, moe_layout_t* L) {
  memset(L, 0, sizeof(*L));
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align256(off + bytes); return o; };
  const size_t R = (size_t)D.R, T = (size_t)D.T;
  L->capacity = D.C;
  L->T_pad = D.T_pad;
  L->rows = D.R;
  L->routed_row0 = D.routed_row0;
  L->max_group_rows = D.max_group_rows;
  L->ctx_logits = take(T * D.E * 4);
  L->ctx_topk_idx = take(T * D.k * 4);
  L->ctx_topk_w = take(T * D.k * 4);
  L->ctx_counts = take((size_t)D.E * 4);
  L->ctx_kept = take((size_t)D.E * 4);
  L->ctx_offsets = take((size_t)(D.E + 1) * 4);
  L->ctx_slot = take(T * D.k * 4);
  L->ctx_row_token = take(R * 4);
  L->ctx_Xd = take(R * D.d * D.elem);
  L->ctx_Gu = take(R * D.F * D.elem);
  L->ctx_Gv = (D.act == MOE_ACT_SWIGLU) ? take(R * D.F * D.elem) : 0;
  L->ctx_H = take(R * D.F * D.elem);
  L->ctx_O = take(R * D.d * D.elem);
  L->ctx_aux_loss = take(4);
  L->ctx_bytes = off;
  L->scratch_bytes = scratch_layout(D).total;
  return MOE_OK;
}

static inline bool misaligned(const void* p) { return ((uintptr_t)p & 15u) != 0; }

// All listed pointers non-null and 16-byte aligned.
static moe_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (misaligned(p)) return MOE_ERR_MISALIGNED;
  }
  return MOE_OK;
}

#define MOE_TRY(expr)                    \
  do {                                   \
    const moe_status s_ = (expr);        \
    if (s_ != MOE_OK) return s_;         \
  } while (0)

// Expert FFN forward: the up-projection GEMM, then the down-projection GEMM.  With
// phase_marks, the profiling event of phase 3 (expert_up) is recorded between the two.
static moe_status expert_fwd(const Dims& D, const void* Xd, const void* x, const int32_t* offsets,
                             const void* W1, const void* W3, const void* W2, void* Gu, void* Gv,
                             void* H, void* O, uint32_t* status, cudaStream_t st,
                             bool phase_marks = false) {
  if (tc_supported(D)) {
    MOE_TRY(launch_expert_up_tc(D, Xd, x, offsets, W1, W3, Gu, Gv, H, status, st));
    if (phase_marks) MOE_TRY(mark_fwd(3, st));
    return launch_expert_down_tc(D, H, offsets, W2, O, status, st);
  }
  MOE_TRY(launch_expert_up_simt(D, Xd, x, offsets, W1, W3, Gu, Gv, H, st));
  if (phase_marks) MOE_TRY(mark_fwd(3, st));
  return launch_expert_down_simt(D, H, offsets, W2, O, st);
}

// Expert FFN backward: dgrad through W2 and the activation, dgrad through W1 (and W3), then the
// weight gradients; with phase_marks, the profiling events of backward phases 3..5 between them.
// The expert GEMMs' backward.  s / S: the scratch area, for the tensor-core path's transposed
// copies of Xd and dO (and of x and dy for shared experts), which its weight gradients read K-major.
static moe_status expert_bwd(const Dims& D, const void* dO, const void* dy, const void* Xd,
                             const void* x, const int32_t* offsets, const void* W1,
                             const void* W3, const void* W2, const void* Gu, const void* Gv,
                             const void* H, void* dU, void* dV, void* dXd, float* dW1, float* dW3,
                             float* dW2, char* s, const ScratchLayout& S, cudaStream_t st,
                             bool phase_marks = false) {
  uint32_t* status = (uint32_t*)(s + S.status);
  if (tc_supported(D)) {
    int* wg_sched = (int*)(s + S.wg_sched);   // the weight gradients' tile counters
    MOE_TRY(launch_dgrad_h_tc(D, dO, dy, offsets, W2, Gu, Gv, dU, dV, nullptr, 0, status, st));
    if (phase_marks) MOE_TRY(mark_bwd(3, st));
    MOE_TRY(launch_dgrad_x_tc(D, dU, dV, offsets, W1, W3, dXd, wg_sched, 4, status, st));
    if (phase_marks) MOE_TRY(mark_bwd(4, st));
    if (!wgrad_kmajor(D)) {
      MOE_TRY(launch_wgrad_w13_tc(D, dU, dV, Xd, x, offsets, dW1, dW3, wg_sched, status, st));
      if (phase_marks) MOE_TRY(mark_bwd(5, st));
      return launch_wgrad_w2_tc(D, H, dO, dy, offsets, dW2, wg_sched + 2, status, st);
    }
    // Xd^T and dO^T over the routed rows (padding rows are zero in both), x^T and dy^T over T_pad
    // columns with zeros past T
    const long long r0 = D.routed_row0, nr = D.R - D.routed_row0;
    TransposeSpec js[4] = {
        {Xd, s + S.Xdt, D.d, D.R, r0, r0, nr, -1, D.d},
        {dO, s + S.dOt, D.d, D.R, r0, r0, nr, -1, D.d}};
    int nj = 2;
    if (D.S > 0) {
      js[nj++] = {x, s + S.xt, D.d, D.T_pad, 0, 0, D.T_pad, D.T, D.d};
      js[nj++] = {dy, s + S.dyt, D.d, D.T_pad, 0, 0, D.T_pad, D.T, D.d};
    }
    MOE_TRY(launch_transpose_bf16(js, nj, st));
    MOE_TRY(launch_wgrad_w13_tc(D, dU, dV, s + S.Xdt, D.S > 0 ? s + S.xt : nullptr, offsets, dW1,
                                dW3, wg_sched, status, st));
    if (phase_marks) MOE_TRY(mark_bwd(5, st));
    MOE_TRY(launch_wgrad_w2_tc(D, H, s + S.dOt, D.S > 0 ? s + S.dyt : nullptr, offsets, dW2,
                               wg_sched + 2, status, st));
    return MOE_OK;
  }
  MOE_TRY(launch_dgrad_h_simt(D, dO, dy, offsets, W2, Gu, Gv, dU, dV, st));
  if (phase_marks) MOE_TRY(mark_bwd(3, st));
  MOE_TRY(launch_dgrad_x_simt(D, dU, dV, offsets, W1, W3, dXd, st));
  if (phase_marks) MOE_TRY(mark_bwd(4, st));
  MOE_TRY(launch_wgrad_w13_simt(D, dU, dV, Xd, x, offsets, dW1, dW3, st));
  if (phase_marks) MOE_TRY(mark_bwd(5, st));
  MOE_TRY(launch_wgrad_w2_simt(D, H, dO, dy, offsets, dW2, st));
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_get_layout(const moe_config_t* cfg, moe_layout_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  return ctx_layout(D, out);
}

moe_status moe_workspace_size(const moe_config_t* cfg, size_t* ctx_bytes, size_t* scratch_bytes) {
  if (!ctx_bytes || !scratch_bytes) return MOE_ERR_INVALID_ARG;
  moe_layout_t L;
  MOE_TRY(moe_get_layout(cfg, &L));
  *ctx_bytes = L.ctx_bytes;
  *scratch_bytes = L.scratch_bytes;
  return MOE_OK;
}

moe_status moe_scratch_grad_offsets(const moe_config_t* cfg, size_t* dg_offset,
                                    size_t* dlogits_offset) {
  if (!dg_offset || !dlogits_offset) return MOE_ERR_INVALID_ARG;
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  const ScratchLayout S = scratch_layout(D);
  *dg_offset = S.dg;
  *dlogits_offset = S.dlogits;
  return MOE_OK;
}

int32_t moe_gemm_engine(const moe_config_t* cfg) {
  Dims D;
  if (resolve_dims(cfg, &D) != MOE_OK) return -1;
  return tc_supported(D) ? 1 : 0;
}

// Router choice: bf16 with d a multiple of 64 takes the tcgen05 kernel (measured faster than the
// warp-per-token kernel from 16 experts up); other shapes with up to 32 experts whose gate matrix
// fits in shared memory take the warp-per-token kernel; the rest the CUDA-core tile kernel.  All
// three end in the same serial softmax + top-k.
static moe_status launch_route(const Dims& D, const void* x, const void* Wg, const float* bias,
                               float* logits, int32_t* idx, float* w, uint32_t* status,
                               cudaStream_t st) {
  if (router_tc_supported(D)) return launch_router_tc(D, x, Wg, bias, logits, idx, w, status, st);
  if (router_warp_supported(D)) return launch_router_warp(D, x, Wg, bias, logits, idx, w, st);
  return launch_router(D, x, Wg, bias, logits, idx, w, st);
}

moe_status moe_route(const moe_config_t* cfg, const void* x, const void* Wg, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({x, Wg, logits, topk_idx, topk_w}));
  if (D.has_bias) MOE_TRY(check_ptrs({bias}));
  return launch_route(D, x, Wg, bias, logits, topk_idx, topk_w, nullptr, (cudaStream_t)stream);
}

moe_status moe_layer_fwd_fused(const moe_config_t* cfg, const void* x, const void* Wg,
                               const float* bias, const void* W1, const void* W3, const void* W2,
                               void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                               moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({x, Wg, W1, W2, y}));
  if (D.act == MOE_ACT_SWIGLU) MOE_TRY(check_ptrs({W3}));
  if (D.has_bias) MOE_TRY(check_ptrs({bias}));
  const bool routing = topk_idx || topk_w || counts;
  if (routing) MOE_TRY(check_ptrs({topk_idx, topk_w, counts}));
  if (!fused_small_supported(D)) return MOE_ERR_UNSUPPORTED;
  return launch_fused_small_fwd(D, x, Wg, bias, W1, W3, W2, y, topk_idx, topk_w, counts,
                                (cudaStream_t)stream);
}

moe_status moe_aux_loss(const moe_config_t* cfg, const float* logits, const int32_t* counts,
                        float* loss, void* scratch, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({logits, counts, loss, scratch}));
  const ScratchLayout S = scratch_layout(D);
  return launch_aux_loss(D, logits, counts, (float*)((char*)scratch + S.aux_part), loss,
                         (cudaStream_t)stream);
}

moe_status moe_route_from_logits(const moe_config_t* cfg, const float* logits, int32_t* topk_idx,
                                 float* topk_w, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({logits, topk_idx, topk_w}));
  return launch_topk_from_logits(D, logits, topk_idx, topk_w, (cudaStream_t)stream);
}

moe_status moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                        int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot,
                        int32_t* row_token, void* Xd, void* scratch, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({x, topk_idx, counts, kept, offsets, slot, row_token, Xd, scratch}));
  const ScratchLayout S = scratch_layout(D);
  return launch_dispatch(D, x, topk_idx, counts, kept, offsets, slot, row_token, Xd,
                         (int32_t*)((char*)scratch + S.blk_counts),
                         (uint32_t*)((char*)scratch + S.status), (cudaStream_t)stream);
}

moe_status moe_expert_ffn(const moe_config_t* cfg, const void* Xd, const void* x,
                          const int32_t* offsets, const void* W1, const void* W3, const void* W2,
                          void* Gu, void* Gv, void* H, void* O, void* scratch,
                          moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({Xd, x, offsets, W1, W2, Gu, H, O, scratch}));
  if (D.act == MOE_ACT_SWIGLU) MOE_TRY(check_ptrs({W3, Gv}));
  const ScratchLayout S = scratch_layout(D);
  return expert_fwd(D, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, O,
                    (uint32_t*)((char*)scratch + S.status), (cudaStream_t)stream);
}

moe_status moe_combine(const moe_config_t* cfg, const void* O, const int32_t* slot,
                       const float* topk_w, void* y, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({O, slot, topk_w, y}));
  return launch_combine(D, O, slot, topk_w, y, (cudaStream_t)stream);
}

moe_status moe_layer_fwd(const moe_config_t* cfg, const void* x, const void* Wg,
                         const float* bias, const void* W1, const void* W3, const void* W2,
                         void* y, void* ctx, void* scratch, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({x, Wg, W1, W2, y, ctx, scratch}));
  if (D.has_bias) MOE_TRY(check_ptrs({bias}));
  if (D.act == MOE_ACT_SWIGLU) MOE_TRY(check_ptrs({W3}));
  moe_layout_t L;
  ctx_layout(D, &L);
  const ScratchLayout S = scratch_layout(D);
  cudaStream_t st = (cudaStream_t)stream;
  char* c = (char*)ctx;
  char* s = (char*)scratch;
  if (cudaMemsetAsync(s + S.status, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  float* logits = (float*)(c + L.ctx_logits);
  int32_t* idx = (int32_t*)(c + L.ctx_topk_idx);
  float* w = (float*)(c + L.ctx_topk_w);
  int32_t* counts = (int32_t*)(c + L.ctx_counts);
  int32_t* kept = (int32_t*)(c + L.ctx_kept);
  int32_t* offsets = (int32_t*)(c + L.ctx_offsets);
  int32_t* slot = (int32_t*)(c + L.ctx_slot);
  int32_t* row_token = (int32_t*)(c + L.ctx_row_token);
  void* Xd = c + L.ctx_Xd;
  void* Gu = c + L.ctx_Gu;
  void* Gv = L.ctx_Gv ? c + L.ctx_Gv : nullptr;
  void* H = c + L.ctx_H;
  void* O = c + L.ctx_O;
  MOE_TRY(mark_fwd(0, st));
  MOE_TRY(launch_route(D, x, Wg, bias, logits, idx, w, (uint32_t*)(s + S.status), st));
  MOE_TRY(mark_fwd(1, st));
  MOE_TRY(launch_dispatch(D, x, idx, counts, kept, offsets, slot, row_token, Xd,
                          (int32_t*)(s + S.blk_counts), (uint32_t*)(s + S.status), st));
  if (D.aux_coef > 0.f)
    MOE_TRY(launch_aux_loss(D, logits, counts, (float*)(s + S.aux_part), (float*)(c + L.ctx_aux_loss),
                            st));
  MOE_TRY(mark_fwd(2, st));
  MOE_TRY(expert_fwd(D, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, O, (uint32_t*)(s + S.status), st,
                     /*phase_marks=*/true));
  MOE_TRY(mark_fwd(4, st));
  MOE_TRY(launch_combine(D, O, slot, w, y, st));
  MOE_TRY(mark_fwd(5, st));
  return MOE_OK;
}

}  // extern "C"

namespace moe {

// Pieces of the backward pass, shared by moe_layer_bwd and the per-step entry points.

// Step 4 backward: dg, dlogits (and their bf16 copy for the tensor-core router backward) into
// scratch, dO = g * dy into the caller's row-space buffer (padding rows zeroed).
static moe_status bwd_combine(const Dims& D, const moe_layout_t& L, const ScratchLayout& S,
                              const char* c, char* s, const void* dy, void* dO, cudaStream_t st) {
  __nv_bfloat16* dl16 = S.dl16 ? (__nv_bfloat16*)(s + S.dl16) : nullptr;
  return launch_combine_bwd(D, dy, c + L.ctx_O, (const int32_t*)(c + L.ctx_slot),
                            (const float*)(c + L.ctx_topk_w), (const int32_t*)(c + L.ctx_topk_idx),
                            (const float*)(c + L.ctx_logits), (const int32_t*)(c + L.ctx_kept),
                            (const int32_t*)(c + L.ctx_offsets), (const int32_t*)(c + L.ctx_counts),
                            (float*)(s + S.dg), (float*)(s + S.dlogits), dl16, dO, st);
}

// Router weight gradient dWg = dl^T x (tensor cores over token chunks for bf16 with d % 64 == 0,
// else CUDA cores), both with fixed-order reductions.
static moe_status bwd_router_wgrad(const Dims& D, const ScratchLayout& S, char* s, const void* x,
                                   float* dWg, cudaStream_t st) {
  float* part = (float*)(s + S.dWg_part);
  if (S.dl16) {
    int n_chunks = 0;
    MOE_TRY(launch_router_wgrad_tc(D, (const __nv_bfloat16*)(s + S.dl16), x, part, &n_chunks,
                                   (uint32_t*)(s + S.status), st));
    return launch_router_wgrad_reduce(D, part, n_chunks, dWg, st);
  }
  return launch_router_wgrad(D, (const float*)(s + S.dlogits), x, part, dWg, st);
}

// Steps 1-2 backward on the token side: dx = dl Wg + the token's routed and shared dXd rows.
static moe_status bwd_router_dx(const Dims& D, const moe_layout_t& L, const ScratchLayout& S,
                                const char* c, char* s, const void* Wg, const void* dXd, void* dx,
                                cudaStream_t st) {
  const int32_t* slot = (const int32_t*)(c + L.ctx_slot);
  if (S.dl16)
    return launch_undispatch_tc(D, (const __nv_bfloat16*)(s + S.dl16), Wg, dXd, slot, dx,
                                (uint32_t*)(s + S.status), st);
  return launch_undispatch(D, (const float*)(s + S.dlogits), Wg, dXd, slot, dx, st);
}

}  // namespace moe

extern "C" {

moe_status moe_layer_bwd(const moe_config_t* cfg, const void* ctx, const void* dy, const void* x,
                         const void* Wg, const void* W1, const void* W3, const void* W2,
                         void* dx, float* dWg, float* dW1, float* dW3, float* dW2, void* scratch,
                         moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({ctx, dy, x, Wg, W1, W2, dx, dWg, dW1, dW2, scratch}));
  if (D.act == MOE_ACT_SWIGLU) MOE_TRY(check_ptrs({W3, dW3}));
  moe_layout_t L;
  ctx_layout(D, &L);
  const ScratchLayout S = scratch_layout(D);
  cudaStream_t st = (cudaStream_t)stream;
  const char* c = (const char*)ctx;
  char* s = (char*)scratch;
  void* dO = s + S.dO;
  void* dXd = s + S.dXd;
  MOE_TRY(mark_bwd(0, st));
  MOE_TRY(bwd_combine(D, L, S, c, s, dy, dO, st));
  MOE_TRY(mark_bwd(1, st));
  MOE_TRY(bwd_router_wgrad(D, S, s, x, dWg, st));
  MOE_TRY(mark_bwd(2, st));
  MOE_TRY(expert_bwd(D, dO, dy, c + L.ctx_Xd, x, (const int32_t*)(c + L.ctx_offsets), W1, W3, W2,
                     c + L.ctx_Gu, L.ctx_Gv ? c + L.ctx_Gv : nullptr, c + L.ctx_H, s + S.dU,
                     S.dV ? s + S.dV : nullptr, dXd, dW1, dW3, dW2, s, S, st,
                     /*phase_marks=*/true));
  MOE_TRY(mark_bwd(6, st));
  MOE_TRY(bwd_router_dx(D, L, S, c, s, Wg, dXd, dx, st));
  MOE_TRY(mark_bwd(7, st));
  return MOE_OK;
}

moe_status moe_layer_step_host(const moe_config_t* cfg, const void* x_host, const void* dy_host,
                               void* y_host, void* dx_host, void* x_dev, void* dy_dev,
                               const void* Wg, const float* bias, const void* W1, const void* W3,
                               const void* W2, void* y_dev, void* dx_dev, float* dWg, float* dW1,
                               float* dW3, float* dW2, void* ctx, void* scratch,
                               moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  if (!x_host || !dy_host || !y_host || !dx_host) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({x_dev, dy_dev, y_dev, dx_dev}));
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)D.T * D.d * D.elem;
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dy_dev, dy_host, bytes, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) {
    note_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  MOE_TRY(moe_layer_fwd(cfg, x_dev, Wg, bias, W1, W3, W2, y_dev, ctx, scratch, stream));
  MOE_TRY(moe_layer_bwd(cfg, ctx, dy_dev, x_dev, Wg, W1, W3, W2, dx_dev, dWg, dW1, dW3, dW2, scratch,
                        stream));
  e = cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dx_host, dx_dev, bytes, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) {
    note_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status moe_combine_bwd(const moe_config_t* cfg, const void* ctx, const void* dy, void* dO,
                           void* scratch, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({ctx, dy, dO, scratch}));
  moe_layout_t L;
  ctx_layout(D, &L);
  const ScratchLayout S = scratch_layout(D);
  return bwd_combine(D, L, S, (const char*)ctx, (char*)scratch, dy, dO, (cudaStream_t)stream);
}

moe_status moe_expert_ffn_bwd(const moe_config_t* cfg, const void* dO, const void* dy,
                              const void* Xd, const void* x, const int32_t* offsets,
                              const void* W1, const void* W3, const void* W2, const void* Gu,
                              const void* Gv, const void* H, void* dXd, float* dW1, float* dW3,
                              float* dW2, void* scratch, moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({dO, Xd, offsets, W1, W2, Gu, H, dXd, dW1, dW2, scratch}));
  if (D.S > 0) MOE_TRY(check_ptrs({dy, x}));
  if (D.act == MOE_ACT_SWIGLU) MOE_TRY(check_ptrs({W3, Gv, dW3}));
  const ScratchLayout S = scratch_layout(D);
  char* s = (char*)scratch;
  // with no shared experts dy and x are never read; any valid pointer stands in for them
  const void* dy_ = D.S > 0 ? dy : dO;
  const void* x_ = D.S > 0 ? x : Xd;
  return expert_bwd(D, dO, dy_, Xd, x_, offsets, W1, W3, W2, Gu, Gv, H, s + S.dU,
                    S.dV ? s + S.dV : nullptr, dXd, dW1, dW3, dW2, s, S, (cudaStream_t)stream);
}

moe_status moe_router_bwd(const moe_config_t* cfg, const void* ctx, const void* x, const void* Wg,
                          const void* dXd, void* dx, float* dWg, void* scratch,
                          moe_stream_t stream) {
  Dims D;
  MOE_TRY(resolve_dims(cfg, &D));
  MOE_TRY(check_ptrs({ctx, x, Wg, dXd, dx, dWg, scratch}));
  moe_layout_t L;
  ctx_layout(D, &L);
  const ScratchLayout S = scratch_layout(D);
  cudaStream_t st = (cudaStream_t)stream;
  char* s = (char*)scratch;
  MOE_TRY(bwd_router_wgrad(D, S, s, x, dWg, st));
  return bwd_router_dx(D, L, S, (const char*)ctx, s, Wg, dXd, dx, st);
}

int64_t moe_kernel_launches(void) {
  return (int64_t)__atomic_load_n(&g_kernel_launches, __ATOMIC_RELAXED);
}

moe_status moe_set_profile_events(void* const* fwd_events, void* const* bwd_events) {
  g_fwd_prof = fwd_events != nullptr;
  g_bwd_prof = bwd_events != nullptr;
  for (int i = 0; g_fwd_prof && i <= MOE_FWD_PHASES; ++i)
    g_fwd_events[i] = (cudaEvent_t)fwd_events[i];   // NULL entries are skipped
  for (int i = 0; g_bwd_prof && i <= MOE_BWD_PHASES; ++i)
    g_bwd_events[i] = (cudaEvent_t)bwd_events[i];
  return MOE_OK;
}

moe_status moe_set_wait_budget_ns(uint64_t budget_ns) {
  if (budget_ns < 1000 || budget_ns > 60ull * 1000000000ull) return MOE_ERR_INVALID_ARG;
  tc::set_wait_budget_ns(budget_ns);
  return MOE_OK;
}

moe_status moe_set_wait_stall(int32_t on) {
  if (on != 0 && on != 1) return MOE_ERR_INVALID_ARG;
  tc::set_wait_stall(on);
  return MOE_OK;
}

moe_status moe_read_status(moe_stream_t stream, void* scratch) {
  if (!scratch) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, scratch, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word != 0) {
    if (cudaMemset(scratch, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_ERR_DEVICE_TIMEOUT;
  }
  return MOE_OK;
}

const char* moe_last_cuda_error(void) { return g_last_cuda_error; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
