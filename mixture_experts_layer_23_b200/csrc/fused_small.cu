// Whole forward of a small MoE layer in one launch (router, capacity dispatch, experts, combine).
//
// Tutorial ch.4 "分布式训练", section "框架": Tutel runs the whole MoE layer as one fused kernel;
// the four steps of section "专家并行" part 二 (gate, send to the experts, expert MLPs, return in
// token order) are the same as on the multi-kernel path.  For layers whose routing is a few
// thousand multiply-adds per token slice, launch latency and the hand-offs between five or six
// kernels dominate; here one kernel does it all.
//
// No grid-wide synchronisation: every CTA recomputes the routing of ALL T tokens -- cheap under
// the size limits below -- so each CTA knows which of its own tokens' assignments survive the
// capacity cut without waiting for any other CTA:
//   1. thread per token: the E logits from the token's row (read in 32-element slices held in
//      registers) against Wg staged in shared memory, fed in expert order to the serial softmax
//      + top-k of route_serial.cuh;
//   2. capacity ranks in priority order (token order, or choice-major by layers j): per expert a
//      warp ballot gives the rank inside the warp, warp totals in shared memory give the rest;
//   3. this CTA's tokens, token by token, through their kept experts (in choice order) and the
//      shared experts: thread per output row of W1 (W3) with the token row in shared memory, the
//      activation, then thread per output column of W2; y_t accumulates g_tj o_tj in order.
// CTA 0 also writes the routing (topk_idx, topk_w, counts) when the caller asks for it.  Bitwise
// deterministic.  Writes no state for a backward pass (inference).
#include "common.cuh"
#include "launch.h"
#include "route_serial.cuh"

namespace moe {
namespace {

constexpr int FS_THREADS = 256;
constexpr int FS_MAX_E = 32;

template <typename T>
__global__ void __launch_bounds__(FS_THREADS)
fused_small_fwd_kernel(const T* __restrict__ x, const T* __restrict__ Wg,
                       const float* __restrict__ bias, const T* __restrict__ W1,
                       const T* __restrict__ W3, const T* __restrict__ W2, int T_, int d, int E,
                       int k, int F, int S, int act, int gate_norm, int choice_major, int64_t C,
                       int tok_per_cta, T* __restrict__ y, int32_t* __restrict__ topk_idx_out,
                       float* __restrict__ topk_w_out, int32_t* __restrict__ counts_out) {
  pdl_prologue();
  extern __shared__ float fs_smem[];
  float* wg = fs_smem;                                               // [E, d] gate matrix
  int32_t* sidx = reinterpret_cast<int32_t*>(wg + (size_t)E * d);    // [T, k] expert ids
  float* sw = reinterpret_cast<float*>(sidx + (size_t)T_ * k);       // [T, k] gate weights
  int32_t* spos = reinterpret_cast<int32_t*>(sw + (size_t)T_ * k);   // [T, k] rank or -1
  float* xs = reinterpret_cast<float*>(spos + (size_t)T_ * k);       // [d] token row
  float* hs = xs + d;                                                // [F] activation
  float* acc = hs + F;                                               // [d] y accumulator
  __shared__ int32_t wcnt[FS_THREADS / 32][FS_MAX_E];                // per-warp expert counts
  __shared__ int32_t run[FS_MAX_E];                                  // running expert totals
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int q = tid; q < E * d; q += FS_THREADS) wg[q] = to_f(Wg[q]);
  __syncthreads();
  // 1. routing, thread per token
  for (int t = tid; t < T_; t += FS_THREADS) {
    const T* xr = x + (int64_t)t * d;
    float lg[FS_MAX_E];
#pragma unroll
    for (int e = 0; e < FS_MAX_E; ++e) lg[e] = 0.f;
    for (int i0 = 0; i0 < d; i0 += 32) {
      float xv[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) xv[i] = (i0 + i < d) ? to_f(xr[i0 + i]) : 0.f;
#pragma unroll
      for (int e = 0; e < FS_MAX_E; ++e)
        if (e < E)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i0 + i < d) lg[e] = fmaf(xv[i], wg[e * d + i0 + i], lg[e]);
    }
    TopK8 st;
    topk_init(st);
#pragma unroll
    for (int e = 0; e < FS_MAX_E; ++e)
      if (e < E) {
        lg[e] += bias ? bias[e] : 0.f;
        topk_push(st, lg[e], e);
      }
    float den = 0.f;
    if (gate_norm == 0)
#pragma unroll
      for (int e = 0; e < FS_MAX_E; ++e)
        if (e < E) den += softmax_term(st, lg[e]);
    topk_finish(st, k, gate_norm, den, sidx + (size_t)t * k, sw + (size_t)t * k);
  }
  if (tid < FS_MAX_E) run[tid] = 0;
  __syncthreads();
  // 2. capacity ranks: layers in priority order (one layer of all choices for token order, one
  //    per choice index for choice-major), tokens in chunks of FS_THREADS, a ballot per expert
  const int L = choice_major ? k : 1;
  for (int layer = 0; layer < L; ++layer) {
    for (int c0 = 0; c0 < T_; c0 += FS_THREADS) {
      const int t = c0 + tid;
      const int j0 = choice_major ? layer : 0, j1 = choice_major ? layer + 1 : k;
      const uint32_t below = (1u << lane) - 1u;
      // per expert: which lanes (tokens) hold it in this layer; a token holds an expert at most
      // once, so its in-warp rank for that choice is the count of lower lanes holding it
      for (int e = 0; e < E; ++e) {
        int hit = -1;
        if (t < T_)
          for (int j = j0; j < j1; ++j)
            if (sidx[(size_t)t * k + j] == e) hit = j;
        const uint32_t m = __ballot_sync(0xffffffffu, hit >= 0);
        if (hit >= 0) spos[(size_t)t * k + hit] = __popc(m & below);
        if (lane == 0) wcnt[warp][e] = __popc(m);
      }
      __syncthreads();
      if (t < T_)
        for (int j = j0; j < j1; ++j) {
          const int e = sidx[(size_t)t * k + j];
          int rank = run[e] + spos[(size_t)t * k + j];
          for (int w = 0; w < warp; ++w) rank += wcnt[w][e];
          spos[(size_t)t * k + j] = (int64_t)rank < C ? rank : -1;
        }
      __syncthreads();
      if (tid < E) {
        int tot = 0;
        for (int w = 0; w < FS_THREADS / 32; ++w) tot += wcnt[w][tid];
        run[tid] += tot;
      }
      __syncthreads();
    }
  }
  if (blockIdx.x == 0 && counts_out && tid < E) counts_out[tid] = run[tid];
  if (blockIdx.x == 0 && topk_idx_out)
    for (int q = tid; q < T_ * k; q += FS_THREADS) {
      topk_idx_out[q] = sidx[q];
      topk_w_out[q] = sw[q];
    }

  // 3. experts and combine for this CTA's tokens
  const int t0 = blockIdx.x * tok_per_cta;
  const int t1 = min(t0 + tok_per_cta, T_);
  const bool swiglu = act == MOE_ACT_SWIGLU;
  for (int t = t0; t < t1; ++t) {
    for (int i = tid; i < d; i += FS_THREADS) {
      xs[i] = to_f(x[(int64_t)t * d + i]);
      acc[i] = 0.f;
    }
    __syncthreads();
    // kept routed choices in order j = 0..k-1, then the shared experts (weight 1)
    for (int c = 0; c < k + S; ++c) {
      int e;
      float g;
      if (c < k) {
        if (spos[(size_t)t * k + c] < 0) continue;   // dropped: contributes nothing
        e = sidx[(size_t)t * k + c];
        g = sw[(size_t)t * k + c];
      } else {
        e = E + (c - k);
        g = 1.f;
      }
      for (int f = tid; f < F; f += FS_THREADS) {
        const T* w1 = W1 + ((int64_t)e * F + f) * d;
        float u = 0.f, v = 0.f;
#pragma unroll 8
        for (int i = 0; i < d; i += 16 / (int)sizeof(T)) {   // 16-byte loads, 8 in flight
          const Vec16<T> a = ld_vec(w1 + i);
#pragma unroll
          for (int q = 0; q < Vec16<T>::N; ++q) u = fmaf(a.get(q), xs[i + q], u);
        }
        if (swiglu) {
          const T* w3 = W3 + ((int64_t)e * F + f) * d;
#pragma unroll 8
          for (int i = 0; i < d; i += 16 / (int)sizeof(T)) {
            const Vec16<T> a = ld_vec(w3 + i);
#pragma unroll
            for (int q = 0; q < Vec16<T>::N; ++q) v = fmaf(a.get(q), xs[i + q], v);
          }
        }
        hs[f] = swiglu ? u * sigmoid_f(u) * v : gelu_f(u);
      }
      __syncthreads();
      for (int i = tid; i < d; i += FS_THREADS) {
        const T* w2 = W2 + ((int64_t)e * d + i) * F;
        float o = 0.f;
#pragma unroll 8
        for (int f = 0; f < F; f += 16 / (int)sizeof(T)) {
          const Vec16<T> a = ld_vec(w2 + f);
#pragma unroll
          for (int q = 0; q < Vec16<T>::N; ++q) o = fmaf(a.get(q), hs[f + q], o);
        }
        acc[i] = fmaf(g, o, acc[i]);
      }
      __syncthreads();
    }
    for (int i = tid; i < d; i += FS_THREADS) y[(int64_t)t * d + i] = from_f<T>(acc[i]);
    __syncthreads();
  }
}

}  // namespace

size_t fused_small_smem_bytes(const Dims& D) {
  return sizeof(float) * ((size_t)D.E * D.d + 3 * (size_t)D.T * D.k + 2 * (size_t)D.d + D.F);
}

// Shapes the fused path takes: at most 32 experts, the redundant routing of all T tokens per CTA
// small (T E d <= 2^19 multiply-adds), and the routing state within shared memory.
bool fused_small_supported(const Dims& D) {
  return D.E <= FS_MAX_E && (int64_t)D.T * D.E * D.d <= (1 << 19) &&
         fused_small_smem_bytes(D) <= 160 * 1024;
}

moe_status launch_fused_small_fwd(const Dims& D, const void* x, const void* Wg, const float* bias,
                                  const void* W1, const void* W3, const void* W2, void* y,
                                  int32_t* topk_idx, float* topk_w, int32_t* counts,
                                  cudaStream_t st) {
  const size_t sm = fused_small_smem_bytes(D);
  const int tok_per_cta = (D.T + 147) / 148 < 1 ? 1 : (D.T + 147) / 148;
  const int grid = (D.T + tok_per_cta - 1) / tok_per_cta;
  const float* b = D.has_bias ? bias : nullptr;
  if (D.dtype == MOE_DTYPE_BF16) {
    using T = __nv_bfloat16;
    auto kern = fused_small_fwd_kernel<T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return MOE_ERR_CUDA;
    return launch_k(kern, grid, FS_THREADS, sm, st, 1, (const T*)x, (const T*)Wg, b, (const T*)W1,
                    (const T*)W3, (const T*)W2, D.T, D.d, D.E, D.k, D.F, D.S, D.act, D.gate_norm,
                    D.choice_major, D.C, tok_per_cta, (T*)y, topk_idx, topk_w, counts);
  }
  auto kern = fused_small_fwd_kernel<float>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_k(kern, grid, FS_THREADS, sm, st, 1, (const float*)x, (const float*)Wg, b,
                  (const float*)W1, (const float*)W3, (const float*)W2, D.T, D.d, D.E, D.k, D.F,
                  D.S, D.act, D.gate_norm, D.choice_major, D.C, tok_per_cta, (float*)y, topk_idx,
                  topk_w, counts);
}

}  // namespace moe
