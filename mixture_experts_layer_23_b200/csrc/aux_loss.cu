// Auxiliary load-balancing loss of the router, forward.
//
// Ch.4 "分布式训练": section "框架" (DeepSpeed's `loss_coef`, the load-balancing loss
// coefficient), section "实践" part 四 (`aux_loss_factor`) and part 七.3 (the auxiliary loss
// should sit near 0 with every expert chosen about equally often).  The pages give no formula;
// the reading taken is
//   loss = coef * E * sum_e f_e * P_e,   f_e = counts[e] / (T k),   P_e = mean_t softmax(l_t)[e]
// (counts before the capacity drop, softmax over all E logits whatever the gate normalisation).
// Its gradient, coef * E / T * p_t * (f - <p_t, f>), is added to dlogits by the combine
// backward (combine.cu).
//
// Two fixed-order levels, so the loss is bitwise reproducible: each CTA sums the probabilities
// of its token chunk (warp per token, lanes over experts; the CTA's eight warps are then summed
// in warp order), and one CTA adds the chunk partials in chunk order and reduces over experts.
#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int AX_THREADS = 256;

__global__ void __launch_bounds__(AX_THREADS)
aux_prob_partial_kernel(const float* __restrict__ logits, int T_, int E, int chunk,
                        float* __restrict__ part) {
  pdl_prologue();
  __shared__ float red[AX_THREADS / 32][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int t0 = blockIdx.x * chunk;
  const int t1 = min(t0 + chunk, T_);
  for (int t = t0 + warp; t < t1; t += AX_THREADS / 32) {
    const float* row = logits + (int64_t)t * E;
    float l[8];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      l[i] = (e < E) ? row[e] : -INFINITY;
      m = fmaxf(m, l[i]);
    }
    m = warp_max(m);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      l[i] = (e < E) ? expf(l[i] - m) : 0.f;
      s += l[i];
    }
    s = warp_sum(s);
    const float inv = 1.f / s;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += l[i] * inv;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e < E) red[warp][e] = acc[i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += AX_THREADS) {
    float v = 0.f;
    for (int w = 0; w < AX_THREADS / 32; ++w) v += red[w][e];
    part[(int64_t)blockIdx.x * E + e] = v;
  }
}

__global__ void __launch_bounds__(AX_THREADS)
aux_loss_final_kernel(const float* __restrict__ part, int n_chunk, const int32_t* __restrict__ counts,
                      int T_, int E, int k, float coef, float* __restrict__ loss) {
  pdl_prologue();
  __shared__ float red[AX_THREADS];
  const int e = threadIdx.x;
  float v = 0.f;
  if (e < E) {
    float P = 0.f;
    for (int c = 0; c < n_chunk; ++c) P += part[(int64_t)c * E + e];
    P /= (float)T_;
    const float f = (float)counts[e] / ((float)T_ * (float)k);
    v = f * P;
  }
  red[e] = v;
  __syncthreads();
  for (int h = AX_THREADS / 2; h > 0; h >>= 1) {
    if (e < h) red[e] += red[e + h];
    __syncthreads();
  }
  if (e == 0) loss[0] = coef * (float)E * red[0];
}

}  // namespace

moe_status launch_aux_loss(const Dims& D, const float* logits, const int32_t* counts, float* part,
                           float* loss, cudaStream_t st) {
  const int chunk = (D.T + D.n_aux - 1) / D.n_aux;
  const int n_chunk = (D.T + chunk - 1) / chunk;
  MOE_TRY_S(launch_k(aux_prob_partial_kernel, n_chunk, AX_THREADS, 0, st, 1, logits, D.T, D.E,
                     chunk, part));
  return launch_k(aux_loss_final_kernel, 1, AX_THREADS, 0, st, 1, (const float*)part, n_chunk,
                  counts, D.T, D.E, D.k, D.aux_coef, loss);
}

}  // namespace moe
