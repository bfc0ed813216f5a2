// Combine (forward) and its backward.
//
// Step 4 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 4: expert results return to their tokens and the sequence order is restored).  Here the
// return trip is a gather: each token reads its kept expert rows and sums them with its gate
// weights, in a fixed order (j ascending, then shared experts), so no atomics are needed and the
// result is bit-reproducible.  The backward kernel is the same gather run in reverse (section
// "专家并行与数据并行的结合", part 三.3: gradients are routed back to the experts): for each kept
// assignment it forms dg = <dy_t, O_row> and writes dO_row = g * dy_t; with every dg of the token
// in hand it then runs the softmax backward of the router and writes the token's logit gradient.
#include "common.cuh"

namespace moe {
namespace {

template <typename T>
__global__ void __launch_bounds__(256)
combine_fwd_kernel(const T* __restrict__ O, const int32_t* __restrict__ slot,
                   const float* __restrict__ topk_w, int T_, int d, int k, int S, int64_t T_pad,
                   T* __restrict__ y) {
  constexpr int VN = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T_) return;
  int my_s = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_s = slot[(int64_t)t * k + lane];
    my_w = topk_w[(int64_t)t * k + lane];
  }
  int s[8];
  float w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s[j] = __shfl_sync(0xffffffffu, my_s, j);
    w[j] = __shfl_sync(0xffffffffu, my_w, j);
  }
  const int nv = d / VN;
  for (int v = lane; v < nv; v += 32) {
    float acc[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && s[j] >= 0) {
        const Vec16<T> o = ld_vec_stream(O + (int64_t)s[j] * d + (int64_t)v * VN);
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = fmaf(w[j], o.get(i), acc[i]);
      }
    }
    for (int sh = 0; sh < S; ++sh) {
      const Vec16<T> o = ld_vec_stream(O + ((int64_t)sh * T_pad + t) * d + (int64_t)v * VN);
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] += o.get(i);
    }
    Vec16<T> out;
#pragma unroll
    for (int i = 0; i < VN; ++i) out.set(i, acc[i]);
    st_vec(y + (int64_t)t * d + (int64_t)v * VN, out);
  }
}

// Softmax backward of one token (warp-cooperative), from its logits row and every lane holding
// dg[0..k-1] (0 at dropped assignments):
//   gate_norm 0: p = softmax(l), dp[e] = sum_j [idx_j = e] dg_j, dl = p * (dp - <p, dp>)
//   gate_norm 1: w = topk_w, dl[idx_j] = w_j * (dg_j - <w, dg>), 0 elsewhere
// No gradient flows through the chosen indices.  Writes the E floats of dl.
__device__ __forceinline__ void dlogits_row(const float* __restrict__ lrow, const int (&e)[8],
                                            const float (&w)[8], const float (&g)[8], int E,
                                            int k, int gate_norm, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  if (gate_norm == 0) {
    float l[8];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      l[i] = (ee < E) ? lrow[ee] : -INFINITY;
      m = fmaxf(m, l[i]);
    }
    m = warp_max(m);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      l[i] = (ee < E) ? expf(l[i] - m) : 0.f;
      s += l[i];
    }
    s = warp_sum(s);
    const float inv = 1.f / s;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      float dp = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && e[j] == ee) dp += g[j];
      l[i] *= inv;       // p
      dot += l[i] * dp;
    }
    dot = warp_sum(dot);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      if (ee < E) {
        float dp = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && e[j] == ee) dp += g[j];
        out[ee] = l[i] * (dp - dot);
      }
    }
  } else {
    float wd = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) wd += w[j] * g[j];
    for (int ee = lane; ee < E; ee += 32) {
      float v = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && e[j] == ee) v = w[j] * (g[j] - wd);
      out[ee] = v;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
combine_bwd_kernel(const T* __restrict__ dy, const T* __restrict__ O,
                   const int32_t* __restrict__ slot, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ topk_idx, const float* __restrict__ logits,
                   const int32_t* __restrict__ kept, const int32_t* __restrict__ offsets, int T_,
                   int d, int E, int k, int gate_norm, int n_tok_blocks, float* __restrict__ dg,
                   float* __restrict__ dlogits, T* __restrict__ dO) {
  constexpr int VN = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int nv = d / VN;
  if ((int)blockIdx.x >= n_tok_blocks) {  // zero the padding rows of expert e in dO
    const int e = blockIdx.x - n_tok_blocks;
    const int r0 = offsets[e] + kept[e], r1 = offsets[e + 1];
    Vec16<T> z;
    z.raw = make_uint4(0, 0, 0, 0);
    for (int r = r0 + (threadIdx.x >> 5); r < r1; r += 8)
      for (int v = lane; v < nv; v += 32) st_vec(dO + (int64_t)r * d + (int64_t)v * VN, z);
    return;
  }
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T_) return;
  int my_s = -1, my_e = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_s = slot[(int64_t)t * k + lane];
    my_w = topk_w[(int64_t)t * k + lane];
    my_e = topk_idx[(int64_t)t * k + lane];
  }
  int s[8], ej[8];
  float w[8], part[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s[j] = __shfl_sync(0xffffffffu, my_s, j);
    w[j] = __shfl_sync(0xffffffffu, my_w, j);
    ej[j] = __shfl_sync(0xffffffffu, my_e, j);
    part[j] = 0.f;
  }
  for (int v = lane; v < nv; v += 32) {
    const Vec16<T> g = ld_vec_stream(dy + (int64_t)t * d + (int64_t)v * VN);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && s[j] >= 0) {
        const Vec16<T> o = ld_vec_stream(O + (int64_t)s[j] * d + (int64_t)v * VN);
        Vec16<T> out;
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          part[j] = fmaf(g.get(i), o.get(i), part[j]);
          out.set(i, w[j] * g.get(i));
        }
        st_vec(dO + (int64_t)s[j] * d + (int64_t)v * VN, out);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) part[j] = (s[j] >= 0) ? warp_sum(part[j]) : 0.f;
  if (lane < k) {
    float mine = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j == lane) mine = part[j];
    dg[(int64_t)t * k + lane] = mine;
  }
  dlogits_row(logits + (int64_t)t * E, ej, w, part, E, k, gate_norm, dlogits + (int64_t)t * E);
}

}  // namespace

moe_status launch_combine(const Dims& D, const void* O, const int32_t* slot, const float* topk_w,
                          void* y, cudaStream_t st) {
  const int grid = (D.T + 7) / 8;
  if (D.dtype == MOE_DTYPE_BF16)
    combine_fwd_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)O, slot, topk_w, D.T, D.d, D.k, D.S, D.T_pad, (__nv_bfloat16*)y);
  else
    combine_fwd_kernel<float><<<grid, 256, 0, st>>>((const float*)O, slot, topk_w, D.T, D.d, D.k,
                                                    D.S, D.T_pad, (float*)y);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_combine_bwd(const Dims& D, const void* dy, const void* O, const int32_t* slot,
                              const float* topk_w, const int32_t* topk_idx, const float* logits,
                              const int32_t* kept, const int32_t* offsets, float* dg,
                              float* dlogits, void* dO, cudaStream_t st) {
  const int n_tok_blocks = (D.T + 7) / 8;
  const int grid = n_tok_blocks + D.E;
  if (D.dtype == MOE_DTYPE_BF16)
    combine_bwd_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)dy, (const __nv_bfloat16*)O, slot, topk_w, topk_idx, logits, kept,
        offsets, D.T, D.d, D.E, D.k, D.gate_norm, n_tok_blocks, dg, dlogits, (__nv_bfloat16*)dO);
  else
    combine_bwd_kernel<float><<<grid, 256, 0, st>>>(
        (const float*)dy, (const float*)O, slot, topk_w, topk_idx, logits, kept, offsets, D.T,
        D.d, D.E, D.k, D.gate_norm, n_tok_blocks, dg, dlogits, (float*)dO);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
