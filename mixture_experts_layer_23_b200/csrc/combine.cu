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

// y_t = sum_j w_j O[slot_j] + sum_s O[s * T_pad + t].  KS >= k + S (a power of two): the
// token's rows are gathered U = max(1, 8 / KS) vectors per lane at a time, all loads in flight
// before the sums.
// Occupancy: 4 CTAs of 256 threads per SM (64 registers) keep a whole T / 8 grid resident in one
// wave for T up to 4736, where 3 (the register count unconstrained) left a tail wave; the
// 16-row form stays at 2 CTAs (it would spill).
template <typename T, int KS>
__global__ void __launch_bounds__(256, KS >= 16 ? 2 : 4)
combine_fwd_kernel(const T* __restrict__ O, const int32_t* __restrict__ slot,
                   const float* __restrict__ topk_w, int T_, int d, int k, int S, int64_t T_pad,
                   T* __restrict__ y) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int U = KS >= 8 ? 1 : 8 / KS;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T_) return;
  // row list: k routed slots (weight topk_w, -1 if dropped) then S shared rows (weight 1)
  int my_s = -1;
  float my_w = 0.f;
  if (lane < k) {
    my_s = slot[(int64_t)t * k + lane];
    my_w = topk_w[(int64_t)t * k + lane];
  } else if (lane < k + S) {
    my_s = (int)((int64_t)(lane - k) * T_pad + t);
    my_w = 1.f;
  }
  int s[KS];
  float w[KS];
#pragma unroll
  for (int j = 0; j < KS; ++j) {
    s[j] = __shfl_sync(0xffffffffu, my_s, j);
    w[j] = __shfl_sync(0xffffffffu, my_w, j);
    if (j >= k + S) s[j] = -1;
  }
  const int nv = d / VN;
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    Vec16<T> o[U][KS];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        const int v = v0 + 32 * u;
        if (v < nv && s[j] >= 0) o[u][j] = ld_vec_stream(O + (int64_t)s[j] * d + (int64_t)v * VN);
      }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v >= nv) break;
      float acc[VN];
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < KS; ++j)
        if (s[j] >= 0) {
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[i] = fmaf(w[j], o[u][j].get(i), acc[i]);
        }
      Vec16<T> out;
#pragma unroll
      for (int i = 0; i < VN; ++i) out.set(i, acc[i]);
      st_vec(y + (int64_t)t * d + (int64_t)v * VN, out);
    }
  }
}

// Softmax backward of one token (warp-cooperative), from its logits row and every lane holding
// dg[0..k-1] (0 at dropped assignments):
//   gate_norm 0: p = softmax(l), dp[e] = sum_j [idx_j = e] dg_j, dl = p * (dp - <p, dp>)
//   gate_norm 1: w = topk_w, dl[idx_j] = w_j * (dg_j - <w, dg>), 0 elsewhere
// No gradient flows through the chosen indices.  With aux_scale = coef * E / T > 0 the gradient
// of the load-balancing loss, aux_scale * p * (f - <p, f>) with p the full softmax of the row and
// f_e = counts[e] * inv_Tk, is added.  Writes the E floats of dl, and when out16 is given also
// their bf16 copy with the row padded by zeros to E8 entries.
__device__ __forceinline__ void dlogits_row(const float* __restrict__ lrow, const int (&e)[8],
                                            const float (&w)[8], const float (&g)[8], int E,
                                            int k, int gate_norm, float* __restrict__ out,
                                            __nv_bfloat16* __restrict__ out16, int E8,
                                            const int32_t* __restrict__ counts, float aux_scale,
                                            float inv_Tk) {
  const int lane = threadIdx.x & 31;
  if (out16 != nullptr)
    for (int ee = E + lane; ee < E8; ee += 32) out16[ee] = __float2bfloat16_rn(0.f);
  float extra[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) extra[i] = 0.f;
  if (aux_scale > 0.f) {
    float p[8], f[8];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      p[i] = (ee < E) ? lrow[ee] : -INFINITY;
      f[i] = (ee < E) ? (float)counts[ee] * inv_Tk : 0.f;
      m = fmaxf(m, p[i]);
    }
    m = warp_max(m);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      p[i] = (ee < E) ? expf(p[i] - m) : 0.f;
      s += p[i];
    }
    s = warp_sum(s);
    const float inv = 1.f / s;
    float pf = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      p[i] *= inv;
      pf += p[i] * f[i];
    }
    pf = warp_sum(pf);
#pragma unroll
    for (int i = 0; i < 8; ++i) extra[i] = aux_scale * p[i] * (f[i] - pf);
  }
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
        const float v = l[i] * (dp - dot) + extra[i];
        out[ee] = v;
        if (out16 != nullptr) out16[ee] = __float2bfloat16_rn(v);
      }
    }
  } else {
    float wd = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k) wd += w[j] * g[j];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      if (ee >= E) break;
      float v = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && e[j] == ee) v = w[j] * (g[j] - wd);
      v += extra[i];
      out[ee] = v;
      if (out16 != nullptr) out16[ee] = __float2bfloat16_rn(v);
    }
  }
}

template <typename T, int KS>
__global__ void __launch_bounds__(256, 4)
combine_bwd_kernel(const T* __restrict__ dy, const T* __restrict__ O,
                   const int32_t* __restrict__ slot, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ topk_idx, const float* __restrict__ logits,
                   const int32_t* __restrict__ kept, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ counts, float aux_scale, float inv_Tk, int T_,
                   int d, int E, int k, int gate_norm, int n_tok_blocks, float* __restrict__ dg,
                   float* __restrict__ dlogits, __nv_bfloat16* __restrict__ dl16, int E8,
                   T* __restrict__ dO) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int U = KS >= 8 ? 1 : 8 / KS;
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
    if (j >= k) s[j] = -1;
    part[j] = 0.f;
  }
  for (int v0 = lane; v0 < nv; v0 += 32 * U) {
    Vec16<T> g[U], o[U][KS];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v < nv) {
        g[u] = ld_vec_stream(dy + (int64_t)t * d + (int64_t)v * VN);
#pragma unroll
        for (int j = 0; j < KS; ++j)
          if (s[j] >= 0) o[u][j] = ld_vec_stream(O + (int64_t)s[j] * d + (int64_t)v * VN);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + 32 * u;
      if (v >= nv) break;
#pragma unroll
      for (int j = 0; j < KS; ++j) {
        if (s[j] >= 0) {
          Vec16<T> out;
#pragma unroll
          for (int i = 0; i < VN; ++i) {
            part[j] = fmaf(g[u].get(i), o[u][j].get(i), part[j]);
            out.set(i, w[j] * g[u].get(i));
          }
          st_vec(dO + (int64_t)s[j] * d + (int64_t)v * VN, out);
        }
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
  dlogits_row(logits + (int64_t)t * E, ej, w, part, E, k, gate_norm, dlogits + (int64_t)t * E,
              dl16 ? dl16 + (int64_t)t * E8 : nullptr, E8, counts, aux_scale, inv_Tk);
}

}  // namespace

// smallest power of two >= n (n <= 16)
static inline int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

template <typename T, int KS>
static moe_status combine_t(const Dims& D, const void* O, const int32_t* slot, const float* topk_w,
                            void* y, cudaStream_t st) {
  return launch_k(combine_fwd_kernel<T, KS>, (D.T + 7) / 8, 256, 0, st, 1, (const T*)O, slot,
                  topk_w, D.T, D.d, D.k, D.S, D.T_pad, (T*)y);
}
template <typename T>
static moe_status combine_ks(const Dims& D, const void* O, const int32_t* slot,
                             const float* topk_w, void* y, cudaStream_t st) {
  switch (pow2_at_least(D.k + D.S)) {
    case 1: case 2: return combine_t<T, 2>(D, O, slot, topk_w, y, st);
    case 4: return combine_t<T, 4>(D, O, slot, topk_w, y, st);
    case 8: return combine_t<T, 8>(D, O, slot, topk_w, y, st);
    default: return combine_t<T, 16>(D, O, slot, topk_w, y, st);
  }
}

moe_status launch_combine(const Dims& D, const void* O, const int32_t* slot, const float* topk_w,
                          void* y, cudaStream_t st) {
  if (D.dtype == MOE_DTYPE_BF16) return combine_ks<__nv_bfloat16>(D, O, slot, topk_w, y, st);
  return combine_ks<float>(D, O, slot, topk_w, y, st);
}

template <typename T, int KS>
static moe_status combine_bwd_t(const Dims& D, const void* dy, const void* O, const int32_t* slot,
                                const float* topk_w, const int32_t* topk_idx,
                                const float* logits, const int32_t* kept, const int32_t* offsets,
                                const int32_t* counts, float* dg, float* dlogits,
                                __nv_bfloat16* dl16, void* dO, cudaStream_t st) {
  const int n_tok_blocks = (D.T + 7) / 8;
  return launch_k(combine_bwd_kernel<T, KS>, n_tok_blocks + D.E, 256, 0, st, 1, (const T*)dy,
                  (const T*)O, slot, topk_w, topk_idx, logits, kept, offsets, counts,
                  D.aux_coef > 0.f ? D.aux_coef * (float)D.E / (float)D.T : 0.f,
                  1.f / ((float)D.T * (float)D.k), D.T, D.d, D.E, D.k,
                  D.gate_norm, n_tok_blocks, dg, dlogits, dl16, (int)round_up(D.E, 8), (T*)dO);
}
template <typename T>
static moe_status combine_bwd_ks(const Dims& D, const void* dy, const void* O, const int32_t* slot,
                                 const float* topk_w, const int32_t* topk_idx,
                                 const float* logits, const int32_t* kept,
                                 const int32_t* offsets, const int32_t* counts, float* dg,
                                 float* dlogits, __nv_bfloat16* dl16, void* dO, cudaStream_t st) {
  switch (pow2_at_least(D.k)) {
    case 1: case 2:
      return combine_bwd_t<T, 2>(D, dy, O, slot, topk_w, topk_idx, logits, kept, offsets,
                                 counts, dg, dlogits, dl16, dO, st);
    case 4:
      return combine_bwd_t<T, 4>(D, dy, O, slot, topk_w, topk_idx, logits, kept, offsets,
                                 counts, dg, dlogits, dl16, dO, st);
    default:
      return combine_bwd_t<T, 8>(D, dy, O, slot, topk_w, topk_idx, logits, kept, offsets,
                                 counts, dg, dlogits, dl16, dO, st);
  }
}

moe_status launch_combine_bwd(const Dims& D, const void* dy, const void* O, const int32_t* slot,
                              const float* topk_w, const int32_t* topk_idx, const float* logits,
                              const int32_t* kept, const int32_t* offsets, const int32_t* counts,
                              float* dg, float* dlogits, __nv_bfloat16* dl16, void* dO,
                              cudaStream_t st) {
  if (D.dtype == MOE_DTYPE_BF16)
    return combine_bwd_ks<__nv_bfloat16>(D, dy, O, slot, topk_w, topk_idx, logits, kept, offsets,
                                         counts, dg, dlogits, dl16, dO, st);
  return combine_bwd_ks<float>(D, dy, O, slot, topk_w, topk_idx, logits, kept, offsets, counts, dg,
                               dlogits, dl16, dO, st);
}

}  // namespace moe
