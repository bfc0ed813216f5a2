// Router: gate logits, softmax and top-k, fused in one kernel.
//
// Step 1 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 1: a small router, replicated on every device, gates the local tokens).  The top-k gate is
// the Tutel gate_type {'type': 'top', 'k': ...} of section "框架".
//
// One CTA owns 64 tokens: it computes their [64 x E] logit tile on CUDA cores (fp32 FMA, x and
// Wg staged through shared memory), adds the constant bias, writes the logits, and then each warp
// runs softmax and a warp-shuffle top-k over its tokens' rows straight from shared memory.
#include "common.cuh"

namespace moe {
namespace {

constexpr int RT_TOK = 64;   // tokens per CTA
constexpr int RT_EC = 64;    // experts per GEMM pass
constexpr int RT_BK = 32;    // d per smem stage
constexpr int RT_THREADS = 256;

// Top-k + gate weights of one token whose E logits are readable at `row` (smem or global).
// Lane l holds logits l, l+32, ...  Selection key: larger logit first, equal logits -> lower
// expert index.  Writes topk_idx / topk_w for this token.
__device__ __forceinline__ void topk_row(const float* row, int E, int k, int gate_norm,
                                         int32_t* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? row[e] : -INFINITY;
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, v[i]);
  m = warp_max(m);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e < E) s += expf(v[i] - m);
  }
  s = warp_sum(s);

  float chosen_l[8];
  int chosen_e[8];
  for (int j = 0; j < k; ++j) {
    // lane-local best among untaken entries (entries scan in increasing expert index)
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u)) {
        if (v[i] > bv || (v[i] == bv && e < be)) { bv = v[i]; be = e; }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    chosen_l[j] = bv;
    chosen_e[j] = be;
  }
  if (lane == 0) {
    if (gate_norm == 0) {
      for (int j = 0; j < k; ++j) {
        idx_out[j] = chosen_e[j];
        w_out[j] = expf(chosen_l[j] - m) / s;
      }
    } else {
      float z = 0.f;
      for (int j = 0; j < k; ++j) z += expf(chosen_l[j] - chosen_l[0]);
      for (int j = 0; j < k; ++j) {
        idx_out[j] = chosen_e[j];
        w_out[j] = expf(chosen_l[j] - chosen_l[0]) / z;
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(RT_THREADS)
router_fwd_kernel(const T* __restrict__ x, const T* __restrict__ Wg,
                  const float* __restrict__ bias, int T_, int d, int E, int k, int gate_norm,
                  float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                  float* __restrict__ topk_w) {
  extern __shared__ float smem[];
  float* xs = smem;                                // [RT_BK][RT_TOK + 4] (k-major)
  float* ws = xs + RT_BK * (RT_TOK + 4);           // [RT_BK][RT_EC + 4]
  float* ls = ws + RT_BK * (RT_EC + 4);            // [RT_TOK][E + 1]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * RT_TOK;
  const int tx = tid & 15, ty = tid >> 4;          // 16 x 16 threads, 4 x 4 outputs each

  for (int e0 = 0; e0 < E; e0 += RT_EC) {
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += RT_BK) {
      // stage x[t0:t0+64, k0:k0+32] and Wg[e0:e0+64, k0:k0+32] transposed (k-major)
      for (int i = tid; i < RT_TOK * RT_BK; i += RT_THREADS) {
        const int r = i / RT_BK, c = i % RT_BK;
        const int t = t0 + r, kk = k0 + c;
        xs[c * (RT_TOK + 4) + r] = (t < T_ && kk < d) ? to_f(x[(int64_t)t * d + kk]) : 0.f;
        const int e = e0 + r;
        ws[c * (RT_EC + 4) + r] = (e < E && kk < d) ? to_f(Wg[(int64_t)e * d + kk]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int c = 0; c < RT_BK; ++c) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = xs[c * (RT_TOK + 4) + ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = ws[c * (RT_EC + 4) + tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = e0 + tx * 4 + j;
        if (e < E) ls[(ty * 4 + i) * (E + 1) + e] = acc[i][j] + (bias ? bias[e] : 0.f);
      }
  }
  __syncthreads();

  // logits out (row-major, coalesced along E)
  for (int i = tid; i < RT_TOK * E; i += RT_THREADS) {
    const int r = i / E, e = i % E;
    if (t0 + r < T_) logits[(int64_t)(t0 + r) * E + e] = ls[r * (E + 1) + e];
  }
  const int warp = tid >> 5;
  for (int r = warp; r < RT_TOK; r += RT_THREADS / 32) {
    const int t = t0 + r;
    if (t >= T_) break;
    topk_row(ls + r * (E + 1), E, k, gate_norm, topk_idx + (int64_t)t * k, topk_w + (int64_t)t * k);
  }
}

__global__ void topk_from_logits_kernel(const float* __restrict__ logits, int T_, int E, int k,
                                        int gate_norm, int32_t* __restrict__ topk_idx,
                                        float* __restrict__ topk_w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= T_) return;
  topk_row(logits + (int64_t)warp * E, E, k, gate_norm, topk_idx + (int64_t)warp * k,
           topk_w + (int64_t)warp * k);
}

}  // namespace

size_t router_smem_bytes(int E) {
  return sizeof(float) * (RT_BK * (RT_TOK + 4) + RT_BK * (RT_EC + 4) + RT_TOK * (E + 1));
}

moe_status launch_router(const Dims& D, const void* x, const void* Wg, const float* bias,
                         float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  const int grid = (D.T + RT_TOK - 1) / RT_TOK;
  const size_t sm = router_smem_bytes(D.E);
  if (D.dtype == MOE_DTYPE_BF16) {
    auto kern = router_fwd_kernel<__nv_bfloat16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return MOE_ERR_CUDA;
    kern<<<grid, RT_THREADS, sm, st>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)Wg,
                                       D.has_bias ? bias : nullptr, D.T, D.d, D.E, D.k,
                                       D.gate_norm, logits, topk_idx, topk_w);
  } else {
    auto kern = router_fwd_kernel<float>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return MOE_ERR_CUDA;
    kern<<<grid, RT_THREADS, sm, st>>>((const float*)x, (const float*)Wg,
                                       D.has_bias ? bias : nullptr, D.T, D.d, D.E, D.k,
                                       D.gate_norm, logits, topk_idx, topk_w);
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_topk_from_logits(const Dims& D, const float* logits, int32_t* topk_idx,
                                   float* topk_w, cudaStream_t st) {
  const int threads = 256;
  const int grid = (int)(((int64_t)D.T * 32 + threads - 1) / threads);
  topk_from_logits_kernel<<<grid, threads, 0, st>>>(logits, D.T, D.E, D.k, D.gate_norm, topk_idx,
                                                    topk_w);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
