// Router: gate logits, softmax and top-k, fused in one kernel.
//
// Step 1 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 1: a small router, replicated on every device, gates the local tokens).  The top-k gate is
// the Tutel gate_type {'type': 'top', 'k': ...} of section "框架".
//
// This is the CUDA-core form (fp32 layers and shapes the tensor-core router does not take): one
// CTA owns 64 tokens, computes their [64 x E] logit tile with fp32 FMA (x and Wg staged through
// shared memory), adds the constant bias and writes the logits; then one thread per token runs
// the serial softmax + top-k of route_serial.cuh over its row in shared memory.
#include <algorithm>

#include "common.cuh"
#include "route_serial.cuh"

namespace moe {
namespace {

constexpr int RT_TOK = 64;   // tokens per CTA
constexpr int RT_EC = 64;    // experts per GEMM pass
constexpr int RT_BK = 32;    // d per smem stage
constexpr int RT_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(RT_THREADS)
router_fwd_kernel(const T* __restrict__ x, const T* __restrict__ Wg,
                  const float* __restrict__ bias, int T_, int d, int E, int k, int gate_norm,
                  float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                  float* __restrict__ topk_w) {
  pdl_prologue();
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
  if (tid < RT_TOK && t0 + tid < T_) {
    const int t = t0 + tid;
    TopK8 st;
    topk_init(st);
    for (int e = 0; e < E; ++e) topk_push(st, ls[tid * (E + 1) + e], e);
    float den = 0.f;
    if (gate_norm == 0)
      for (int e = 0; e < E; ++e) den += softmax_term(st, ls[tid * (E + 1) + e]);
    topk_finish(st, k, gate_norm, den, topk_idx + (int64_t)t * k, topk_w + (int64_t)t * k);
  }
}

__global__ void topk_from_logits_kernel(const float* __restrict__ logits, int T_, int E, int k,
                                        int gate_norm, int32_t* __restrict__ topk_idx,
                                        float* __restrict__ topk_w) {
  pdl_prologue();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T_) return;
  const float* row = logits + (int64_t)t * E;
  TopK8 st;
  topk_init(st);
  for (int e = 0; e < E; ++e) topk_push(st, row[e], e);
  float den = 0.f;
  if (gate_norm == 0)
    for (int e = 0; e < E; ++e) den += softmax_term(st, row[e]);
  topk_finish(st, k, gate_norm, den, topk_idx + (int64_t)t * k, topk_w + (int64_t)t * k);
}

// Few experts: one warp per token.  The CTA stages the whole gate matrix Wg [E, d] in shared
// memory; a warp reads its token's row once (16-byte vectors, lane-strided), keeps EP partial
// dot products per lane, and folds them across the warp with a transposing butterfly (each
// exchange halves the values a lane keeps), after which lane l holds the logit of expert
// l >> (5 - log2 EP).  Lane 0 then runs the serial softmax + top-k of route_serial.cuh.
constexpr int RW_THREADS = 512;

template <int EP>
__device__ __forceinline__ float transpose_reduce(float (&acc)[EP], int lane) {
  int n = EP;
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int off = 16 >> s;
    if (n > 1) {
      const int h = n >> 1;
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < EP / 2; ++i)
        if (i < h) {
          const float send = up ? acc[i] : acc[i + h];
          const float keep = up ? acc[i + h] : acc[i];
          acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      n = h;
    } else {
      acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
    }
  }
  return acc[0];
}

template <typename T, int EP>
__global__ void __launch_bounds__(RW_THREADS)
router_warp_kernel(const T* __restrict__ x, const T* __restrict__ Wg,
                   const float* __restrict__ bias, int T_, int d, int E, int k, int gate_norm,
                   float* __restrict__ logits, int32_t* __restrict__ topk_idx,
                   float* __restrict__ topk_w) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int SH = (EP >= 32) ? 0 : (EP >= 16) ? 1 : (EP >= 8) ? 2 : (EP >= 4) ? 3 : (EP >= 2) ? 4 : 5;
  extern __shared__ uint4 rw_smem[];
  const int nv = d / VN;
  const uint4* wsrc = reinterpret_cast<const uint4*>(Wg);
  for (int q = threadIdx.x; q < E * nv; q += RW_THREADS) rw_smem[q] = __ldg(wsrc + q);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = RW_THREADS / 32;
  const int e_l = lane >> SH;   // expert whose logit this lane ends up with
  const float b_l = (bias != nullptr && e_l < E) ? bias[e_l] : 0.f;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T_; t += gridDim.x * warps) {
    float acc[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[e] = 0.f;
    const T* xr = x + (int64_t)t * d;
    for (int v = lane; v < nv; v += 32) {
      const Vec16<T> xv = ld_vec_stream(xr + (int64_t)v * VN);
      float xf[VN];
#pragma unroll
      for (int i = 0; i < VN; ++i) xf[i] = xv.get(i);
#pragma unroll
      for (int e = 0; e < EP; ++e)
        if (e < E) {
          Vec16<T> w;
          w.raw = rw_smem[e * nv + v];
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[e] = fmaf(xf[i], w.get(i), acc[e]);
        }
    }
    const float lg = transpose_reduce<EP>(acc, lane) + b_l;
    if ((lane & ((1 << SH) - 1)) == 0 && e_l < E) logits[(int64_t)t * E + e_l] = lg;
    TopK8 st;
    topk_init(st);
    for (int e = 0; e < E; ++e) {
      const float v = __shfl_sync(0xffffffffu, lg, e << SH);
      if (lane == 0) topk_push(st, v, e);
    }
    float den = 0.f;
    if (gate_norm == 0)
      for (int e = 0; e < E; ++e) {
        const float v = __shfl_sync(0xffffffffu, lg, e << SH);
        if (lane == 0) den += softmax_term(st, v);
      }
    if (lane == 0)
      topk_finish(st, k, gate_norm, den, topk_idx + (int64_t)t * k, topk_w + (int64_t)t * k);
  }
}

template <typename T, int EP>
static moe_status router_warp_t(const Dims& D, const void* x, const void* Wg, const float* bias,
                                float* logits, int32_t* topk_idx, float* topk_w,
                                cudaStream_t st) {
  const size_t sm = (size_t)D.E * D.d * sizeof(T);
  auto kern = router_warp_kernel<T, EP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int grid = (int)std::min<int64_t>((D.T + RW_THREADS / 32 - 1) / (RW_THREADS / 32), 148);
  return launch_k(kern, grid, RW_THREADS, sm, st, 1, (const T*)x, (const T*)Wg, bias, D.T, D.d,
                  D.E, D.k, D.gate_norm, logits, topk_idx, topk_w);
}

template <typename T>
static moe_status router_warp_e(const Dims& D, const void* x, const void* Wg, const float* bias,
                                float* logits, int32_t* topk_idx, float* topk_w,
                                cudaStream_t st) {
  if (D.E <= 4) return router_warp_t<T, 4>(D, x, Wg, bias, logits, topk_idx, topk_w, st);
  if (D.E <= 8) return router_warp_t<T, 8>(D, x, Wg, bias, logits, topk_idx, topk_w, st);
  if (D.E <= 16) return router_warp_t<T, 16>(D, x, Wg, bias, logits, topk_idx, topk_w, st);
  return router_warp_t<T, 32>(D, x, Wg, bias, logits, topk_idx, topk_w, st);
}

}  // namespace

bool router_warp_supported(const Dims& D) {
  const int esz = D.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  return D.E <= 32 && D.d % (16 / esz) == 0 && (size_t)D.E * D.d * esz <= (size_t)96 * 1024;
}

moe_status launch_router_warp(const Dims& D, const void* x, const void* Wg, const float* bias,
                              float* logits, int32_t* topk_idx, float* topk_w, cudaStream_t st) {
  const float* b = D.has_bias ? bias : nullptr;
  if (D.dtype == MOE_DTYPE_BF16)
    return router_warp_e<__nv_bfloat16>(D, x, Wg, b, logits, topk_idx, topk_w, st);
  return router_warp_e<float>(D, x, Wg, b, logits, topk_idx, topk_w, st);
}

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
    return launch_k(kern, grid, RT_THREADS, sm, st, 1, (const __nv_bfloat16*)x,
                    (const __nv_bfloat16*)Wg, D.has_bias ? bias : nullptr, D.T, D.d, D.E, D.k,
                    D.gate_norm, logits, topk_idx, topk_w);
  } else {
    auto kern = router_fwd_kernel<float>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return MOE_ERR_CUDA;
    return launch_k(kern, grid, RT_THREADS, sm, st, 1, (const float*)x, (const float*)Wg,
                    D.has_bias ? bias : nullptr, D.T, D.d, D.E, D.k, D.gate_norm, logits,
                    topk_idx, topk_w);
  }
}

moe_status launch_topk_from_logits(const Dims& D, const float* logits, int32_t* topk_idx,
                                   float* topk_w, cudaStream_t st) {
  const int threads = 128;
  const int grid = (D.T + threads - 1) / threads;
  return launch_k(topk_from_logits_kernel, grid, threads, 0, st, 1, logits, D.T, D.E, D.k,
                  D.gate_norm, topk_idx, topk_w);
}

}  // namespace moe
