// Backward of the router and of the dispatch ("un-dispatch").
//
// Section "专家并行与数据并行的结合", part 三.3 of tutorial ch.4 "分布式训练": in the backward pass the
// gradients travel back along the routes the tokens took; expert weight gradients are computed
// where the experts are, and the replicated router (part 三.2) gets its gradient like any
// other replicated parameter.  Selection and drops are piecewise constant, so no gradient flows
// through the chosen indices:
//   (the softmax backward, dl from dg, runs inside the combine backward kernel)
//   dWg = dl^T x (two-level fixed-order reduction, bit-reproducible)
//   dx  = dl Wg + sum_j dXd[slot_j] + sum_s dXd[shared row of t]   (a gather, no atomics)
#include "common.cuh"

namespace moe {
namespace {

// Partial dWg over one chunk of tokens and 64 columns of d: part[c][e][i] = sum_t dl[t,e] x[t,i].
template <typename T>
__global__ void __launch_bounds__(256)
router_wgrad_partial_kernel(const float* __restrict__ dl, const T* __restrict__ x, int T_, int d,
                            int E, float* __restrict__ part) {
  __shared__ float ds[32][68];
  __shared__ float xs[32][68];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int c = blockIdx.x, i0 = blockIdx.y * 64;
  const int t_begin = c * kRouterBwdTokensPerChunk;
  const int t_end = min(T_, t_begin + kRouterBwdTokensPerChunk);
  for (int e0 = 0; e0 < E; e0 += 64) {
    float acc[4][4] = {};
    for (int tb = t_begin; tb < t_end; tb += 32) {
      for (int q = tid; q < 32 * 64; q += 256) {
        const int r = q / 64, col = q % 64;
        const int t = tb + r;
        ds[r][col] = (t < t_end && e0 + col < E) ? dl[(int64_t)t * E + e0 + col] : 0.f;
        xs[r][col] = (t < t_end && i0 + col < d) ? to_f(x[(int64_t)t * d + i0 + col]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int r = 0; r < 32; ++r) {
        float a[4], b[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) a[q] = ds[r][ty * 4 + q];
#pragma unroll
        for (int q = 0; q < 4; ++q) b[q] = xs[r][tx * 4 + q];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = e0 + ty * 4 + p, i = i0 + tx * 4 + q;
        if (e < E && i < d) part[((int64_t)c * E + e) * d + i] = acc[p][q];
      }
  }
}

__global__ void router_wgrad_reduce_kernel(const float* __restrict__ part, int n_chunk,
                                           int64_t n, float* __restrict__ dWg) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float s = 0.f;
  for (int c = 0; c < n_chunk; ++c) s += part[(int64_t)c * n + i];
  dWg[i] = s;
}

// dx for a tile of 64 tokens x 64 columns: dl Wg (K = E on CUDA cores) plus the gathered rows.
template <typename T>
__global__ void __launch_bounds__(256)
undispatch_kernel(const float* __restrict__ dl, const T* __restrict__ Wg,
                  const T* __restrict__ dXd, const int32_t* __restrict__ slot, int T_, int d,
                  int E, int k, int S, int64_t T_pad, T* __restrict__ dx) {
  __shared__ float ds[64][33];
  __shared__ float ws[32][68];
  __shared__ int32_t ss[64][8];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * 64, i0 = blockIdx.y * 64;
  for (int q = tid; q < 64 * 8; q += 256) {
    const int r = q / 8, j = q % 8;
    ss[r][j] = (t0 + r < T_ && j < k) ? slot[(int64_t)(t0 + r) * k + j] : -1;
  }
  float acc[4][4] = {};
  for (int e0 = 0; e0 < E; e0 += 32) {
    for (int q = tid; q < 64 * 32; q += 256) {
      const int r = q / 32, e = q % 32;
      ds[r][e] = (t0 + r < T_ && e0 + e < E) ? dl[(int64_t)(t0 + r) * E + e0 + e] : 0.f;
      const int er = q / 64, col = q % 64;
      ws[er][col] = (e0 + er < E && i0 + col < d) ? to_f(Wg[(int64_t)(e0 + er) * d + i0 + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int e = 0; e < 32; ++e) {
      float a[4], b[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) a[p] = ds[ty * 4 + p][e];
#pragma unroll
      for (int q = 0; q < 4; ++q) b[q] = ws[e][tx * 4 + q];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int r = ty * 4 + p, t = t0 + r;
    if (t >= T_) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = i0 + tx * 4 + q;
      if (i >= d) continue;
      float v = acc[p][q];
      for (int j = 0; j < k; ++j) {
        const int s = ss[r][j];
        if (s >= 0) v += to_f(dXd[(int64_t)s * d + i]);
      }
      for (int sh = 0; sh < S; ++sh) v += to_f(dXd[((int64_t)sh * T_pad + t) * d + i]);
      dx[(int64_t)t * d + i] = from_f<T>(v);
    }
  }
}

}  // namespace

moe_status launch_router_wgrad(const Dims& D, const float* dlogits, const void* x, float* part,
                               float* dWg, cudaStream_t st) {
  dim3 grid(D.n_tchunk, (D.d + 63) / 64);
  if (D.dtype == MOE_DTYPE_BF16)
    router_wgrad_partial_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        dlogits, (const __nv_bfloat16*)x, D.T, D.d, D.E, part);
  else
    router_wgrad_partial_kernel<float><<<grid, 256, 0, st>>>(dlogits, (const float*)x, D.T, D.d,
                                                             D.E, part);
  MOE_LAUNCH_CHECK();
  const int64_t n = (int64_t)D.E * D.d;
  router_wgrad_reduce_kernel<<<(int)((n + 255) / 256), 256, 0, st>>>(part, D.n_tchunk, n, dWg);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

moe_status launch_undispatch(const Dims& D, const float* dlogits, const void* Wg, const void* dXd,
                             const int32_t* slot, void* dx, cudaStream_t st) {
  dim3 grid((D.T + 63) / 64, (D.d + 63) / 64);
  if (D.dtype == MOE_DTYPE_BF16)
    undispatch_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        dlogits, (const __nv_bfloat16*)Wg, (const __nv_bfloat16*)dXd, slot, D.T, D.d, D.E, D.k,
        D.S, D.T_pad, (__nv_bfloat16*)dx);
  else
    undispatch_kernel<float><<<grid, 256, 0, st>>>(dlogits, (const float*)Wg, (const float*)dXd,
                                                   slot, D.T, D.d, D.E, D.k, D.S, D.T_pad,
                                                   (float*)dx);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

}  // namespace moe
