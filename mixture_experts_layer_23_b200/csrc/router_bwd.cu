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
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

// Partial dWg over one chunk of tokens: part[c][e][i] = sum_{t in chunk c} dl[t,e] x[t,i].
// A CTA of 128 threads covers 256 columns (two per thread) and 16 experts at a time (32
// accumulators per thread).  For every 64 tokens (32 for fp32) it stages the x tile in shared memory
// with 16-byte loads that are all in flight together, and the matching dl values; the products
// are then read from shared memory (x as each thread's two columns, dl as broadcasts).
constexpr int WG_COLS = 256, WG_EC = 16;

template <typename T>
__global__ void __launch_bounds__(128)
router_wgrad_partial_kernel(const float* __restrict__ dl, const T* __restrict__ x, int T_, int d,
                            int E, int chunk, float* __restrict__ part) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int WG_TS = 128 / (int)sizeof(T);  // 64 bf16 or 32 fp32 token rows: a 32 KB tile
  __shared__ __align__(16) T xs[WG_TS][WG_COLS];
  __shared__ float ds[WG_TS][WG_EC];
  const int c = blockIdx.x;
  const int c0 = blockIdx.y * WG_COLS;
  const int i = 2 * threadIdx.x;           // column inside the slice
  const int t_begin = c * chunk;
  const int t_end = min(T_, t_begin + chunk);
  const bool col_ok = c0 + i < d;
  for (int e0 = 0; e0 < E; e0 += WG_EC) {
    float acc0[WG_EC], acc1[WG_EC];
#pragma unroll
    for (int e = 0; e < WG_EC; ++e) acc0[e] = acc1[e] = 0.f;
    for (int tb = t_begin; tb < t_end; tb += WG_TS) {
      __syncthreads();
      constexpr int VPR = WG_COLS / VN;   // 16-byte vectors per tile row
#pragma unroll 4
      for (int q = threadIdx.x; q < WG_TS * VPR; q += 128) {
        const int r = q / VPR, v = q % VPR;
        const int t = tb + r, col = c0 + v * VN;
        Vec16<T> val;
        val.raw = make_uint4(0, 0, 0, 0);
        if (t < t_end && col < d) val = ld_vec(x + (int64_t)t * d + col);
        st_vec(&xs[r][v * VN], val);
      }
      for (int q = threadIdx.x; q < WG_TS * WG_EC; q += 128) {
        const int r = q / WG_EC, e = q % WG_EC;
        const int t = tb + r;
        ds[r][e] = (t < t_end && e0 + e < E) ? dl[(int64_t)t * E + e0 + e] : 0.f;
      }
      __syncthreads();
      const int nt = min(WG_TS, t_end - tb);
#pragma unroll 4
      for (int r = 0; r < nt; ++r) {
        const float x0 = to_f(xs[r][i]), x1 = to_f(xs[r][i + 1]);
#pragma unroll
        for (int e = 0; e < WG_EC; ++e) {
          acc0[e] = fmaf(ds[r][e], x0, acc0[e]);
          acc1[e] = fmaf(ds[r][e], x1, acc1[e]);
        }
      }
    }
    if (col_ok) {
#pragma unroll
      for (int e = 0; e < WG_EC; ++e)
        if (e0 + e < E)
          *reinterpret_cast<float2*>(part + ((int64_t)c * E + e0 + e) * d + c0 + i) =
              make_float2(acc0[e], acc1[e]);
    }
  }
}

__global__ void router_wgrad_reduce_kernel(const float* __restrict__ part, int n_chunk,
                                           int64_t n, float* __restrict__ dWg) {
  pdl_prologue();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float s = 0.f;
  for (int c = 0; c < n_chunk; ++c) s += part[(int64_t)c * n + i];
  dWg[i] = s;
}

// dx for 32 tokens x (32 * VN) columns: warp w takes tokens w, w+8, w+16, w+24, two at a time;
// lane l owns the VN columns at 16-byte vector l.  dx = dl Wg (K = E from shared memory) + the
// token's gathered dXd rows (routed slots in order, then shared experts), a fixed-order sum.  The
// four tokens' slots are fetched together, and each pair's gathers are issued before the K = E
// contraction so that their latency overlaps it.
template <typename T>
__global__ void __launch_bounds__(256)
undispatch_kernel(const float* __restrict__ dl, const T* __restrict__ Wg,
                  const T* __restrict__ dXd, const int32_t* __restrict__ slot, int T_, int d,
                  int E, int k, int S, int64_t T_pad, T* __restrict__ dx) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int COLS = 32 * VN;
  extern __shared__ uint4 ud_smem[];
  T* ws = reinterpret_cast<T*>(ud_smem);                       // [E][COLS]
  float* dls = reinterpret_cast<float*>(ws + (size_t)E * COLS); // [32][E]
  const int t0 = blockIdx.x * 32, c0 = blockIdx.y * COLS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nvec_row = COLS / VN;  // 32
  for (int q = threadIdx.x; q < E * nvec_row; q += 256) {
    const int e = q / nvec_row, v = q % nvec_row;
    const int col = c0 + v * VN;
    Vec16<T> w;
    w.raw = make_uint4(0, 0, 0, 0);
    if (col < d) w = ld_vec(Wg + (int64_t)e * d + col);
    st_vec(ws + (size_t)e * COLS + v * VN, w);
  }
  for (int q = threadIdx.x; q < 32 * E; q += 256) {
    const int r = q / E, e = q % E;
    dls[q] = (t0 + r < T_) ? dl[(int64_t)(t0 + r) * E + e] : 0.f;
  }
  // slots of this warp's four tokens: lane q < 4k holds slot (token q / k, choice q % k)
  int my_slot = -1;
  if (lane < 4 * k) {
    const int t = t0 + warp + 8 * (lane / k);
    if (t < T_) my_slot = slot[(int64_t)t * k + (lane % k)];
  }
  __syncthreads();
  const int col = c0 + lane * VN;
  const bool col_ok = col < d;  // lanes past d stay in the warp: they source slot shuffles
#pragma unroll 1
  for (int p = 0; p < 2; ++p) {
    const int ra = warp + 16 * p, rb = ra + 8;    // the pair's two tokens
    const int ta = t0 + ra, tb = t0 + rb;
    if (ta >= T_) break;
    const bool hb = tb < T_;
    Vec16<T> ga[8], gb[8];
    int sa[8], sb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sa[j] = __shfl_sync(0xffffffffu, my_slot, (2 * p) * k + j);
      sb[j] = __shfl_sync(0xffffffffu, my_slot, (2 * p + 1) * k + j);
      if (j >= k || !col_ok) sa[j] = sb[j] = -1;
      if (!hb) sb[j] = -1;
      if (sa[j] >= 0) ga[j] = ld_vec_stream(dXd + (int64_t)sa[j] * d + col);
      if (sb[j] >= 0) gb[j] = ld_vec_stream(dXd + (int64_t)sb[j] * d + col);
    }
    float acc_a[VN], acc_b[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc_a[i] = acc_b[i] = 0.f;
    for (int sj = 0; sj < (col_ok ? S : 0); ++sj) {
      const Vec16<T> ha = ld_vec_stream(dXd + ((int64_t)sj * T_pad + ta) * d + col);
#pragma unroll
      for (int i = 0; i < VN; ++i) acc_a[i] += ha.get(i);
      if (hb) {
        const Vec16<T> hbv = ld_vec_stream(dXd + ((int64_t)sj * T_pad + tb) * d + col);
#pragma unroll
        for (int i = 0; i < VN; ++i) acc_b[i] += hbv.get(i);
      }
    }
    float ca[VN], cb[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) ca[i] = cb[i] = 0.f;
    const float* dla = dls + ra * E;
    const float* dlb = dls + rb * E;
    for (int e = 0; e < E; ++e) {
      const Vec16<T> wv = *reinterpret_cast<const Vec16<T>*>(ws + (size_t)e * COLS + lane * VN);
      const float wa = dla[e], wb = dlb[e];
#pragma unroll
      for (int i = 0; i < VN; ++i) {
        ca[i] = fmaf(wa, wv.get(i), ca[i]);
        cb[i] = fmaf(wb, wv.get(i), cb[i]);
      }
    }
    // fixed order: dl Wg, routed rows j = 0..k-1, shared rows
    Vec16<T> oa, ob;
#pragma unroll
    for (int i = 0; i < VN; ++i) {
      float va = ca[i], vb = cb[i];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (sa[j] >= 0) va += ga[j].get(i);
        if (sb[j] >= 0) vb += gb[j].get(i);
      }
      oa.set(i, va + acc_a[i]);
      ob.set(i, vb + acc_b[i]);
    }
    if (col_ok) {
      st_vec(dx + (int64_t)ta * d + col, oa);
      if (hb) st_vec(dx + (int64_t)tb * d + col, ob);
    }
  }
}

// Few experts (the gate matrix fits in shared memory): one warp per token, persistent CTAs.  The
// CTA stages Wg [E, d] once; a warp loads its token's k routed and S shared dXd rows, U = 8 / KR
// vectors per lane at a time with all loads in flight together, and the dl row (lane e holds
// dl[t, e], broadcast by shuffles).  Per element: (sum_e dl_e Wg_e) + routed rows j = 0..k-1 +
// (sum of shared rows), a fixed order.
constexpr int UW_THREADS = 512;

template <typename T, int KR>
__global__ void __launch_bounds__(UW_THREADS)
undispatch_warp_kernel(const float* __restrict__ dl, const T* __restrict__ Wg,
                       const T* __restrict__ dXd, const int32_t* __restrict__ slot, int T_, int d,
                       int E, int k, int S, int64_t T_pad, T* __restrict__ dx) {
  pdl_prologue();
  constexpr int VN = Vec16<T>::N;
  constexpr int U = KR >= 8 ? 1 : 8 / KR;
  extern __shared__ uint4 uw_smem[];
  const int nv = d / VN;
  const uint4* wsrc = reinterpret_cast<const uint4*>(Wg);
  for (int q = threadIdx.x; q < E * nv; q += UW_THREADS) uw_smem[q] = __ldg(wsrc + q);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = UW_THREADS / 32;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T_; t += gridDim.x * warps) {
    int my_s = -1;
    if (lane < k)
      my_s = slot[(int64_t)t * k + lane];
    else if (lane < k + S)
      my_s = (int)((int64_t)(lane - k) * T_pad + t);
    const float my_dl = lane < E ? dl[(int64_t)t * E + lane] : 0.f;
    int s[KR];
#pragma unroll
    for (int j = 0; j < KR; ++j) {
      s[j] = __shfl_sync(0xffffffffu, my_s, j);
      if (j >= k + S) s[j] = -1;
    }
    // the loop bounds are the same for every lane (the dl shuffles need the whole warp)
    for (int base = 0; base < nv; base += 32 * U) {
      const int v0 = base + lane;
      Vec16<T> g[U][KR];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          const int v = v0 + 32 * u;
          if (v < nv && s[j] >= 0) g[u][j] = ld_vec_stream(dXd + (int64_t)s[j] * d + (int64_t)v * VN);
        }
      float acc[U][VN];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[u][i] = 0.f;
      for (int e = 0; e < E; ++e) {
        const float w = __shfl_sync(0xffffffffu, my_dl, e);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < nv) {
            Vec16<T> wv;
            wv.raw = uw_smem[e * nv + v];
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[u][i] = fmaf(w, wv.get(i), acc[u][i]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + 32 * u;
        if (v >= nv) break;
        Vec16<T> out;
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          float r = acc[u][i], sh = 0.f;
#pragma unroll
          for (int j = 0; j < KR; ++j)
            if (s[j] >= 0) {
              if (j < k) r += g[u][j].get(i);
              else sh += g[u][j].get(i);
            }
          out.set(i, r + sh);
        }
        st_vec(dx + (int64_t)t * d + (int64_t)v * VN, out);
      }
    }
  }
}

}  // namespace

moe_status launch_router_wgrad_reduce(const Dims& D, const float* part, int n_chunks, float* dWg,
                                      cudaStream_t st) {
  const int64_t n = (int64_t)D.E * D.d;
  return launch_k(router_wgrad_reduce_kernel, (int)((n + 255) / 256), 256, 0, st, 1, part,
                  n_chunks, n, dWg);
}

bool undispatch_warp_supported(const Dims& D) {
  const int esz = D.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  return D.E <= 32 && D.k + D.S <= 16 && (size_t)D.E * D.d * esz <= (size_t)96 * 1024;
}

template <typename T, int KR>
static moe_status undispatch_warp_t(const Dims& D, const float* dlogits, const void* Wg,
                                    const void* dXd, const int32_t* slot, void* dx,
                                    cudaStream_t st) {
  const size_t sm = (size_t)D.E * D.d * sizeof(T);
  auto kern = undispatch_warp_kernel<T, KR>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int wpc = UW_THREADS / 32;
  const int grid = (int)std::min<int64_t>((D.T + wpc - 1) / wpc, 148);
  return launch_k(kern, grid, UW_THREADS, sm, st, 1, dlogits, (const T*)Wg, (const T*)dXd, slot,
                  D.T, D.d, D.E, D.k, D.S, D.T_pad, (T*)dx);
}

template <typename T>
static moe_status undispatch_warp_kr(const Dims& D, const float* dlogits, const void* Wg,
                                     const void* dXd, const int32_t* slot, void* dx,
                                     cudaStream_t st) {
  const int r = D.k + D.S;
  if (r <= 2) return undispatch_warp_t<T, 2>(D, dlogits, Wg, dXd, slot, dx, st);
  if (r <= 4) return undispatch_warp_t<T, 4>(D, dlogits, Wg, dXd, slot, dx, st);
  if (r <= 8) return undispatch_warp_t<T, 8>(D, dlogits, Wg, dXd, slot, dx, st);
  return undispatch_warp_t<T, 16>(D, dlogits, Wg, dXd, slot, dx, st);
}

moe_status launch_router_wgrad(const Dims& D, const float* dlogits, const void* x, float* part,
                               float* dWg, cudaStream_t st) {
  const int chunk = (D.T + D.n_tchunk - 1) / D.n_tchunk;
  dim3 grid(D.n_tchunk, (D.d + WG_COLS - 1) / WG_COLS);
  if (D.dtype == MOE_DTYPE_BF16)
    MOE_TRY_S(launch_k(router_wgrad_partial_kernel<__nv_bfloat16>, grid, 128, 0, st, 1, dlogits,
                       (const __nv_bfloat16*)x, D.T, D.d, D.E, chunk, part));
  else
    MOE_TRY_S(launch_k(router_wgrad_partial_kernel<float>, grid, 128, 0, st, 1, dlogits,
                       (const float*)x, D.T, D.d, D.E, chunk, part));
  const int64_t n = (int64_t)D.E * D.d;
  return launch_k(router_wgrad_reduce_kernel, (int)((n + 255) / 256), 256, 0, st, 1,
                  (const float*)part, D.n_tchunk, n, dWg);
}

template <typename T>
static moe_status undispatch_t(const Dims& D, const float* dlogits, const void* Wg, const void* dXd,
                               const int32_t* slot, void* dx, cudaStream_t st) {
  constexpr int COLS = 32 * Vec16<T>::N;
  const size_t smem = (size_t)D.E * COLS * sizeof(T) + 32 * (size_t)D.E * sizeof(float);
  auto kern = undispatch_kernel<T>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  dim3 grid((D.T + 31) / 32, (D.d + COLS - 1) / COLS);
  return launch_k(kern, grid, 256, smem, st, 1, dlogits, (const T*)Wg, (const T*)dXd, slot, D.T,
                  D.d, D.E, D.k, D.S, D.T_pad, (T*)dx);
}

moe_status launch_undispatch(const Dims& D, const float* dlogits, const void* Wg, const void* dXd,
                             const int32_t* slot, void* dx, cudaStream_t st) {
  if (undispatch_warp_supported(D)) {
    if (D.dtype == MOE_DTYPE_BF16)
      return undispatch_warp_kr<__nv_bfloat16>(D, dlogits, Wg, dXd, slot, dx, st);
    return undispatch_warp_kr<float>(D, dlogits, Wg, dXd, slot, dx, st);
  }
  if (D.dtype == MOE_DTYPE_BF16)
    return undispatch_t<__nv_bfloat16>(D, dlogits, Wg, dXd, slot, dx, st);
  return undispatch_t<float>(D, dlogits, Wg, dXd, slot, dx, st);
}

}  // namespace moe
