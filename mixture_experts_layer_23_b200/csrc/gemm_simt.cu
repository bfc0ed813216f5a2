// Grouped expert GEMMs on CUDA cores (fp32 FMA, fp32 accumulate).
//
// Step 3 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 3: each device runs its local experts on the tokens it received; part 一: each expert is
// an MLP) and its backward (section "专家并行与数据并行的结合", part 三.3: expert weight gradients
// are computed locally).
//
// This engine serves the fp32 layers (tf32 tensor cores would not hold fp32 accuracy) and shapes
// the tensor-core engine does not take.  Every kernel is one 64x64 output tile per CTA of one
// group (expert): 256 threads, 4x4 outputs each, operands staged through shared memory as
// float.  Groups: routed expert e owns rows [offsets[e], offsets[e+1]) of the row space and
// reads the dispatched buffer; shared expert s owns rows [s*T_pad, s*T_pad + T_pad) and reads
// the token buffer (x or dy) directly, rows >= T reading as zero.
#include "common.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

// A view of a matrix: element (r, c) = p[r * sr + c * sc], zero outside r < nr, c < nc.
template <typename T>
struct View {
  const T* p;
  int64_t sr, sc;
  int64_t nr, nc;
  __device__ __forceinline__ float at(int64_t r, int64_t c) const {
    return (r < nr && c < nc) ? to_f(p[r * sr + c * sc]) : 0.f;
  }
};

struct Group {
  int64_t rows, a_row, o_row;
  int w;
  bool shared;
};

__device__ __forceinline__ Group group_of(int g, int E, const int32_t* offsets, int64_t T_pad) {
  Group G;
  if (g < E) {
    G.a_row = offsets[g];
    G.o_row = G.a_row;
    G.rows = offsets[g + 1] - G.a_row;
    G.shared = false;
  } else {
    G.a_row = 0;
    G.o_row = (int64_t)(g - E) * T_pad;
    G.rows = T_pad;
    G.shared = true;
  }
  G.w = g;
  return G;
}

// acc[i][j] += sum_k A(m0 + ty*4 + i, k) * B(n0 + tx*4 + j, k), k < K.
template <typename TA, typename TB>
__device__ __forceinline__ void mainloop(const View<TA>& A, const View<TB>& B, int64_t m0,
                                         int64_t n0, int64_t K, float (*As)[BM + 4],
                                         float (*Bs)[BN + 4], float acc[4][4]) {
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int64_t k0 = 0; k0 < K; k0 += BK) {
    for (int q = tid; q < BM * BK; q += 256) {
      // consecutive threads walk the operand's contiguous dimension
      int r, c;
      if (A.sc == 1) { r = q / BK; c = q % BK; } else { r = q % BM; c = q / BM; }
      As[c][r] = (k0 + c < K) ? A.at(m0 + r, k0 + c) : 0.f;
      int rb, cb;
      if (B.sc == 1) { rb = q / BK; cb = q % BK; } else { rb = q % BN; cb = q / BN; }
      Bs[cb][rb] = (k0 + cb < K) ? B.at(n0 + rb, k0 + cb) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < BK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[c][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[c][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

// u = A W1^T (and v = A W3^T); H = gelu(u) or silu(u) * v.  Instead of u and v, the factors the
// backward needs are stored: U <- Gu = gelu'(u), or Gu = v s (1 + u (1 - s)) and V <- Gv = silu(u)
// with s = sigmoid(u).
template <typename T>
__global__ void __launch_bounds__(256)
up_kernel(const T* __restrict__ Xd, const T* __restrict__ x, const int32_t* __restrict__ offsets,
          const T* __restrict__ W1, const T* __restrict__ W3, int T_, int d, int F, int E,
          int64_t T_pad, int act, T* __restrict__ U, T* __restrict__ V, T* __restrict__ H) {
  pdl_prologue();
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  const Group G = group_of(blockIdx.z, E, offsets, T_pad);
  const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
  if (m0 >= G.rows) return;
  View<T> A = G.shared ? View<T>{x, d, 1, T_, d} : View<T>{Xd + G.a_row * d, d, 1, G.rows, d};
  View<T> B1{W1 + (int64_t)G.w * F * d, d, 1, F, d};
  float au[4][4] = {}, av[4][4] = {};
  mainloop(A, B1, m0, n0, d, As, Bs, au);
  if (act == MOE_ACT_SWIGLU) {
    View<T> B3{W3 + (int64_t)G.w * F * d, d, 1, F, d};
    mainloop(A, B3, m0, n0, d, As, Bs, av);
  }
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= G.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= F) continue;
      const int64_t o = (G.o_row + m) * F + n;
      const float u = au[i][j];
      if (act == MOE_ACT_GELU) {
        U[o] = from_f<T>(gelu_grad_f(u));                  // Gu = GELU'(u)
        H[o] = from_f<T>(gelu_f(u));
      } else {
        const float v = av[i][j];
        const float s = sigmoid_f(u);
        U[o] = from_f<T>(v * s * (1.f + u * (1.f - s)));   // Gu
        V[o] = from_f<T>(u * s);                           // Gv = silu(u)
        H[o] = from_f<T>(u * s * v);
      }
    }
  }
}

// O = H W2^T
template <typename T>
__global__ void __launch_bounds__(256)
down_kernel(const T* __restrict__ H, const int32_t* __restrict__ offsets,
            const T* __restrict__ W2, int d, int F, int E, int64_t T_pad, T* __restrict__ O) {
  pdl_prologue();
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  const Group G = group_of(blockIdx.z, E, offsets, T_pad);
  const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
  if (m0 >= G.rows) return;
  View<T> A{H + G.o_row * F, F, 1, G.rows, F};
  View<T> B{W2 + (int64_t)G.w * d * F, F, 1, d, F};
  float acc[4][4] = {};
  mainloop(A, B, m0, n0, F, As, Bs, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= G.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n < d) O[(G.o_row + m) * d + n] = from_f<T>(acc[i][j]);
    }
  }
}

// dH = dO W2 (B = W2_e read N-contiguous), then dU = dH * Gu (and dV = dH * Gv).
template <typename T>
__global__ void __launch_bounds__(256)
dgrad_h_kernel(const T* __restrict__ dO, const T* __restrict__ dy,
               const int32_t* __restrict__ offsets, const T* __restrict__ W2,
               const T* __restrict__ U, const T* __restrict__ V, int T_, int d, int F, int E,
               int64_t T_pad, int act, T* __restrict__ dU, T* __restrict__ dV) {
  pdl_prologue();
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  const Group G = group_of(blockIdx.z, E, offsets, T_pad);
  const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
  if (m0 >= G.rows) return;
  View<T> A = G.shared ? View<T>{dy, d, 1, T_, d} : View<T>{dO + G.a_row * d, d, 1, G.rows, d};
  View<T> B{W2 + (int64_t)G.w * d * F, 1, F, F, d};  // B(n=f, k=i) = W2[i][f]
  float acc[4][4] = {};
  mainloop(A, B, m0, n0, d, As, Bs, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= G.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= F) continue;
      const int64_t o = (G.o_row + m) * F + n;
      const float dh = acc[i][j];
      dU[o] = from_f<T>(dh * to_f(U[o]));                  // dU = dH * Gu
      if (act == MOE_ACT_SWIGLU) dV[o] = from_f<T>(dh * to_f(V[o]));   // dV = dH * Gv
    }
  }
}

// dXd = dU W1 (+ dV W3)  (B = W1_e read N-contiguous)
template <typename T>
__global__ void __launch_bounds__(256)
dgrad_x_kernel(const T* __restrict__ dU, const T* __restrict__ dV,
               const int32_t* __restrict__ offsets, const T* __restrict__ W1,
               const T* __restrict__ W3, int d, int F, int E, int64_t T_pad, int act,
               T* __restrict__ dXd) {
  pdl_prologue();
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  const Group G = group_of(blockIdx.z, E, offsets, T_pad);
  const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
  if (m0 >= G.rows) return;
  float acc[4][4] = {};
  mainloop(View<T>{dU + G.o_row * F, F, 1, G.rows, F},
           View<T>{W1 + (int64_t)G.w * F * d, 1, d, d, F}, m0, n0, F, As, Bs, acc);
  if (act == MOE_ACT_SWIGLU)
    mainloop(View<T>{dV + G.o_row * F, F, 1, G.rows, F},
             View<T>{W3 + (int64_t)G.w * F * d, 1, d, d, F}, m0, n0, F, As, Bs, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= G.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n < d) dXd[(G.o_row + m) * d + n] = from_f<T>(acc[i][j]);
    }
  }
}

// Weight gradients, K = the group's rows:
//   which 0: dW1[w][f][i] = sum_r dU[r][f] * X[r][i]
//   which 1: dW3[w][f][i] = sum_r dV[r][f] * X[r][i]
//   which 2: dW2[w][i][f] = sum_r dOut[r][i] * H[r][f]
template <typename T>
__global__ void __launch_bounds__(256)
wgrad_kernel(int which, const T* __restrict__ Gf /* dU, dV or H */, const T* __restrict__ Xd_or_dO,
             const T* __restrict__ tok /* x or dy */, const int32_t* __restrict__ offsets, int T_,
             int d, int F, int E, int64_t T_pad, float* __restrict__ dW) {
  pdl_prologue();
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  const Group G = group_of(blockIdx.z, E, offsets, T_pad);
  const int64_t m0 = (int64_t)blockIdx.x * BM, n0 = (int64_t)blockIdx.y * BN;
  const int64_t Mdim = (which == 2) ? d : F, Ndim = (which == 2) ? F : d;
  if (m0 >= Mdim || n0 >= Ndim) return;
  // row-space operand (indexed by the group's own rows) and token-side operand
  View<T> Rv{Gf + G.o_row * F, 1, F, F, G.rows};       // (f, r)
  View<T> Tv = G.shared ? View<T>{tok, 1, d, d, T_}     // (i, r)
                        : View<T>{Xd_or_dO + G.a_row * d, 1, d, d, G.rows};
  float acc[4][4] = {};
  if (which == 2) mainloop(Tv, Rv, m0, n0, G.rows, As, Bs, acc);
  else mainloop(Rv, Tv, m0, n0, G.rows, As, Bs, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float* out = dW + (int64_t)G.w * F * d;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= Mdim) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n < Ndim) out[m * Ndim + n] = acc[i][j];
    }
  }
}

}  // namespace

#define MOE_SIMT_DISPATCH(D, CALL)                                   \
  ((D).dtype == MOE_DTYPE_BF16 ? [&] { using T = __nv_bfloat16; return CALL; }() \
                               : [&] { using T = float; return CALL; }())
#define SIMT_LAUNCH(KERN, GRID, ...) launch_k(KERN, GRID, 256, 0, st, 1, __VA_ARGS__)

moe_status launch_expert_up_simt(const Dims& D, const void* Xd, const void* x,
                                 const int32_t* offsets, const void* W1, const void* W3, void* U,
                                 void* V, void* H, cudaStream_t st) {
  const int mt = (int)((D.max_group_rows + BM - 1) / BM);
  const dim3 grid(mt, (D.F + BN - 1) / BN, D.E_tot);
  return MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(up_kernel<T>, grid,
      (const T*)Xd, (const T*)x, offsets, (const T*)W1, (const T*)W3, D.T, D.d, D.F, D.E,
      D.T_pad, D.act, (T*)U, (T*)V, (T*)H));
}

moe_status launch_expert_down_simt(const Dims& D, const void* H, const int32_t* offsets,
                                   const void* W2, void* O, cudaStream_t st) {
  const int mt = (int)((D.max_group_rows + BM - 1) / BM);
  const dim3 grid(mt, (D.d + BN - 1) / BN, D.E_tot);
  return MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(down_kernel<T>, grid,
      (const T*)H, offsets, (const T*)W2, D.d, D.F, D.E, D.T_pad, (T*)O));
}

moe_status launch_dgrad_h_simt(const Dims& D, const void* dO, const void* dy,
                               const int32_t* offsets, const void* W2, const void* U,
                               const void* V, void* dU, void* dV, cudaStream_t st) {
  const int mt = (int)((D.max_group_rows + BM - 1) / BM);
  const dim3 grid(mt, (D.F + BN - 1) / BN, D.E_tot);
  return MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(dgrad_h_kernel<T>, grid,
      (const T*)dO, (const T*)dy, offsets, (const T*)W2, (const T*)U, (const T*)V, D.T, D.d, D.F,
      D.E, D.T_pad, D.act, (T*)dU, (T*)dV));
}

moe_status launch_dgrad_x_simt(const Dims& D, const void* dU, const void* dV,
                               const int32_t* offsets, const void* W1, const void* W3, void* dXd,
                               cudaStream_t st) {
  const int mt = (int)((D.max_group_rows + BM - 1) / BM);
  const dim3 grid(mt, (D.d + BN - 1) / BN, D.E_tot);
  return MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(dgrad_x_kernel<T>, grid,
      (const T*)dU, (const T*)dV, offsets, (const T*)W1, (const T*)W3, D.d, D.F, D.E, D.T_pad,
      D.act, (T*)dXd));
}

moe_status launch_wgrad_w13_simt(const Dims& D, const void* dU, const void* dV, const void* Xd,
                                 const void* x, const int32_t* offsets, float* dW1, float* dW3,
                                 cudaStream_t st) {
  const dim3 g1((D.F + BM - 1) / BM, (D.d + BN - 1) / BN, D.E_tot);
  MOE_TRY_S(MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(wgrad_kernel<T>, g1,
      0, (const T*)dU, (const T*)Xd, (const T*)x, offsets, D.T, D.d, D.F, D.E, D.T_pad, dW1)));
  if (D.act == MOE_ACT_SWIGLU)
    MOE_TRY_S(MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(wgrad_kernel<T>, g1,
        1, (const T*)dV, (const T*)Xd, (const T*)x, offsets, D.T, D.d, D.F, D.E, D.T_pad, dW3)));
  return MOE_OK;
}

moe_status launch_wgrad_w2_simt(const Dims& D, const void* H, const void* dO, const void* dy,
                                const int32_t* offsets, float* dW2, cudaStream_t st) {
  const dim3 g2((D.d + BM - 1) / BM, (D.F + BN - 1) / BN, D.E_tot);
  return MOE_SIMT_DISPATCH(D, SIMT_LAUNCH(wgrad_kernel<T>, g2,
      2, (const T*)H, (const T*)dO, (const T*)dy, offsets, D.T, D.d, D.F, D.E, D.T_pad, dW2));
}

}  // namespace moe
