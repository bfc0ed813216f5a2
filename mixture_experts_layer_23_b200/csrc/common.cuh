// Device and host helpers shared by the MoE kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_ROW_ALIGN 128  // every dispatched segment is a multiple of the GEMM M tile

// Status word kept at the start of scratch (see moe_read_status).
#define MOE_STATUS_TIMEOUT 0x1u

namespace moe {

// Scratch layout: fixed-size header then per-call areas.  All offsets 256-byte aligned.
struct ScratchLayout {
  size_t status;        // uint32 status word
  size_t blk_counts;    // [n_blk, E] int32, per-block expert histograms of dispatch
  size_t local_rank;    // [T, k] int32, rank of each assignment inside its block
  size_t groups;        // [E_tot] int4 group table {rows, a_row, o_row, w}
  size_t dO;            // [R, d] act
  size_t dU;            // [R, F] act
  size_t dV;            // [R, F] act
  size_t dXd;           // [R, d] act
  size_t dg;            // [T, k] float
  size_t dlogits;       // [T, E] float
  size_t dWg_part;      // [n_tchunk, E, d] float
  size_t dl16;          // [T, E8] bf16 copy of dlogits (tensor-core router backward), or 0
  size_t wg_sched;      // [4] int32 tile counters of the tensor-core weight gradients (dW1, dW3, dW2)
  size_t aux_part;      // [n_aux, E] float partial probability sums of the load-balancing loss
  // column-major copies read K-major by the tensor-core weight gradients (0 on the CUDA-core path)
  size_t Xdt;           // [d, R] bf16: Xd^T (routed columns)
  size_t dOt;           // [d, R] bf16: dO^T (routed columns)
  size_t xt;            // [d, T_pad] bf16: x^T, zero past T (shared experts only, else 0)
  size_t dyt;           // [d, T_pad] bf16: dy^T, zero past T (shared experts only, else 0)
  size_t total;
};

struct Dims {
  int T, d, E, k, F, S, E_tot;
  int act, gate_norm, dtype, has_bias;
  int64_t C;            // capacity or MOE_DROPLESS
  int64_t T_pad, R, routed_row0, max_group_rows;
  int elem;             // bytes per activation element
  int n_blk;            // dispatch blocks
  int n_tchunk;         // token chunks of the router-weight gradient (two-level reduction)
  float aux_coef;       // weight of the load-balancing loss (0: off)
  int choice_major;     // dispatch drop priority: 0 token order, 1 choice index then token
  int n_layers;         // histogram layers of the dispatch: k when choice-major, else 1
  int n_aux;            // token chunks of the load-balancing loss's probability sums
};

constexpr int kDispatchTokensPerBlock = 256;
constexpr int kAuxTokensPerChunk = 64;   // load-balancing loss: tokens per CTA of the first level
constexpr int kAuxMaxChunks = 296;       // and at most this many CTAs (more tokens per CTA)

__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// ----------------------------------------------------------------------------- device helpers

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 16-byte vector of activations: 8 bf16 or 4 float.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  uint4 raw;
  __device__ __forceinline__ float get(int i) const {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(&raw);
    return __bfloat162float(p[i]);
  }
  __device__ __forceinline__ void set(int i, float v) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(&raw);
    p[i] = __float2bfloat16_rn(v);
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  uint4 raw;
  __device__ __forceinline__ float get(int i) const {
    return reinterpret_cast<const float*>(&raw)[i];
  }
  __device__ __forceinline__ void set(int i, float v) { reinterpret_cast<float*>(&raw)[i] = v; }
};

template <typename T>
__device__ __forceinline__ Vec16<T> ld_vec(const T* p) {
  Vec16<T> v;
  v.raw = __ldg(reinterpret_cast<const uint4*>(p));
  return v;
}
template <typename T>
__device__ __forceinline__ Vec16<T> ld_vec_stream(const T* p) {  // read-once data
  Vec16<T> v;
  v.raw = __ldcs(reinterpret_cast<const uint4*>(p));
  return v;
}
template <typename T>
__device__ __forceinline__ void st_vec(T* p, const Vec16<T>& v) {
  *reinterpret_cast<uint4*>(p) = v.raw;
}

// Programmatic dependent launch: every kernel of this library is launched so that it may start
// while its predecessor on the stream drains.  It first waits until the predecessor grid has
// completed and its writes are visible (a no-op without the launch attribute), then lets its own
// successor start launching.  Nothing global is touched before the wait.
__device__ __forceinline__ void pdl_prologue() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float gelu_f(float u) {
  return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
}
__device__ __forceinline__ float gelu_grad_f(float u) {
  const float Phi = 0.5f * (1.0f + erff(u * 0.70710678118654752f));
  const float phi = 0.39894228040143268f * expf(-0.5f * u * u);
  return Phi + u * phi;
}
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }

}  // namespace moe

// ----------------------------------------------------------------------------- host plumbing

namespace moe {
moe_status resolve_dims(const moe_config_t* cfg, Dims* out);
ScratchLayout scratch_layout(const Dims& D);
moe_status ctx_layout(const Dims& D, moe_layout_t* L);
}  // namespace moe

namespace moe {
extern unsigned long long g_kernel_launches;  // counted by MOE_LAUNCH_CHECK after each launch
void note_cuda_error(cudaError_t e);          // remembered for moe_last_cuda_error
}

#define MOE_LAUNCH_CHECK()                                                   \
  do {                                                                       \
    __atomic_fetch_add(&moe::g_kernel_launches, 1ull, __ATOMIC_RELAXED);     \
    cudaError_t e_ = cudaGetLastError();                                     \
    if (e_ != cudaSuccess) {                                                 \
      moe::note_cuda_error(e_);                                              \
      return MOE_ERR_CUDA;                                                   \
    }                                                                        \
  } while (0)

namespace moe {
// Status of the launch just made (counts it, like MOE_LAUNCH_CHECK).
inline moe_status launch_status() {
  __atomic_fetch_add(&g_kernel_launches, 1ull, __ATOMIC_RELAXED);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MOE_OK;
  note_cuda_error(e);
  return MOE_ERR_CUDA;
}
}  // namespace moe

namespace moe {
// Whether launches carry the programmatic-dependent-launch attribute (default on; the environment
// variable MOE_DISABLE_PDL=1 turns it off).
bool pdl_enabled();

// Launch `kern` on `st` with the programmatic-dependent-launch attribute (and, when cluster_x > 1,
// a cluster dimension); counts the launch and records a failure like launch_status().
template <typename... KArgs, typename... Args>
inline moe_status launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t st, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  __atomic_fetch_add(&g_kernel_launches, 1ull, __ATOMIC_RELAXED);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    note_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
}  // namespace moe

#define MOE_TRY_S(expr)                 \
  do {                                  \
    const moe_status s_ = (expr);       \
    if (s_ != MOE_OK) return s_;        \
  } while (0)
