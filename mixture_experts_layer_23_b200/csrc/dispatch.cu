// Capacity-limited dispatch of token rows into expert-contiguous buffers.
//
// Step 2 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 2) and the exchange of section "All-to-All 通信模式", part 二 (device i sends the subset
// S_ik of its tokens to expert k's device).  On one GPU the exchange is a permutation in HBM;
// the expert-contiguous buffer it fills is exactly what an all-to-all would send.
//
// Ranking rule: within one expert, assignments are ordered by token index; the first C are kept
// ("drop by token order").  The rank must be bit-exact and deterministic, so it is computed as a
// stable counting sort in three launches, none of which waits on another CTA:
//   1. rank:    each CTA takes 256 tokens; per warp, a shared-memory bitmask per expert marks the
//               lanes (tokens) that chose it, so a popcount of the lower lanes gives each
//               assignment's rank inside the warp; warp bases make it a rank inside the CTA.
//               The CTA's per-expert histogram goes to scratch.  Choice-major priority
//               (drop_order 1) repeats this per choice index j: k histogram layers, and each
//               assignment's rank inside its CTA's layer.
//   2. scan:    one warp per expert turns its histogram column into exclusive bases (over rank
//               CTAs in token order; choice-major: over layers first, then rank CTAs), in place,
//               and writes counts and kept = min(counts, C);
//   3. scatter: every CTA derives the 128-row aligned offsets from kept; one warp per token
//               finalises its slots (its rank CTA's base + its rank inside the CTA) and copies its
//               x row, read once and written to each kept slot (bulk copies through a shared-memory
//               buffer, or 16-byte register copies for rows too long for the buffers); extra CTAs
//               zero padding rows.
#include <mutex>

#include "common.cuh"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int DT = kDispatchTokensPerBlock;  // 256 tokens = 8 warps x 32 lanes
static_assert(DT == 256, "rank kernel assumes 8 warps of 32 tokens");

template <bool CM>
__global__ void __launch_bounds__(256)
dispatch_rank_kernel(const int32_t* __restrict__ topk_idx, int T_, int E, int k,
                     int32_t* __restrict__ blk_counts, int32_t* __restrict__ local_rank) {
  pdl_prologue();
  __shared__ uint32_t mask[8][256];
  __shared__ int32_t wbase[8][256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = blockIdx.x * DT + tid;
  int e_of[8];
  if (t < T_)
    for (int j = 0; j < k; ++j) e_of[j] = topk_idx[(int64_t)t * k + j];
  const uint32_t below = (1u << lane) - 1u;
  // token order: one pass over all choices; choice-major: one pass (layer) per choice index
  for (int layer = 0; layer < (CM ? k : 1); ++layer) {
    for (int i = tid; i < 8 * 256; i += 256) (&mask[0][0])[i] = 0u;
    __syncthreads();
    if (t < T_)
      for (int j = CM ? layer : 0; j < (CM ? layer + 1 : k); ++j)
        if ((unsigned)e_of[j] < (unsigned)E) atomicOr(&mask[warp][e_of[j]], 1u << lane);
    __syncthreads();
    for (int e = tid; e < E; e += 256) {
      int run = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        wbase[w][e] = run;
        run += __popc(mask[w][e]);
      }
      blk_counts[((int64_t)blockIdx.x * (CM ? k : 1) + layer) * E + e] = run;
    }
    __syncthreads();
    if (t < T_)
      for (int j = CM ? layer : 0; j < (CM ? layer + 1 : k); ++j) {
        const int e = e_of[j];
        local_rank[(int64_t)t * k + j] =
            ((unsigned)e < (unsigned)E) ? wbase[warp][e] + __popc(mask[warp][e] & below) : 0;
      }
    __syncthreads();   // wbase and mask are reused by the next layer
  }
}

// Scan: one warp per expert turns that expert's column of the rank CTAs' histograms into
// exclusive bases in drop-priority order (token order: rank CTAs in order; choice-major: choice
// layers first, then rank CTAs), in place, and writes counts (the total) and kept = min(counts, C).
__global__ void __launch_bounds__(256)
dispatch_scan_kernel(int32_t* __restrict__ blk /* in: block counts, out: exclusive bases */,
                     int n_blk, int E, int L, int64_t C, int32_t* __restrict__ counts_out,
                     int32_t* __restrict__ kept_out) {
  pdl_prologue();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= E) return;
  const int n = n_blk * L;
  int carry = 0;
#pragma unroll 4
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int layer = i / n_blk, b = i - layer * n_blk;
    const int64_t at = ((int64_t)b * L + layer) * E + e;
    const int v = (i < n) ? blk[at] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (i < n) blk[at] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    counts_out[e] = carry;
    kept_out[e] = (int64_t)carry < C ? carry : (int)C;
  }
}

// Scatter.  Every CTA turns kept into the 128-row aligned segment offsets (an exclusive prefix
// over at most 256 experts; CTA 0 also writes them out).  Then one warp per token finalises its
// slots (base of its rank CTA from the scan + its rank inside that CTA) and copies its x row
// (16-byte vectors, read once, written to each kept slot); the last E + 1 CTAs zero the padding
// rows and mark shared rows in row_token.
constexpr int SC_TOK = 32;   // tokens per scatter CTA (four per warp)
static_assert(DT % SC_TOK == 0, "a scatter CTA must not straddle two rank CTAs");

// BULK: rows move through shared memory by bulk copies (one warp lane issues them): each warp
// keeps SC_NB row buffers, loading token i + SC_NB while token i's row is stored to its slots.
// Measured against 16-byte register copies (kernel bench, L2 flushed): 90.1 -> 79.1 us on the
// Mixtral-style layer, 74.8 -> 71.3 us DeepSeek-style, 22.8 -> 18.2 us GPT-2-style.  Rows too
// long for 8 warps x SC_NB buffers in shared memory (over kBulkMaxSmem) take the register copies.
constexpr int SC_NB = 2;
constexpr size_t kBulkMaxSmem = 200 * 1024;

// The slot of this lane's assignment (lanes < k) of token t: its rank CTA's base + its rank inside
// that CTA, kept if below C; writes slot[] and row_token[].  Returns -1 for dropped assignments.
template <bool CM>
__device__ __forceinline__ int finalise_slot(const int32_t* __restrict__ topk_idx,
                                             const int32_t* __restrict__ blk_base,
                                             const int32_t* s_off, int t, int E, int k, int64_t C,
                                             int my_blk, int32_t* __restrict__ slot,
                                             int32_t* __restrict__ row_token, int lane) {
  int my_slot = -1;
  if (lane < k) {
    const int L = CM ? k : 1;
    const int e = topk_idx[(int64_t)t * k + lane];
    const bool valid = (unsigned)e < (unsigned)E;  // an out-of-range id is never kept
    const int layer = CM ? lane : 0;
    const int pos = valid ? blk_base[((int64_t)my_blk * L + layer) * E + e] +
                                slot[(int64_t)t * k + lane]
                          : 0;
    if (valid && (int64_t)pos < C) {
      my_slot = s_off[e] + pos;
      row_token[my_slot] = t;
    }
    slot[(int64_t)t * k + lane] = my_slot;
  }
  return my_slot;
}

// Bulk-copy form of the row copies: warp w takes tokens w, w + 8, w + 16, w + 24 of the CTA.  Lane 0
// loads each token's row into one of the warp's SC_NB shared-memory buffers (an mbarrier per
// buffer), stores it to each kept slot, and reloads the buffer for the token SC_NB later once those
// stores have read it.  Every wait is bounded: when one runs out the warp stops, lets its copies in
// flight land, and the status word (if any) reports MOE_STATUS_TIMEOUT.
template <typename T, bool CM>
__device__ __forceinline__ void scatter_rows_bulk(
    const T* __restrict__ x, const int32_t* __restrict__ topk_idx,
    const int32_t* __restrict__ blk_base, const int32_t* s_off, int T_, int d, int E, int k,
    int64_t C, int my_blk, int32_t* __restrict__ slot, int32_t* __restrict__ row_token,
    T* __restrict__ Xd, uint32_t* __restrict__ status, unsigned long long budget) {
  extern __shared__ __align__(128) uint8_t sc_rows[];   // [8 warps][SC_NB][row bytes], barriers
  __shared__ int sc_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t rb = (uint32_t)d * (uint32_t)sizeof(T);
  uint8_t* buf = sc_rows + (size_t)warp * SC_NB * rb;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sc_rows + (size_t)8 * SC_NB * rb) + warp * SC_NB;
  if (threadIdx.x == 0) sc_abort = 0;
  if (lane == 0) {
    for (int b = 0; b < SC_NB; ++b) tc::mbar_init(&bars[b], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort_flag = &sc_abort;
  const int t0 = blockIdx.x * SC_TOK + warp;
  int n = 0;   // this warp's tokens: t0 + 8 i, i < n
  while (n < SC_TOK / 8 && t0 + 8 * n < T_) ++n;
  int pend[SC_NB];   // token (index i) whose load into buffer b is in flight, -1 if none
#pragma unroll
  for (int b = 0; b < SC_NB; ++b) pend[b] = -1;
  if (lane == 0)
    for (int i = 0; i < n && i < SC_NB; ++i) {
      tc::mbar_expect_tx(&bars[i], rb);
      tc::bulk_g2s(buf + (size_t)i * rb, x + (int64_t)(t0 + 8 * i) * d, rb, &bars[i]);
      pend[i] = i;
    }
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    const int t = t0 + 8 * i;
    const int my_slot = finalise_slot<CM>(topk_idx, blk_base, s_off, t, E, k, C, my_blk, slot,
                                          row_token, lane);
    int sl[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sl[j] = __shfl_sync(0xffffffffu, my_slot, j);
    if (lane == 0 && ok) {
      const int b = i % SC_NB;
      if (!tc::wait_bounded(&bars[b], (uint32_t)(i / SC_NB) & 1u, abort_flag, budget)) {
        ok = false;
      } else {
        pend[b] = -1;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && sl[j] >= 0) tc::bulk_s2g(Xd + (int64_t)sl[j] * d, buf + (size_t)b * rb, rb);
        tc::bulk_commit();
        if (i + SC_NB < n) {
          tc::bulk_wait_read<0>();   // this buffer's stores have read it
          tc::mbar_expect_tx(&bars[b], rb);
          tc::bulk_g2s(buf + (size_t)b * rb, x + (int64_t)(t + 8 * SC_NB) * d, rb, &bars[b]);
          pend[b] = i + SC_NB;
        }
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    // loads still in flight after an abort land before the CTA exits (bounded), then every store
    // has completed
#pragma unroll
    for (int b = 0; b < SC_NB; ++b)
      if (pend[b] >= 0) {
        volatile int never = 0;
        tc::wait_bounded(&bars[b], (uint32_t)(pend[b] / SC_NB) & 1u, &never, 20000000ull);
      }
    tc::bulk_wait<0>();
    if (!ok && status) atomicOr(status, MOE_STATUS_TIMEOUT);
  }
}

template <typename T, bool CM, bool BULK>
__global__ void __launch_bounds__(256)
dispatch_scatter_kernel(const T* __restrict__ x, const int32_t* __restrict__ topk_idx,
                        const int32_t* __restrict__ blk_base, const int32_t* __restrict__ kept,
                        int T_, int d, int E, int k, int64_t C, int routed_row0, int n_tok_blocks,
                        int shared_rows, int32_t* __restrict__ offsets_out,
                        int32_t* __restrict__ slot /* in: local rank, out: slot */,
                        int32_t* __restrict__ row_token, T* __restrict__ Xd,
                        uint32_t* __restrict__ status, unsigned long long budget) {
  pdl_prologue();
  __shared__ int32_t s_kept[256];
  __shared__ int32_t s_off[257];
  constexpr int VN = Vec16<T>::N;
  const int nv = d / VN;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool tok_cta = (int)blockIdx.x < n_tok_blocks;
  const int my_blk = tok_cta ? (int)(blockIdx.x * SC_TOK / DT) : 0;
  for (int e = threadIdx.x; e < E; e += 256) {
    const int kp = kept[e];
    s_kept[e] = kp;
    s_off[e + 1] = (int)round_up(kp, MOE_ROW_ALIGN);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix of the segment sizes
    int carry = routed_row0;
    for (int base = 0; base < E; base += 32) {
      const int i = base + lane;
      int v = (i < E) ? s_off[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (i < E) s_off[i + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) s_off[0] = routed_row0;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += 256) offsets_out[e] = s_off[e];

  if (!tok_cta) {
    // padding rows of routed expert e (or, for the last CTA, the shared rows' row_token)
    const int e = blockIdx.x - n_tok_blocks;
    if (e < E) {
      const int r0 = s_off[e] + s_kept[e], r1 = s_off[e + 1];
      Vec16<T> z;
      z.raw = make_uint4(0, 0, 0, 0);
      for (int r = r0 + warp; r < r1; r += 8) {
        if (lane == 0) row_token[r] = -1;
        for (int v = lane; v < nv; v += 32) st_vec(Xd + (int64_t)r * d + (int64_t)v * VN, z);
      }
    } else {
      for (int r = threadIdx.x; r < shared_rows; r += blockDim.x) row_token[r] = -1;
    }
    return;
  }
  if constexpr (BULK) {
    scatter_rows_bulk<T, CM>(x, topk_idx, blk_base, s_off, T_, d, E, k, C, my_blk, slot,
                             row_token, Xd, status, budget);
  } else {
    for (int tt = warp; tt < SC_TOK; tt += 8) {
      const int t = blockIdx.x * SC_TOK + tt;
      if (t >= T_) break;
      const int my_slot = finalise_slot<CM>(topk_idx, blk_base, s_off, t, E, k, C, my_blk, slot,
                                            row_token, lane);
      int sl[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) sl[j] = __shfl_sync(0xffffffffu, my_slot, j);
      const T* src = x + (int64_t)t * d;
#pragma unroll 8
      for (int v = lane; v < nv; v += 32) {
        const Vec16<T> val = ld_vec_stream(src + (int64_t)v * VN);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && sl[j] >= 0) st_vec(Xd + (int64_t)sl[j] * d + (int64_t)v * VN, val);
      }
    }
  }
}

}  // namespace

template <typename T, bool CM>
static moe_status dispatch_t(const Dims& D, const void* x, const int32_t* topk_idx,
                             int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* slot,
                             int32_t* row_token, void* Xd, int32_t* blk_counts, uint32_t* status,
                             cudaStream_t st) {
  MOE_TRY_S(launch_k(dispatch_rank_kernel<CM>, D.n_blk, 256, 0, st, 1, topk_idx, D.T, D.E, D.k,
                     blk_counts, slot));
  MOE_TRY_S(launch_k(dispatch_scan_kernel, (D.E + 7) / 8, 256, 0, st, 1, blk_counts, D.n_blk, D.E,
                     D.n_layers, D.C, counts, kept));
  const int n_tok_blocks = (D.T + SC_TOK - 1) / SC_TOK;
  const int grid = n_tok_blocks + D.E + 1;
  const size_t smem = (size_t)8 * SC_NB * D.d * sizeof(T) + 8 * SC_NB * 8;
  if (smem <= kBulkMaxSmem) {
    static size_t smem_set = 48 * 1024;
    if (smem > smem_set) {
      if (cudaFuncSetAttribute(dispatch_scatter_kernel<T, CM, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MOE_ERR_CUDA;
      smem_set = smem;
    }
    return launch_k(dispatch_scatter_kernel<T, CM, true>, grid, 256, smem, st, 1, (const T*)x,
                    topk_idx, (const int32_t*)blk_counts, (const int32_t*)kept, D.T, D.d, D.E,
                    D.k, D.C, (int)D.routed_row0, n_tok_blocks, (int)D.routed_row0, offsets, slot,
                    row_token, (T*)Xd, status, tc::wait_budget_ns());
  }
  return launch_k(dispatch_scatter_kernel<T, CM, false>, grid, 256, 0, st, 1, (const T*)x,
                  topk_idx, (const int32_t*)blk_counts, (const int32_t*)kept, D.T, D.d, D.E, D.k,
                  D.C, (int)D.routed_row0, n_tok_blocks, (int)D.routed_row0, offsets, slot,
                  row_token, (T*)Xd, status, tc::wait_budget_ns());
}

moe_status launch_dispatch(const Dims& D, const void* x, const int32_t* topk_idx, int32_t* counts,
                           int32_t* kept, int32_t* offsets, int32_t* slot, int32_t* row_token,
                           void* Xd, int32_t* blk_counts, uint32_t* status, cudaStream_t st) {
  if (D.dtype == MOE_DTYPE_BF16) {
    if (D.choice_major)
      return dispatch_t<__nv_bfloat16, true>(D, x, topk_idx, counts, kept, offsets, slot,
                                             row_token, Xd, blk_counts, status, st);
    return dispatch_t<__nv_bfloat16, false>(D, x, topk_idx, counts, kept, offsets, slot,
                                            row_token, Xd, blk_counts, status, st);
  }
  if (D.choice_major)
    return dispatch_t<float, true>(D, x, topk_idx, counts, kept, offsets, slot, row_token, Xd,
                                   blk_counts, status, st);
  return dispatch_t<float, false>(D, x, topk_idx, counts, kept, offsets, slot, row_token, Xd,
                                  blk_counts, status, st);
}

// ----------------------------------------------------------------------------- no-allocation form
//
// moe_dispatch_noalloc: the same dispatch for callers that cannot allocate device memory.  The
// per-CTA expert histograms (the only scratch the dispatch needs) live in a fixed array inside
// this library instead of a caller-supplied buffer.  Every device that loads the library holds the
// array (256 KB) until the process exits.  All calls share it, so calls that overlap on the GPU
// race; it keeps the last call's contents, and needs no clearing because the rank kernel writes
// every entry a call reads before the scan reads it.

constexpr int kNoAllocMaxHistogram = 1 << 16;  // int32 entries: ceil(T / 256) * E (* k when
                                               // choice-major) must fit
static __device__ __align__(256) int32_t g_noalloc_histogram[kNoAllocMaxHistogram];

// The CUDA context current on this thread (through the runtime's driver entry point, so the
// library does not link libcuda); null if it cannot be read.
static void* current_context() {
  typedef int (*CtxGetCurrentFn)(void**);
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the array on the current device, looked up once per device (with that device
// current, on its first call) and again whenever that device's context has changed since (after a
// cudaDeviceReset the module is loaded anew and the array may sit elsewhere).  In host code the
// array's name is only a host-side stand-in, so the kernels must be given this address, never the
// name.
static moe_status noalloc_histogram(int32_t** out) {
  constexpr int kMaxDevices = 64;
  static int32_t* addr[kMaxDevices] = {};
  static void* ctx_of[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  void* ctx = current_context();   // null before the runtime has made a context current
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || !ctx || ctx != ctx_of[dev]) {
    void* p = nullptr;
    // (this call also makes the device's primary context current on this thread)
    if (cudaGetSymbolAddress(&p, g_noalloc_histogram) != cudaSuccess || !p) return MOE_ERR_CUDA;
    addr[dev] = static_cast<int32_t*>(p);
    ctx_of[dev] = current_context();
  }
  *out = addr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" moe_status moe_dispatch_noalloc(const moe_config_t* cfg, const void* x,
                                           const int32_t* topk_idx, int32_t* counts, int32_t* kept,
                                           int32_t* offsets, int32_t* slot, int32_t* row_token,
                                           void* Xd, moe_stream_t stream) {
  moe::Dims D;
  const moe_status s = moe::resolve_dims(cfg, &D);
  if (s != MOE_OK) return s;
  const void* ptrs[] = {x, topk_idx, counts, kept, offsets, slot, row_token, Xd};
  for (const void* p : ptrs) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)p & 15u) != 0) return MOE_ERR_MISALIGNED;
  }
  if ((int64_t)D.n_blk * D.n_layers * D.E > moe::kNoAllocMaxHistogram)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  int32_t* hist = nullptr;
  const moe_status h = moe::noalloc_histogram(&hist);
  if (h != MOE_OK) return h;
  return moe::launch_dispatch(D, x, topk_idx, counts, kept, offsets, slot, row_token, Xd, hist,
                              nullptr, (cudaStream_t)stream);
}
