// Router on tcgen05 tensor cores: gate logits, softmax and top-k fused in one kernel.
//
// Step 1 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 1: a small router, replicated on every device, gates the local tokens; top-k gate of
// section "框架").  The gate is a thin GEMM (N = E experts) that must run at the speed of reading
// x once from HBM: with E = 64 its 2*T*d*E FLOPs are more than the CUDA cores deliver in that
// time, so the contraction runs on the tensor cores and everything after it stays on chip.
//
// One CTA per 128 tokens (192 threads): warp 0 streams x tiles [128 x 64] and the whole gate
// matrix slice [E_pad x 64] (E rounded up to 16, zero rows from TMA's out-of-bounds fill) through
// a ring of up to 16 stages (as many as shared memory holds: with d <= 1024 and few experts the
// whole token tile is in flight at once, since a CTA has only one tile to load); one lane of warp 1 issues tcgen05.mma (M = 128, N = E_pad) into a TMEM
// accumulator; warps 2..5 read it back with tcgen05.ld, so each thread holds the E logits of one
// token, adds the bias, writes the logits and runs the serial softmax + top-k of route_serial.cuh.
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "route_serial.cuh"
#include "tc_host.h"
#include "tc_ptx.cuh"

namespace moe {
namespace tc {
namespace {

constexpr int MAX_RSTAGES = 16;
constexpr size_t RSMEM_BUDGET = 200 * 1024;   // stage ring bytes
constexpr uint32_t RA_BYTES = 128 * 64 * 2;  // x tile

struct alignas(64) RouterParams {
  CUtensorMap x_map;  // x [T, d], box {64, 128}
  CUtensorMap w_map;  // Wg [E, d], box {64, E_pad}
  const float* bias;
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  uint32_t* status;   // may be null (no status word to report a timeout into)
  unsigned long long timeout_ns;
  int T, d, E, E_pad, k, gate_norm;
  uint32_t idesc, tmem_cols, stage_bytes;
  int nstages;
  int stall;          // failure-path test: the MMA issuer first waits on a barrier nothing arrives on
};

__global__ void __launch_bounds__(192, 1) router_tc_kernel(const __grid_constant__ RouterParams P) {
  pdl_prologue();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const int RSTAGES = P.nstages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RSTAGES * P.stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + RSTAGES;
  uint64_t* tfull = bars + 2 * RSTAGES;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < RSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, P.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m0 = blockIdx.x * 128;
  const int nk = P.d / 64;
  const unsigned long long budget = P.timeout_ns;

  uint32_t outstanding = 0, out_phase = 0;   // producer: stages loaded and not seen consumed
  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, budget)) break;
      outstanding &= ~(1u << stage);
      mbar_expect_tx(&full[stage], P.stage_bytes);
      uint8_t* sA = smem + stage * P.stage_bytes;
      tma_load_2d(sA, &P.x_map, &full[stage], kb * 64, m0);
      tma_load_2d(sA + RA_BYTES, &P.w_map, &full[stage], kb * 64, 0);
      outstanding |= 1u << stage;
      out_phase = (out_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == RSTAGES) { stage = 0; phase ^= 1u; }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    bool issued = false, ok = true;
    // test hook: `drain` gets no arrival before an abort, so this wait runs out after `budget`
    if (P.stall && !wait_bounded(drain, 0u, abort_flag, budget)) ok = false;
    for (int kb = 0; ok && kb < nk; ++kb) {
      if (!wait_bounded(&full[stage], phase, abort_flag, budget)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + stage * P.stage_bytes);
      const uint32_t sb = sa + RA_BYTES;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_bf16(tmem_base, sw128_desc(sa + k * 32, 16, 1024), sw128_desc(sb + k * 32, 16, 1024),
                  P.idesc, (kb > 0 || k > 0) ? 1u : 0u);
      issued = true;
      umma_commit(&empty[stage]);
      if (++stage == RSTAGES) { stage = 0; phase ^= 1u; }
    }
    if (ok) umma_commit(tfull);
    if (*abort_flag && issued) {
      umma_commit(drain);
      volatile int never = 0;
      wait_bounded(drain, 0, &never, 20000000ull);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    if (wait_bounded(tfull, 0, abort_flag, budget)) {
      __syncwarp();
      tc_fence_after();
      const int t = m0 + quarter * 32 + lane;
      const bool live = t < P.T;
      TopK8 st;
      topk_init(st);
      float v[16];
      for (int c = 0; c < P.E_pad / 16; ++c) {
        tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(c * 16), v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c * 16 + i;
          if (e < P.E) {
            const float l = v[i] + (P.bias ? P.bias[e] : 0.f);
            if (live) P.logits[(size_t)t * P.E + e] = l;
            topk_push(st, l, e);
          }
        }
      }
      if (live)
        topk_finish(st, P.k, P.gate_norm, P.topk_idx + (size_t)t * P.k,
                    P.topk_w + (size_t)t * P.k);
    } else {
      // the accumulator never arrived (a wait ran out): write a well-formed placeholder routing
      // (experts 0..k-1, weight 0, logits 0) so the kernels after this one stay in bounds; the
      // status word reports the timeout
      const int t = m0 + quarter * 32 + lane;
      if (t < P.T) {
        for (int e = 0; e < P.E; ++e) P.logits[(size_t)t * P.E + e] = 0.f;
        for (int j = 0; j < P.k; ++j) {
          P.topk_idx[(size_t)t * P.k + j] = j;
          P.topk_w[(size_t)t * P.k + j] = 0.f;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();   // every role has finished (the abort flag is final)
  if (*abort_flag && warp == 0 && lane == 0) {
    // TMA loads of an aborted CTA may still be in flight: let them land before it exits
    for (int s = 0; s < RSTAGES; ++s)
      if (outstanding & (1u << s)) {
        volatile int never = 0;
        wait_bounded(&full[s], (out_phase >> s) & 1u, &never, 20000000ull);
      }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && P.status) atomicOr(P.status, MOE_STATUS_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

}  // namespace
}  // namespace tc

bool router_tc_supported(const Dims& D) {
  return D.dtype == MOE_DTYPE_BF16 && D.d % 64 == 0 && D.E <= 256 && tc::encoder() != nullptr;
}

moe_status launch_router_tc(const Dims& D, const void* x, const void* Wg, const float* bias,
                            float* logits, int32_t* topk_idx, float* topk_w, uint32_t* status,
                            cudaStream_t st) {
  using namespace tc;
  RouterParams P;
  memset(&P, 0, sizeof(P));
  const int E_pad = (int)round_up(D.E, 16);
  if (!map2(&P.x_map, x, D.d, D.T, 64, 128) || !map2(&P.w_map, Wg, D.d, D.E, 64, E_pad))
    return MOE_ERR_CUDA;
  P.bias = D.has_bias ? bias : nullptr;
  P.logits = logits;
  P.topk_idx = topk_idx;
  P.topk_w = topk_w;
  P.status = status;
  P.timeout_ns = tc::wait_budget_ns();
  P.stall = tc::wait_stall();
  P.T = D.T;
  P.d = D.d;
  P.E = D.E;
  P.E_pad = E_pad;
  P.k = D.k;
  P.gate_norm = D.gate_norm;
  P.idesc = idesc_bf16_m128(E_pad, false, false);
  uint32_t cols = 32;
  while ((int)cols < E_pad) cols <<= 1;
  P.tmem_cols = cols;
  P.stage_bytes = RA_BYTES + (uint32_t)E_pad * 128u;
  P.nstages = (int)std::min<size_t>(std::min<size_t>(MAX_RSTAGES, RSMEM_BUDGET / P.stage_bytes),
                                    (size_t)(D.d / 64));
  const size_t smem = 1024 + (size_t)P.nstages * P.stage_bytes + 512;
  if (cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_k(router_tc_kernel, (D.T + 127) / 128, 192, smem, st, 1, P);
}

}  // namespace moe
