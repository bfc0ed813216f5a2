// Router on tcgen05 tensor cores: gate logits, softmax and top-k fused in one kernel.
//
// Step 1 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 1: a small router, replicated on every device, gates the local tokens; top-k gate of
// section "框架").  The gate is a thin GEMM (N = E experts) that must run at the speed of reading
// x once from HBM: with E = 64 its 2*T*d*E FLOPs are more than the CUDA cores deliver in that
// time, so the contraction runs on the tensor cores and everything after it stays on chip.
//
// One CTA per tile of at most 128 tokens (192 threads).  Warp 0 streams x tiles [rows x 64] and the
// gate matrix slice [E_pad x 64] (E rounded up to 16, zero rows from TMA's out-of-bounds fill)
// through a ring of up to 16 stages: as many as shared memory holds, so with d <= 1024 and few
// experts the whole token tile is in flight at once (a CTA has only one tile to load).  One lane of
// warp 1 issues tcgen05.mma (M = 128, N = E_pad) into a TMEM accumulator.  Warps 2..5 read it back
// with tcgen05.ld, one token per thread, add the bias, write the logits and run the softmax + top-k
// of route_serial.cuh (k slots per token, the softmax denominator in a second pass).
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
// x loads leave in groups of this many consecutive k blocks (see the producer loop).  Measured with
// the router alone, L2 flushed between launches: groups of 2 took 4-6 % off every bf16 layer size
// (Mixtral-style 35.6 -> 33.6 us, DeepSeek-style 37.4 -> 35.7 us); groups of 4 and 8 were slower
// than 2, since the producer then holds back more free stages.
#ifndef MOE_ROUTER_ISSUE_GROUP
#define MOE_ROUTER_ISSUE_GROUP 2
#endif
constexpr uint32_t RA_BYTES = 128 * 64 * 2;  // x tile
constexpr int STAGE_MAX_EPAD = 64;            // rows of at most 64 logits are staged in shared memory

// Shared memory per CTA: the router keeps up to ~200 KB of loads in flight; the router weight
// gradient stays within 112 KB so that two of its CTAs share an SM.
constexpr size_t RSMEM_WHOLE = 226 * 1024;
constexpr size_t RSMEM_SPLIT = 112 * 1024;

struct alignas(64) RouterParams {
  CUtensorMap x_map;  // x [T, d], box {64, rows}
  CUtensorMap w_map;  // Wg [E, d], box {64, E_pad}
  const float* bias;
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  uint32_t* status;   // may be null (no status word to report a timeout into)
  unsigned long long timeout_ns;
  int T, d, E, E_pad, k, gate_norm;
  int rows;           // tokens per CTA (<= 128): the tiles are balanced over the SMs
  uint32_t idesc, tmem_cols, stage_bytes;
  int nstages;
  uint32_t region;    // bytes before the barriers: the load ring, which the staged rows reuse
  int stall;          // failure-path test: the MMA issuer first waits on a barrier nothing arrives on
};

__device__ __forceinline__ void epi_bar() {   // the 128 epilogue threads (warps 2..5)
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// the same barrier, returning whether `v` holds in every epilogue thread
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// One CTA per token tile contracts the whole of d.  A tile holds `rows` <= 128 tokens, chosen on
// the host so that the tiles come out close to a whole number of waves over the SMs (T = 16384:
// 147 tiles of 112 tokens instead of 128 tiles of 128, which left 20 SMs idle); the MMA still
// runs M = 128, and the accumulator lanes past `rows` (zero rows of A) are never read.
// (Splitting the contraction over a cluster, with the partial logits added over distributed
// shared memory, measured slower at every layer size and was dropped.)
// Rows of at most 64 logits are staged in shared memory with the expert ids and gate weights, and
// leave as contiguous rows.
// KS: top-k slots kept per token (>= k), so the insertion work per expert scales with k, not 8.
template <int KS>
__global__ void __launch_bounds__(192, 1) router_tc_kernel(const __grid_constant__ RouterParams P) {
  pdl_prologue();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const int RSTAGES = P.nstages;
  const bool small = P.E_pad <= STAGE_MAX_EPAD;   // rows staged in shared memory
  // staging row stride (floats): odd, so the 32 lanes' scalar accesses to their own rows (column
  // e of rows 32q..32q+31) hit 32 distinct banks
  const int PS = P.E_pad + 1;
  // The staged rows reuse the load ring: they are written only once every MMA of the tile, the
  // ring's last reader, has completed (so no load is in flight either), which leaves the whole
  // ring to loads in flight until then.
  float* part = reinterpret_cast<float*>(smem);                             // [128][PS]
  int32_t* sidx = reinterpret_cast<int32_t*>(part + (small ? 128 * PS : 0));  // [128][9]
  float* sw = reinterpret_cast<float*>(sidx + 128 * 9);                     // [128][9]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.region);
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
  // A rows [rows, 128) of the stages are never loaded and hold whatever shared memory held: each
  // accumulator lane depends only on its own A row, and lanes past the tile's tokens are not stored.
  // (Zeroing them cost 3.6 us per launch on the GPT-2-style layer, 32-token tiles.)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m0 = blockIdx.x * P.rows;
  const int nk = P.d / 64;
  const unsigned long long budget = P.timeout_ns;

  uint32_t outstanding = 0, out_phase = 0;   // producer: stages loaded and not seen consumed
  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    // loads leave in groups of G consecutive k blocks: the producer waits until G stages are free,
    // then issues them back to back, so that the G 128-byte pieces of each token row reach the
    // memory system together
    const int G = min(MOE_ROUTER_ISSUE_GROUP, RSTAGES);
    bool ok = true;
    for (int kb0 = 0; ok && kb0 < nk; kb0 += G) {
      const int gn = min(G, nk - kb0);
      int s = stage;
      uint32_t ph = phase;
      for (int j = 0; j < gn; ++j) {
        if (!wait_bounded(&empty[s], ph ^ 1u, abort_flag, budget)) { ok = false; break; }
        outstanding &= ~(1u << s);
        if (++s == RSTAGES) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      for (int kb = kb0; kb < kb0 + gn; ++kb) {
        mbar_expect_tx(&full[stage], (uint32_t)(P.rows + P.E_pad) * 128u);
        uint8_t* sA = smem + stage * P.stage_bytes;
        tma_load_2d(sA, &P.x_map, &full[stage], kb * 64, m0);
        tma_load_2d(sA + RA_BYTES, &P.w_map, &full[stage], kb * 64, 0);
        outstanding |= 1u << stage;
        out_phase = (out_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == RSTAGES) { stage = 0; phase ^= 1u; }
      }
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
  }

  // ---- epilogue: warps 2..5, one token (TMEM lane) per thread
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;          // token row inside the tile
  const int t = m0 + row;
  const bool epi = warp >= 2;
  const int nrow = min(P.rows, P.T - m0);       // the tile's tokens
  bool have = false;                             // this warp holds its accumulator rows
  if (epi) {
    // warp-uniform: the TMEM loads below need the whole warp
    have = __all_sync(0xffffffffu, wait_bounded(tfull, 0, abort_flag, budget));
  }
  if (have) tc_fence_after();
  if (epi) {
    // a placeholder routing (experts 0..k-1, weight 0, logits 0) when any wait of the tile ran
    // out, so that the kernels after this one stay in bounds; the status word reports it
    const bool ok = have && !*abort_flag;
    const bool live = row < nrow;
    // staging only when every epilogue thread saw the tile complete: otherwise loads may still be
    // landing in the ring, and the placeholders go straight to global memory
    const bool staged = small && epi_bar_and(ok);
    if (small && !staged) {
      if (live) {
        for (int e = 0; e < P.E; ++e) P.logits[(size_t)t * P.E + e] = 0.f;
        for (int j = 0; j < P.k; ++j) {
          P.topk_idx[(size_t)t * P.k + j] = j;
          P.topk_w[(size_t)t * P.k + j] = 0.f;
        }
      }
    } else if (small) {
      // the row's logits (+ bias) go to its staging row 16 at a time, then the serial softmax +
      // top-k reads them back from there: a short loop body instead of E unrolled steps, whose
      // code outgrew the instruction cache at 64 experts
      float* prow = part + row * PS;
      const uint32_t ta = tmem_base + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < P.E_pad / 16; ++c) {
        float v[16];
        tmem_ld16(ta + (uint32_t)(c * 16), v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c * 16 + i;
          if (e < P.E) prow[e] = v[i] + (P.bias ? P.bias[e] : 0.f);
        }
      }
      TopK<KS> st;
      topk_init(st);
#pragma unroll 4
      for (int e = 0; e < P.E; ++e) topk_push(st, prow[e], e);
      float den = 0.f;
      if (P.gate_norm == 0) {
#pragma unroll 8
        for (int e = 0; e < P.E; ++e) den += softmax_term(st, prow[e]);
      }
      topk_finish(st, P.k, P.gate_norm, den, sidx + row * 9, sw + row * 9);
      epi_bar();
      // the tile's rows are contiguous in logits, topk_idx and topk_w: coalesced stores
      const int tid = threadIdx.x - 64;
      for (int i = tid; i < nrow * P.E; i += 128)
        P.logits[(size_t)m0 * P.E + i] = part[(i / P.E) * PS + i % P.E];
      for (int i = tid; i < nrow * P.k; i += 128) {
        P.topk_idx[(size_t)m0 * P.k + i] = sidx[(i / P.k) * 9 + i % P.k];
        P.topk_w[(size_t)m0 * P.k + i] = sw[(i / P.k) * 9 + i % P.k];
      }
    } else if (ok) {
      // wide rows (more than 64 experts): stream them out of TMEM 16 at a time
      TopK<KS> st;
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
      float den = 0.f;
      if (P.gate_norm == 0) {   // second pass over the accumulator for the softmax denominator
        for (int c = 0; c < P.E_pad / 16; ++c) {
          tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(c * 16), v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = c * 16 + i;
            if (e < P.E) den += softmax_term(st, v[i] + (P.bias ? P.bias[e] : 0.f));
          }
        }
      }
      if (live)
        topk_finish(st, P.k, P.gate_norm, den, P.topk_idx + (size_t)t * P.k,
                    P.topk_w + (size_t)t * P.k);
    } else if (live) {
      for (int e = 0; e < P.E; ++e) P.logits[(size_t)t * P.E + e] = 0.f;
      for (int j = 0; j < P.k; ++j) {
        P.topk_idx[(size_t)t * P.k + j] = j;
        P.topk_w[(size_t)t * P.k + j] = 0.f;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();             // every role has finished (the abort flag is final)
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

// ----------------------------------------------------------------------------- router weight gradient
//
// dWg = dl^T x, computed as its transpose dWg^T = x^T dl so that the long side, d, is the MMA's M:
// each CTA takes 128 columns of d (M = 128, x read MN-major) and one chunk of tokens (K), against
// every expert at once (N = E rounded up to 64, dl16 read MN-major, one 64-expert swizzle atom per
// 64 experts).  The MMA work is then 2 d N T flops, a few percent of the time it takes to read x,
// and x is read exactly once.  Each CTA writes its chunk's partial dWg[e][d] in fp32 (a warp's lanes
// hold 32 consecutive columns: coalesced); router_wgrad_reduce adds the chunks in order.  The chunks
// are sized so that all CTAs fit in one wave at two per SM.  (Folding the sum into this kernel, the
// last CTA of each 128-column tile adding every chunk's partial, measured slower: on the
// DeepSeek-style layer that CTA's E x 128 x chunks loads took 136 against 30 us for both launches.)

struct alignas(64) RWParams {
  CUtensorMap x_map;   // x [T, d], box {64 (d), 64 (tokens)}
  CUtensorMap l_map;   // dl16 [T, E8], box {64 (experts), 64 (tokens)}; narrow: {16, 64}, 32 B swizzle
  float* part;         // [n_chunks][E][d]
  uint32_t* status;
  unsigned long long timeout_ns;
  int T, d, E, N, chunk, n_dt;
  uint32_t idesc, tmem_cols, stage_bytes;
  int nstages, stall;
  int narrow;          // E <= 16: N = 16, dl16 rows of 32 bytes
};

// Shared-memory descriptor of an MN-major operand in the 32-byte swizzle: atoms of 8 K rows x 32
// bytes (16 bf16 along MN), `sbo` bytes between consecutive 8-row groups.  The operand is a single
// 16-element chunk along MN, so the leading-byte offset (the stride between such chunks) is unused.
__device__ __forceinline__ uint64_t sw32_desc(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((2048u >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 6ull << 61;   // SWIZZLE_32B
  return d;
}

__global__ void __launch_bounds__(192, 1) router_wgrad_tc_kernel(const __grid_constant__ RWParams P) {
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
  const int dt = blockIdx.x % P.n_dt, c = blockIdx.x / P.n_dt;
  const int d0 = dt * 128, t0 = c * P.chunk;
  const int t1 = min(P.T, t0 + P.chunk);
  const int nk = (t1 - t0 + 63) / 64;   // chunks are multiples of 64 tokens: only T ends one early
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
      uint8_t* sB = sA + 16384;
      const int tk = t0 + kb * 64;
      tma_load_2d(sA, &P.x_map, &full[stage], d0, tk);
      tma_load_2d(sA + 8192, &P.x_map, &full[stage], d0 + 64, tk);
      if (P.narrow) tma_load_2d(sB, &P.l_map, &full[stage], 0, tk);
      else
        for (int j = 0; j < P.N / 64; ++j)
          tma_load_2d(sB + j * 8192, &P.l_map, &full[stage], 64 * j, tk);
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
      const uint32_t sb = sa + 16384;
#pragma unroll
      for (int k = 0; k < 4; ++k)   // both operands MN-major: a K step of 16 rows is 2 KB (B narrow: 512 B)
        umma_bf16(tmem_base, sw128_desc(sa + k * 2048, 8192, 1024),
                  P.narrow ? sw32_desc(sb + k * 512, 256) : sw128_desc(sb + k * 2048, 8192, 1024),
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
    const int col = d0 + quarter * 32 + lane;   // this thread's TMEM lane = column of d
    if (__all_sync(0xffffffffu, wait_bounded(tfull, 0, abort_flag, budget))) {
      tc_fence_after();
      float* out = P.part + (size_t)c * P.E * P.d;
      for (int e0 = 0; e0 < P.E; e0 += 16) {
        float v[16];
        tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)e0, v);
        if (col < P.d) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (e0 + i < P.E) out[(size_t)(e0 + i) * P.d + col] = v[i];
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

template <int KS>
static moe_status launch_router_ks(const tc::RouterParams& P, int n_tiles, size_t smem,
                                   cudaStream_t st) {
  static int smem_set = 0;
  if ((int)smem > smem_set) {
    if (cudaFuncSetAttribute(tc::router_tc_kernel<KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    smem_set = (int)smem;
  }
  return launch_k(tc::router_tc_kernel<KS>, n_tiles, 192, smem, st, 1, P);
}

moe_status launch_router_tc(const Dims& D, const void* x, const void* Wg, const float* bias,
                            float* logits, int32_t* topk_idx, float* topk_w, uint32_t* status,
                            cudaStream_t st) {
  using namespace tc;
  RouterParams P;
  memset(&P, 0, sizeof(P));
  const int E_pad = (int)round_up(D.E, 16);
  // tokens per CTA: the fewest waves of 128-token tiles over the SMs, then tiles just large
  // enough to cover T in that many waves (at least 16 tokens, so the per-CTA setup and the gate
  // matrix reads stay small next to the token rows)
  const int n_sm = num_sms();
  const int waves = (D.T + 128 * n_sm - 1) / (128 * n_sm);
  const int rows = (int)round_up(
      std::max(std::min(16, D.T), std::min(128, (D.T + waves * n_sm - 1) / (waves * n_sm))), 8);
  if (!map2(&P.x_map, x, D.d, D.T, 64, (uint32_t)rows) || !map2(&P.w_map, Wg, D.d, D.E, 64, E_pad))
    return MOE_ERR_CUDA;
  P.rows = rows;
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
  const int n_tiles = (D.T + rows - 1) / rows;
  const int nk_cta = D.d / 64;
  const size_t stage_rows = E_pad <= STAGE_MAX_EPAD ? (size_t)128 * (E_pad + 8) * 4 : 0;
  // alignment slack, staged rows, expert ids and weights, barriers (2 per stage + 2), TMEM slot
  // alignment slack, barriers (2 per stage + 2), TMEM slot and abort flag; the staged rows, expert
  // ids and weights reuse the ring
  const size_t fixed = 1024 + 2 * 8 + 16;
  const size_t fit = (RSMEM_WHOLE - fixed) / (P.stage_bytes + 2 * 8);
  P.nstages = (int)std::max<size_t>(
      1, std::min<size_t>(std::min<size_t>(MAX_RSTAGES, fit), (size_t)nk_cta));
  const size_t staged = stage_rows + 2 * 128 * 9 * 4;
  P.region = (uint32_t)round_up(std::max<size_t>((size_t)P.nstages * P.stage_bytes, staged), 8);
  const size_t smem = fixed + P.region + (size_t)P.nstages * 2 * 8;
  return P.k <= 2   ? launch_router_ks<2>(P, n_tiles, smem, st)
         : P.k <= 4 ? launch_router_ks<4>(P, n_tiles, smem, st)
         : P.k <= 6 ? launch_router_ks<6>(P, n_tiles, smem, st)
                    : launch_router_ks<8>(P, n_tiles, smem, st);
}

moe_status launch_router_wgrad_tc(const Dims& D, const __nv_bfloat16* dl16, const void* x,
                                  float* part, int* n_chunks, uint32_t* status, cudaStream_t st) {
  using namespace tc;
  RWParams P;
  memset(&P, 0, sizeof(P));
  const int E8 = (int)round_up(D.E, 8);
  // At most 16 experts: N = 16 MMAs (their cost grows with N) over dl16 rows fetched as 16-element
  // boxes in the 32-byte swizzle, instead of N = 64 with 56 or 48 zero columns.
  P.narrow = E8 <= 16;
  if (!map2(&P.x_map, x, D.d, D.T, 64, 64) ||
      !(P.narrow ? map2_sw32(&P.l_map, dl16, E8, D.T, 16, 64)
                 : map2(&P.l_map, dl16, E8, D.T, 64, 64)))
    return MOE_ERR_CUDA;
  P.part = part;
  P.status = status;
  P.timeout_ns = tc::wait_budget_ns();
  P.stall = tc::wait_stall();
  P.T = D.T;
  P.d = D.d;
  P.E = D.E;
  P.N = P.narrow ? 16 : (int)round_up(D.E, 64);   // 16, or 64..256
  P.n_dt = (D.d + 127) / 128;
  // token chunks: at most two CTAs per SM in all (one wave: a partial second wave of a few CTAs
  // would double the time), within the partial buffer (D.n_tchunk chunks)
  int nc = 2 * num_sms() / P.n_dt;
  nc = std::max(1, std::min(nc, std::min(D.n_tchunk, (D.T + 63) / 64)));
  P.chunk = (int)round_up((D.T + nc - 1) / nc, 64);
  nc = (D.T + P.chunk - 1) / P.chunk;
  P.idesc = idesc_bf16_m128(P.N, true, true);
  uint32_t cols = 64;
  while ((int)cols < P.N) cols <<= 1;
  P.tmem_cols = cols;
  P.stage_bytes = 16384u + (P.narrow ? 64u * 32u : (uint32_t)P.N * 128u);   // x, then dl16
  const int nk_cta = P.chunk / 64;
  const size_t fixed = 1024 + 2 * 8 + 16;
  const size_t fit = (RSMEM_SPLIT - fixed) / (P.stage_bytes + 2 * 8);
  P.nstages = (int)std::max<size_t>(1, std::min<size_t>(std::min<size_t>(8, fit), (size_t)nk_cta));
  const size_t smem = fixed + (size_t)P.nstages * (P.stage_bytes + 2 * 8);
  static int smem_set = 0;
  if ((int)smem > smem_set) {
    if (cudaFuncSetAttribute(router_wgrad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    smem_set = (int)smem;
  }
  *n_chunks = nc;
  return launch_k(router_wgrad_tc_kernel, P.n_dt * nc, 192, smem, st, 1, P);
}

}  // namespace moe
