// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA).
//
// Step 3 of the expert-parallel workflow (tutorial ch.4 "分布式训练", section "专家并行", part 二,
// step 3: each device runs its local experts on the tokens it received; part 一: each expert is
// an MLP) and its backward (section "专家并行与数据并行的结合", part 三.3: expert weight gradients
// are computed locally).  The Piper digest ("关键贡献", "关键要点") singles out thin expert GEMMs as
// a cause of low GPU utilisation; here every expert's GEMM is one slice of a single persistent
// launch, so a thin expert only costs its own tiles.
//
// One kernel, five kinds of grouped GEMM over the dispatched row space (bf16 in, fp32 accumulate):
//   UP      : u (and v) = A W1^T (W3^T); epilogue H = gelu(u) or silu(u) * v, plus the factors
//             the backward needs: Gu = gelu'(u), or Gu = v s (1 + u (1 - s)) and Gv = silu(u)
//             with s = sigmoid(u)                                             A = Xd (or x)
//   DOWN    : O = H W2^T
//   DGRAD_H : dH = A W2, epilogue dU = dH * Gu (and dV = dH * Gv)             A = dO (or dy)
//   DGRAD_X : dXd = dU W1 (+ dV W3)
//   WGRAD   : dW1 = dU^T Xd, dW3 = dV^T Xd (which 0)  or  dW2 = dO^T H (which 2), fp32 out
// Tiles are 256 x 256 (M x N) computed by a pair of CTAs on two SMs with tcgen05.mma.cta_group::2:
// each CTA stages its own 128 rows of A and its half (128 rows) of B, the pair's leader issues the
// MMA, and each CTA's TMEM receives its own 128 rows of the fp32 accumulator.  K advances in
// blocks of 64 (one 128-byte swizzle atom of bf16).
//
// CTA organisation (one CTA per SM, clusters of 2, persistent over tiles; see Cfg for the per-kind
// numbers of epilogue warps and stages):
//   warp 0      TMA producer: loads this CTA's A and B halves into a 4- to 6-stage ring;
//               completion is counted on the leader CTA's barrier (cta_group::2 loads)
//   warp 1      owns 512 TMEM columns (two 128x256 fp32 accumulators, allocated pair-wide); on the
//               leader, one lane issues the MMAs and commits each stage back to both producers
//   warps 2..    epilogue: tcgen05.ld the finished accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31 = tile rows; with 8 epilogue warps, the two warps of a lane
//               quarter take its 64-column chunks in turn), apply the fused activation, store
//               via TMA
// The two accumulators let the epilogue of one tile overlap the main loop of the next.
// Every mbarrier wait is bounded: on timeout the kernel records MOE_STATUS_TIMEOUT in the status
// word, drains its own copies and MMAs (with a bound), frees TMEM and returns.
#include <cuda.h>  // CUtensorMap and its enums (types only; the encoder is fetched at run time)
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "tc_host.h"
#include "tc_ptx.cuh"
#include "act_fast.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;           // rows per CTA
constexpr int BMP = 2 * BM;        // rows per CTA-pair tile (MMA M)
constexpr int BN = 256;            // MMA N (accumulator columns)
constexpr int BNH = BN / 2;        // B rows staged by each CTA
constexpr int BK = 64;
constexpr uint32_t A_BYTES = BM * BK * 2;           // 16 KB
constexpr uint32_t B_BYTES = BNH * BK * 2;          // 16 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES; // per CTA
constexpr uint32_t TMEM_COLS = 2 * BN;              // two accumulators
constexpr int MAX_GROUPS = 264;
#ifndef MOE_HALF_N_EDGE
#define MOE_HALF_N_EDGE 1   // N = 128 MMAs for tiles with at most 128 valid columns (see half_n)
#endif
#ifndef MOE_WGRAD_TRANSPOSED_W13
#define MOE_WGRAD_TRANSPOSED_W13 1   // dW1, dW3 computed transposed when F ends in a short tile
#endif
#ifndef MOE_TILE_GROUP_M
#define MOE_TILE_GROUP_M 16
#endif
constexpr int TILE_GROUP_M = MOE_TILE_GROUP_M;  // m tiles per band of the tile order (see decode)
// Epilogue staging: each epilogue warp owns a ring of Cfg::NSLOT 4 KB slots (32 rows x 128 B, laid out
// in the 128-byte swizzle TMA expects); finished chunks leave through TMA tile stores.
constexpr uint32_t SLOT_BYTES = 32 * 128;
constexpr size_t MISC_BYTES = 1536;   // barriers, TMEM slot, abort flag, tile prefix

enum Kind { UP = 0, DOWN = 1, DGRAD_H = 2, DGRAD_X = 3, WGRAD = 4, UNDISPATCH = 5 };

// UNDISPATCH epilogue gathers: per epilogue warp, buffers of 32 rows x 64 bf16 columns, rows 144
// bytes apart (16-byte reads of a row by 8 lanes at a time hit 8 distinct bank groups), filled by
// 16-byte asynchronous copies.  (TMA gathers of four rows each into the 128-byte swizzled layout
// measured slower: 213 against 191 us on the Mixtral-style layer, 256 against 202 us on the
// DeepSeek-style layer.)  The kind has 8 epilogue warps (MOE_UNDISPATCH_SPLIT = 2), two per TMEM
// lane quarter taking alternate 64-column chunks, with 3 gather buffers each and one load stage:
// 190 -> 155 us on the Mixtral-style layer and 205 -> 150 us on the DeepSeek-style layer against 4
// warps with 6 buffers each (MOE_UNDISPATCH_SPLIT = 1), whose single warp per SM sub-partition
// could not keep its gathers in flight.
#ifndef MOE_UNDISPATCH_SPLIT
#define MOE_UNDISPATCH_SPLIT 2
#endif
constexpr uint32_t GROW = 144;
constexpr uint32_t GATHER_BUF_BYTES = 32 * GROW;

// Per-kind balance of epilogue warps against pipeline stages (shared memory holds both).  The
// up-projection's activation epilogue is the heaviest per output, so it gets 8 epilogue warps (two
// per TMEM lane quarter, taking the tile's 64-column chunks in turn) and 5 stages (12 warps with
// 4 stages measured slower); the others keep 4 epilogue warps and 6 stages of loads in flight, except the
// activation-gradient GEMM, whose epilogue reads the saved factors Gu (Gv) through TMA into NIN
// input slots per warp: two slots (one chunk's Gu and Gv ahead) and 5 stages measured 6-8 % faster
// on the Mixtral- and DeepSeek-style layers than four slots and 4 stages.  Warps are spread over the SM's four
// sub-partitions by warp index and each sub-partition has a quarter of the register file
// (16384 registers): 10 warps put 3 on one sub-partition, capping threads at 168 registers;
// 6 warps allow 255.
#ifndef MOE_GEMM_DIRECT_STORE
#define MOE_GEMM_DIRECT_STORE 0
#endif
#ifndef MOE_UP_STAGES
#define MOE_UP_STAGES 5        // load stages of the up-projection GEMM
#endif
#ifndef MOE_UP_EPI_WARPS
#define MOE_UP_EPI_WARPS 8     // its epilogue warps (4 or 8)
#endif
#ifndef MOE_DGRAD_H_STAGES
#define MOE_DGRAD_H_STAGES 5   // load stages of the activation-gradient GEMM
#endif
#ifndef MOE_DGRAD_H_NIN
#define MOE_DGRAD_H_NIN 2      // its epilogue input slots per warp
#endif

template <int KIND>
struct Cfg {
  static constexpr int EPI_WARPS = (KIND == UP) ? MOE_UP_EPI_WARPS : (KIND == UNDISPATCH) ? 4 * MOE_UNDISPATCH_SPLIT : 4;
  static constexpr int SPLIT = EPI_WARPS / 4;   // epilogue warps per TMEM lane quarter
  // plain-output kinds may store straight from registers, which frees the staging ring for a
  // seventh stage of loads in flight
  static constexpr bool DIRECT =
      MOE_GEMM_DIRECT_STORE && (KIND == DOWN || KIND == DGRAD_X || KIND == WGRAD);
  // UNDISPATCH contracts K = E (at most 4 k blocks): two stages are plenty, and the room goes to
  // the gather buffers of its epilogue
  static constexpr int STAGES = DIRECT ? 7 : (KIND == UP) ? MOE_UP_STAGES : (KIND == DGRAD_H) ? MOE_DGRAD_H_STAGES
                                       : (KIND == UNDISPATCH) ? (MOE_UNDISPATCH_SPLIT > 1 ? 1 : 2) : 6;
  static constexpr int NIN = (KIND == DGRAD_H) ? MOE_DGRAD_H_NIN : 0;   // epilogue input slots per warp
  static constexpr int NGATH = (KIND == UNDISPATCH) ? (MOE_UNDISPATCH_SPLIT > 1 ? 3 : 6) : 0;   // gather buffers per warp
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int NSLOT = 2;                          // output staging slots per warp
  static constexpr uint32_t RING_BYTES = DIRECT ? 0 : EPI_WARPS * NSLOT * SLOT_BYTES;
  static constexpr uint32_t IN_BYTES = EPI_WARPS * NIN * SLOT_BYTES;
  static constexpr uint32_t GATH_BYTES = EPI_WARPS * NGATH * GATHER_BUF_BYTES;
  // WGRAD takes its tiles from a queue (longest first, claimed by the pair that is free first): its
  // tiles' K is the group's row count, which differs tenfold between shared and routed experts
  static constexpr int QD = (KIND == WGRAD) ? 8 : 0;         // tile-queue slots
  static constexpr int NBARS = 2 * STAGES + 5 + EPI_WARPS * NIN + EPI_WARPS * NGATH + 2 * QD;
  static constexpr size_t SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + RING_BYTES + IN_BYTES + GATH_BYTES + MISC_BYTES;
  static_assert(SMEM_BYTES <= 232448, "over the 227 KB per-CTA shared memory limit");
  static_assert(8 * NBARS + 16 + 4 * (MAX_GROUPS + 1) + 4 * QD <= MISC_BYTES, "misc too small");
};

struct alignas(64) Params {
  CUtensorMap a_main, a_alt, b_main, b_alt;
  CUtensorMap o0, o1, o2;  // output tensor maps (TMA stores), see the epilogue of each kind
  CUtensorMap i0, i1;      // DGRAD_H epilogue inputs Gu, Gv (TMA loads, 64 x 32 boxes)
  const int32_t* offsets;
  uint32_t* status;
  unsigned long long timeout_ns;
  long long T_pad;
  int E, S, T;
  int N;                 // output columns (row GEMMs: F or d; WGRAD: columns of the weight grad)
  int Mw;                // WGRAD: rows of the weight grad
  int K;                 // row GEMMs: inner dimension (d or F)
  int act;
  int which;             // WGRAD: 0 -> A = dU|dV (row space), B = Xd|x;  2 -> A = dO|dy, B = H
  int kmajor;            // WGRAD: B (which 0) or A (which 2) read K-major from its transposed copy
  int wtrans;            // WGRAD: the tiles are of the weight gradient's transpose (stored transposed)
  int chunk;             // > 0: the groups are fixed chunks of this many token rows (router
                         // backward) instead of the experts' row ranges
  int stall;             // failure-path test: the MMA issuer first waits on a barrier that
                         // nothing arrives on, so the wait runs out and the CTA aborts
  int dynamic;           // WGRAD: tiles from the queue, shared experts' groups first
  int* sched;            // dynamic: the launch's tile counter (zero before the launch)
  int* zero;             // set zero[0..zero_n) to 0 first (the next launches' tile counters)
  int zero_n;
  void* out;              // the output's base and row stride (elements), for direct stores
  long long out_ld;
  // UNDISPATCH: the rows its epilogue gathers and adds
  const __nv_bfloat16* gsrc;   // dXd [rows, gd]
  const int32_t* gslot;        // slot [T, gk]: routed row of each assignment, -1 if dropped
  int gk, gS, gd;              // routed choices, shared experts (rows s * T_pad + t), row length
};

// Instruction descriptor of the pair MMA: bf16 x bf16 -> fp32, M = 256 (two CTAs), N = BN.
__host__ __device__ constexpr uint32_t make_idesc(bool a_mn, bool b_mn) {
  return idesc_bf16(BMP, BN, a_mn, b_mn);
}

// ----------------------------------------------------------------------------- scheduling

struct Tile {
  int g, m, n;           // group, m tile (256 rows), n tile
  int a_row, o_row;      // first row of the group in input- / output-indexed buffers
  int rows;              // group rows (multiple of 128)
  int mrow;              // first row of this CTA's half, relative to the group (m * 256 + 128 * rank)
  bool live;             // this CTA's half holds rows of the group
  bool shared;
};

// N columns one tile covers: a SwiGLU up-projection tile holds 128 columns of U and the same
// 128 columns of V side by side.
template <int KIND>
__device__ __forceinline__ int tile_n(const Params& P) {
  return (KIND == UP && P.act == MOE_ACT_SWIGLU) ? BN / 2 : BN;
}

template <int KIND>
__device__ __forceinline__ int m_tiles(const Params& P, int rows) {
  return ((KIND == WGRAD ? P.Mw : rows) + BMP - 1) / BMP;
}

template <int KIND>
__device__ __forceinline__ int group_tiles(const Params& P, int rows) {
  const int nt = (P.N + tile_n<KIND>(P) - 1) / tile_n<KIND>(P);
  return m_tiles<KIND>(P, rows) * nt;
}

__device__ __forceinline__ void group_rows(const Params& P, int g, int& a_row, int& o_row,
                                           int& rows, bool& shared) {
  if (P.chunk > 0) {   // token chunk g: rows [g * chunk, min((g + 1) * chunk, T)), K-padded to 64
    a_row = g * P.chunk;
    o_row = a_row;
    const int n = P.T - a_row < P.chunk ? P.T - a_row : P.chunk;
    rows = (int)round_up(n, BK);
    shared = false;
  } else if (g < P.E) {
    a_row = P.offsets[g];
    o_row = a_row;
    rows = P.offsets[g + 1] - a_row;
    shared = false;
  } else {
    a_row = 0;
    o_row = (int)((g - P.E) * P.T_pad);
    rows = (int)P.T_pad;
    shared = true;
  }
}

// The group at position v of the tile order: groups in index order, or (dynamic) the shared
// experts' groups first, whose K = T_pad is the longest, then the routed ones.
__device__ __forceinline__ int group_at(const Params& P, int v) {
  if (!P.dynamic || P.S == 0) return v;
  return v < P.S ? P.E + v : v - P.S;
}

template <int KIND>
__device__ __forceinline__ Tile decode(const Params& P, const int* tile_start, int n_groups, int t,
                                       int rank) {
  int lo = 0, hi = n_groups - 1;  // last position v with tile_start[v] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile T;
  const int g = group_at(P, lo);
  T.g = g;
  group_rows(P, g, T.a_row, T.o_row, T.rows, T.shared);
  // Tile order inside the group: bands of TILE_GROUP_M m tiles, each walked m-fastest across all
  // n tiles.  The CTA pairs run consecutive tile indices at the same time, so one wave of pairs
  // touches about TILE_GROUP_M A slices and (pairs / TILE_GROUP_M) B slices, which stay in L2;
  // walking all m tiles first would stream the whole A operand from DRAM once per wave when it
  // is larger than L2 (the weight gradients of a 14336-wide expert).
  const int local = t - tile_start[lo];
  const int mt = m_tiles<KIND>(P, T.rows);
  const int nt = (P.N + tile_n<KIND>(P) - 1) / tile_n<KIND>(P);
  const int band = local / (TILE_GROUP_M * nt);
  const int m0 = band * TILE_GROUP_M;
  const int gm = mt - m0 < TILE_GROUP_M ? mt - m0 : TILE_GROUP_M;
  const int r = local - band * TILE_GROUP_M * nt;
  T.m = m0 + r % gm;
  T.n = r / gm;
  T.mrow = T.m * BMP + rank * BM;
  T.live = T.mrow < (KIND == WGRAD ? P.Mw : T.rows);
  return T;
}

template <int KIND>
__device__ __forceinline__ int k_blocks(const Params& P, const Tile& t) {
  if (KIND == WGRAD) return t.rows / BK;
  if (KIND == DGRAD_X && P.act == MOE_ACT_SWIGLU) return 2 * (P.K / BK);
  return P.K / BK;
}

// A tile whose valid columns fit in half of BN (the last N tile of, for example, F = 1408) runs
// N = 128 MMAs with each CTA staging 64 rows of B, instead of a full 256-column tile half of which
// is zero.  Only kinds whose B is read MN-major in 64-row boxes.
template <int KIND>
__device__ __forceinline__ bool half_n(const Params& P, const Tile& t) {
  const bool kinds = KIND == DGRAD_H || KIND == DGRAD_X ||
                     (KIND == WGRAD && !(P.kmajor && P.which == 0));
  return MOE_HALF_N_EDGE && kinds && P.N - t.n * BN <= BNH;
}

// ----------------------------------------------------------------------------- producer
//
// Each CTA loads its own half: A rows [mrow, mrow + 128) and B rows [nb, nb + 128) with
// nb = n0 + 128 * rank (for the SwiGLU up-projection: CTA 0 loads W1 rows, CTA 1 the same rows of
// W3, which makes accumulator columns 0..127 U and 128..255 V).  bar: the leader's full barrier.

template <int KIND>
__device__ __forceinline__ void issue_loads(const Params& P, const Tile& t, int kb, int rank,
                                            uint8_t* sA, uint8_t* sB, uint32_t bar) {
  const bool swiglu = P.act == MOE_ACT_SWIGLU;
  const int k0 = kb * BK;
  const bool hn = half_n<KIND>(P, t);
  const int nb = t.n * BN + rank * (hn ? BNH / 2 : BNH);
  const int nbj = hn ? 1 : BNH / 64;   // 64-row B boxes of an MN-major B
  if (KIND == UP) {
    if (t.shared) tma_load_2d_pair(sA, &P.a_alt, bar, k0, t.mrow);
    else tma_load_2d_pair(sA, &P.a_main, bar, k0, t.a_row + t.mrow);
    if (swiglu) tma_load_3d_pair(sB, rank ? &P.b_alt : &P.b_main, bar, k0, t.n * BNH, t.g);
    else tma_load_3d_pair(sB, &P.b_main, bar, k0, nb, t.g);
  } else if (KIND == DOWN) {
    tma_load_2d_pair(sA, &P.a_main, bar, k0, t.o_row + t.mrow);
    tma_load_3d_pair(sB, &P.b_main, bar, k0, nb, t.g);
  } else if (KIND == DGRAD_H) {
    if (t.shared) tma_load_2d_pair(sA, &P.a_alt, bar, k0, t.mrow);
    else tma_load_2d_pair(sA, &P.a_main, bar, k0, t.a_row + t.mrow);
    for (int j = 0; j < nbj; ++j)
      tma_load_3d_pair(sB + j * 8192, &P.b_main, bar, nb + 64 * j, k0, t.g);
  } else if (KIND == DGRAD_X || KIND == UNDISPATCH) {
    const int nkF = P.K / BK;
    const bool second = kb >= nkF;
    const int kk = (second ? kb - nkF : kb) * BK;
    tma_load_2d_pair(sA, second ? &P.a_alt : &P.a_main, bar, kk, t.o_row + t.mrow);
    for (int j = 0; j < nbj; ++j)
      tma_load_3d_pair(sB + j * 8192, second ? &P.b_alt : &P.b_main, bar, nb + 64 * j, kk, t.g);
  } else if (P.kmajor) {
    // WGRAD, K over the group's rows, one operand read through its column-major copy (K-major,
    // one 128-row box), the other straight from the token-major rows (MN-major, two 64-column
    // boxes): with both MN-major the MMAs ran about a third slower per clock
    if (P.which == 0) {
      // A = dU|dV rows of the group (row space, MN-major); B = Xd^T (routed) or x^T (shared)
#pragma unroll
      for (int j = 0; j < BM / 64; ++j)
        tma_load_2d_pair(sA + j * 8192, &P.a_main, bar, t.mrow + 64 * j, t.o_row + k0);
      if (t.shared) tma_load_2d_pair(sB, &P.b_alt, bar, k0, nb);
      else tma_load_2d_pair(sB, &P.b_main, bar, t.a_row + k0, nb);
    } else {
      // A = dO^T (routed) or dy^T (shared), K-major; B = H rows of the group (MN-major)
      if (t.shared) tma_load_2d_pair(sA, &P.a_alt, bar, k0, t.mrow);
      else tma_load_2d_pair(sA, &P.a_main, bar, t.a_row + k0, t.mrow);
      for (int j = 0; j < nbj; ++j)
        tma_load_2d_pair(sB + j * 8192, &P.b_main, bar, nb + 64 * j, t.o_row + k0);
    }
  } else {  // WGRAD, both operands straight from the token-major rows (MN-major)
    if (P.which == 0) {
      // A = dU|dV rows of the group (row space), B = Xd rows (routed) or x (shared)
#pragma unroll
      for (int j = 0; j < BM / 64; ++j)
        tma_load_2d_pair(sA + j * 8192, &P.a_main, bar, t.mrow + 64 * j, t.o_row + k0);
      for (int j = 0; j < nbj; ++j) {
        if (t.shared) tma_load_2d_pair(sB + j * 8192, &P.b_alt, bar, nb + 64 * j, k0);
        else tma_load_2d_pair(sB + j * 8192, &P.b_main, bar, nb + 64 * j, t.a_row + k0);
      }
    } else {
      // A = dO rows (routed) or dy (shared), B = H rows of the group
#pragma unroll
      for (int j = 0; j < BM / 64; ++j) {
        if (t.shared) tma_load_2d_pair(sA + j * 8192, &P.a_alt, bar, t.mrow + 64 * j, k0);
        else tma_load_2d_pair(sA + j * 8192, &P.a_main, bar, t.mrow + 64 * j, t.a_row + k0);
      }
      for (int j = 0; j < nbj; ++j)
        tma_load_2d_pair(sB + j * 8192, &P.b_main, bar, nb + 64 * j, t.o_row + k0);
    }
  }
}

// ----------------------------------------------------------------------------- epilogue
//
// Warp q (TMEM lane quarter) owns rows 32q..32q+31 of the tile; lane = row.  A chunk is 64 bf16
// (or 32 fp32) columns: each lane writes its 128-byte row into a staging slot with the 128-byte
// swizzle (16-byte unit c of row r lands at unit c ^ (r % 8): conflict-free), the warp fences the
// writes into the async proxy, and lane 0 hands the 32 x 128 B box to a TMA store.  Stores that
// fall outside the tensor (a partial last N tile) are clipped by TMA.

// A bounded wait taken by a whole warp: every lane returns the same answer (the warp goes on only
// when all its lanes saw the phase complete), so the warp never splits between success and abort.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long budget) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, budget));
}

template <int NSLOT>
struct Ring {
  uint8_t* base;
  int next;  // slots taken so far; slot = next % NSLOT.  Stores are issued in take order.
};

// Take the next slot.  AHEAD = slots taken earlier whose stores are not issued yet.  Take j
// reuses the slot of take j - NSLOT, whose store must have finished reading shared memory; at
// this point j - AHEAD stores have been issued, so at most NSLOT - 1 - AHEAD may still be pending.
template <int AHEAD = 0, int NSLOT>
__device__ __forceinline__ uint8_t* ring_take(Ring<NSLOT>& r, int lane) {
  static_assert(AHEAD < NSLOT, "more slots held than the ring has");
  if (r.next >= NSLOT && lane == 0) bulk_wait_read<NSLOT - 1 - AHEAD>();
  __syncwarp();
  uint8_t* p = r.base + (r.next % NSLOT) * SLOT_BYTES;
  ++r.next;
  return p;
}
__device__ __forceinline__ void ring_store_2d(const CUtensorMap* map, uint8_t* slot, int c0,
                                              int c1, int lane) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, slot, c0, c1);
    bulk_commit();
  }
}
// two slots written at the same coordinates of two tensors, behind one proxy fence
__device__ __forceinline__ void ring_store_2d_two(const CUtensorMap* m0, uint8_t* s0,
                                                  const CUtensorMap* m1, uint8_t* s1, int c0,
                                                  int c1, int lane) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(m0, s0, c0, c1);
    bulk_commit();
    tma_store_2d(m1, s1, c0, c1);
    bulk_commit();
  }
}
__device__ __forceinline__ void ring_store_3d(const CUtensorMap* map, uint8_t* slot, int c0,
                                              int c1, int c2, int lane) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(map, slot, c0, c1, c2);
    bulk_commit();
  }
}

// Epilogue input slots (DGRAD_H): 32 x 64 bf16 boxes of Gu / Gv loaded by TMA in the same
// swizzled layout the output slots use, one mbarrier per slot.  Loads are consumed in issue order,
// so load j uses slot j % NIN with parity (j / NIN) & 1; a slot is refilled only after the chunk
// that read it has been computed.
struct InRing {
  uint8_t* base;
  uint64_t* bars;
  int issued, consumed;
};
template <int NIN>
__device__ __forceinline__ void in_issue(InRing& r, const CUtensorMap* map, int c0, int c1,
                                         int lane) {
  const int s = r.issued % NIN;
  if (lane == 0) {
    fence_async_smem();   // earlier generic reads of this slot before the async-proxy write
    mbar_expect_tx(&r.bars[s], SLOT_BYTES);
    tma_load_2d(r.base + s * SLOT_BYTES, map, &r.bars[s], c0, c1);
  }
  ++r.issued;
}
template <int NIN>
__device__ __forceinline__ const uint8_t* in_wait(InRing& r, volatile int* abort_flag,
                                                  unsigned long long budget) {
  const int j = r.consumed;
  if (!warp_wait(&r.bars[j % NIN], (uint32_t)(j / NIN) & 1u, abort_flag, budget))
    return nullptr;   // still counted as in flight: the exit path waits for it
  ++r.consumed;
  return r.base + (j % NIN) * SLOT_BYTES;
}
// 32 columns (half h) of row r of an input slot -> fp32
__device__ __forceinline__ void slot_get_bf16_half(const uint8_t* slot, int r, int h, float* v) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int cc = 4 * h + c;
    const uint4 w = *reinterpret_cast<const uint4*>(slot + r * 128 + ((cc ^ (r & 7)) << 4));
    const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * c + 2 * i] = __uint_as_float(q[i] << 16);
      v[8 * c + 2 * i + 1] = __uint_as_float(q[i] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// 16-byte unit cc of row r of a slot <- 8 values as bf16
__device__ __forceinline__ void slot_put8(uint8_t* slot, int r, int cc, const float* v) {
  *reinterpret_cast<uint4*>(slot + r * 128 + ((cc ^ (r & 7)) << 4)) =
      make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                 pack_bf16(v[6], v[7]));
}
// row r of a slot <- 64 values as bf16
__device__ __forceinline__ void slot_put_bf16(uint8_t* slot, int r, const float* v) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(slot + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_uint4(pack_bf16(v[8 * c + 0], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                   pack_bf16(v[8 * c + 4], v[8 * c + 5]), pack_bf16(v[8 * c + 6], v[8 * c + 7]));
}
// half h (32 columns) of row r of a slot <- 32 values as bf16
__device__ __forceinline__ void slot_put_bf16_half(uint8_t* slot, int r, int h, const float* v) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int cc = 4 * h + c;
    *reinterpret_cast<uint4*>(slot + r * 128 + ((cc ^ (r & 7)) << 4)) =
        make_uint4(pack_bf16(v[8 * c + 0], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                   pack_bf16(v[8 * c + 4], v[8 * c + 5]), pack_bf16(v[8 * c + 6], v[8 * c + 7]));
  }
}
// row r of a slot <- 32 fp32 values
__device__ __forceinline__ void slot_put_f32(uint8_t* slot, int r, const float* v) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4*>(slot + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// 64 accumulator columns starting at taddr (two loads, one wait)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t a[32], b[32];
  tmem_ld32_async(taddr, a);
  tmem_ld32_async(taddr + 32, b);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __uint_as_float(a[i]);
    v[32 + i] = __uint_as_float(b[i]);
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* v) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Straight from registers to global memory: 64 bf16 / 32 fp32 values (128 bytes) of one row.
__device__ __forceinline__ void st_row_bf16(void* base, long long ld, long long row, int col,
                                            const float* v) {
  uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + row * ld + col);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    p[c] = make_uint4(pack_bf16(v[8 * c + 0], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                      pack_bf16(v[8 * c + 4], v[8 * c + 5]), pack_bf16(v[8 * c + 6], v[8 * c + 7]));
}
__device__ __forceinline__ void st_row_f32(void* base, long long ld, long long row, int col,
                                           const float* v) {
  float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + row * ld + col);
#pragma unroll
  for (int c = 0; c < 8; ++c) p[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// First chunk of warp `sub` (of `split` warps sharing a TMEM lane quarter) when `before` chunks
// of the quarter were dealt before this tile: chunk c goes to warp (before + c) % split.
__device__ __forceinline__ int q_sub_first(int sub, int before, int split) {
  return ((sub - before) % split + split) % split;
}

// Warp (q, sub) covers rows 32q..32q+31 of the tile; with SPLIT > 1 warps per quarter (UP) it
// takes the 64-column chunks q_sub_first deals to it.  Returns false if the wait for the
// accumulator timed out.
// The tiles of one CTA pair, for code that looks ahead to the pair's next tiles.
struct Sched {
  const int* tile_start;
  int n_groups, n_tiles, n_pairs, rank;
};

// a[j] for a runtime j < 16, through selects: indexing the array with j itself would move it from
// registers to local memory, which a CTA with ~210 KB of shared memory reaches only through L2
__device__ __forceinline__ int pick16(const int (&a)[16], int j) {
  int r = a[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) r = (j == i) ? a[i] : r;
  return r;
}

// UNDISPATCH: one epilogue warp's stream of gathers, (tile, chunk, source) in the order its
// epilogue consumes them, so that they can be issued ahead across tile boundaries.
struct GCursor {
  int t;          // tile (>= n_tiles: the stream has ended)
  int ch, j;      // chunk and source inside the tile
  int sub;        // the warp's chunks of a tile are sub, sub + SPLIT, ...
  int nch;        // 64-column chunks of the tile in this warp's rows (0: none)
  int n0, row0;   // first column and first row of the warp's slab
  int src[16];    // gathered row of each source for this lane's token, -1 when there is none
};

template <int KIND>
__device__ __forceinline__ void gcursor_load(const Params& P, const Sched& S, int q, int lane,
                                             GCursor& c) {
  c.ch = c.sub;
  c.j = 0;
  c.nch = 0;
  if (c.t >= S.n_tiles) return;
  const Tile tl = decode<KIND>(P, S.tile_start, S.n_groups, c.t, S.rank);
  c.row0 = tl.o_row + tl.mrow + q * 32;
  c.n0 = tl.n * BN;
  if (tl.live)
    for (int ch = 0; ch < BN / 64 && c.n0 + ch * 64 < P.N; ++ch) ++c.nch;
  const int tok = c.row0 + lane;
  const bool live_row = tl.live && tok < P.T;
  const int nsrc = P.gk + P.gS;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    int r = -1;
    if (j < nsrc && live_row)
      r = (j < P.gk) ? P.gslot[(size_t)tok * P.gk + j] : (int)((j - P.gk) * P.T_pad + tok);
    c.src[j] = r;
  }
}

// Issue the cursor's gather into the next buffer of the ring and advance it (past tiles whose
// rows are not this warp's).  The warp copies the 32 rows' 128-byte pieces with eight 16-byte
// asynchronous copies per lane, eight lanes to a row (each copy instruction moves four whole
// 128-byte lines); the buffer's mbarrier completes once all 32 lanes' copies have landed.
template <int KIND>
__device__ __forceinline__ void gcursor_issue(const Params& P, const Sched& S, int q, int lane,
                                              GCursor& c, InRing& gr) {
  constexpr int NG = Cfg<KIND>::NGATH;
  const int b = gr.issued % NG;
  const int r = pick16(c.src, c.j);
  uint8_t* buf = gr.base + b * GATHER_BUF_BYTES + (lane & 7) * 16;
  const int col = c.n0 + c.ch * 64 + (lane & 7) * 8;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int row = 4 * u + (lane >> 3);                 // token row of the warp's 32
    const int rr = __shfl_sync(0xffffffffu, r, row);     // its gathered row, -1 if none
    if (rr >= 0) cp_async16(buf + row * GROW, P.gsrc + (size_t)rr * P.gd + col);
  }
  cp_async_arrive_noinc(&gr.bars[b]);
  ++gr.issued;
  if (++c.j == P.gk + P.gS) {
    c.j = 0;
    c.ch += Cfg<KIND>::SPLIT;
    if (c.ch >= c.nch) {
      do {
        c.t += S.n_pairs;
        gcursor_load<KIND>(P, S, q, lane, c);
      } while (c.t < S.n_tiles && c.ch >= c.nch);
    }
  }
}

template <int KIND>
__device__ __forceinline__ bool epilogue_tile(const Params& P, const Tile& t, uint32_t tacc, int nk,
                                              int q, int sub, int lane,
                                              Ring<Cfg<KIND>::NSLOT>& ring,
                                              InRing& inr, InRing& gr, GCursor& gc, const Sched& S,
                                              int tcount, uint64_t* tfull,
                                              uint32_t parity, volatile int* abort_flag) {
  constexpr int SPLIT = Cfg<KIND>::SPLIT;
  const uint32_t tl = tacc + ((uint32_t)(q * 32) << 16);
  const bool swiglu = P.act == MOE_ACT_SWIGLU;
  float a[64];
  if (KIND == WGRAD) {
    if (!warp_wait(tfull, parity, abort_flag, P.timeout_ns)) return false;
    __syncwarp();
    tc_fence_after();
    if (!t.live) return true;  // this CTA's half of the pair tile lies past the weight rows
    const int m_row0 = t.mrow + q * 32;
    if (m_row0 >= P.Mw) return true;  // this warp's 32 rows lie past the weight rows
#pragma unroll 1
    for (int c = sub * (BN / 32 / SPLIT); c < (sub + 1) * (BN / 32 / SPLIT); ++c) {
      const int n = t.n * BN + c * 32;
      if (n >= P.N) break;
      if (nk > 0) {
        uint32_t r[32];
        tmem_ld32_async(tl + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = __uint_as_float(r[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = 0.f;
      }
      if constexpr (Cfg<KIND>::DIRECT) {
        st_row_f32(P.out, P.out_ld, (long long)t.g * P.Mw + m_row0 + lane, n, a);
      } else if (P.wtrans) {
        // the accumulator holds the transpose of the weight gradient's tile (rows = its columns):
        // lane l writes its 32 values down column l of the 32 x 32 box, in the 128-byte swizzle
        // the TMA store reads (16-byte unit u of row r at unit u ^ (r % 8): conflict-free)
        uint8_t* slot = ring_take(ring, lane);
#pragma unroll
        for (int f = 0; f < 32; ++f)
          *reinterpret_cast<float*>(slot + f * 128 + ((((lane >> 2) ^ (f & 7)) << 4)) +
                                    (lane & 3) * 4) = a[f];
        ring_store_3d(&P.o0, slot, m_row0, n, t.g, lane);
      } else {
        uint8_t* slot = ring_take(ring, lane);
        slot_put_f32(slot, lane, a);
        ring_store_3d(&P.o0, slot, n, m_row0, t.g, lane);
      }
    }
    return true;
  }
  const int row0 = t.o_row + t.mrow + q * 32;  // first output row of this warp's slab
  if constexpr (KIND == DGRAD_H) {
    // 64-column chunks; each chunk's Gu (and Gv) box is loaded by TMA into an input slot, the
    // first chunks' loads issued before the wait for the accumulator.
    constexpr int NIN = Cfg<KIND>::NIN;
    const int F = P.N;
    const int per = swiglu ? 2 : 1;              // input slots per chunk
    const int depth = NIN / per;                 // chunks in flight
    const int ch0 = sub * (BN / 64 / SPLIT), ch1 = (sub + 1) * (BN / 64 / SPLIT);
    int nch = 0;                                 // chunks of this warp inside [0, F)
    for (int ch = ch0; ch < ch1 && t.n * BN + ch * 64 < F; ++ch) ++nch;
    if (!t.live) nch = 0;
    auto issue_chunk = [&](int i) {
      const int n = t.n * BN + (ch0 + i) * 64;
      in_issue<NIN>(inr, &P.i0, n, row0, lane);
      if (swiglu) in_issue<NIN>(inr, &P.i1, n, row0, lane);
    };
    for (int i = 0; i < nch && i < depth; ++i) issue_chunk(i);
    if (!warp_wait(tfull, parity, abort_flag, P.timeout_ns)) return false;
    __syncwarp();
    tc_fence_after();
#pragma unroll 1
    for (int i = 0; i < nch; ++i) {
      const int n = t.n * BN + (ch0 + i) * 64;
      const uint8_t* gu = in_wait<NIN>(inr, abort_flag, P.timeout_ns);
      const uint8_t* gv = swiglu ? in_wait<NIN>(inr, abort_flag, P.timeout_ns) : nullptr;
      if (gu == nullptr || (swiglu && gv == nullptr)) return false;
      uint8_t* su = ring_take(ring, lane);
      uint8_t* sv = swiglu ? ring_take<1>(ring, lane) : nullptr;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tmem_ld32_async(tl + (ch0 + i) * 64 + h * 32, r);
        float u[32];
        slot_get_bf16_half(gu, lane, h, u);
        tmem_wait_ld();
        if (!swiglu) {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = __uint_as_float(r[j]) * u[j];   // dU = dH * Gu
          slot_put_bf16_half(su, lane, h, a);
        } else {
          float v[32];
          slot_get_bf16_half(gv, lane, h, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float dh = __uint_as_float(r[j]);
            a[j] = dh * u[j];   // dU = dH * Gu
            v[j] = dh * v[j];   // dV = dH * Gv
          }
          slot_put_bf16_half(su, lane, h, a);
          slot_put_bf16_half(sv, lane, h, v);
        }
      }
      __syncwarp();   // every lane has read this chunk's input slots
      if (i + depth < nch) issue_chunk(i + depth);
      if (swiglu)
        ring_store_2d_two(&P.o0, su, &P.o1, sv, n, row0, lane);
      else
        ring_store_2d(&P.o0, su, n, row0, lane);
    }
    return true;
  }
  if constexpr (KIND == UNDISPATCH) {
    // dx = dl Wg (the accumulator) + the token's kept routed rows of dXd (choices 0..k-1) + its
    // shared experts' rows, summed in that fixed order.  The rows arrive through the warp's
    // gather stream (gcursor_issue), which runs up to NGATH buffers ahead of this consumer, across
    // tile boundaries, so the next tile's gathers are in flight while this one finishes.
    constexpr int NG = Cfg<KIND>::NGATH;
    const int nsrc = P.gk + P.gS;
    // this tile as the consumer sees it: its chunks, and which of this lane's sources exist
    const int n0 = t.n * BN;
    int nch = 0;
    if (t.live)
      for (int ch = 0; ch < BN / 64 && n0 + ch * 64 < P.N; ++ch) ++nch;
    uint32_t have_src = 0;   // bit j: source j of this lane's token is a row
    {
      const int tok = row0 + lane;
      const bool live_row = t.live && tok < P.T;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < nsrc && live_row &&
            (j >= P.gk || P.gslot[(size_t)tok * P.gk + j] >= 0))
          have_src |= 1u << j;
    }
    if (!warp_wait(tfull, parity, abort_flag, P.timeout_ns)) return false;
    __syncwarp();
    tc_fence_after();
#pragma unroll 1
    for (int ch = sub; ch < nch; ch += SPLIT) {
      const int n = n0 + ch * 64;
      tmem_ld64(tl + ch * 64, a);
#pragma unroll 1
      for (int j = 0; j < nsrc; ++j) {
        const int b = gr.consumed % NG;
        if (!warp_wait(&gr.bars[b], (uint32_t)(gr.consumed / NG) & 1u, abort_flag,
                       P.timeout_ns))
          return false;   // still counted as in flight: the exit path waits for it
        ++gr.consumed;
        if ((have_src >> j) & 1u) {
          const uint8_t* row = gr.base + b * GATHER_BUF_BYTES + lane * GROW;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float v[8];
            unpack_bf16x8(*reinterpret_cast<const uint4*>(row + c * 16), v);
#pragma unroll
            for (int i = 0; i < 8; ++i) a[8 * c + i] += v[i];
          }
        }
        __syncwarp();   // every lane has read this buffer before it is refilled
        if (gc.t < S.n_tiles) gcursor_issue<KIND>(P, S, q, lane, gc, gr);
      }
      uint8_t* slot = ring_take(ring, lane);
      slot_put_bf16(slot, lane, a);
      ring_store_2d(&P.o0, slot, n, row0, lane);
    }
    return true;
  }
  if (!warp_wait(tfull, parity, abort_flag, P.timeout_ns)) return false;
  __syncwarp();
  tc_fence_after();
  if (!t.live) return true;  // this CTA's half of the pair tile lies past the group's rows
  if (KIND == UP) {
    const int F = P.N;
    // this warp's chunks: the quarter's chunks are dealt round robin over its SPLIT warps,
    // continuing from the previous tile (tcount tiles of nch chunks each came before)
    const int nch = swiglu ? 2 : BN / 64;
    const int first = (q_sub_first(sub, tcount * nch, SPLIT));
    if (!swiglu) {
#pragma unroll 1
      for (int ch = first; ch < nch; ch += SPLIT) {
        const int n = t.n * BN + ch * 64;
        if (n >= F) break;
        // Gu = GELU'(u) (what the backward needs) and H = GELU(u) from one erf evaluation,
        // 8 columns at a time into two slots
        uint8_t* sg = ring_take(ring, lane);
        uint8_t* sh = ring_take<1>(ring, lane);
        // both 32-column halves are read from TMEM before the math, one wait for the two loads
        // (BERT-style layer 155 -> 146 us against a load and a wait per half)
        uint32_t rr[2][32];
        tmem_ld32_async(tl + ch * 64, rr[0]);
        tmem_ld32_async(tl + ch * 64 + 32, rr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float g8[8], h8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float u = __uint_as_float(rr[h][8 * c + i]);
              const fast::ErfParts e = fast::erf_parts(u);
              const float phi_cdf = fmaf(0.5f, copysignf(e.erf_abs, u), 0.5f);   // Phi(u)
              g8[i] = fmaf(u, 0.39894228040143268f * e.e, phi_cdf);              // GELU'(u)
              h8[i] = u * phi_cdf;                                               // GELU(u)
            }
            slot_put8(sg, lane, 4 * h + c, g8);
            slot_put8(sh, lane, 4 * h + c, h8);
          }
        }
        ring_store_2d_two(&P.o0, sg, &P.o2, sh, n, row0, lane);   // Gu, H
      }
    } else {
      // u (accumulator columns [0, 128)) and v (columns [128, 256)) of one 64-column chunk.
      // Outputs: Gu = v s (1 + u (1 - s)) and Gv = u s (the backward's factors, s = sigmoid(u)),
      // then H = u s v in a second pass over TMEM, so that two staging slots are enough.
#pragma unroll 1
      for (int ch = first; ch < nch; ch += SPLIT) {
        const int n = t.n * (BN / 2) + ch * 64;
        if (n >= F) break;
        const uint32_t tu = tl + ch * 64, tv = tl + BN / 2 + ch * 64;
        uint8_t* sa = ring_take(ring, lane);
        uint8_t* sb = ring_take<1>(ring, lane);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t ru[32], rv[32];
          tmem_ld32_async(tu + 32 * h, ru);
          tmem_ld32_async(tv + 32 * h, rv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float gu8[8], gv8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float u = __uint_as_float(ru[8 * c + i]), v = __uint_as_float(rv[8 * c + i]);
              const float sg = fast::sigmoid(u);
              gu8[i] = v * sg * fmaf(u, 1.f - sg, 1.f);   // Gu
              gv8[i] = u * sg;                            // Gv
            }
            slot_put8(sa, lane, 4 * h + c, gu8);
            slot_put8(sb, lane, 4 * h + c, gv8);
          }
        }
        ring_store_2d_two(&P.o0, sa, &P.o1, sb, n, row0, lane);   // Gu, Gv
        uint8_t* sh = ring_take(ring, lane);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t ru[32], rv[32];
          tmem_ld32_async(tu + 32 * h, ru);
          tmem_ld32_async(tv + 32 * h, rv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float h8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float u = __uint_as_float(ru[8 * c + i]);
              h8[i] = u * fast::sigmoid(u) * __uint_as_float(rv[8 * c + i]);   // H
            }
            slot_put8(sh, lane, 4 * h + c, h8);
          }
        }
        ring_store_2d(&P.o2, sh, n, row0, lane);   // H
      }
    }
    return true;
  }
  // DOWN, DGRAD_X: plain bf16 output
#pragma unroll 1
  for (int ch = sub * (BN / 64 / SPLIT); ch < (sub + 1) * (BN / 64 / SPLIT); ++ch) {
    const int n = t.n * BN + ch * 64;
    if (n >= P.N) break;
    tmem_ld64(tl + ch * 64, a);
    if constexpr (Cfg<KIND>::DIRECT) {
      st_row_bf16(P.out, P.out_ld, row0 + lane, n, a);
    } else {
      uint8_t* slot = ring_take(ring, lane);
      slot_put_bf16(slot, lane, a);
      ring_store_2d(&P.o0, slot, n, row0, lane);
    }
  }
  return true;
}

// ----------------------------------------------------------------------------- tile queue

// The static tile sequence of a pair: pair, pair + n_pairs, ... (-1 past the last tile).
__device__ __forceinline__ int static_next(int it, int t, int pair, int n_pairs, int n_tiles) {
  const int n = it == 0 ? pair : t + n_pairs;
  return n < n_tiles ? n : -1;
}
//
// With P.dynamic (WGRAD) the pair's tiles come from a queue instead of the static sequence pair,
// pair + n_pairs, ...: the leader's producer takes tile `pair` first and then claims tiles from the
// launch's counter (n_pairs + atomicAdd), and publishes each in slot pos % QD of both CTAs' queues;
// the leader's MMA issuer and epilogue warps and the second CTA's producer and epilogue warps read
// the slots in order and free them on the leader's q_empty.  -1 ends the sequence.  So the pair
// that is free first takes the next tile, and the longest tiles (the shared experts' groups, first
// in the tile order) are spread over the pairs before the short ones fill in.
struct TileQueue {
  int* tile;                 // this CTA's slots
  uint64_t* full;            // this CTA's q_full
  uint64_t* empty;           // this CTA's q_empty (the leader's are the ones used)
  uint32_t own_tile, own_full, peer_tile, peer_full, leader_empty;   // shared::cluster addresses
  int pos;                   // tiles taken so far
};

__device__ __forceinline__ TileQueue make_queue(int* tile, uint64_t* full, uint64_t* empty,
                                                int rank) {
  TileQueue q;
  q.tile = tile;
  q.full = full;
  q.empty = empty;
  q.own_tile = mapa_shared(smem_u32(tile), rank);
  q.own_full = mapa_shared(smem_u32(full), rank);
  q.peer_tile = mapa_shared(smem_u32(tile), rank ^ 1);
  q.peer_full = mapa_shared(smem_u32(full), rank ^ 1);
  q.leader_empty = mapa_shared(smem_u32(empty), 0);
  q.pos = 0;
  return q;
}

// the leader's producer: publish `t` in the next slot of both CTAs' queues
template <int QD>
__device__ __forceinline__ bool q_publish(TileQueue& q, int t, volatile int* abort_flag,
                                          unsigned long long budget) {
  const int s = q.pos % QD;
  if (!wait_bounded_cluster(&q.empty[s], ((uint32_t)(q.pos / QD) & 1u) ^ 1u, abort_flag, budget))
    return false;
  st_cluster_u32(q.own_tile + 4 * s, t);
  st_cluster_u32(q.peer_tile + 4 * s, t);
  mbar_arrive_cluster(q.own_full + 8 * s);
  mbar_arrive_cluster(q.peer_full + 8 * s);
  ++q.pos;
  return true;
}

// a single reading thread: the next tile (-1: none), or false if the wait ran out
template <int QD>
__device__ __forceinline__ bool q_take(TileQueue& q, int& t, volatile int* abort_flag,
                                       unsigned long long budget) {
  const int s = q.pos % QD;
  if (!wait_bounded_cluster(&q.full[s], (uint32_t)(q.pos / QD) & 1u, abort_flag, budget))
    return false;
  t = *reinterpret_cast<volatile int*>(&q.tile[s]);
  mbar_arrive_cluster(q.leader_empty + 8 * s);
  ++q.pos;
  return true;
}

// a reading warp (every lane gets the same answer; lane 0 frees the slot)
template <int QD>
__device__ __forceinline__ bool q_take_warp(TileQueue& q, int& t, int lane, volatile int* abort_flag,
                                            unsigned long long budget) {
  const int s = q.pos % QD;
  if (!__all_sync(0xffffffffu, wait_bounded_cluster(&q.full[s], (uint32_t)(q.pos / QD) & 1u,
                                                    abort_flag, budget)))
    return false;
  t = *reinterpret_cast<volatile int*>(&q.tile[s]);
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(q.leader_empty + 8 * s);
  ++q.pos;
  return true;
}

// ----------------------------------------------------------------------------- kernel

template <int KIND>
__global__ void __launch_bounds__(Cfg<KIND>::THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ Params P) {
  pdl_prologue();
  constexpr int STAGES = Cfg<KIND>::STAGES;
  constexpr int NUM_THREADS = Cfg<KIND>::THREADS;
  constexpr int NUM_EPI_WARPS = Cfg<KIND>::EPI_WARPS;
  constexpr uint32_t RING_BYTES = Cfg<KIND>::RING_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* tiles = smem;
  uint8_t* ring_base = smem + STAGES * STAGE_BYTES;            // epilogue warps x NSLOT slots
  constexpr int NIN = Cfg<KIND>::NIN;
  uint8_t* in_base = ring_base + RING_BYTES;                     // epilogue warps x NIN slots
  constexpr int NG = Cfg<KIND>::NGATH;
  uint8_t* g_base = in_base + Cfg<KIND>::IN_BYTES;               // epilogue warps x NG buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(g_base + Cfg<KIND>::GATH_BYTES);
  uint64_t* full = bars;                 // [STAGES]  (the leader's are the ones used)
  uint64_t* empty = bars + STAGES;       // [STAGES]
  uint64_t* tfull = bars + 2 * STAGES;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]       (the leader's are the ones used)
  uint64_t* drain = tempty + 2;          // [1]
  uint64_t* in_bars = drain + 1;         // [EPI_WARPS * NIN]
  uint64_t* g_bars = in_bars + NUM_EPI_WARPS * NIN;   // [EPI_WARPS * NG]
  constexpr int QD = Cfg<KIND>::QD;
  uint64_t* q_full = g_bars + NUM_EPI_WARPS * NG;      // [QD] tile-queue slot written
  uint64_t* q_empty = q_full + QD;                     // [QD] slot read by all (the leader's used)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + QD);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* tile_start = reinterpret_cast<int*>(tmem_slot + 4);   // [MAX_GROUPS + 1]
  int* q_tile = tile_start + MAX_GROUPS + 1;                 // [QD]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();   // 0 = leader of the pair
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_groups = P.E + P.S;

  if (P.zero && blockIdx.x == 0 && (int)threadIdx.x < P.zero_n) P.zero[threadIdx.x] = 0;
  // per-group tile counts in tile order, then an exclusive prefix (warp 0)
  for (int v = threadIdx.x; v < n_groups; v += NUM_THREADS) {
    int a_row, o_row, rows;
    bool sh;
    group_rows(P, group_at(P, v), a_row, o_row, rows, sh);
    tile_start[v + 1] = group_tiles<KIND>(P, rows);
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    tile_start[0] = 0;
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * NUM_EPI_WARPS);   // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int i = 0; i < NUM_EPI_WARPS * NIN; ++i) mbar_init(&in_bars[i], 1);
    // gather buffers: one arrival per lane (asynchronous copies) or one armed arrival (TMA gathers)
    for (int i = 0; i < NUM_EPI_WARPS * NG; ++i) mbar_init(&g_bars[i], 32);
    // tile queue: written by the leader's producer (one arrival in each CTA), read by the leader's
    // MMA issuer and epilogue warps and by the second CTA's producer and epilogue warps
    for (int i = 0; i < QD; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 2 + 2 * NUM_EPI_WARPS);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 1; base <= n_groups; base += 32) {
      const int i = base + lane;
      int v = (i <= n_groups) ? tile_start[i] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (i <= n_groups) tile_start[i] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = tile_start[n_groups];
  const unsigned long long budget = P.timeout_ns;
  // operand layouts: MN-major for the weights in the dgrads; in the weight gradients, both
  // operands MN-major, or (P.kmajor) dU|dV (dW1, dW3: P.which 0) or H (dW2) MN-major and the
  // partner read K-major from its transposed copy
  const bool A_MN = (KIND == WGRAD) && (P.which == 0 || !P.kmajor);
  const bool B_MN = (KIND == DGRAD_H || KIND == DGRAD_X || KIND == UNDISPATCH) ||
                    ((KIND == WGRAD) && (P.which != 0 || !P.kmajor));
  const uint32_t IDESC = make_idesc(A_MN, B_MN);
  const uint32_t IDESC_HALF = idesc_bf16(BMP, BN / 2, A_MN, B_MN);   // N = 128 edge tiles

  // producer bookkeeping, read again after every role has finished (abort drain)
  uint32_t outstanding = 0;            // stages with a load issued and not yet seen consumed
  uint32_t out_phase = 0;              // bit s: phase parity of stage s's last issued load
  const bool dyn = QD > 0 && P.dynamic;
  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (both CTAs; with the tile queue, the leader's publishes)
    int stage = 0;
    uint32_t phase = 0;
    TileQueue q = make_queue(q_tile, q_full, q_empty, rank);
    int t = -1, t_next = pair < n_tiles ? pair : -1;   // the leader claims one tile ahead
    for (int it = 0; !*abort_flag; ++it) {
      if constexpr (QD > 0) {
        if (dyn && rank == 0) {
          t = t_next;
          if (!q_publish<QD>(q, t, abort_flag, budget)) break;
          if (t >= 0) {
            const int c = n_pairs + atomicAdd(P.sched, 1);
            t_next = c < n_tiles ? c : -1;
          }
        } else if (dyn) {
          if (!q_take<QD>(q, t, abort_flag, budget)) break;
        } else {
          t = static_next(it, t, pair, n_pairs, n_tiles);
        }
      } else {
        t = static_next(it, t, pair, n_pairs, n_tiles);
      }
      if (t < 0) break;
      const Tile tl = decode<KIND>(P, tile_start, n_groups, t, rank);
      const int nk = k_blocks<KIND>(P, tl);
      const bool hn = half_n<KIND>(P, tl);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, budget)) { ok = false; break; }
        outstanding &= ~(1u << stage);
        if (rank == 0) mbar_expect_tx(&full[stage], hn ? 2 * (A_BYTES + B_BYTES / 2) : 2 * STAGE_BYTES);
        uint8_t* sA = tiles + stage * STAGE_BYTES;
        issue_loads<KIND>(P, tl, kb, rank, sA, sA + A_BYTES, mapa_shared(smem_u32(&full[stage]), 0));
        outstanding |= 1u << stage;
        out_phase = (out_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------- MMA issuer (leader CTA only)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t a_step = A_MN ? 2048u : 32u;   // bytes per UMMA_K = 16 step
    const uint32_t b_step = B_MN ? 2048u : 32u;
    const uint32_t a_lbo = A_MN ? 8192u : 16u, b_lbo = B_MN ? 8192u : 16u;
    bool issued_any = false;
    // test hook: `drain` gets no arrival before an abort, so this wait runs out after `budget`
    // and raises the abort flag before any MMA is issued
    if (P.stall) wait_bounded(drain, 0u, abort_flag, budget);
    TileQueue q = make_queue(q_tile, q_full, q_empty, rank);
    int t = -1;
    for (int it = 0; !*abort_flag; ++it) {
      if constexpr (QD > 0) {
        if (dyn) {
          if (!q_take<QD>(q, t, abort_flag, budget)) break;
        } else {
          t = static_next(it, t, pair, n_pairs, n_tiles);
        }
      } else {
        t = static_next(it, t, pair, n_pairs, n_tiles);
      }
      if (t < 0) break;
      const Tile tl = decode<KIND>(P, tile_start, n_groups, t, rank);
      const int nk = k_blocks<KIND>(P, tl);
      if (!wait_bounded_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag, budget)) break;
      tc_fence_after();
      const uint32_t dtm = tmem_base + (uint32_t)(acc * BN);
      const uint32_t idesc = half_n<KIND>(P, tl) ? IDESC_HALF : IDESC;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_bounded(&full[stage], phase, abort_flag, budget)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(tiles + stage * STAGE_BYTES);
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t ad = sw128_desc(sa + k * a_step, a_lbo, 1024);
          const uint64_t bd = sw128_desc(sb + k * b_step, b_lbo, 1024);
          umma_bf16_pair(dtm, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
        }
        issued_any = true;
        umma_commit_pair(&empty[stage], 0x3);   // frees this stage in both CTAs
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit_pair(&tfull[acc], 0x3);       // accumulator ready in both CTAs
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (*abort_flag && issued_any) {
      umma_commit_pair_local(drain);
      volatile int never = 0;
      wait_bounded(drain, 0, &never, 20000000ull);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs)
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;   // which of the quarter's SPLIT warps
    Ring<Cfg<KIND>::NSLOT> ring{ring_base + (warp - 2) * Cfg<KIND>::NSLOT * SLOT_BYTES, 0};
    InRing inr{in_base + (warp - 2) * NIN * SLOT_BYTES, in_bars + (warp - 2) * NIN, 0, 0};
    InRing gr{g_base + (warp - 2) * NG * GATHER_BUF_BYTES, g_bars + (warp - 2) * NG, 0, 0};
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0),
                                       mapa_shared(smem_u32(&tempty[1]), 0)};
    int acc = 0, tcount = 0;
    uint32_t acc_phase = 0;
    const Sched sched{tile_start, n_groups, n_tiles, n_pairs, rank};
    GCursor gc;   // UNDISPATCH: the warp's gather stream, started NGATH buffers ahead
    gc.t = n_tiles;
    gc.sub = sub;
    if constexpr (KIND == UNDISPATCH) {
      gc.t = pair;
      gcursor_load<KIND>(P, sched, quarter, lane, gc);
      while (gc.t < n_tiles && gc.ch >= gc.nch) {
        gc.t += n_pairs;
        gcursor_load<KIND>(P, sched, quarter, lane, gc);
      }
      for (int i = 0; i < NG && gc.t < n_tiles; ++i) gcursor_issue<KIND>(P, sched, quarter, lane, gc, gr);
    }
    TileQueue q = make_queue(q_tile, q_full, q_empty, rank);
    int t = -1;
    for (int it = 0; !*abort_flag; ++it, ++tcount) {
      if constexpr (QD > 0) {
        if (dyn) {
          if (!q_take_warp<QD>(q, t, lane, abort_flag, budget)) break;
        } else {
          t = static_next(it, t, pair, n_pairs, n_tiles);
        }
      } else {
        t = static_next(it, t, pair, n_pairs, n_tiles);
      }
      if (t < 0) break;
      const Tile tl = decode<KIND>(P, tile_start, n_groups, t, rank);
      const int nk = k_blocks<KIND>(P, tl);
      if (!epilogue_tile<KIND>(P, tl, tmem_base + (uint32_t)(acc * BN), nk, quarter, sub, lane,
                               ring, inr, gr, gc, sched, tcount, &tfull[acc], acc_phase,
                               abort_flag))
        break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait<0>();  // this warp's stores have completed
    // on abort, let input loads still in flight land before the CTA exits
    for (int j = inr.consumed; j < inr.issued; ++j) {
      volatile int never = 0;
      wait_bounded(&inr.bars[j % (NIN > 0 ? NIN : 1)], (uint32_t)(j / (NIN > 0 ? NIN : 1)) & 1u,
                   &never, 20000000ull);
    }
    for (int j = gr.consumed; j < gr.issued; ++j) {
      volatile int never = 0;
      wait_bounded(&gr.bars[j % (NG > 0 ? NG : 1)], (uint32_t)(j / (NG > 0 ? NG : 1)) & 1u,
                   &never, 20000000ull);
    }
    __syncwarp();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();   // every role of both CTAs has finished (the abort flag is final)
  if (*abort_flag && warp == 0 && lane == 0 && outstanding) {
    // An aborted CTA may still have TMA loads in flight into its shared memory: they must land
    // before it exits.  The leader sees the pair's copies complete on its full barriers; the
    // second CTA's copies are counted on the leader's barriers, so it waits a fixed grace period
    // (far longer than a copy takes) instead.
    if (rank == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (outstanding & (1u << s)) {
          volatile int never = 0;
          wait_bounded(&full[s], (out_phase >> s) & 1u, &never, 20000000ull);
        }
    } else {
      const unsigned long long t0 = globaltimer();
      while (globaltimer() - t0 < 200000ull) {
      }
    }
  }
  __syncwarp();
  cluster_sync();   // the pair's MMAs, copies and TMEM reads are over before either CTA moves on
  if (*abort_flag && threadIdx.x == 0) atomicOr(P.status, MOE_STATUS_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------- host side


// Persistent launch: one CTA pair (cluster of 2) per two SMs, at most one pair per tile.
template <int KIND>
static moe_status launch(const Params& P, int max_tiles, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    const cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<KIND>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)Cfg<KIND>::SMEM_BYTES);
    if (e != cudaSuccess) {
      note_cuda_error(e);
      return MOE_ERR_CUDA;
    }
    attr_done = true;
  }
  const int max_pairs = num_sms() / 2;
  const int pairs = max_tiles < max_pairs ? (max_tiles > 0 ? max_tiles : 1) : max_pairs;
  return launch_k(grouped_gemm_kernel<KIND>, dim3(2 * pairs, 1, 1), dim3(Cfg<KIND>::THREADS, 1, 1),
                  Cfg<KIND>::SMEM_BYTES, st, 2, P);
}

static Params base_params(const Dims& D, const int32_t* offsets, uint32_t* status) {
  Params P;
  memset(&P, 0, sizeof(P));
  P.offsets = offsets;
  P.status = status;
  P.timeout_ns = wait_budget_ns();
  P.stall = wait_stall();
  P.T_pad = D.T_pad;
  P.E = D.E;
  P.S = D.S;
  P.T = D.T;
  P.act = D.act;
  return P;
}

// Upper bound on the pair tiles of a row GEMM: a group of r rows (a multiple of 128) has
// ceil(r / 256) <= r / 128 m tiles.
static int row_tiles_bound(const Dims& D, int n_tiles_n) {
  return (int)((D.R / BM) * n_tiles_n);
}

}  // namespace tc

bool tc_supported(const Dims& D) {
  return D.dtype == MOE_DTYPE_BF16 && D.d % 64 == 0 && D.F % 64 == 0 && D.E + D.S <= tc::MAX_GROUPS &&
         tc::encoder() != nullptr;
}

// Weight gradients with one operand read K-major from a transposed copy: worth its copies (two
// [rows, d] arrays read and written) only when the experts take long batches.  Measured: the
// Mixtral-style layer (T k / E = 4096 rows per expert) gains 1.2 ms of its 30.6 ms step; the
// DeepSeek-style (1536), BERT- and GPT-2-style (512) layers lost 0.1-0.25 ms, their weight
// gradients being short or bound by writing their fp32 output.
bool wgrad_kmajor(const Dims& D) {
  return tc_supported(D) && (long long)D.T * D.k >= 2048LL * D.E;
}

// Weight-gradient tiles from the queue (claimed by the pair free first, longest first) only when the
// layer has shared experts, whose tiles are T_pad rows long against the routed experts' share of
// T k: measured on the DeepSeek-style layer (K 16384 against ~1000) 1430 -> 1348 us for dW1|dW3 and
// 729 -> 685 us for dW2; with tiles of equal length the queue's per-tile hand-offs cost more than they
// balance (GPT-2-style layer 57 -> 65 us, BERT-style 165 -> 182 us).
static bool wgrad_queue(const Dims& D) { return D.S > 0; }


using namespace tc;

moe_status launch_expert_up_tc(const Dims& D, const void* Xd, const void* x, const int32_t* offsets,
                               const void* W1, const void* W3, void* U, void* V, void* H,
                               uint32_t* status, cudaStream_t st) {
  Params P = base_params(D, offsets, status);
  const bool sw = D.act == MOE_ACT_SWIGLU;
  bool ok = map2(&P.a_main, Xd, D.d, D.R, 64, BM) && map2(&P.a_alt, x, D.d, D.T, 64, BM) &&
            map3(&P.b_main, W1, D.d, D.F, D.E_tot, 64, BNH);
  if (sw) ok = ok && map3(&P.b_alt, W3, D.d, D.F, D.E_tot, 64, BNH);
  if (!ok) return MOE_ERR_CUDA;
  ok = map2(&P.o0, U, D.F, D.R, 64, 32) && map2(&P.o2, H, D.F, D.R, 64, 32);
  if (sw) ok = ok && map2(&P.o1, V, D.F, D.R, 64, 32);
  if (!ok) return MOE_ERR_CUDA;
  P.N = D.F;
  P.K = D.d;
  const int tn = sw ? BN / 2 : BN;
  return launch<UP>(P, row_tiles_bound(D, (D.F + tn - 1) / tn), st);
}

moe_status launch_expert_down_tc(const Dims& D, const void* H, const int32_t* offsets,
                                 const void* W2, void* O, uint32_t* status, cudaStream_t st) {
  Params P = base_params(D, offsets, status);
  if (!(map2(&P.a_main, H, D.F, D.R, 64, BM) && map3(&P.b_main, W2, D.F, D.d, D.E_tot, 64, BNH)))
    return MOE_ERR_CUDA;
  if (!map2(&P.o0, O, D.d, D.R, 64, 32)) return MOE_ERR_CUDA;
  P.out = O;
  P.out_ld = D.d;
  P.N = D.d;
  P.K = D.F;
  return launch<DOWN>(P, row_tiles_bound(D, (D.d + BN - 1) / BN), st);
}

moe_status launch_dgrad_h_tc(const Dims& D, const void* dO, const void* dy, const int32_t* offsets,
                             const void* W2, const void* U, const void* V, void* dU, void* dV,
                             int* zero, int zero_n, uint32_t* status, cudaStream_t st) {
  Params P = base_params(D, offsets, status);
  P.zero = zero;
  P.zero_n = zero_n;
  if (!(map2(&P.a_main, dO, D.d, D.R, 64, BM) && map2(&P.a_alt, dy, D.d, D.T, 64, BM) &&
        map3(&P.b_main, W2, D.F, D.d, D.E_tot, 64, 64)))
    return MOE_ERR_CUDA;
  if (!map2(&P.i0, U, D.F, D.R, 64, 32)) return MOE_ERR_CUDA;
  if (D.act == MOE_ACT_SWIGLU && !map2(&P.i1, V, D.F, D.R, 64, 32)) return MOE_ERR_CUDA;
  if (!map2(&P.o0, dU, D.F, D.R, 64, 32)) return MOE_ERR_CUDA;
  if (D.act == MOE_ACT_SWIGLU && !map2(&P.o1, dV, D.F, D.R, 64, 32)) return MOE_ERR_CUDA;
  P.N = D.F;
  P.K = D.d;
  return launch<DGRAD_H>(P, row_tiles_bound(D, (D.F + BN - 1) / BN), st);
}

moe_status launch_dgrad_x_tc(const Dims& D, const void* dU, const void* dV, const int32_t* offsets,
                             const void* W1, const void* W3, void* dXd, int* zero, int zero_n,
                             uint32_t* status, cudaStream_t st) {
  Params P = base_params(D, offsets, status);
  P.zero = zero;
  P.zero_n = zero_n;
  bool ok = map2(&P.a_main, dU, D.F, D.R, 64, BM) && map3(&P.b_main, W1, D.d, D.F, D.E_tot, 64, 64);
  if (D.act == MOE_ACT_SWIGLU)
    ok = ok && map2(&P.a_alt, dV, D.F, D.R, 64, BM) && map3(&P.b_alt, W3, D.d, D.F, D.E_tot, 64, 64);
  if (!ok) return MOE_ERR_CUDA;
  if (!map2(&P.o0, dXd, D.d, D.R, 64, 32)) return MOE_ERR_CUDA;
  P.out = dXd;
  P.out_ld = D.d;
  P.N = D.d;
  P.K = D.F;
  return launch<DGRAD_X>(P, row_tiles_bound(D, (D.d + BN - 1) / BN), st);
}

// dW1 (and dW3) = dU^T X  -- M = F, N = d, K = the group's rows.  With wgrad_kmajor(D), B comes
// K-major from Xdt [d][R] (routed groups) or xt [d][T_pad] (shared experts); otherwise Xd and x
// are read MN-major as they are.
moe_status launch_wgrad_w13_tc(const Dims& D, const void* dU, const void* dV, const void* X,
                               const void* xs, const int32_t* offsets, float* dW1, float* dW3,
                               int* sched, uint32_t* status, cudaStream_t st) {
  const bool km = wgrad_kmajor(D);
  // dW1^T = X^T dU when F ends in a partial N tile of at most 128 columns and d fills its M tiles:
  // the dW2 form (A = X, B = dU|dV), edge tiles of N = 128, tiles stored transposed.  In the direct
  // orientation the last M tile of F = 1408 would be half empty (the pair computing 256 rows for 128).
  const bool swap = MOE_WGRAD_TRANSPOSED_W13 && !MOE_GEMM_DIRECT_STORE && D.F % BMP != 0 && D.F % BMP <= BNH && D.d % BMP == 0;
  for (int pass = 0; swap && pass < (D.act == MOE_ACT_SWIGLU ? 2 : 1); ++pass) {
    Params P = base_params(D, offsets, status);
    P.kmajor = km ? 1 : 0;
    P.dynamic = wgrad_queue(D) ? 1 : 0;
    P.sched = sched + pass;
    P.wtrans = 1;
    bool ok = map2(&P.b_main, pass ? dV : dU, D.F, D.R, 64, 64);
    if (km)
      ok = ok && map2(&P.a_main, X, D.R, D.d, 64, BM) &&
           (D.S == 0 || map2(&P.a_alt, xs, D.T_pad, D.d, 64, BM));
    else
      ok = ok && map2(&P.a_main, X, D.d, D.R, 64, 64) && map2(&P.a_alt, xs, D.d, D.T, 64, 64);
    if (!ok) return MOE_ERR_CUDA;
    if (!map3_f32(&P.o0, pass ? dW3 : dW1, D.d, D.F, D.E_tot, 32, 32)) return MOE_ERR_CUDA;
    P.out = pass ? dW3 : dW1;
    P.out_ld = D.d;
    P.Mw = D.d;
    P.N = D.F;
    P.which = 2;   // the dW2 form: A's rows are the expert's routed rows, B's the row space
    const int tiles = D.E_tot * ((D.d + BMP - 1) / BMP) * ((D.F + BN - 1) / BN);
    const moe_status s = launch<WGRAD>(P, tiles, st);
    if (s != MOE_OK) return s;
  }
  for (int pass = 0; !swap && pass < (D.act == MOE_ACT_SWIGLU ? 2 : 1); ++pass) {
    Params P = base_params(D, offsets, status);
    P.kmajor = km ? 1 : 0;
    P.dynamic = wgrad_queue(D) ? 1 : 0;
    P.sched = sched + pass;
    bool ok = map2(&P.a_main, pass ? dV : dU, D.F, D.R, 64, 64);
    if (km)
      ok = ok && map2(&P.b_main, X, D.R, D.d, 64, BNH) &&
           (D.S == 0 || map2(&P.b_alt, xs, D.T_pad, D.d, 64, BNH));
    else
      ok = ok && map2(&P.b_main, X, D.d, D.R, 64, 64) && map2(&P.b_alt, xs, D.d, D.T, 64, 64);
    if (!ok) return MOE_ERR_CUDA;
    if (!map3_f32(&P.o0, pass ? dW3 : dW1, D.d, D.F, D.E_tot, 32, 32)) return MOE_ERR_CUDA;
    P.out = pass ? dW3 : dW1;
    P.out_ld = D.d;
    P.Mw = D.F;
    P.N = D.d;
    P.which = 0;
    const int tiles = D.E_tot * ((D.F + BMP - 1) / BMP) * ((D.d + BN - 1) / BN);
    const moe_status s = launch<WGRAD>(P, tiles, st);
    if (s != MOE_OK) return s;
  }
  return MOE_OK;
}

// dW2 = dO^T H  -- M = d, N = F.  With wgrad_kmajor(D), A comes K-major from dOt [d][R] (routed
// groups) or dyt [d][T_pad] (shared experts); otherwise dO and dy are read MN-major as they are.
moe_status launch_wgrad_w2_tc(const Dims& D, const void* H, const void* G, const void* gs,
                              const int32_t* offsets, float* dW2, int* sched, uint32_t* status,
                              cudaStream_t st) {
  const bool km = wgrad_kmajor(D);
  Params P = base_params(D, offsets, status);
  P.kmajor = km ? 1 : 0;
  P.dynamic = wgrad_queue(D) ? 1 : 0;
  P.sched = sched;
  bool ok = map2(&P.b_main, H, D.F, D.R, 64, 64);
  if (km)
    ok = ok && map2(&P.a_main, G, D.R, D.d, 64, BM) &&
         (D.S == 0 || map2(&P.a_alt, gs, D.T_pad, D.d, 64, BM));
  else
    ok = ok && map2(&P.a_main, G, D.d, D.R, 64, 64) && map2(&P.a_alt, gs, D.d, D.T, 64, 64);
  if (!ok) return MOE_ERR_CUDA;
  if (!map3_f32(&P.o0, dW2, D.F, D.d, D.E_tot, 32, 32)) return MOE_ERR_CUDA;
  P.out = dW2;
  P.out_ld = D.F;
  P.Mw = D.d;
  P.N = D.F;
  P.which = 2;
  const int tiles = D.E_tot * ((D.d + BMP - 1) / BMP) * ((D.F + BN - 1) / BN);
  return launch<WGRAD>(P, tiles, st);
}

// ----------------------------------------------------------------------------- router backward
//
// The router's two backward contractions are GEMMs worth the tensor cores (2 T E d FLOPs each;
// 4.3 GFLOP for T = 16384, E = 64, d = 2048; measured faster than the CUDA-core kernels from
// E = 16 up, by 2x at E = 32).  Both read a bf16 copy of dlogits, dl16 [T, E8] (E8 = E rounded up
// to 8, zero padded).  dl Wg reuses the grouped kernel with all T rows as one group (DGRAD_X form,
// UNDISPATCH epilogue): dx = dl16 Wg + the gathered dXd rows, K = E.  (The weight gradient dWg has
// its own kernel next to the router's, router_tc.cu.)

bool router_bwd_tc_supported(const Dims& D) {
  return D.dtype == MOE_DTYPE_BF16 && D.d % 64 == 0 && tc::encoder() != nullptr;
}

// dx = dl16 Wg + the token's kept routed rows of dXd + its shared experts' rows, in one launch:
// the DGRAD_X-form contraction over one chunk of all T rows (K = E), whose epilogue gathers and
// adds the rows (UNDISPATCH), so dl Wg never goes through memory.
moe_status launch_undispatch_tc(const Dims& D, const __nv_bfloat16* dl16, const void* Wg,
                                const void* dXd, const int32_t* slot, void* dx, uint32_t* status,
                                cudaStream_t st) {
  using namespace tc;
  Params P = base_params(D, nullptr, status);
  P.act = MOE_ACT_GELU;   // one operand pair per K block (not the SwiGLU pair of DGRAD_X)
  const int E8 = (int)round_up(D.E, 8);
  if (!(map2(&P.a_main, dl16, E8, D.T, 64, BM) && map3(&P.b_main, Wg, D.d, D.E, 1, 64, 64) &&
        map2(&P.o0, dx, D.d, D.T, 64, 32)))
    return MOE_ERR_CUDA;
  if (D.k + D.S > 16) return MOE_ERR_UNSUPPORTED;
  P.E = 1;
  P.S = 0;                 // one token chunk is the only group
  P.chunk = (int)round_up(D.T, BK);
  P.N = D.d;
  P.K = (int)round_up(D.E, BK);
  P.gsrc = (const __nv_bfloat16*)dXd;
  P.gslot = slot;
  P.gk = D.k;
  P.gS = D.S;
  P.gd = D.d;
  const int tiles = (int)(((D.T + BMP - 1) / BMP) * ((D.d + BN - 1) / BN));
  return launch<UNDISPATCH>(P, tiles, st);
}

}  // namespace moe
