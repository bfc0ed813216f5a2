// Token-major activations transposed for the weight-gradient GEMMs.
//
// The weight gradients contract over token rows: dW1 = dU^T Xd, dW3 = dV^T Xd, dW2 = dO^T H.  Every
// activation is stored token-major ([rows, cols], a row per token), so both operands of these
// GEMMs would reach the tensor cores with K (the token index) as their outer dimension, the
// MN-major operand layout; measured on the Mixtral-style layer, tcgen05 MMAs with both operands
// MN-major ran about a third slower per clock than with both K-major.  These kernels write
// column-major copies ([cols, rows]: a row per feature, tokens contiguous) so that the weight
// gradients read both operands K-major.
//
// One launch handles a table of jobs.  A job copies src[row0 + r][c] to dst[c][col0 + r] for
// r < nrows, c < cols (cols a multiple of 64, 16-byte aligned rows), reading rows r >= nvalid as
// zeros (padding columns of the destination that the source does not have).  A CTA moves one
// 64 x 64 tile:
// 128 threads read its 64 rows as 128-byte segments (eight 16-byte loads per row), park them in
// shared memory with the 16-byte chunks of each row rotated by (row / 8) (so the transposed reads
// below hit 16 distinct banks), then write 64 output rows of 128 bytes.  Rows of a ragged last
// tile are read as zeros, and their group of 8 output columns is written whole: a job's
// destination must hold round_up(nrows, 8) columns from col0 on.
#include <string.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr int kMaxTransposeJobs = 8;

struct TransposeJob {
  const __nv_bfloat16* src;
  __nv_bfloat16* dst;
  long long src_ld, dst_ld;   // row strides in elements
  long long row0, col0;
  int nrows, nvalid, cols;
  int tile0;                  // first tile of this job in the launch's tile numbering
  int row_tiles;              // ceil(nrows / 64)
};

struct TransposeJobs {
  TransposeJob job[kMaxTransposeJobs];
  int n;
};

__global__ void __launch_bounds__(128) transpose64_kernel(const __grid_constant__ TransposeJobs J) {
  pdl_prologue();
  __shared__ uint4 tile[64 * 8];   // 64 rows x 8 chunks of 16 bytes (8 bf16)
  const int b = blockIdx.x;
  int j = 0;
  while (j + 1 < J.n && b >= J.job[j + 1].tile0) ++j;
  const TransposeJob& jb = J.job[j];
  const int local = b - jb.tile0;
  const int rt = local % jb.row_tiles, ct = local / jb.row_tiles;
  const int r_base = rt * 64, c_base = ct * 64;
  const int tid = threadIdx.x;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int q = it * 128 + tid;
    const int r = q >> 3, ch = q & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r_base + r < jb.nvalid)
      v = __ldcs(reinterpret_cast<const uint4*>(jb.src + (jb.row0 + r_base + r) * jb.src_ld +
                                                c_base + ch * 8));
    tile[r * 8 + (ch ^ ((r >> 3) & 7))] = v;
  }
  __syncthreads();
  const uint16_t* t16 = reinterpret_cast<const uint16_t*>(tile);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int q = it * 128 + tid;
    const int c = q >> 3, rg = q & 7;   // output row c (a column of the tile), its rows 8 rg..8 rg+7
    if (r_base + rg * 8 >= jb.nrows) continue;
    const int cpos = (((c >> 3) ^ rg) << 3) + (c & 7);   // element c of a row of group rg
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = rg * 8 + 2 * i;
      w[i] = (uint32_t)t16[r * 64 + cpos] | ((uint32_t)t16[(r + 1) * 64 + cpos] << 16);
    }
    *reinterpret_cast<uint4*>(jb.dst + (long long)(c_base + c) * jb.dst_ld + jb.col0 + r_base +
                              rg * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

moe_status launch_transpose_bf16(const TransposeSpec* specs, int n, cudaStream_t st) {
  if (n < 1 || n > kMaxTransposeJobs) return MOE_ERR_INVALID_ARG;
  TransposeJobs J;
  memset(&J, 0, sizeof(J));
  int tiles = 0;
  for (int i = 0; i < n; ++i) {
    const TransposeSpec& s = specs[i];
    if (s.cols % 64 != 0 || s.nrows < 0 || s.nvalid > s.nrows) return MOE_ERR_INVALID_ARG;
    TransposeJob& jb = J.job[J.n];
    jb.src = static_cast<const __nv_bfloat16*>(s.src);
    jb.dst = static_cast<__nv_bfloat16*>(s.dst);
    jb.src_ld = s.src_ld;
    jb.dst_ld = s.dst_ld;
    jb.row0 = s.row0;
    jb.col0 = s.col0;
    jb.nrows = (int)s.nrows;
    jb.nvalid = (int)(s.nvalid < 0 ? s.nrows : s.nvalid);
    jb.cols = (int)s.cols;
    jb.row_tiles = (int)((s.nrows + 63) / 64);
    jb.tile0 = tiles;
    if (jb.row_tiles == 0) continue;
    tiles += jb.row_tiles * (int)(s.cols / 64);
    ++J.n;
  }
  if (tiles == 0) return MOE_OK;
  return launch_k(transpose64_kernel, tiles, 128, 0, st, 1, J);
}

}  // namespace moe
