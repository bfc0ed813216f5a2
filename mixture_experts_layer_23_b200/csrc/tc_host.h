// Host-side helpers of the tcgen05 kernels (see tc_host.cu).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {
namespace tc {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encoder();
// Tensor map with 128-byte swizzle (32-byte with swz32) over bf16 (elem 2) or fp32 (elem 4) data;
// dims and box innermost first, rank 2 or 3.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint32_t* box,
              int elem = 2, bool swz32 = false);
bool map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
          uint32_t box_rows);
// bf16, 32-byte swizzle: boxes 16 elements wide
bool map2_sw32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows);
bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
          uint32_t box_inner, uint32_t box_mid);
bool map3_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
              uint32_t box_inner, uint32_t box_mid);
int num_sms();
// Time budget of every bounded device wait in the tcgen05 kernels (default 2 s).
unsigned long long wait_budget_ns();
void set_wait_budget_ns(unsigned long long ns);
// Failure-path test hook: when set, the tcgen05 kernels launched afterwards first wait on a
// barrier that nothing arrives on (moe_set_wait_stall).
int wait_stall();
void set_wait_stall(int on);

}  // namespace tc
}  // namespace moe
