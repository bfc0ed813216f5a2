// Host-side helpers of the tcgen05 kernels: TMA tensor-map encoding (the driver's encoder is
// fetched through the runtime, so the library does not link libcuda) and the SM count.
#include "tc_host.h"

namespace moe {
namespace tc {

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 map, 128-byte swizzle (32-byte with swz32).  dims/box innermost first; rank 2 or 3.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint32_t* box, int elem, bool swz32) {
  EncodeTiledFn enc = encoder();
  if (!enc || !base) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  gs[0] = dims[0] * elem;
  if (rank == 3) gs[1] = dims[0] * dims[1] * elem;
  return enc(m, elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             swz32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                 uint32_t box_rows) {
  const uint64_t d[2] = {inner, rows};
  const uint32_t b[2] = {box_inner, box_rows};
  return make_map(m, base, 2, d, b);
}
bool map2_sw32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
               uint32_t box_inner, uint32_t box_rows) {
  const uint64_t d[2] = {inner, rows};
  const uint32_t b[2] = {box_inner, box_rows};
  return make_map(m, base, 2, d, b, 2, true);
}
bool map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                 uint32_t box_inner, uint32_t box_mid) {
  const uint64_t d[3] = {inner, mid, outer};
  const uint32_t b[3] = {box_inner, box_mid, 1};
  return make_map(m, base, 3, d, b);
}

bool map3_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
              uint32_t box_inner, uint32_t box_mid) {
  const uint64_t d[3] = {inner, mid, outer};
  const uint32_t b[3] = {box_inner, box_mid, 1};
  return make_map(m, base, 3, d, b, 4);
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

static unsigned long long g_wait_budget_ns = 2000000000ull;
static int g_wait_stall = 0;
unsigned long long wait_budget_ns() { return g_wait_budget_ns; }
void set_wait_budget_ns(unsigned long long ns) { g_wait_budget_ns = ns; }
int wait_stall() { return g_wait_stall; }
void set_wait_stall(int on) { g_wait_stall = on ? 1 : 0; }

}  // namespace tc
}  // namespace moe
