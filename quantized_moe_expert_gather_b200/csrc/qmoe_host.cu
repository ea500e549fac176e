// Host-side plumbing: launch counter, SM count cache, TMA descriptor encoding.
#include <atomic>
#include <cudaTypedefs.h>
#include <mutex>

#include "qmoe_internal.h"
#include "qmoe_tma.h"

namespace qmoe {

namespace {
std::atomic<uint64_t> g_launches{0};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base,
                      int64_t inner, int64_t rows, int box_inner, int box_rows, bool swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner * esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 1;
  }
  return cache[dev];
}

cudaError_t make_tmap_2d_u32(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                             int box_inner, int box_rows, bool swizzle128) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, base, inner, rows, box_inner,
                   box_rows, swizzle128);
}
cudaError_t make_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                              int box_inner, int box_rows, bool swizzle128) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, rows, box_inner,
                   box_rows, swizzle128);
}

}  // namespace qmoe

extern "C" uint64_t qmoe_launch_count(void) { return qmoe::g_launches.load(); }
