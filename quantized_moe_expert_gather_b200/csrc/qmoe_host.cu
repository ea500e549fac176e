// Host-side plumbing: launch counter, SM count cache, TMA descriptor encoding.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <cudaTypedefs.h>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

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

cudaError_t make_tmap_colblocks(CUtensorMap* map, const void* base, int64_t words, int64_t rows,
                                int box_rows, int box_blocks) {
  auto fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (words % 32 != 0) return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {32, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(words / 32)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(words * 4), 128};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_blocks)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QMOE_PDL");
    return !(v != nullptr && v[0] == '0');
  }();
  return on;
}

namespace {
struct TimingState {
  std::mutex mu;
  ProfSlot* slots = nullptr;
  int64_t capacity = 0;
  std::vector<std::string> names;  // kernel name of each used slot
};
TimingState& timing() {
  static TimingState* t = new TimingState();  // never destroyed: safe at process exit
  return *t;
}
}  // namespace

LaunchTimer::LaunchTimer(const char* kernel, cudaStream_t stream) {
  TimingState& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  if (t.slots == nullptr || static_cast<int64_t>(t.names.size()) >= t.capacity) return;
  ProfSlot* s = t.slots + t.names.size();
  if (cudaMemsetAsync(s, 0, sizeof(ProfSlot), stream) != cudaSuccess) return;
  t.names.emplace_back(kernel);
  slot_ = s;
}

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
cudaError_t make_tmap_3d_u32_colblocks(CUtensorMap* map, const void* base, int64_t words,
                                       int64_t rows, int box_rows, int box_blocks) {
  return make_tmap_colblocks(map, base, words, rows, box_rows, box_blocks);
}
cudaError_t make_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                              int box_inner, int box_rows, bool swizzle128) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, rows, box_inner,
                   box_rows, swizzle128);
}

}  // namespace qmoe

extern "C" {

uint64_t qmoe_launch_count(void) { return qmoe::g_launches.load(); }

int qmoe_timing_enable(void* slots, int64_t capacity) {
  auto& t = qmoe::timing();
  std::lock_guard<std::mutex> g(t.mu);
  t.names.clear();
  t.slots = capacity > 0 ? static_cast<qmoe::ProfSlot*>(slots) : nullptr;
  t.capacity = t.slots ? capacity : 0;
  return QMOE_OK;
}

int qmoe_timing_read(const char* kernel, double* total_ms, uint64_t* launches) {
  if (kernel == nullptr || total_ms == nullptr || launches == nullptr) return QMOE_ERR_ARG;
  auto& t = qmoe::timing();
  std::lock_guard<std::mutex> g(t.mu);
  *total_ms = 0.0;
  *launches = 0;
  if (t.slots == nullptr || t.names.empty()) return QMOE_OK;
  std::vector<qmoe::ProfSlot> host(t.names.size());
  if (cudaMemcpy(host.data(), t.slots, host.size() * sizeof(qmoe::ProfSlot),
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return QMOE_ERR_CUDA;
  for (size_t i = 0; i < host.size(); ++i) {
    if (t.names[i] != kernel || host[i].end == 0 || host[i].start_inv == 0) continue;
    const unsigned long long start = ~host[i].start_inv;
    if (host[i].end < start) continue;
    *total_ms += static_cast<double>(host[i].end - start) * 1e-6;
    *launches += 1;
  }
  return QMOE_OK;
}

}  // extern "C"
