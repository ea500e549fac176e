// Host-side plumbing: launch counter, SM count cache, TMA descriptor encoding.
#include <atomic>
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
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

namespace {
struct TimingState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;  // free events
  std::map<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>> recs;
  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  void clear() {
    for (auto& kv : recs)
      for (auto& pr : kv.second) {
        pool.push_back(pr.first);
        pool.push_back(pr.second);
      }
    recs.clear();
  }
};
TimingState& timing() {
  static TimingState* t = new TimingState();  // never destroyed: safe at process exit
  return *t;
}
}  // namespace

LaunchTimer::LaunchTimer(const char* kernel, cudaStream_t stream) : name_(kernel), stream_(stream) {
  TimingState& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  if (!t.on) return;
  cudaEvent_t e = t.take();
  if (e != nullptr && cudaEventRecord(e, stream_) == cudaSuccess) start_ = e;
}

LaunchTimer::~LaunchTimer() {
  if (start_ == nullptr) return;
  TimingState& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  cudaEvent_t e = t.take();
  if (e != nullptr && cudaEventRecord(e, stream_) == cudaSuccess)
    t.recs[name_].emplace_back(static_cast<cudaEvent_t>(start_), e);
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
cudaError_t make_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                              int box_inner, int box_rows, bool swizzle128) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, rows, box_inner,
                   box_rows, swizzle128);
}

}  // namespace qmoe

extern "C" {

uint64_t qmoe_launch_count(void) { return qmoe::g_launches.load(); }

int qmoe_timing_enable(int on) {
  auto& t = qmoe::timing();
  std::lock_guard<std::mutex> g(t.mu);
  if (on) t.clear();
  t.on = on != 0;
  return QMOE_OK;
}

int qmoe_timing_read(const char* kernel, double* total_ms, uint64_t* launches) {
  if (kernel == nullptr || total_ms == nullptr || launches == nullptr) return QMOE_ERR_ARG;
  auto& t = qmoe::timing();
  std::lock_guard<std::mutex> g(t.mu);
  *total_ms = 0.0;
  *launches = 0;
  auto it = t.recs.find(kernel);
  if (it == t.recs.end()) return QMOE_OK;
  for (auto& pr : it->second) {
    if (cudaEventSynchronize(pr.second) != cudaSuccess) return QMOE_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess) return QMOE_ERR_CUDA;
    *total_ms += ms;
    *launches += 1;
  }
  return QMOE_OK;
}

}  // extern "C"
