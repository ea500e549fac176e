// qmoe_gather_qmm_noalloc: gather_qmm for callers that cannot allocate device memory.
//
// The ordinary qmoe_gather_qmm needs a caller-provided workspace for its routing
// metadata (expert sort, inverse permutation, expert offsets, tile table).  Some
// callers cannot provide one: a plugin that is handed only its input and output
// tensors by a host framework that owns every device allocation, or a serving loop
// that must not call cudaMalloc (which can synchronise the whole device) between
// requests.  This entry point keeps that metadata in a fixed array in device
// memory that is part of the library image instead, and otherwise runs the same
// kernels as qmoe_gather_qmm's streaming path.
//
// Limits: at most kMaxRows routed rows (B*M) and kMaxExperts experts per call.
// Every call shares the one array, so calls that overlap on the GPU (on different
// streams, or from different threads without ordering) race on it; serialise them.
#include <algorithm>
#include <mutex>

#include "qmoe_internal.h"

namespace {

constexpr int64_t kMaxRows = 4096;
constexpr int64_t kMaxExperts = 1024;
constexpr size_t kScratchBytes = 128 * 1024;

// Routing metadata of one call.  Each GPU that loads the library holds its own copy
// of this array until the process exits.  The route kernels overwrite every entry a
// call reads before reading it, so nothing here has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch per device ordinal, looked up once per device
// with that device current (the first call on a device does it).  The address is
// kept for the life of the process: it is not looked up again after a device reset
// or anything else that destroys and recreates the device's primary context.
void* scratch_for_current_device(int* status) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = QMOE_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> g(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *status = QMOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

// Lays the routing metadata out in the scratch array (256-byte aligned pieces).
struct Layout {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(int64_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += static_cast<size_t>(std::max<int64_t>(n, 0)) * sizeof(T);
    return p;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int qmoe_gather_qmm_noalloc(const qmoe_bf16* x, int64_t x_batches, int64_t M,
                                       int64_t K, const uint32_t* codes,
                                       const qmoe_bf16* scales, const qmoe_bf16* biases,
                                       int64_t E, int64_t N, int group, int bits,
                                       const uint32_t* lhs_indices,
                                       const uint32_t* rhs_indices, int64_t B,
                                       int sorted_indices, qmoe_bf16* y, int* d_status,
                                       qmoe_stream stream) {
  using namespace qmoe;
  if (!((bits == 4 || bits == 8) && (group == 32 || group == 64 || group == 128)))
    return QMOE_ERR_UNSUPPORTED;
  if (K <= 0 || K % group != 0) return QMOE_ERR_ARG;
  if (x_batches <= 0 || M < 0 || B < 0 || E <= 0 || N <= 0) return QMOE_ERR_ARG;
  if (B == 0 || M == 0) return QMOE_OK;
  if (!x || !codes || !scales || !biases || !y) return QMOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases))
    return QMOE_ERR_ARG;
  const int64_t R = B * M;
  if (R > kMaxRows || E > kMaxExperts) return QMOE_ERR_TOO_LARGE;

  const int64_t touched = std::max<int64_t>(1, std::min(E, R));
  const int bm = R / touched > 8 ? 16 : 8;
  const int64_t max_tiles = (R + bm - 1) / bm + std::min(E, R) + 1;
  Layout probe{nullptr};
  probe.take<char>(static_cast<int64_t>(route_workspace_bytes(R, E)));
  probe.take<uint32_t>(R);
  probe.take<uint32_t>(R);
  probe.take<uint32_t>(E + 1);
  probe.take<uint32_t>(R);
  probe.take<uint32_t>(1);
  probe.take<uint32_t>(3 * max_tiles);
  if (probe.off > kScratchBytes) return QMOE_ERR_TOO_LARGE;

  int status = QMOE_OK;
  void* scratch = scratch_for_current_device(&status);
  if (scratch == nullptr) return status;
  Layout lay{static_cast<char*>(scratch)};
  void* route_ws = lay.take<char>(static_cast<int64_t>(route_workspace_bytes(R, E)));
  uint32_t* order = lay.take<uint32_t>(R);
  uint32_t* inv = lay.take<uint32_t>(R);
  uint32_t* offsets = lay.take<uint32_t>(E + 1);
  uint32_t* src_row = lay.take<uint32_t>(R);
  uint32_t* num_tiles = lay.take<uint32_t>(1);
  uint32_t* tiles = lay.take<uint32_t>(3 * max_tiles);

  RouteArgs ra;
  ra.rhs = rhs_indices;
  ra.lhs = lhs_indices;
  ra.B = B;
  ra.M = M;
  ra.x_batches = x_batches;
  ra.E = E;
  ra.bm = bm;
  ra.order = order;
  ra.inv_order = inv;
  ra.offsets = offsets;
  ra.src_row = src_row;
  ra.tiles = tiles;
  ra.num_tiles = num_tiles;
  ra.max_tiles = max_tiles;
  ra.zero_out = y;
  ra.zero_cols = N;
  ra.zero_by_pos = false;
  ra.check_sorted = sorted_indices != 0;
  ra.d_status = d_status;
  auto s = static_cast<cudaStream_t>(stream);
  if (launch_route(ra, route_ws, s) != cudaSuccess) return QMOE_ERR_CUDA;

  GemmArgs a;
  a.w[0] = QWeight{codes, scales, biases};
  a.nmat = 1;
  a.E = E;
  a.N = N;
  a.K = K;
  a.group = group;
  a.bits = bits;
  a.x = x;
  a.src_row = src_row;
  a.y = y;
  a.dst_row = order;
  a.tiles = tiles;
  a.num_tiles = num_tiles;
  a.max_tiles = max_tiles;
  a.bm = bm;
  a.d_status = d_status;
  return launch_qmv(a, s) == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}
