// The C ABI (include/qmoe.h): host-side validation, workspace carving and kernel
// dispatch.  Every numerical step runs in the library's CUDA kernels.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "qmoe_internal.h"

using namespace qmoe;

namespace {

bool group_ok(int group) { return group == 32 || group == 64 || group == 128; }
// quantize / dequantize: every width of the quantisation tests (7 is rejected there)
bool codec_ok(int group, int bits) {
  return (bits >= 1 && bits <= 8 && bits != 7) && group_ok(group);
}
// the matmul calls: every codec width (4- and 8-bit codes, and 2-bit codes in groups of
// 64 or 128, on the MMA kernels; 1-, 3-, 5- and 6-bit codes and 2-bit codes in groups of
// 32 on the bit-stream kernel)
bool matmul_codec_ok(int group, int bits) { return codec_ok(group, bits); }

// K must be a positive multiple of the group size.
int check_codec(int64_t K, int group, int bits) {
  if (!matmul_codec_ok(group, bits)) return QMOE_ERR_UNSUPPORTED;
  if (K <= 0 || K % group != 0) return QMOE_ERR_ARG;
  return QMOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA; }

enum class Kernel { Auto, Qmv, Tc };

// QMOE_FORCE_KERNEL=qmv|tc pins the gathered matmul to one kernel (tests use it
// to cover both kernels on the same shapes).
Kernel forced_kernel() {
  const char* s = std::getenv("QMOE_FORCE_KERNEL");
  if (s == nullptr) return Kernel::Auto;
  if (std::strcmp(s, "qmv") == 0) return Kernel::Qmv;
  if (std::strcmp(s, "tc") == 0) return Kernel::Tc;
  return Kernel::Auto;
}

// Bump allocator over the caller's workspace (256-byte aligned pieces).  With a
// null base it only measures.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(int64_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += static_cast<size_t>(std::max<int64_t>(n, 0)) * sizeof(T);
    return p;
  }
};

int64_t max_tiles_for(int64_t R, int64_t E, int bm) {
  return (R + bm - 1) / bm + std::min<int64_t>(E, R) + 1;
}

constexpr int kTcBm = 128;

// Which kernel serves a gathered matmul of R routed rows over E experts.  The tile
// tables are built on the device, so the host plans from the most rows one expert can
// receive (`max_rows`), not from an average: with skewed routing one expert may take
// most rows even when the average is a few.  Up to 16 rows per expert the streaming
// kernel (weights read once per tile of 8 or 16 rows) wins; beyond that one 128-row
// tensor-core tile costs less than the streamed tiles it replaces.
struct Plan {
  bool tc;
  int bm;
  bool ts = false;    // tensor cores with the weights in tensor memory (tiles of 192 rows)
};
// QMOE_PREFILL=tc keeps the tensor-core plan on the kernel that stages dequantised
// weights in shared memory (tiles of 128 rows) where the tensor-memory one applies.
bool ts_allowed() {
  const char* v = std::getenv("QMOE_PREFILL");
  return v == nullptr || std::strcmp(v, "tc") != 0;
}
Plan plan_for(int64_t R, int64_t E, int64_t max_rows, bool tc_ok, bool ts_ok = false) {
  const Kernel k = forced_kernel();
  const int64_t touched = std::max<int64_t>(1, std::min(E, R));
  Plan stream{false, R / touched > 8 ? 16 : 8};
  if (!(tc_ok || ts_ok) || k == Kernel::Qmv) return stream;
  if (k == Kernel::Tc || max_rows > 16) {
    if (ts_ok && ts_allowed()) return Plan{true, kTsTileRows, true};
    if (tc_ok) return Plan{true, kTcBm};
  }
  return stream;
}

struct RouteBufs {
  void* route_ws;
  uint32_t* order;
  uint32_t* inv;
  uint32_t* offsets;
  uint32_t* src_row;
  uint32_t* num_tiles;
  uint32_t* tiles;
  int64_t max_tiles;
};

RouteBufs carve_route(Carver& c, int64_t R, int64_t E, bool own_inv) {
  RouteBufs b{};
  b.route_ws = c.take<char>(static_cast<int64_t>(route_workspace_bytes(R, E)));
  b.order = c.take<uint32_t>(R);
  b.inv = own_inv ? c.take<uint32_t>(R) : nullptr;
  b.offsets = c.take<uint32_t>(E + 1);
  b.src_row = c.take<uint32_t>(R);
  b.num_tiles = c.take<uint32_t>(1);
  b.max_tiles = max_tiles_for(R, E, 8);
  b.tiles = c.take<uint32_t>(3 * b.max_tiles);
  return b;
}

int validate_qweight(const qmoe_qweight* w) {
  if (w == nullptr || w->codes == nullptr || w->scales == nullptr || w->biases == nullptr)
    return QMOE_ERR_ARG;
  if (w->E <= 0 || w->N <= 0) return QMOE_ERR_ARG;
  if (!aligned16(w->codes) || !aligned16(w->scales) || !aligned16(w->biases)) return QMOE_ERR_ARG;
  return check_codec(w->K, w->group, w->bits);
}

QWeight qw(const qmoe_qweight* w) { return QWeight{w->codes, w->scales, w->biases}; }

}  // namespace

extern "C" {

const char* qmoe_status_string(int status) {
  switch (status) {
    case QMOE_OK: return "QMOE_OK";
    case QMOE_ERR_ARG: return "QMOE_ERR_ARG: invalid argument (shape, size, pointer or index count)";
    case QMOE_ERR_DTYPE: return "QMOE_ERR_DTYPE: unsupported dtype";
    case QMOE_ERR_UNSUPPORTED: return "QMOE_ERR_UNSUPPORTED: unsupported bits/group/K combination";
    case QMOE_ERR_WORKSPACE: return "QMOE_ERR_WORKSPACE: workspace missing or too small";
    case QMOE_ERR_CUDA: return "QMOE_ERR_CUDA: kernel launch failed";
    case QMOE_ERR_TOO_LARGE:
      return "QMOE_ERR_TOO_LARGE: problem exceeds the fixed scratch capacity (B*M <= 4096, E <= 1024)";
    default: return "unknown qmoe status";
  }
}

int qmoe_quantize(const void* w, int w_dtype, int64_t rows, int64_t cols, int group, int bits,
                  uint32_t* codes, void* scales, void* biases, qmoe_stream stream) {
  if (w_dtype != QMOE_DTYPE_BF16 && w_dtype != QMOE_DTYPE_F32) return QMOE_ERR_DTYPE;
  if (!codec_ok(group, bits)) return QMOE_ERR_UNSUPPORTED;
  if (rows < 0 || cols <= 0 || cols % group != 0) return QMOE_ERR_ARG;
  if (rows == 0) return QMOE_OK;
  if (!w || !codes || !scales || !biases) return QMOE_ERR_ARG;
  return cuda_status(launch_quantize(w, w_dtype == QMOE_DTYPE_F32, rows, cols, group, bits, codes,
                                     scales, biases, static_cast<cudaStream_t>(stream)));
}

int qmoe_dequantize(const uint32_t* codes, const void* scales, const void* biases, int sb_dtype,
                    int64_t rows, int64_t cols, int group, int bits, void* out, int out_dtype,
                    qmoe_stream stream) {
  if ((sb_dtype != QMOE_DTYPE_BF16 && sb_dtype != QMOE_DTYPE_F32) ||
      (out_dtype != QMOE_DTYPE_BF16 && out_dtype != QMOE_DTYPE_F32))
    return QMOE_ERR_DTYPE;
  if (!codec_ok(group, bits)) return QMOE_ERR_UNSUPPORTED;
  if (rows < 0 || cols <= 0 || cols % group != 0) return QMOE_ERR_ARG;
  if (rows == 0) return QMOE_OK;
  if (!codes || !scales || !biases || !out) return QMOE_ERR_ARG;
  return cuda_status(launch_dequantize(codes, scales, biases, sb_dtype == QMOE_DTYPE_F32, rows,
                                       cols, group, bits, out, out_dtype == QMOE_DTYPE_F32,
                                       static_cast<cudaStream_t>(stream)));
}

int qmoe_qmm(const qmoe_bf16* x, int64_t M, const uint32_t* codes, const qmoe_bf16* scales,
             const qmoe_bf16* biases, int64_t N, int64_t K, int group, int bits, qmoe_bf16* y,
             int* d_status, qmoe_stream stream) {
  const int c = check_codec(K, group, bits);
  if (c != QMOE_OK) return c;
  if (M < 0 || N <= 0) return QMOE_ERR_ARG;
  if (M == 0) return QMOE_OK;
  if (!x || !codes || !scales || !biases || !y) return QMOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases))
    return QMOE_ERR_ARG;
  GemmArgs a;
  a.w[0] = QWeight{codes, scales, biases};
  a.nmat = 1;
  a.E = 1;
  a.N = N;
  a.K = K;
  a.group = group;
  a.bits = bits;
  a.x = x;
  a.x_rows = M;
  a.y = y;
  a.dense_rows = M;
  a.d_status = d_status;
  // one weight matrix: tensor cores from 32 rows, else the streaming kernel
  auto s = static_cast<cudaStream_t>(stream);
  if (qmv_bits_needed(bits, group)) {  // bit-stream widths: one kernel at every row count
    a.bm = M > 8 ? 16 : 8;
    a.max_tiles = (M + a.bm - 1) / a.bm;
    return cuda_status(launch_qmv_bits(a, s));
  }
  const Kernel k = forced_kernel();
  const bool big = k == Kernel::Tc || (k == Kernel::Auto && M >= 32);
  const bool ts = big && ts_allowed() && qmm_ts_supported(a);
  const bool tc = !ts && big && qmm_tc_supported(a);
  a.bm = ts ? kTsTileRows : tc ? kTcBm : (M > 8 ? 16 : 8);
  a.max_tiles = (M + a.bm - 1) / a.bm;
  if (ts) return cuda_status(launch_qmm_ts(a, s));
  return cuda_status(tc ? launch_qmm_tc(a, s) : launch_qmv(a, s));
}

size_t qmoe_gather_qmm_workspace_size(int64_t B, int64_t M, int64_t E, int64_t N, int64_t K) {
  (void)N;
  const int64_t R = std::max<int64_t>(B, 0) * std::max<int64_t>(M, 0);
  Carver c(nullptr);
  carve_route(c, R, std::max<int64_t>(E, 1), true);
  c.take<uint16_t>(R * std::max<int64_t>(K, 0));  // activation rows in expert order
  return c.off + 256;
}

int qmoe_gather_qmm(const qmoe_bf16* x, int64_t x_batches, int64_t M, int64_t K,
                    const uint32_t* codes, const qmoe_bf16* scales, const qmoe_bf16* biases,
                    int64_t E, int64_t N, int group, int bits, const uint32_t* lhs_indices,
                    const uint32_t* rhs_indices, int64_t B, int sorted_indices, void* workspace,
                    size_t workspace_bytes, qmoe_bf16* y, int* d_status, qmoe_stream stream) {
  // sorted_indices is a promise about rhs: the expert sort makes the result independent
  // of it; a broken promise is flagged (QMOE_DEV_UNSORTED).
  const int c = check_codec(K, group, bits);
  if (c != QMOE_OK) return c;
  if (x_batches <= 0 || M < 0 || B < 0 || E <= 0 || N <= 0) return QMOE_ERR_ARG;
  if (B == 0 || M == 0) return QMOE_OK;
  if (!x || !codes || !scales || !biases || !y) return QMOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(biases))
    return QMOE_ERR_ARG;
  if (workspace == nullptr || workspace_bytes < qmoe_gather_qmm_workspace_size(B, M, E, N, K))
    return QMOE_ERR_WORKSPACE;
  const int64_t R = B * M;
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255)));
  RouteBufs rb = carve_route(cv, R, E, true);
  uint16_t* x_sorted = cv.take<uint16_t>(R * K);

  GemmArgs a;
  a.w[0] = QWeight{codes, scales, biases};
  a.nmat = 1;
  a.E = E;
  a.N = N;
  a.K = K;
  a.group = group;
  a.bits = bits;
  a.y = y;
  a.x_rows = R;  // the tensor-core path reads the expert-ordered copy of x
  a.dst_row = rb.order;
  a.tiles = rb.tiles;
  a.num_tiles = rb.num_tiles;
  a.d_status = d_status;
  // Any expert may receive every routed row; below one 128-row tile the streaming
  // kernel serves every expert.
  GemmArgs a_sorted = a;  // as the tensor-core streaming kernel would read x
  a_sorted.x = x_sorted;
  a_sorted.src_row = nullptr;
  const Plan pl = plan_for(R, E, R > kTcBm ? R : 16, qmm_tc_supported(a),
                           qmm_ts_supported(a_sorted));
  a.bm = pl.bm;
  a.max_tiles = max_tiles_for(R, E, pl.bm);

  RouteArgs ra;
  ra.rhs = rhs_indices;
  ra.lhs = lhs_indices;
  ra.B = B;
  ra.M = M;
  ra.x_batches = x_batches;
  ra.E = E;
  ra.bm = pl.bm;
  ra.order = rb.order;
  ra.inv_order = rb.inv;
  ra.offsets = rb.offsets;
  ra.src_row = rb.src_row;
  ra.tiles = rb.tiles;
  ra.num_tiles = rb.num_tiles;
  ra.max_tiles = a.max_tiles;
  ra.zero_out = y;
  ra.zero_cols = N;
  ra.zero_by_pos = false;
  ra.check_sorted = sorted_indices != 0;
  ra.d_status = d_status;
  auto s = static_cast<cudaStream_t>(stream);
  if (launch_route(ra, rb.route_ws, s) != cudaSuccess) return QMOE_ERR_CUDA;
  if (pl.tc) {
    if (launch_gather_rows(x, rb.src_row, R, K, x_sorted, s) != cudaSuccess) return QMOE_ERR_CUDA;
    a.x = x_sorted;  // row tiles over the expert-ordered rows
    a.src_row = nullptr;
    return cuda_status(pl.ts ? launch_qmm_ts(a, s) : launch_qmm_tc(a, s));
  }
  a.x = x;  // the streaming kernels read x through src_row
  a.src_row = rb.src_row;
  return cuda_status(qmv_bits_needed(bits, group) ? launch_qmv_bits(a, s) : launch_qmv(a, s));
}

size_t qmoe_gather_mm_workspace_size(int64_t B, int64_t M, int64_t E, int64_t N, int64_t K) {
  return qmoe_gather_qmm_workspace_size(B, M, E, N, K);
}

int qmoe_gather_mm(const qmoe_bf16* x, int64_t x_batches, int64_t M, int64_t K, const qmoe_bf16* w,
                   int64_t E, int64_t N, const uint32_t* lhs_indices, const uint32_t* rhs_indices,
                   int64_t B, int sorted_indices, void* workspace, size_t workspace_bytes,
                   qmoe_bf16* y, int* d_status, qmoe_stream stream) {
  // sorted_indices is a promise about rhs: the expert sort makes the result independent
  // of it; a broken promise is flagged (QMOE_DEV_UNSORTED).
  if (K <= 0 || x_batches <= 0 || M < 0 || B < 0 || E <= 0 || N <= 0) return QMOE_ERR_ARG;
  if (K % 64 != 0) return QMOE_ERR_UNSUPPORTED;
  if (B == 0 || M == 0) return QMOE_OK;
  if (!x || !w || !y) return QMOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return QMOE_ERR_ARG;
  if (workspace == nullptr || workspace_bytes < qmoe_gather_mm_workspace_size(B, M, E, N, K))
    return QMOE_ERR_WORKSPACE;
  const int64_t R = B * M;
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255)));
  RouteBufs rb = carve_route(cv, R, E, true);
  uint16_t* x_sorted = cv.take<uint16_t>(R * K);

  GemmArgs a;
  a.w[0] = QWeight{reinterpret_cast<const uint32_t*>(w), nullptr, nullptr};
  a.nmat = 1;
  a.E = E;
  a.N = N;
  a.K = K;
  a.group = 64;  // no groups: bf16 weights
  a.bits = 16;
  a.y = y;
  a.x = x_sorted;
  a.x_rows = R;
  a.dst_row = rb.order;
  a.tiles = rb.tiles;
  a.num_tiles = rb.num_tiles;
  a.bm = kTcBm;
  a.max_tiles = max_tiles_for(R, E, kTcBm);
  a.d_status = d_status;

  RouteArgs ra;
  ra.rhs = rhs_indices;
  ra.lhs = lhs_indices;
  ra.B = B;
  ra.M = M;
  ra.x_batches = x_batches;
  ra.E = E;
  ra.bm = kTcBm;
  ra.order = rb.order;
  ra.inv_order = rb.inv;
  ra.offsets = rb.offsets;
  ra.src_row = rb.src_row;
  ra.tiles = rb.tiles;
  ra.num_tiles = rb.num_tiles;
  ra.max_tiles = a.max_tiles;
  ra.zero_out = y;
  ra.zero_cols = N;
  ra.zero_by_pos = false;
  ra.check_sorted = sorted_indices != 0;
  ra.d_status = d_status;
  auto s = static_cast<cudaStream_t>(stream);
  if (launch_route(ra, rb.route_ws, s) != cudaSuccess) return QMOE_ERR_CUDA;
  if (launch_gather_rows(x, rb.src_row, R, K, x_sorted, s) != cudaSuccess) return QMOE_ERR_CUDA;
  return cuda_status(launch_qmm_tc(a, s));
}

size_t qmoe_sort_by_expert_workspace_size(int64_t R, int64_t E) {
  return route_workspace_bytes(std::max<int64_t>(R, 0), std::max<int64_t>(E, 1)) + 256;
}

int qmoe_sort_by_expert(const uint32_t* indices, int64_t R, int64_t E, uint32_t* order,
                        uint32_t* inv_order, uint32_t* offsets, void* workspace,
                        size_t workspace_bytes, int* d_status, qmoe_stream stream) {
  if (R < 0 || E <= 0) return QMOE_ERR_ARG;
  if (!offsets) return QMOE_ERR_ARG;
  if (R > 0 && (!indices || !order || !inv_order)) return QMOE_ERR_ARG;
  if (workspace == nullptr || workspace_bytes < qmoe_sort_by_expert_workspace_size(R, E))
    return QMOE_ERR_WORKSPACE;
  RouteArgs ra;
  ra.rhs = indices;
  ra.B = R;
  ra.M = 1;
  ra.x_batches = 1;
  ra.E = E;
  ra.order = order;
  ra.inv_order = inv_order;
  ra.offsets = offsets;
  ra.d_status = d_status;
  void* ws = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  return cuda_status(launch_route(ra, ws, static_cast<cudaStream_t>(stream)));
}

int qmoe_tile_table(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                    int64_t max_tiles, uint32_t* num_tiles, int* d_status, qmoe_stream stream) {
  if (E <= 0 || bm <= 0 || max_tiles < 0 || !offsets || !num_tiles) return QMOE_ERR_ARG;
  if (max_tiles > 0 && !tiles) return QMOE_ERR_ARG;
  return cuda_status(launch_tile_table(offsets, E, bm, tiles, max_tiles, num_tiles, d_status,
                                       static_cast<cudaStream_t>(stream)));
}

size_t qmoe_switch_glu_workspace_size(int64_t T, int top_k, const qmoe_qweight* up,
                                      const qmoe_qweight* gate, const qmoe_qweight* down) {
  (void)gate;
  if (up == nullptr || down == nullptr) return 0;
  const int64_t R = std::max<int64_t>(T, 0) * std::max(top_k, 0);
  Carver c(nullptr);
  carve_route(c, R, std::max<int64_t>(up->E, 1), true);
  c.take<uint16_t>(R * up->N);   // h in expert order
  c.take<uint16_t>(R * up->K);   // x rows in expert order
  return c.off + 256;
}

int qmoe_switch_glu(const qmoe_bf16* x, const uint32_t* indices, int64_t T, int top_k,
                    const qmoe_qweight* up, const qmoe_qweight* gate, const qmoe_qweight* down,
                    int mode, void* workspace, size_t workspace_bytes, qmoe_bf16* y,
                    uint32_t* inv_order, int* d_status, qmoe_stream stream) {
  int c = validate_qweight(up);
  if (c == QMOE_OK) c = validate_qweight(gate);
  if (c == QMOE_OK) c = validate_qweight(down);
  if (c != QMOE_OK) return c;
  if (T < 0 || top_k <= 0 || (mode != 0 && mode != 1)) return QMOE_ERR_ARG;
  const int64_t H = up->K, I = up->N, E = up->E;
  if (gate->K != H || gate->N != I || gate->E != E || gate->group != up->group ||
      gate->bits != up->bits)
    return QMOE_ERR_ARG;
  if (down->K != I || down->N != H || down->E != E) return QMOE_ERR_ARG;
  if (T == 0) return QMOE_OK;
  if (!x || !indices || !y || (mode == 1 && !inv_order)) return QMOE_ERR_ARG;
  if (!aligned16(x)) return QMOE_ERR_ARG;
  if (workspace == nullptr ||
      workspace_bytes < qmoe_switch_glu_workspace_size(T, top_k, up, gate, down))
    return QMOE_ERR_WORKSPACE;
  const int64_t R = T * top_k;
  Carver cv(reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255)));
  RouteBufs rb = carve_route(cv, R, E, true);
  uint16_t* h = cv.take<uint16_t>(R * I);
  uint16_t* x_sorted = cv.take<uint16_t>(R * H);
  uint32_t* inv = mode == 1 ? inv_order : rb.inv;

  GemmArgs ug;
  ug.w[0] = qw(up);
  ug.w[1] = qw(gate);
  ug.nmat = 2;
  ug.E = E;
  ug.N = I;
  ug.K = H;
  ug.group = up->group;
  ug.bits = up->bits;
  ug.y = h;
  ug.x_rows = R;
  ug.tiles = rb.tiles;
  ug.num_tiles = rb.num_tiles;
  ug.d_status = d_status;
  GemmArgs dn;
  dn.w[0] = qw(down);
  dn.nmat = 1;
  dn.E = E;
  dn.N = H;
  dn.K = I;
  dn.group = down->group;
  dn.bits = down->bits;
  dn.x = h;
  dn.x_rows = R;
  dn.y = y;
  dn.dst_row = mode == 0 ? rb.order : nullptr;
  dn.tiles = rb.tiles;
  dn.num_tiles = rb.num_tiles;
  dn.tiles_ready = true;  // written by the routing kernel, before the up/gate launch
  dn.d_status = d_status;
  // With distinct experts per token one expert receives at most T rows.  The bound only
  // picks the plan: any routing is served correctly by either kernel.
  GemmArgs ug_sorted = ug;  // as the tensor-core streaming kernel would read x
  ug_sorted.src_row = nullptr;
  const bool bits_ug = qmv_bits_needed(ug.bits, ug.group);
  const bool bits_dn = qmv_bits_needed(dn.bits, dn.group);
  const bool mma_only = !bits_ug && !bits_dn;  // tensor-core plans take no bit-stream width
  const Plan pl = plan_for(R, E, T, mma_only && qmm_tc_supported(ug) && qmm_tc_supported(dn),
                           mma_only && qmm_ts_supported(ug_sorted) && qmm_ts_supported(dn));
  ug.bm = dn.bm = pl.bm;
  ug.max_tiles = dn.max_tiles = max_tiles_for(R, E, pl.bm);

  RouteArgs ra;
  ra.rhs = indices;
  ra.B = R;
  ra.M = 1;
  ra.x_batches = T;
  ra.E = E;
  ra.bm = pl.bm;
  ra.order = rb.order;
  ra.inv_order = inv;
  ra.offsets = rb.offsets;
  ra.src_row = rb.src_row;
  ra.tiles = rb.tiles;
  ra.num_tiles = rb.num_tiles;
  ra.max_tiles = ug.max_tiles;
  ra.zero_out = y;
  ra.zero_cols = H;
  ra.zero_by_pos = mode == 1;
  ra.d_status = d_status;
  auto s = static_cast<cudaStream_t>(stream);
  if (launch_route(ra, rb.route_ws, s) != cudaSuccess) return QMOE_ERR_CUDA;
  if (pl.tc) {
    if (launch_gather_rows(x, rb.src_row, R, H, x_sorted, s) != cudaSuccess) return QMOE_ERR_CUDA;
    ug.x = x_sorted;
    ug.src_row = nullptr;
    if (pl.ts) {
      if (launch_qmm_ts(ug, s) != cudaSuccess) return QMOE_ERR_CUDA;
      return cuda_status(launch_qmm_ts(dn, s));
    }
    if (launch_qmm_tc(ug, s) != cudaSuccess) return QMOE_ERR_CUDA;
    return cuda_status(launch_qmm_tc(dn, s));
  }
  ug.x = x;
  ug.src_row = rb.src_row;
  if ((bits_ug ? launch_qmv_bits(ug, s) : launch_qmv(ug, s)) != cudaSuccess) return QMOE_ERR_CUDA;
  return cuda_status(bits_dn ? launch_qmv_bits(dn, s) : launch_qmv(dn, s));
}

int qmoe_moe_combine(const qmoe_bf16* y_sorted, const uint32_t* inv_order, const float* scores,
                     const qmoe_bf16* shared, const qmoe_bf16* x, const qmoe_bf16* w_shared_gate,
                     int64_t T, int top_k, int64_t H, qmoe_bf16* out, int* d_status,
                     qmoe_stream stream) {
  if (T < 0 || top_k <= 0 || H <= 0) return QMOE_ERR_ARG;
  if (H % 8 != 0) return QMOE_ERR_UNSUPPORTED;
  if ((x == nullptr) != (w_shared_gate == nullptr)) return QMOE_ERR_ARG;
  if (w_shared_gate != nullptr && shared == nullptr) return QMOE_ERR_ARG;
  if (T == 0) return QMOE_OK;
  if (!y_sorted || !inv_order || !scores || !out) return QMOE_ERR_ARG;
  if (!aligned16(y_sorted) || !aligned16(out) || (shared && !aligned16(shared)) ||
      (x && !aligned16(x)) || (w_shared_gate && !aligned16(w_shared_gate)))
    return QMOE_ERR_ARG;
  return cuda_status(launch_combine(y_sorted, inv_order, scores, shared, x, w_shared_gate, T,
                                    top_k, H, out, d_status, static_cast<cudaStream_t>(stream)));
}

int qmoe_moe_combine_stock(const qmoe_bf16* y_sorted, const uint32_t* inv_order,
                           const float* scores, const qmoe_bf16* shared,
                           const qmoe_bf16* shared_gate_logit, int64_t T, int top_k, int64_t H,
                           qmoe_bf16* out, int* d_status, qmoe_stream stream) {
  if (T < 0 || top_k <= 0 || H <= 0) return QMOE_ERR_ARG;
  if (H % 8 != 0) return QMOE_ERR_UNSUPPORTED;
  if (shared_gate_logit != nullptr && shared == nullptr) return QMOE_ERR_ARG;
  if (T == 0) return QMOE_OK;
  if (!y_sorted || !inv_order || !scores || !out) return QMOE_ERR_ARG;
  if (!aligned16(y_sorted) || !aligned16(out) || (shared && !aligned16(shared))) return QMOE_ERR_ARG;
  return cuda_status(launch_combine_stock(y_sorted, inv_order, scores, shared, shared_gate_logit,
                                          T, top_k, H, out, d_status,
                                          static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
