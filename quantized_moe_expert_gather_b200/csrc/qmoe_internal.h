// Host-side interfaces between the library's translation units.  Not part of the
// public ABI (include/qmoe.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

#include "../../include/qmoe.h"

namespace qmoe {

void count_launch(int n = 1);
int sm_count();
// Programmatic dependent launch on (default) or off (environment QMOE_PDL=0).
bool pdl_enabled();

// Launches `kernel` with programmatic stream serialization (when enabled): the kernel
// may run its prologue, up to griddep_wait(), while the previous kernel on the stream
// finishes.  Inside CUDA graph capture this becomes a programmatic dependency edge.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Device-side timing record of one launch: ~(earliest CTA start) and the latest
// CTA end, in global-timer nanoseconds, both combined with atomicMax.
struct ProfSlot {
  unsigned long long start_inv;
  unsigned long long end;
};

// While qmoe_timing_enable() is in effect, reserves the next timing slot for one
// launch of `kernel` and zeroes it on `stream`; slot() is null otherwise.  Pass
// slot() to the kernel.
class LaunchTimer {
 public:
  LaunchTimer(const char* kernel, cudaStream_t stream);
  ProfSlot* slot() const { return slot_; }

 private:
  ProfSlot* slot_ = nullptr;
};

// ----------------------------------------------------------------- quantisation
cudaError_t launch_quantize(const void* w, bool w_f32, int64_t rows, int64_t cols, int group,
                            int bits, uint32_t* codes, void* scales, void* biases,
                            cudaStream_t stream);
cudaError_t launch_dequantize(const uint32_t* codes, const void* scales, const void* biases,
                              bool sb_f32, int64_t rows, int64_t cols, int group, int bits,
                              void* out, bool out_f32, cudaStream_t stream);

// --------------------------------------------------------------- route metadata
// Routed row r = b*M + m (b in [0, B), m in [0, M)) has expert key rhs(b) and reads
// x row lhs(b)*M + m, with the NULL-index defaults of qmoe_gather_qmm.
struct RouteArgs {
  const uint32_t* rhs = nullptr;   // [B] or null
  const uint32_t* lhs = nullptr;   // [B] or null
  int64_t B = 0, M = 1, x_batches = 1, E = 1;
  int bm = 8;                      // rows per tile of the tile table
  // outputs (workspace or caller memory)
  uint32_t* order = nullptr;       // [R]
  uint32_t* inv_order = nullptr;   // [R]
  uint32_t* offsets = nullptr;     // [E+1]; offsets[E] = number of valid rows
  uint32_t* src_row = nullptr;     // [R] x row of each sorted position (nullable)
  uint32_t* tiles = nullptr;       // [max_tiles*3] (nullable)
  uint32_t* num_tiles = nullptr;   // [1] (nullable)
  int64_t max_tiles = 0;
  // Rows with an invalid index are zeroed in this output: row = by_pos ? sorted
  // position : r, `zero_cols` bf16 wide.  Nullable.
  uint16_t* zero_out = nullptr;
  int64_t zero_cols = 0;
  bool zero_by_pos = false;
  // The caller promised sorted rhs indices: flag QMOE_DEV_UNSORTED where they decrease.
  bool check_sorted = false;
  int* d_status = nullptr;
};
size_t route_workspace_bytes(int64_t R, int64_t E);
cudaError_t launch_route(const RouteArgs& a, void* ws, cudaStream_t stream);
cudaError_t launch_tile_table(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                              int64_t max_tiles, uint32_t* num_tiles, int* d_status,
                              cudaStream_t stream);
// x_sorted[p] = x[src_row[p]] for p < rows (rows of `cols` bf16).
cudaError_t launch_gather_rows(const uint16_t* x, const uint32_t* src_row, int64_t rows,
                               int64_t cols, uint16_t* out, cudaStream_t stream);

// ------------------------------------------------------- gathered quantised matmul
struct QWeight {
  const uint32_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
};
// One streaming (small rows per expert) or tensor-core (many rows) launch over the
// expert-aligned tile table.  NMAT = 2 fuses two weight stacks (up, gate) with the
// silu(gate)*up epilogue.
struct GemmArgs {
  QWeight w[2];
  int nmat = 1;
  int64_t E = 1, N = 0, K = 0;
  int group = 64, bits = 4;
  const uint16_t* x = nullptr;       // activation rows, K wide
  int64_t x_rows = 0;                // rows of x (bound of the activation tensor map)
  const uint32_t* src_row = nullptr; // sorted position -> x row (null: identity)
  uint16_t* y = nullptr;             // output rows, N wide
  const uint32_t* dst_row = nullptr; // sorted position -> y row (null: identity)
  const uint32_t* tiles = nullptr;   // (row_start, expert, valid) triples
  const uint32_t* num_tiles = nullptr;
  int64_t dense_rows = 0;            // > 0: no tile table, rows [0, dense_rows), expert 0
  int64_t max_tiles = 0;             // host upper bound of the tile count
  int bm = 8;                        // rows per tile the table was built with
  // The tile table was written before the kernel launched just before this one (the
  // down projection after the up/gate launch): with the weights, it may be read before
  // that kernel completes.
  bool tiles_ready = false;
  int* d_status = nullptr;
};
// Test hook of the bounded waits (qmoe_debug_skip_stage): the stage the next streaming
// launch's last CTA leaves unissued, or -1.  Read and cleared by that launch.
int64_t take_skip_stage();
cudaError_t launch_qmv(const GemmArgs& a, cudaStream_t stream);   // tiles of <= 16 rows
// Bit-stream code widths (1, 3, 5, 6 bits; 2 bits in groups of 32): CUDA-core streaming
// kernel over tiles of <= 16 rows.  qmv_bits_needed: the codec has no MMA kernel.
bool qmv_bits_needed(int bits, int group);
cudaError_t launch_qmv_bits(const GemmArgs& a, cudaStream_t stream);
cudaError_t launch_qmm_tc(const GemmArgs& a, cudaStream_t stream); // tiles of 128 rows
bool qmm_tc_supported(const GemmArgs& a);
// Tensor-core kernel with the dequantised weights as the MMA A operand in tensor memory,
// for tiles of up to kTsTileRows rows: 4-bit codes, activations already in tile order.
#ifndef QMOE_TS_TILE_ROWS
#define QMOE_TS_TILE_ROWS 192
#endif
constexpr int kTsTileRows = QMOE_TS_TILE_ROWS;
bool qmm_ts_supported(const GemmArgs& a);
cudaError_t launch_qmm_ts(const GemmArgs& a, cudaStream_t stream);

// ------------------------------------------------------------------------ combine
cudaError_t launch_combine(const uint16_t* y_sorted, const uint32_t* inv_order,
                           const float* scores, const uint16_t* shared, const uint16_t* x,
                           const uint16_t* w_sg, int64_t T, int top_k, int64_t H, uint16_t* out,
                           int* d_status, cudaStream_t stream);
// The same tail with the stock block's bf16 rounding points (see qmoe_moe_combine_stock).
cudaError_t launch_combine_stock(const uint16_t* y_sorted, const uint32_t* inv_order,
                                 const float* scores, const uint16_t* shared,
                                 const uint16_t* gate_logit, int64_t T, int top_k, int64_t H,
                                 uint16_t* out, int* d_status, cudaStream_t stream);

}  // namespace qmoe
