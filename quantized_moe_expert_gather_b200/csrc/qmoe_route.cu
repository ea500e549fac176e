// Route metadata: stable counting sort of routed rows by expert, the inverse
// permutation, per-expert offsets and the expert-aligned tile table.
//
// MLX PR #4567 "[Metal] Gather mm improvement", Proposed changes: tiles are cut
// per expert from offsets precomputed from rhs_indices, each tile carrying the row
// it starts from, the expert it loads and its number of valid rows, so no tile
// spans two experts.  MTPLX PR #558, Change: the sorted chain sorts rows by expert
// (`_gather_sort`) and keeps the inverse permutation to unsort later.
//
// Integer work, bit-exact with the oracle: equal experts keep ascending row order.
// Three phases over chunks of 1024 rows: (1) per-chunk histogram and stable local
// ranks (warp match + per-warp counts), (2) one CTA turns the chunk histograms into
// global bases, offsets and the tile table, (3) scatter.  Up to one chunk the three
// phases run in a single CTA (one launch); beyond that as three launches.
#include <algorithm>

#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

constexpr int kChunk = 1024;          // rows per chunk = threads per CTA
constexpr uint32_t kNoRow = 0xFFFFFFFFu;

struct RouteDev {
  const uint32_t* rhs;
  const uint32_t* lhs;
  int64_t B, M, x_batches, E, R;
  int bm;
  uint32_t* lrank;   // [R]
  uint32_t* hist;    // [nchunks][E+1]: chunk histogram, then global base
  uint32_t* order;
  uint32_t* inv_order;
  uint32_t* offsets;  // [E+1]
  uint32_t* src_row;
  uint32_t* tiles;
  uint32_t* num_tiles;
  int64_t max_tiles;
  uint16_t* zero_out;
  int64_t zero_cols;
  bool zero_by_pos;
  bool check_sorted;  // flag rhs indices that decrease (the caller promised sorted ones)
  int* d_status;
  ProfSlot* prof;
};

// With check_sorted, a batch whose expert index is below the previous batch's breaks
// the caller's promise of sorted rhs indices: flag it (the result does not depend on
// the promise, the rows are sorted here anyway).
__device__ __forceinline__ void check_rhs_order(const RouteDev& d, int64_t r) {
  if (!d.check_sorted || d.rhs == nullptr || r % d.M != 0) return;
  const int64_t b = r / d.M;
  if (b > 0 && d.rhs[b] < d.rhs[b - 1]) set_status(d.d_status, QMOE_DEV_UNSORTED);
}

// Expert key of routed row r (E for an invalid expert or x row) and its x row.
__device__ __forceinline__ uint32_t row_key(const RouteDev& d, int64_t r, uint32_t* xrow) {
  const int64_t b = r / d.M;
  const int64_t m = r % d.M;
  const uint64_t e = d.rhs ? d.rhs[b] : static_cast<uint64_t>((b * d.E) / d.B);
  const uint64_t l = d.lhs ? d.lhs[b] : static_cast<uint64_t>((b * d.x_batches) / d.B);
  const bool ok = e < static_cast<uint64_t>(d.E) && l < static_cast<uint64_t>(d.x_batches);
  *xrow = ok ? static_cast<uint32_t>(l * d.M + m) : 0u;
  return ok ? static_cast<uint32_t>(e) : static_cast<uint32_t>(d.E);
}

// Phase 1 for one chunk: keys, stable ranks within the chunk, chunk histogram.
// `cnt` is shared scratch of 32*(E+1) bytes.
__device__ void phase_count(const RouteDev& d, int64_t chunk, uint8_t* cnt) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nb = d.E + 1;
  for (int64_t i = tid; i < 32 * nb; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int64_t r = chunk * kChunk + tid;
  uint32_t key = kNoRow, xrow = 0;
  if (r < d.R) {
    key = row_key(d, r, &xrow);
    check_rhs_order(d, r);
  }
  const uint32_t mask = __match_any_sync(0xFFFFFFFFu, key);
  const uint32_t lt = (1u << lane) - 1u;
  const uint32_t rank = __popc(mask & lt);
  if (key != kNoRow && rank == 0) cnt[warp * nb + key] = static_cast<uint8_t>(__popc(mask));
  __syncthreads();
  if (key != kNoRow) {
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += cnt[w * nb + key];
    d.lrank[r] = before + rank;
  }
  for (int64_t e = tid; e < nb; e += blockDim.x) {
    uint32_t tot = 0;
    for (int w = 0; w < 32; ++w) tot += cnt[w * nb + e];
    d.hist[chunk * nb + e] = tot;
  }
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = sh[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;
  }
  __syncthreads();
  const uint32_t warp_base = warp ? sh[warp - 1] : 0u;
  *total = sh[31];
  __syncthreads();
  return warp_base + x - v;
}

// Tile table from offsets[0..E]: ceil(count_e/bm) tiles per expert, in order.
__device__ void write_tiles(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                            int64_t max_tiles, uint32_t* num_tiles, int* d_status,
                            uint32_t* sh) {
  const int tid = threadIdx.x;
  uint32_t carry = 0;
  for (int64_t e0 = 0; e0 < E; e0 += blockDim.x) {
    const int64_t e = e0 + tid;
    uint32_t cnt = 0, start = 0;
    if (e < E) {
      start = offsets[e];
      cnt = offsets[e + 1] - start;
    }
    const uint32_t nt = (cnt + bm - 1) / bm;
    uint32_t total;
    const uint32_t t0 = carry + block_exclusive_scan(nt, sh, &total);
    for (uint32_t i = 0; i < nt; ++i) {
      const int64_t ti = static_cast<int64_t>(t0) + i;
      if (ti < max_tiles) {
        const uint32_t rs = start + i * bm;
        tiles[3 * ti + 0] = rs;
        tiles[3 * ti + 1] = static_cast<uint32_t>(e);
        tiles[3 * ti + 2] = min(static_cast<uint32_t>(bm), start + cnt - rs);
      } else {
        set_status(d_status, QMOE_DEV_BAD_INDEX);
      }
    }
    carry += total;
  }
  if (tid == 0) *num_tiles = static_cast<uint32_t>(imin64(carry, max_tiles));
}

// Phase 2 (one CTA): chunk histograms -> global bases, offsets, tile table.
__device__ void phase_scan(const RouteDev& d, int64_t nchunks, uint32_t* sh) {
  const int tid = threadIdx.x;
  const int64_t nb = d.E + 1;
  uint32_t carry = 0;
  for (int64_t e0 = 0; e0 < nb; e0 += blockDim.x) {
    const int64_t e = e0 + tid;
    uint32_t tot = 0;
    if (e < nb)
      for (int64_t c = 0; c < nchunks; ++c) tot += d.hist[c * nb + e];
    uint32_t total;
    const uint32_t off = carry + block_exclusive_scan(tot, sh, &total);
    if (e < nb) {
      d.offsets[e] = off;
      uint32_t run = off;
      for (int64_t c = 0; c < nchunks; ++c) {
        const uint32_t h = d.hist[c * nb + e];
        d.hist[c * nb + e] = run;
        run += h;
      }
    }
    carry += total;
  }
  __syncthreads();
  if (d.tiles != nullptr)
    write_tiles(d.offsets, d.E, d.bm, d.tiles, d.max_tiles, d.num_tiles, d.d_status, sh);
}

// Phase 3 for one chunk: scatter order / inv_order / src_row; zero invalid rows.
__device__ void phase_scatter(const RouteDev& d, int64_t chunk) {
  const int64_t nb = d.E + 1;
  const int64_t r = chunk * kChunk + threadIdx.x;
  if (r < d.R) {
    uint32_t xrow;
    const uint32_t key = row_key(d, r, &xrow);
    const uint32_t pos = d.hist[chunk * nb + key] + d.lrank[r];
    d.order[pos] = static_cast<uint32_t>(r);
    d.inv_order[r] = pos;
    if (d.src_row) d.src_row[pos] = xrow;
    if (key == static_cast<uint32_t>(d.E)) set_status(d.d_status, QMOE_DEV_BAD_INDEX);
    if (key == static_cast<uint32_t>(d.E) && d.zero_out != nullptr) {
      const int64_t row = d.zero_by_pos ? static_cast<int64_t>(pos) : r;
      uint16_t* dst = d.zero_out + row * d.zero_cols;
      for (int64_t c = 0; c < d.zero_cols; ++c) dst[c] = 0;
    }
  }
}

__global__ void __launch_bounds__(kChunk) route_count_kernel(RouteDev d) {
  extern __shared__ uint8_t cnt[];
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(d.prof);
  phase_count(d, blockIdx.x, cnt);
  __syncthreads();
  if (threadIdx.x == 0) prof_end(d.prof);
}
__global__ void __launch_bounds__(kChunk) route_scan_kernel(RouteDev d, int64_t nchunks) {
  __shared__ uint32_t sh[32];
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(d.prof);
  phase_scan(d, nchunks, sh);
  __syncthreads();
  if (threadIdx.x == 0) prof_end(d.prof);
}
__global__ void __launch_bounds__(kChunk) route_scatter_kernel(RouteDev d) {
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(d.prof);
  phase_scatter(d, blockIdx.x);
  __syncthreads();
  if (threadIdx.x == 0) prof_end(d.prof);
}
// R <= 1024: all three phases in one CTA.
__global__ void __launch_bounds__(kChunk) route_fused_kernel(RouteDev d) {
  // Shared scratch: per-warp counts [32][E+1] bytes, then the expert bases [E+1].
  // Every thread keeps its own row's key, x row and stable rank in registers across
  // the phases, so nothing round-trips through global memory inside the CTA.
  extern __shared__ uint8_t dyn[];
  __shared__ uint32_t sh[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nb = d.E + 1;
  uint8_t* cnt = dyn;
  uint32_t* base = reinterpret_cast<uint32_t*>(dyn + ((32 * nb + 15) & ~int64_t(15)));
  griddep_wait();  // the indices may come from the kernel before this one
  griddep_launch_dependents();
  if (tid == 0) prof_start(d.prof);
  for (int64_t i = tid; i < 32 * nb; i += blockDim.x) cnt[i] = 0;
  const int64_t r = tid;
  uint32_t key = kNoRow, xrow = 0;
  if (r < d.R) {
    key = row_key(d, r, &xrow);
    check_rhs_order(d, r);
  }
  __syncthreads();
  // stable rank: rank inside the warp's equal keys + equal keys of earlier warps
  const uint32_t mask = __match_any_sync(0xFFFFFFFFu, key);
  const uint32_t rank = __popc(mask & ((1u << lane) - 1u));
  if (key != kNoRow && rank == 0) cnt[warp * nb + key] = static_cast<uint8_t>(__popc(mask));
  __syncthreads();
  uint32_t lrank = rank;
  if (key != kNoRow)
    for (int w = 0; w < warp; ++w) lrank += cnt[w * nb + key];
  // expert totals -> exclusive scan -> bases (shared) and offsets (global)
  uint32_t carry = 0;
  for (int64_t e0 = 0; e0 < nb; e0 += blockDim.x) {
    const int64_t e = e0 + tid;
    uint32_t tot = 0;
    if (e < nb)
      for (int w = 0; w < 32; ++w) tot += cnt[w * nb + e];
    uint32_t total;
    const uint32_t off = carry + block_exclusive_scan(tot, sh, &total);
    if (e < nb) {
      base[e] = off;
      d.offsets[e] = off;
    }
    carry += total;
  }
  __syncthreads();
  if (d.tiles != nullptr)
    write_tiles(base, d.E, d.bm, d.tiles, d.max_tiles, d.num_tiles, d.d_status, sh);
  // scatter
  if (r < d.R) {
    const uint32_t pos = base[key] + lrank;
    d.order[pos] = static_cast<uint32_t>(r);
    d.inv_order[r] = pos;
    if (d.src_row) d.src_row[pos] = xrow;
    if (key == static_cast<uint32_t>(d.E)) {
      set_status(d.d_status, QMOE_DEV_BAD_INDEX);
      if (d.zero_out != nullptr) {
        const int64_t row = d.zero_by_pos ? static_cast<int64_t>(pos) : r;
        uint16_t* dst = d.zero_out + row * d.zero_cols;
        for (int64_t c = 0; c < d.zero_cols; ++c) dst[c] = 0;
      }
    }
  }
  __syncthreads();
  if (tid == 0) prof_end(d.prof);
}
__global__ void __launch_bounds__(kChunk)
    tile_table_kernel(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                      int64_t max_tiles, uint32_t* num_tiles, int* d_status) {
  __shared__ uint32_t sh[32];
  write_tiles(offsets, E, bm, tiles, max_tiles, num_tiles, d_status, sh);
}

__global__ void gather_rows_kernel(const uint16_t* __restrict__ x,
                                   const uint32_t* __restrict__ src_row, int64_t rows,
                                   int64_t cols, uint16_t* __restrict__ out, ProfSlot* prof) {
  griddep_wait();  // src_row comes from the route kernel
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(prof);
  // cols is a multiple of 8: 16-byte vectors.
  const int64_t vec_per_row = cols / 8;
  const int64_t n = rows * vec_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = i / vec_per_row, v = i % vec_per_row;
    const int64_t sr = src_row[p];
    reinterpret_cast<uint4*>(out + p * cols)[v] =
        reinterpret_cast<const uint4*>(x + sr * cols)[v];
  }
  __syncthreads();
  if (threadIdx.x == 0) prof_end(prof);
}

inline int64_t align256(int64_t b) { return (b + 255) & ~int64_t(255); }

}  // namespace

size_t route_workspace_bytes(int64_t R, int64_t E) {
  const int64_t nchunks = (R + kChunk - 1) / kChunk;
  return static_cast<size_t>(align256(4 * R) + align256(4 * std::max<int64_t>(nchunks, 1) * (E + 1)));
}

cudaError_t launch_route(const RouteArgs& a, void* ws, cudaStream_t stream) {
  const int64_t R = a.B * a.M;
  RouteDev d{};
  d.rhs = a.rhs;
  d.lhs = a.lhs;
  d.B = a.B;
  d.M = a.M;
  d.x_batches = a.x_batches;
  d.E = a.E;
  d.R = R;
  d.bm = a.bm;
  char* p = static_cast<char*>(ws);
  d.lrank = reinterpret_cast<uint32_t*>(p);
  p += align256(4 * R);
  d.hist = reinterpret_cast<uint32_t*>(p);
  d.order = a.order;
  d.inv_order = a.inv_order;
  d.offsets = a.offsets;
  d.src_row = a.src_row;
  d.tiles = a.tiles;
  d.num_tiles = a.num_tiles;
  d.max_tiles = a.max_tiles;
  d.zero_out = a.zero_out;
  d.zero_cols = a.zero_cols;
  d.zero_by_pos = a.zero_by_pos;
  d.check_sorted = a.check_sorted;
  d.d_status = a.d_status;
  const int64_t nchunks = (R + kChunk - 1) / kChunk;
  const size_t cnt_bytes = static_cast<size_t>(32 * (a.E + 1));
  const size_t fused_bytes = ((cnt_bytes + 15) & ~size_t(15)) + 4 * static_cast<size_t>(a.E + 1);
  if (cnt_bytes > 200 * 1024) return cudaErrorInvalidValue;  // E above ~6400 experts
  if (cnt_bytes > 48 * 1024)
    cudaFuncSetAttribute(route_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(cnt_bytes));
  if (nchunks <= 1 && fused_bytes <= 220 * 1024) {
    if (fused_bytes > 48 * 1024)
      cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(fused_bytes));
    LaunchTimer timer("route", stream);
    d.prof = timer.slot();
    if (launch_pdl(route_fused_kernel, dim3(1), dim3(kChunk), fused_bytes, stream, d) != cudaSuccess)
      return cudaGetLastError();
    count_launch();
  } else {
    {
      LaunchTimer timer("route", stream);
      d.prof = timer.slot();
      if (launch_pdl(route_count_kernel, dim3(static_cast<unsigned>(nchunks)), dim3(kChunk),
                     cnt_bytes, stream, d) != cudaSuccess)
        return cudaGetLastError();
    }
    {
      LaunchTimer timer("route", stream);
      d.prof = timer.slot();
      if (launch_pdl(route_scan_kernel, dim3(1), dim3(kChunk), 0, stream, d, nchunks) != cudaSuccess)
        return cudaGetLastError();
    }
    {
      LaunchTimer timer("route", stream);
      d.prof = timer.slot();
      if (launch_pdl(route_scatter_kernel, dim3(static_cast<unsigned>(nchunks)), dim3(kChunk), 0,
                     stream, d) != cudaSuccess)
        return cudaGetLastError();
    }
    count_launch(3);
  }
  return cudaGetLastError();
}

cudaError_t launch_tile_table(const uint32_t* offsets, int64_t E, int bm, uint32_t* tiles,
                              int64_t max_tiles, uint32_t* num_tiles, int* d_status,
                              cudaStream_t stream) {
  tile_table_kernel<<<1, kChunk, 0, stream>>>(offsets, E, bm, tiles, max_tiles, num_tiles,
                                               d_status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* x, const uint32_t* src_row, int64_t rows,
                               int64_t cols, uint16_t* out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t n = rows * (cols / 8);
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
  LaunchTimer timer("gather_rows", stream);
  if (launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream,
                 x, src_row, rows, cols, out, timer.slot()) != cudaSuccess)
    return cudaGetLastError();
  count_launch();
  return cudaGetLastError();
}

}  // namespace qmoe
