// Gathered quantised matmul for the bit-stream code widths without a tensor-core or
// mma.sync kernel of their own: 1, 3, 5 and 6 bits in any group, and 2 bits in groups of
// 32 (nuvec-core 0.4.0 tests/quantized.rs, round_trip_error_is_about_half_a_step and the
// quantized_matmul / gather_qmm tests over `const BITS = [1, 2, 3, 4, 5, 6, 8]`).
//
//   y[row, n] = x[row] . dequantize(W[e])[n]^T, and with two weight stacks the SwitchGLU
//   epilogue h = silu(gate) * up (MLX issue #4509 repro script, `moe`),
//
// over the expert-aligned tile table of MLX PR #4567 (Proposed changes): a unit is one
// tile of at most 16 routed rows of one expert and 32 output channels; every unit reads
// those channels' packed codes once.
//
// The codes of a row form one least-significant-bit-first bit stream, code j at stream
// bits [j*bits, (j+1)*bits).  32 consecutive codes occupy exactly `bits` words and start
// on a word boundary for every width, and they lie in one quantisation group (groups
// are multiples of 32).  A lane takes such runs of 32 codes, extracts each code with a
// constant funnel shift (a 3-, 5- or 6-bit code may straddle two words), dequantises
// w = q * s + b in fp32 (the product of a code and a bf16 scale is exact), and
// accumulates x * w for each routed row of the tile in fp32 on the CUDA cores.  The 32
// lanes of a warp then sum their partials in a fixed butterfly order, so a row's result
// does not depend on the other rows of its tile.
#include <algorithm>

#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

constexpr int kWarps = 8;        // warps per CTA
constexpr int kUnitRows = 32;    // output channels per unit: four per warp
constexpr int kTileMax = 16;     // routed rows per tile

struct BitsParams {
  const uint32_t* codes[2];
  const uint16_t* scales[2];
  const uint16_t* biases[2];
  const uint16_t* x;
  const uint32_t* src_row;
  const uint32_t* dst_row;
  uint16_t* y;
  const uint32_t* tiles;
  const uint32_t* num_tiles;
  int64_t dense_rows;
  int64_t N, K;
  int group;
  int bm;
  ProfSlot* prof;
};

// Code i (0..31) of a run of 32 codes held in words w[0..BITS-1].
template <int BITS>
__device__ __forceinline__ uint32_t run_code(const uint32_t (&w)[BITS], int i) {
  const int o = i * BITS, j = o >> 5, sh = o & 31;
  uint32_t v;
  if (sh + BITS <= 32 || j + 1 >= BITS)
    v = w[j] >> sh;
  else
    v = __funnelshift_r(w[j], w[j + 1], sh);
  return v & ((1u << BITS) - 1u);
}

template <int BITS, int NMAT>
__global__ void __launch_bounds__(kWarps * 32) qmv_bits_kernel(const __grid_constant__ BitsParams p) {
  griddep_wait();  // activations and the tile table come from the kernels before this one
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(p.prof);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t runs = p.K / 32;                   // runs of 32 codes per row
  const int64_t words_row = p.K * BITS / 32;
  const int64_t groups_row = p.K / p.group;
  const int64_t NB = (p.N + kUnitRows - 1) / kUnitRows;
  const int64_t ntiles = p.dense_rows > 0 ? (p.dense_rows + p.bm - 1) / p.bm : *p.num_tiles;
  const int64_t units = ntiles * NB;

  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t j = u / NB;
    uint32_t row_start, expert, valid;
    if (p.dense_rows > 0) {
      row_start = static_cast<uint32_t>(j * p.bm);
      expert = 0;
      valid = static_cast<uint32_t>(imin64(p.bm, p.dense_rows - j * p.bm));
    } else {
      row_start = p.tiles[3 * j];
      expert = p.tiles[3 * j + 1];
      valid = min(p.tiles[3 * j + 2], static_cast<uint32_t>(kTileMax));
    }
    const uint16_t* xr[kTileMax];
#pragma unroll
    for (int v = 0; v < kTileMax; ++v) {
      xr[v] = nullptr;
      if (static_cast<uint32_t>(v) < valid) {
        const uint32_t pos = row_start + v;
        const uint32_t sr = p.src_row ? p.src_row[pos] : pos;
        xr[v] = p.x + static_cast<int64_t>(sr) * p.K;
      }
    }
    for (int r = warp; r < kUnitRows; r += kWarps) {
      const int64_t n = (u % NB) * kUnitRows + r;
      if (n >= p.N) break;
      const int64_t wrow = static_cast<int64_t>(expert) * p.N + n;
      float acc[NMAT][kTileMax];
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int v = 0; v < kTileMax; ++v) acc[m][v] = 0.f;
      for (int64_t c = lane; c < runs; c += 32) {
        const int64_t grp = c * 32 / p.group;
        float wv[NMAT][32];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          uint32_t w[BITS];
          const uint32_t* src = p.codes[m] + wrow * words_row + c * BITS;
#pragma unroll
          for (int k = 0; k < BITS; ++k) w[k] = src[k];
          const float s = bf16_to_f32(p.scales[m][wrow * groups_row + grp]);
          const float b = bf16_to_f32(p.biases[m][wrow * groups_row + grp]);
#pragma unroll
          for (int i = 0; i < 32; ++i) wv[m][i] = fmaf(static_cast<float>(run_code<BITS>(w, i)), s, b);
        }
#pragma unroll
        for (int v = 0; v < kTileMax; ++v) {
          if (static_cast<uint32_t>(v) >= valid) break;
          const uint4* xp = reinterpret_cast<const uint4*>(xr[v] + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 xq = __ldg(xp + q);
            const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float x0 = __uint_as_float(xw[h] << 16);
              const float x1 = __uint_as_float(xw[h] & 0xFFFF0000u);
#pragma unroll
              for (int m = 0; m < NMAT; ++m) {
                acc[m][v] = fmaf(x0, wv[m][8 * q + 2 * h], acc[m][v]);
                acc[m][v] = fmaf(x1, wv[m][8 * q + 2 * h + 1], acc[m][v]);
              }
            }
          }
        }
      }
      // fixed-order butterfly over the lanes, then lane 0 writes the tile's rows
#pragma unroll
      for (int v = 0; v < kTileMax; ++v) {
        if (static_cast<uint32_t>(v) >= valid) break;
        float out[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          float t = acc[m][v];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
          out[m] = t;
        }
        if (lane == 0) {
          const uint32_t pos = row_start + v;
          const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
          float val = out[0];
          if constexpr (NMAT == 2) val = out[0] * (out[1] / (1.0f + expf(-out[1])));
          p.y[static_cast<int64_t>(dr) * p.N + n] = f32_to_bf16(val);
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) prof_end(p.prof);
}

template <int BITS>
cudaError_t launch_bits(const BitsParams& prm, int nmat, cudaStream_t stream) {
  const int64_t NB = (prm.N + kUnitRows - 1) / kUnitRows;
  const int64_t max_units =
      (prm.dense_rows > 0 ? (prm.dense_rows + prm.bm - 1) / prm.bm : 1) * NB;
  // enough CTAs to fill the GPU several times over, never more than the units of a
  // dense call (a gathered call's tile count is known only on the device)
  int64_t grid = static_cast<int64_t>(sm_count()) * 8;
  if (prm.dense_rows > 0) grid = std::min(grid, max_units);
  if (grid < 1) grid = 1;
  const dim3 g(static_cast<unsigned>(grid)), b(kWarps * 32);
  if (nmat == 2) return launch_pdl(qmv_bits_kernel<BITS, 2>, g, b, 0, stream, prm);
  return launch_pdl(qmv_bits_kernel<BITS, 1>, g, b, 0, stream, prm);
}

}  // namespace

bool qmv_bits_needed(int bits, int group) {
  return !((bits == 4 || bits == 8) || (bits == 2 && group != 32));
}

cudaError_t launch_qmv_bits(const GemmArgs& a, cudaStream_t stream) {
  BitsParams prm{};
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
    prm.codes[m] = wm.codes;
    prm.scales[m] = wm.scales;
    prm.biases[m] = wm.biases;
  }
  prm.x = a.x;
  prm.src_row = a.src_row;
  prm.dst_row = a.dst_row;
  prm.y = a.y;
  prm.tiles = a.tiles;
  prm.num_tiles = a.num_tiles;
  prm.dense_rows = a.dense_rows;
  prm.N = a.N;
  prm.K = a.K;
  prm.group = a.group;
  prm.bm = std::min(a.bm, kTileMax);
  LaunchTimer timer(a.nmat == 2 ? "qmv_glu" : "qmv", stream);
  prm.prof = timer.slot();
  cudaError_t e;
  switch (a.bits) {
    case 1: e = launch_bits<1>(prm, a.nmat, stream); break;
    case 2: e = launch_bits<2>(prm, a.nmat, stream); break;
    case 3: e = launch_bits<3>(prm, a.nmat, stream); break;
    case 5: e = launch_bits<5>(prm, a.nmat, stream); break;
    case 6: e = launch_bits<6>(prm, a.nmat, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace qmoe
