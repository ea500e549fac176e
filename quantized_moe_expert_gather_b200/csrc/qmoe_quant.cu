// Affine group quantisation and dequantisation (nuvec-core 0.4.0 tests/quantized.rs:
// round_trip_error_is_about_half_a_step, quantize_snaps_zero_and_handles_constant_
// and_one_signed_groups, and the `reference` helper).
//
// Weight preparation, off the timed path: one thread per group.  Every float step
// is an explicit IEEE round-to-nearest intrinsic (no contraction), so codes,
// scales, biases and dequantised values are bit-exact with the CPU oracle.
#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

template <typename T>
__device__ __forceinline__ float load_val(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_val<uint16_t>(const uint16_t* p, int64_t i) {
  return bf16_to_f32(p[i]);
}
template <>
__device__ __forceinline__ float load_val<float>(const float* p, int64_t i) {
  return p[i];
}

template <typename T>
__device__ __forceinline__ void store_val(T* p, int64_t i, float v);
template <>
__device__ __forceinline__ void store_val<uint16_t>(uint16_t* p, int64_t i, float v) {
  p[i] = f32_to_bf16(v);
}
template <>
__device__ __forceinline__ void store_val<float>(float* p, int64_t i, float v) {
  p[i] = v;
}

template <typename T>
__device__ __forceinline__ float round_to_storage(float v);
template <>
__device__ __forceinline__ float round_to_storage<uint16_t>(float v) {
  return bf16_to_f32(f32_to_bf16(v));
}
template <>
__device__ __forceinline__ float round_to_storage<float>(float v) {
  return v;
}

template <typename T, int BITS>
__global__ void quantize_kernel(const T* __restrict__ w, int64_t rows, int64_t cols, int group,
                                uint32_t* __restrict__ codes, T* __restrict__ scales,
                                T* __restrict__ biases) {
  const int64_t groups_per_row = cols / group;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= rows * groups_per_row) return;
  const int64_t row = gid / groups_per_row;
  const int64_t g = gid % groups_per_row;
  const T* src = w + row * cols + g * group;
  float lo = load_val(src, 0), hi = lo;
  for (int i = 1; i < group; ++i) {
    const float v = load_val(src, i);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  const float n = static_cast<float>((1 << BITS) - 1);
  const float delta = fmaxf(__fdiv_rn(__fsub_rn(hi, lo), n), 1e-7f);
  const bool neg = fabsf(lo) > fabsf(hi);
  const float edge = neg ? lo : hi;
  const float step0 = neg ? delta : -delta;
  const float q0 = rintf(__fdiv_rn(edge, step0));
  float scale, bias;
  if (q0 != 0.0f) {
    scale = __fdiv_rn(edge, q0);
    bias = edge;
  } else {
    scale = step0;
    bias = 0.0f;
  }
  const float s_st = round_to_storage<T>(scale);
  const float b_st = round_to_storage<T>(bias);
  store_val(scales, gid, scale);
  store_val(biases, gid, bias);
  // The row's codes are one least-significant-bit-first bit stream (code j at stream
  // bits [j*BITS, (j+1)*BITS)); a group of a multiple of 32 codes fills whole words, so
  // each thread writes its own words.
  uint32_t* dst = codes + (row * cols + g * group) * BITS / 32;
  uint64_t acc = 0;
  int nacc = 0;
  for (int i = 0; i < group; ++i) {
    const float v = load_val(src, i);
    float q = rintf(__fdiv_rn(__fsub_rn(v, b_st), s_st));
    q = fminf(fmaxf(q, 0.0f), n);
    acc |= static_cast<uint64_t>(q) << nacc;
    nacc += BITS;
    if (nacc >= 32) {
      *dst++ = static_cast<uint32_t>(acc);
      acc >>= 32;
      nacc -= 32;
    }
  }
}

template <typename S, typename O, int BITS>
__global__ void dequantize_kernel(const uint32_t* __restrict__ codes, const S* __restrict__ scales,
                                  const S* __restrict__ biases, int64_t rows, int64_t cols,
                                  int group, O* __restrict__ out) {
  constexpr int PER = 32 / BITS;
  const int64_t words_per_row = cols / PER;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (wid >= rows * words_per_row) return;
  const int64_t row = wid / words_per_row;
  const int64_t col0 = (wid % words_per_row) * PER;
  const int64_t gidx = row * (cols / group) + col0 / group;
  const float s = load_val(scales, gidx);
  const float b = load_val(biases, gidx);
  const uint32_t word = codes[wid];
  for (int j = 0; j < PER; ++j) {
    const float q = static_cast<float>((word >> (j * BITS)) & ((1u << BITS) - 1));
    store_val(out, row * cols + col0 + j, __fadd_rn(__fmul_rn(q, s), b));
  }
}

// Any width: one thread per element, reading the (up to two) words its code spans.
template <typename S, typename O>
__global__ void dequantize_stream_kernel(const uint32_t* __restrict__ codes,
                                         const S* __restrict__ scales,
                                         const S* __restrict__ biases, int64_t rows, int64_t cols,
                                         int group, int bits, O* __restrict__ out) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t row = idx / cols, j = idx % cols;
  const uint32_t* rw = codes + row * (cols * bits / 32);
  const int64_t bit = j * bits;
  const int64_t w = bit >> 5;
  const int o = static_cast<int>(bit & 31);
  uint64_t v = rw[w];
  if (o + bits > 32) v |= static_cast<uint64_t>(rw[w + 1]) << 32;
  const float q = static_cast<float>((v >> o) & ((1ull << bits) - 1));
  const int64_t gidx = row * (cols / group) + j / group;
  store_val(out, idx, __fadd_rn(__fmul_rn(q, load_val(scales, gidx)), load_val(biases, gidx)));
}

template <typename T>
cudaError_t launch_quantize_t(const T* wp, int64_t rows, int64_t cols, int group, int bits,
                              uint32_t* codes, T* sp, T* bp, unsigned blocks, int threads,
                              cudaStream_t stream) {
  switch (bits) {
    case 1: quantize_kernel<T, 1><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 2: quantize_kernel<T, 2><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 3: quantize_kernel<T, 3><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 4: quantize_kernel<T, 4><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 5: quantize_kernel<T, 5><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 6: quantize_kernel<T, 6><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    case 8: quantize_kernel<T, 8><<<blocks, threads, 0, stream>>>(wp, rows, cols, group, codes, sp, bp); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_quantize(const void* w, bool w_f32, int64_t rows, int64_t cols, int group,
                            int bits, uint32_t* codes, void* scales, void* biases,
                            cudaStream_t stream) {
  const int64_t n = rows * (cols / group);
  if (n == 0) return cudaSuccess;
  const int threads = 128;
  const unsigned blocks = static_cast<unsigned>((n + threads - 1) / threads);
  const cudaError_t e =
      w_f32 ? launch_quantize_t(static_cast<const float*>(w), rows, cols, group, bits, codes,
                                static_cast<float*>(scales), static_cast<float*>(biases), blocks,
                                threads, stream)
            : launch_quantize_t(static_cast<const uint16_t*>(w), rows, cols, group, bits, codes,
                                static_cast<uint16_t*>(scales), static_cast<uint16_t*>(biases),
                                blocks, threads, stream);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

namespace {
template <typename S, typename O>
void dequant_dispatch(const uint32_t* codes, const void* s, const void* b, int64_t rows,
                      int64_t cols, int group, int bits, void* out, cudaStream_t stream) {
  const int threads = 256;
  if (bits != 4 && bits != 8) {
    const int64_t ne = rows * cols;
    dequantize_stream_kernel<S, O><<<static_cast<unsigned>((ne + threads - 1) / threads), threads,
                                     0, stream>>>(codes, static_cast<const S*>(s),
                                                  static_cast<const S*>(b), rows, cols, group,
                                                  bits, static_cast<O*>(out));
    return;
  }
  const int64_t n = rows * (cols * bits / 32);
  const unsigned blocks = static_cast<unsigned>((n + threads - 1) / threads);
  if (bits == 4)
    dequantize_kernel<S, O, 4><<<blocks, threads, 0, stream>>>(
        codes, static_cast<const S*>(s), static_cast<const S*>(b), rows, cols, group,
        static_cast<O*>(out));
  else
    dequantize_kernel<S, O, 8><<<blocks, threads, 0, stream>>>(
        codes, static_cast<const S*>(s), static_cast<const S*>(b), rows, cols, group,
        static_cast<O*>(out));
}
}  // namespace

cudaError_t launch_dequantize(const uint32_t* codes, const void* scales, const void* biases,
                              bool sb_f32, int64_t rows, int64_t cols, int group, int bits,
                              void* out, bool out_f32, cudaStream_t stream) {
  if (rows * cols == 0) return cudaSuccess;
  if (sb_f32 && out_f32)
    dequant_dispatch<float, float>(codes, scales, biases, rows, cols, group, bits, out, stream);
  else if (sb_f32)
    dequant_dispatch<float, uint16_t>(codes, scales, biases, rows, cols, group, bits, out, stream);
  else if (out_f32)
    dequant_dispatch<uint16_t, float>(codes, scales, biases, rows, cols, group, bits, out, stream);
  else
    dequant_dispatch<uint16_t, uint16_t>(codes, scales, biases, rows, cols, group, bits, out,
                                         stream);
  count_launch();
  return cudaGetLastError();
}

}  // namespace qmoe
