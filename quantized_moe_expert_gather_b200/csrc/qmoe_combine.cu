// One-pass MoE combine (MTPLX PR #558 "One-kernel MoE combine for Qwen3.5/3.6 MoE
// prefill on the invariant lane", Summary and Motivation): the expert-sorted
// outputs, their inverse permutation, the routing scores and the gated shared
// expert are combined in a single pass instead of materialising three
// [rows, top_k, hidden] tensors:
//
//   out[t] = sum_k scores[t,k] * y_sorted[inv_order[t*top_k+k]]
//            + sigmoid(x[t] . w_shared_gate) * shared[t]
//
// One CTA per token, 16-byte vectors, fp32 accumulation, one bf16 rounding.
// HBM-bound: per token it reads top_k + 2 rows and the gate vector, writes one row.
#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kThreads) combine_kernel(
    const uint16_t* __restrict__ y_sorted, const uint32_t* __restrict__ inv_order,
    const float* __restrict__ scores, const uint16_t* __restrict__ shared,
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ w_sg, int64_t T, int top_k,
    int64_t H, uint16_t* __restrict__ out, int* d_status, ProfSlot* prof) {
  __shared__ float red[kThreads / 32];
  __shared__ float gate_sh;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) prof_start(prof);
  const int64_t nvec = H / 8;
  const int64_t R = T * top_k;

  float gate = 1.0f;
  if (shared != nullptr && w_sg != nullptr) {
    float dot = 0.f;
    for (int64_t v = tid; v < nvec; v += kThreads) {
      float a[8], b[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(x + t * H)[v], a);
      bf16x8_to_f32(reinterpret_cast<const uint4*>(w_sg)[v], b);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(a[i], b[i], dot);
    }
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
    if ((tid & 31) == 0) red[tid >> 5] = dot;
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) s += red[w];
      gate_sh = 1.0f / (1.0f + expf(-s));
    }
    __syncthreads();
    gate = gate_sh;
  }

  for (int64_t v = tid; v < nvec; v += kThreads) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < top_k; ++k) {
      const uint32_t pos = inv_order[t * top_k + k];
      if (pos >= R) {
        if (v == tid) set_status(d_status, QMOE_DEV_BAD_INDEX);
        continue;
      }
      const float s = scores[t * top_k + k];
      float yv[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(y_sorted + static_cast<int64_t>(pos) * H)[v], yv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(s, yv[i], acc[i]);
    }
    if (shared != nullptr) {
      float sv[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(shared + t * H)[v], sv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(gate, sv[i], acc[i]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(out + t * H)[v] = o;
  }
  __syncthreads();
  if (tid == 0) prof_end(prof);
}

}  // namespace

cudaError_t launch_combine(const uint16_t* y_sorted, const uint32_t* inv_order,
                           const float* scores, const uint16_t* shared, const uint16_t* x,
                           const uint16_t* w_sg, int64_t T, int top_k, int64_t H, uint16_t* out,
                           int* d_status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  LaunchTimer timer("combine", stream);
  combine_kernel<<<static_cast<unsigned>(T), kThreads, 0, stream>>>(
      y_sorted, inv_order, scores, shared, x, w_sg, T, top_k, H, out, d_status, timer.slot());
  count_launch();
  return cudaGetLastError();
}

}  // namespace qmoe
