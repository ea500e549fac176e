// One-pass MoE combine (MTPLX PR #558 "One-kernel MoE combine for Qwen3.5/3.6 MoE
// prefill on the invariant lane", Summary and Motivation): the expert-sorted
// outputs, their inverse permutation, the routing scores and the gated shared
// expert are combined in a single pass instead of materialising three
// [rows, top_k, hidden] tensors:
//
//   out[t] = sum_k scores[t,k] * y_sorted[inv_order[t*top_k+k]]
//            + sigmoid(x[t] . w_shared_gate) * shared[t]
//
// Grid: tokens x slices of the hidden dimension (one 16-byte vector per thread), so
// that a handful of decode tokens still spreads over many SMs.  A CTA stages the
// token's expert positions and scores in shared memory and issues the loads of up to
// eight expert rows before it accumulates them, instead of walking a chain of
// dependent index and row loads.  fp32 accumulation in k order, one bf16 rounding.
// HBM-bound: per token it reads top_k + 2 rows and the gate vector, writes one row.
#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

constexpr int kThreads = 128;
constexpr int kKChunk = 32;   // expert slots staged in shared memory at a time
constexpr int kKBatch = 8;    // expert rows loaded before they are accumulated

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
  __shared__ uint32_t pos_sh[kKChunk];
  __shared__ float score_sh[kKChunk];
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  griddep_wait();  // the expert outputs come from the kernel before this one
  griddep_launch_dependents();
  if (tid == 0) prof_start(prof);
  const int64_t nvec = H / 8;
  const int64_t v = static_cast<int64_t>(blockIdx.y) * kThreads + tid;  // this thread's vector
  const bool live = v < nvec;
  const uint32_t R = static_cast<uint32_t>(T * top_k);

  // shared-expert gate: sigmoid(x[t] . w_sg), reduced over the whole row by every CTA
  float gate = 1.0f;
  if (shared != nullptr && w_sg != nullptr) {
    float dot = 0.f;
    for (int64_t w = tid; w < nvec; w += kThreads) {
      float a[8], b[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(x + t * H)[w], a);
      bf16x8_to_f32(reinterpret_cast<const uint4*>(w_sg)[w], b);
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

  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < top_k; k0 += kKChunk) {
    const int kn = min(kKChunk, top_k - k0);
    if (tid < kn) {
      const uint32_t pos = inv_order[t * top_k + k0 + tid];
      if (pos >= R && blockIdx.y == 0) set_status(d_status, QMOE_DEV_BAD_INDEX);
      pos_sh[tid] = pos;
      score_sh[tid] = scores[t * top_k + k0 + tid];
    }
    __syncthreads();
    if (live) {
      for (int kb = 0; kb < kn; kb += kKBatch) {
        uint4 yv[kKBatch];
#pragma unroll
        for (int j = 0; j < kKBatch; ++j) {
          yv[j] = make_uint4(0, 0, 0, 0);
          const uint32_t pos = kb + j < kn ? pos_sh[kb + j] : R;
          if (pos < R)  // an out-of-range position contributes nothing (status set above)
            yv[j] = reinterpret_cast<const uint4*>(y_sorted + static_cast<int64_t>(pos) * H)[v];
        }
#pragma unroll
        for (int j = 0; j < kKBatch; ++j) {
          if (kb + j < kn && pos_sh[kb + j] < R) {
            const float s = score_sh[kb + j];
            float yf[8];
            bf16x8_to_f32(yv[j], yf);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(s, yf[i], acc[i]);
          }
        }
      }
    }
    __syncthreads();  // before the next chunk overwrites pos_sh / score_sh
  }
  if (live) {
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

// bf16 rounding (nearest even) of an fp32 value, returned as fp32.
__device__ __forceinline__ float round_bf16(float v) {
  return __uint_as_float(static_cast<uint32_t>(f32_to_bf16(v)) << 16);
}

// The tail with the stock block's rounding: each product, the top_k sum, the gate and
// the shared term are rounded to bf16 where the stock block materialises them; the
// top_k sum runs in fp32 in k order.  Same grid and row batching as combine_kernel.
__global__ void __launch_bounds__(kThreads) combine_stock_kernel(
    const uint16_t* __restrict__ y_sorted, const uint32_t* __restrict__ inv_order,
    const float* __restrict__ scores, const uint16_t* __restrict__ shared,
    const uint16_t* __restrict__ gate_logit, int64_t T, int top_k, int64_t H,
    uint16_t* __restrict__ out, int* d_status, ProfSlot* prof) {
  __shared__ uint32_t pos_sh[kKChunk];
  __shared__ float score_sh[kKChunk];
  __shared__ float gate_sh;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  griddep_wait();  // the expert outputs come from the kernel before this one
  griddep_launch_dependents();
  if (tid == 0) {
    prof_start(prof);
    float g = 1.0f;
    if (gate_logit != nullptr) {
      const double z = static_cast<double>(bf16_to_f32(gate_logit[t]));
      g = round_bf16(static_cast<float>(1.0 / (1.0 + exp(-z))));
    }
    gate_sh = g;  // read after the first barrier below
  }
  const int64_t nvec = H / 8;
  const int64_t v = static_cast<int64_t>(blockIdx.y) * kThreads + tid;
  const bool live = v < nvec;
  const uint32_t R = static_cast<uint32_t>(T * top_k);

  float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < top_k; k0 += kKChunk) {
    const int kn = min(kKChunk, top_k - k0);
    if (tid < kn) {
      const uint32_t pos = inv_order[t * top_k + k0 + tid];
      if (pos >= R && blockIdx.y == 0) set_status(d_status, QMOE_DEV_BAD_INDEX);
      pos_sh[tid] = pos;
      score_sh[tid] = round_bf16(scores[t * top_k + k0 + tid]);
    }
    __syncthreads();
    if (live) {
      for (int kb = 0; kb < kn; kb += kKBatch) {
        uint4 yv[kKBatch];
#pragma unroll
        for (int j = 0; j < kKBatch; ++j) {
          yv[j] = make_uint4(0, 0, 0, 0);
          const uint32_t pos = kb + j < kn ? pos_sh[kb + j] : R;
          if (pos < R)
            yv[j] = reinterpret_cast<const uint4*>(y_sorted + static_cast<int64_t>(pos) * H)[v];
        }
#pragma unroll
        for (int j = 0; j < kKBatch; ++j) {
          if (kb + j < kn && pos_sh[kb + j] < R) {
            const float sk = score_sh[kb + j];
            float yf[8];
            bf16x8_to_f32(yv[j], yf);
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] = __fadd_rn(r[i], round_bf16(__fmul_rn(yf[i], sk)));
          }
        }
      }
    }
    __syncthreads();  // before the next chunk overwrites pos_sh / score_sh
  }
  if (live) {
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = round_bf16(r[i]);
    if (shared != nullptr) {
      const float g = gate_sh;
      float sv[8];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(shared + t * H)[v], sv);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __fadd_rn(o[i], round_bf16(__fmul_rn(g, sv[i])));
    }
    uint4 w;
    w.x = pack_bf16x2(o[0], o[1]);
    w.y = pack_bf16x2(o[2], o[3]);
    w.z = pack_bf16x2(o[4], o[5]);
    w.w = pack_bf16x2(o[6], o[7]);
    reinterpret_cast<uint4*>(out + t * H)[v] = w;
  }
  __syncthreads();
  if (tid == 0) prof_end(prof);
}

}  // namespace

cudaError_t launch_combine_stock(const uint16_t* y_sorted, const uint32_t* inv_order,
                                 const float* scores, const uint16_t* shared,
                                 const uint16_t* gate_logit, int64_t T, int top_k, int64_t H,
                                 uint16_t* out, int* d_status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (T > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const int64_t slices = (H / 8 + kThreads - 1) / kThreads;
  if (slices > 65535) return cudaErrorInvalidValue;
  LaunchTimer timer("combine", stream);
  const dim3 grid(static_cast<unsigned>(T), static_cast<unsigned>(slices));
  if (launch_pdl(combine_stock_kernel, grid, dim3(kThreads), 0, stream, y_sorted, inv_order, scores,
                 shared, gate_logit, T, top_k, H, out, d_status, timer.slot()) != cudaSuccess)
    return cudaGetLastError();
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* y_sorted, const uint32_t* inv_order,
                           const float* scores, const uint16_t* shared, const uint16_t* x,
                           const uint16_t* w_sg, int64_t T, int top_k, int64_t H, uint16_t* out,
                           int* d_status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (T > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const int64_t slices = (H / 8 + kThreads - 1) / kThreads;
  if (slices > 65535) return cudaErrorInvalidValue;
  LaunchTimer timer("combine", stream);
  const dim3 grid(static_cast<unsigned>(T), static_cast<unsigned>(slices));
  if (launch_pdl(combine_kernel, grid, dim3(kThreads), 0, stream, y_sorted, inv_order, scores, shared,
                 x, w_sg, T, top_k, H, out, d_status, timer.slot()) != cudaSuccess)
    return cudaGetLastError();
  count_launch();
  return cudaGetLastError();
}

}  // namespace qmoe
