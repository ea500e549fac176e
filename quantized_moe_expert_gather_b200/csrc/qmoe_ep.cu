// Expert-parallel dispatch packing: the rows a rank sends to the experts' owners.
//
// MTPLX PR #558 (Change): the sorted chain gathers the routed rows in expert order and
// keeps the inverse permutation to unsort the expert outputs in the combine.  With the
// experts partitioned contiguously over ranks (expert e on rank e / E_local), the rows in
// expert order are also grouped by owner rank, so one all-to-all of this buffer sends
// every row to its expert, and the same all-to-all in reverse brings the outputs back in
// expert order, ready for the one-pass combine.
//
//   x_send[p] = x[order[p] / top_k]           (the activation row of sorted routed row p)
//   e_send[p] = indices[order[p]] mod E_local  (its expert, numbered on the owner rank)
//
// Bandwidth-bound copy: 16-byte vectors, a grid of several CTAs per SM.
#include <algorithm>

#include "qmoe_common.cuh"
#include "qmoe_internal.h"

namespace qmoe {
namespace {

__global__ void ep_pack_kernel(const uint16_t* __restrict__ x, int64_t H, int top_k,
                               const uint32_t* __restrict__ indices,
                               const uint32_t* __restrict__ order, int64_t R, int64_t T,
                               int64_t E_local, uint16_t* __restrict__ x_send,
                               uint32_t* __restrict__ e_send, int* d_status) {
  griddep_wait();  // order comes from the expert sort before this kernel
  griddep_launch_dependents();
  const int64_t vec_per_row = H / 8;
  const int64_t n = R * vec_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t p = i / vec_per_row, v = i % vec_per_row;
    const uint32_t r = order[p];
    const int64_t t = r / static_cast<uint32_t>(top_k);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t < T) {
      val = reinterpret_cast<const uint4*>(x + t * H)[v];
    } else if (v == 0) {
      set_status(d_status, QMOE_DEV_BAD_INDEX);
    }
    reinterpret_cast<uint4*>(x_send + p * H)[v] = val;
    if (v == 0) e_send[p] = t < T ? indices[r] % static_cast<uint32_t>(E_local) : 0u;
  }
}

}  // namespace
}  // namespace qmoe

extern "C" int qmoe_ep_pack(const qmoe_bf16* x, int64_t T, int64_t H, int top_k,
                            const uint32_t* indices, const uint32_t* order, int64_t E_local,
                            qmoe_bf16* x_send, uint32_t* e_send, int* d_status,
                            qmoe_stream stream) {
  using namespace qmoe;
  if (T < 0 || H <= 0 || top_k <= 0 || E_local <= 0) return QMOE_ERR_ARG;
  if (H % 8 != 0) return QMOE_ERR_UNSUPPORTED;
  const int64_t R = T * top_k;
  if (R == 0) return QMOE_OK;
  if (!x || !indices || !order || !x_send || !e_send) return QMOE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_send) & 15u))
    return QMOE_ERR_ARG;
  const int threads = 256;
  const int64_t n = R * (H / 8);
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 148 * 8);
  auto s = static_cast<cudaStream_t>(stream);
  if (launch_pdl(ep_pack_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s, x, H,
                 top_k, indices, order, R, T, E_local, x_send, e_send, d_status) != cudaSuccess)
    return QMOE_ERR_CUDA;
  count_launch();
  return cudaGetLastError() == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA;
}
