// Device helpers shared by the qmoe kernels (sm_100a): bf16 bits, mbarriers with
// bounded waits, TMA / bulk / cp.async copies, warp-level MMA and status flags.
//
// Every wait in this library is bounded: a wait that runs out sets
// QMOE_DEV_TIMEOUT in the caller's status word and returns false, and the
// calling kernel then finishes without touching the data it was waiting for.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/qmoe.h"

namespace qmoe {

// ----------------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// Two floats -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ----------------------------------------------------------------- status word
__device__ __forceinline__ void set_status(int* d_status, int bits) {
  if (d_status != nullptr) atomicOr(d_status, bits);
}

// -------------------------------------------------------------- launch timing
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Call from one thread per CTA at its start / after its last work.
template <typename Slot>
__device__ __forceinline__ void prof_start(Slot* p) {
  if (p != nullptr) atomicMax(&p->start_inv, ~global_ns());
}
template <typename Slot>
__device__ __forceinline__ void prof_end(Slot* p) {
  if (p != nullptr) atomicMax(&p->end, global_ns());
}

// --------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while the kernel
// before it on the stream is still running.  griddep_wait() blocks until that kernel has
// completed and its memory is visible; every read of inputs another kernel produced
// comes after it (it is a no-op for ordinary launches).  griddep_launch_dependents()
// lets the next kernel start its own prologue once every CTA of this grid has issued it.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------- mbarriers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
// Makes mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// One test of the phase.  With kSuspend the thread may be suspended until the phase
// completes or for up to kWaitHintNs, so a waiting warp does not keep issuing while it
// waits; without it the test returns at once.  Measured per kernel: suspending helps the
// tensor-memory prefill kernel (T=4123 layer 0.432 -> 0.407 ms) and costs the kernel with
// shared-memory weight tiles (T=4096 layer 0.551 -> 0.585 ms), which therefore tests
// without it.
constexpr uint32_t kWaitHintNs = 1000;
template <bool kSuspend = true>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  if constexpr (kSuspend) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
  }
  return ok != 0;
}

// Spin limit for every mbarrier wait: about a second with the back-off below (up to a few
// seconds when every test is suspended for its full hint).
constexpr uint32_t kWaitSpins = 1u << 22;

// Waits until the phase of `bar` with parity `parity` has completed.  Returns
// false (and flags QMOE_DEV_TIMEOUT) if it did not complete within the limit.
template <bool kSuspend = true>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* d_status) {
  for (uint32_t i = 0; i < kWaitSpins; ++i) {
    if (mbar_try_wait<kSuspend>(bar, parity)) return true;
    if (i > 64) __nanosleep(i > 4096 ? 256 : 32);
  }
  set_status(d_status, QMOE_DEV_TIMEOUT);
  return false;
}

// ---------------------------------------------------------------------- copies
// 2-D TMA tile load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// 3-D TMA tile load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
// 1-D bulk copy (no multicast) of `bytes` contiguous bytes global -> shared, completing
// on `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 2-D TMA tile store from shared memory (after fence_proxy_async_smem of the writes),
// tracked by the issuing thread's bulk groups.  Coordinates are never negative.
__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* src, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(x), "r"(y), "r"(smem_u32(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The issuing thread's committed bulk stores have read their shared-memory sources.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// The issuing thread's committed bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
// Asynchronous global -> shared copies of 4, 8 or 16 bytes (both addresses
// aligned to the size).
template <int BYTES>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
  if constexpr (BYTES == 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
  } else {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "n"(BYTES)
                 : "memory");
  }
}
// Arrive on `bar` once every cp.async this thread issued so far has landed.  The
// arrival is not pre-counted (.noinc): the barrier's expected count includes it.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Read-only 16-byte global load that bypasses L1 allocation for streaming data.
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

// --------------------------------------------------------------------- barriers
// Named barrier ID (an immediate, so the compiler sees every barrier a kernel uses).
template <int ID>
__device__ __forceinline__ void named_bar_sync(int nthreads) {
  static_assert(ID > 0 && ID < 16, "named barrier id");
  asm volatile("bar.sync %0, %1;" ::"n"(ID), "r"(nthreads) : "memory");
}
// Named barrier that also returns, to every participant, whether any of them passed
// `pred` true: a decision all of them take together.
template <int ID>
__device__ __forceinline__ bool named_bar_any(int nthreads, bool pred) {
  static_assert(ID > 0 && ID < 16, "named barrier id");
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "n"(ID), "r"(nthreads)
      : "memory");
  return r != 0;
}

// --------------------------------------------------------------- warp-level MMA
// D = A(16x16, row) * B(16x8, col) + C, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// (v & mask) | magic in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t v, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(magic));
  return r;
}

}  // namespace qmoe
