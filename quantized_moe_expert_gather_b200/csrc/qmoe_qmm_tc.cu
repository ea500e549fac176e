// Tensor-core gathered quantised matmul for many rows per expert (prefill).
//
// MLX PR #4567 "[Metal] Gather mm improvement", Proposed changes: rows are sorted by
// expert and cut into expert-aligned tiles (row start, expert, valid rows), so every
// tile runs one K loop against one expert's weights.  Each tile of 128 expert-sorted
// activation rows is multiplied by dequantize(W[e])^T (nuvec-core 0.4.0
// tests/quantized.rs, gather_qmm_selects_batches) on the 5th-generation tensor cores;
// with two weight stacks the SwitchGLU epilogue h = silu(gate) * up is fused (MLX
// issue #4509 repro script, `moe`).
//
// One persistent CTA per SM walks a contiguous range of units (tile, block of output
// channels).  A unit owns two 128x128 fp32 accumulators in tensor memory: (up, gate)
// for the SwitchGLU, or two adjacent 128-channel blocks of one weight stack.  Warps:
//   0-3   epilogue: tcgen05.ld of the finished accumulators (one TMEM lane = one row),
//         silu*mul, bf16 stores to the routed rows;
//   4     producer: 2-D TMA of the activation tile (128 rows x 64 k, 128B-swizzled)
//         for every k stage; every 128/(8*bits) k stages, 128 bytes of packed codes of
//         each of the 128 rows per stack (128B-swizzled, own two-slot ring); every 8
//         groups, the scales and biases;
//   5     MMA issuer: owns 512 TMEM columns (two double-buffered unit accumulators),
//         one elected lane issues tcgen05.mma kind::f16 (M=128, N=256, K=16) and
//         commits to mbarriers;
//   6-13  dequant: one thread per (stack, row) turns 64 packed codes into bf16
//         q*scale + bias (one rounding) and writes them in the 128B-swizzled K-major
//         layout the MMA descriptors read.
// Every mbarrier wait is bounded; a timeout sets QMOE_DEV_TIMEOUT, stops all roles,
// drains the copies and MMAs in flight and frees the tensor memory.
#include <algorithm>
#include <cudaTypedefs.h>
#include <mutex>

#include "qmoe_common.cuh"
#include "qmoe_internal.h"
#include "qmoe_tcgen05.cuh"
#include "qmoe_tma.h"

namespace qmoe {
namespace {

constexpr int kBM = 128;            // rows per tile = TMEM lanes
constexpr int kBN = 128;            // output channels per accumulator
constexpr int kBK = 64;             // k per stage: one 128-byte swizzle atom of bf16
constexpr int kEpiWarps = 4, kProdWarp = 4, kMmaWarp = 5, kDqWarp0 = 6, kDqWarps = 8;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;  // 448
constexpr int kTmemCols = 512;      // 2 buffers x 2 accumulators x 128 columns
constexpr int kSbGroups = 8;        // groups per scale/bias TMA box (16 bytes of bf16)

template <int BITS>
struct TcCfg {
#ifndef QMOE_TC_S1_4BIT
#define QMOE_TC_S1_4BIT 5
#define QMOE_TC_S2_4BIT 2
#endif
  // BITS == 16: unquantized bf16 weights, copied by TMA straight into the weight ring
  // (no packed codes, scales or dequant warps); that ring takes their space.
  static constexpr bool WBF16 = BITS == 16;
  static constexpr int S1 = BITS == 4 ? QMOE_TC_S1_4BIT : (WBF16 ? 5 : 4);  // activation ring
  static constexpr int S2 = BITS == 4 ? QMOE_TC_S2_4BIT : (WBF16 ? 4 : 2);  // weight ring
  static constexpr int A_BYTES = kBM * kBK * 2;                  // 16 KB
  static constexpr int P_ROW = kBK * BITS / 8;                   // packed bytes per row per stage
  static constexpr int PK = WBF16 ? 1 : 128 / P_ROW;             // stages per packed-code load
  static constexpr int SP = WBF16 ? 0 : 2;                       // packed-code ring
  static constexpr int P_SLOT = 2 * kBM * 128;                   // two stacks, 128 B per row
  static constexpr int B_BYTES = 2 * kBN * kBK * 2;              // two stacks, bf16
  static constexpr int SB_BYTES = WBF16 ? 0 : 2 * 2 * kBM * kSbGroups * 2;  // [stack][s|b][row][8]
  static constexpr int OFF_A = 0;
  static constexpr int OFF_P = OFF_A + S1 * A_BYTES;
  static constexpr int OFF_B = OFF_P + SP * P_SLOT;
  static constexpr int OFF_SB = OFF_B + S2 * B_BYTES;
  static constexpr int OFF_BAR = OFF_SB + 2 * SB_BYTES;
  static constexpr int SMEM = OFF_BAR + 256;
  static_assert(SMEM + 1024 <= 227 * 1024, "shared memory budget");
  static_assert(OFF_P % 1024 == 0 && OFF_B % 1024 == 0 && OFF_SB % 1024 == 0, "alignment");
};

struct alignas(64) TcParams {
  CUtensorMap tm_a;        // activation rows [x_rows, K] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tm_w[2];     // packed codes [E*N, K*bits/32] u32, box {32, 128}, 128B swizzle;
                           // bf16 weights [E*N, K], box {64, 128}, 128B swizzle
  CUtensorMap tm_sb[2][2]; // scales / biases [E*N, K/group] bf16, box {8, 128}
  uint16_t* y;
  const uint32_t* dst_row;
  const uint32_t* tiles;
  const uint32_t* num_tiles;
  int64_t dense_rows;
  int64_t N, K;
  int pair;                // 1: one stack, the two accumulators are adjacent channel blocks
  int sb_groups;           // > 0: a row has fewer than 8 groups; the unit's scales and
                           // biases ([128 rows][sb_groups] each) come by 1-D bulk copies
  const uint16_t* scales[2];
  const uint16_t* biases[2];
  int* d_status;
  ProfSlot* prof;
};

struct Tile {
  uint32_t row_start, expert, valid;
};

__device__ __forceinline__ Tile tc_tile(const TcParams& p, int64_t j) {
  Tile t;
  if (p.dense_rows > 0) {
    t.row_start = static_cast<uint32_t>(j * kBM);
    t.expert = 0;
    t.valid = static_cast<uint32_t>(imin64(kBM, p.dense_rows - j * kBM));
  } else {
    t.row_start = p.tiles[3 * j];
    t.expert = p.tiles[3 * j + 1];
    t.valid = min(p.tiles[3 * j + 2], static_cast<uint32_t>(kBM));
  }
  return t;
}

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, M=128,
// N=256: one MMA covers both weight tiles of a stage (they are contiguous in shared
// memory with the same 1024-byte 8-row stride) and both accumulators (adjacent TMEM
// columns).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (uint32_t((2 * kBN) >> 3) << 17) | (uint32_t(kBM >> 4) << 24);

__device__ __forceinline__ uint32_t bf16x2_of(float lo, float hi) { return pack_bf16x2(lo, hi); }

// 4 packed 8-bit codes -> 4 bf16 of q*s + b (fp32 fma, then one rounding to bf16).
__device__ __forceinline__ uint2 dequant_word8(uint32_t w, float s, float b) {
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t f = prmt(w, 0x4B000000u, k | (4 << 4) | (4 << 8) | (7 << 12));  // 2^23 + q
    const float q = __uint_as_float(f) - 8388608.0f;
    v[k] = fmaf(q, s, b);
  }
  return make_uint2(bf16x2_of(v[0], v[1]), bf16x2_of(v[2], v[3]));
}

template <int BITS, int GS, bool SB_WHOLE>
__global__ void __launch_bounds__(kThreads, 1) qmm_tc_kernel(const __grid_constant__ TcParams p) {
  using C = TcCfg<BITS>;
  constexpr int kS1 = C::S1;
  constexpr int kS2 = C::S2;
  // stages covered by one scale/bias box of kSbGroups groups
  constexpr int KS_SB_BOX = kSbGroups * GS / kBK;
  static_assert(KS_SB_BOX >= 1 && (kSbGroups * GS) % kBK == 0, "group size");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full1 = bars;                 // [kS1] TMA tx (activation + packed)
  uint64_t* empty1 = full1 + kS1;         // [kS1] MMA commit + dequant warps
  uint64_t* full2 = empty1 + kS1;         // [kS2] dequant warps
  uint64_t* empty2 = full2 + kS2;         // [kS2] MMA commit
  uint64_t* full_sb = empty2 + kS2;       // [2] TMA tx
  uint64_t* empty_sb = full_sb + 2;       // [2] dequant warps
  uint64_t* tfull = empty_sb + 2;         // [2] MMA commit: accumulator ready
  uint64_t* tempty = tfull + 2;           // [2] epilogue warps: accumulator drained
  uint64_t* drain = tempty + 2;           // [1] final MMA commit on the abort path
  uint64_t* fullP = drain + 1;            // [SP] TMA tx (packed codes)
  uint64_t* emptyP = fullP + C::SP;       // [SP] dequant warps
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(emptyP + C::SP);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS1; ++s) {
      mbar_init(&full1[s], 1);
      mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < C::SP; ++s) {
      mbar_init(&fullP[s], 1);
      mbar_init(&emptyP[s], kDqWarps);
    }
    for (int s = 0; s < kS2; ++s) {
      mbar_init(&full2[s], C::WBF16 ? 1 : kDqWarps);  // TMA tx, or the dequant warps
      mbar_init(&empty2[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full_sb[s], 1);
      mbar_init(&empty_sb[s], kDqWarps);
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_sh;
  // inputs (tile table, activations) may come from the kernel before this one
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(p.prof);

  const int64_t KS = p.K / kBK;  // k stages per unit
  // Scale/bias window: one box of 8 groups (KS_SB_BOX stages), or the whole row when it
  // has fewer groups.  Only compile-time divisors appear in the per-stage tests.
  constexpr bool sb_whole = SB_WHOLE;  // p.sb_groups > 0
  const int sb_stride = sb_whole ? p.sb_groups : kSbGroups;  // groups per smem row
  auto sb_first = [&](int64_t ks) { return sb_whole ? ks == 0 : ks % KS_SB_BOX == 0; };
  auto sb_last = [&](int64_t ks) {
    return ks == KS - 1 || (!sb_whole && ks % KS_SB_BOX == KS_SB_BOX - 1);
  };
  const int unit_n = p.pair ? 2 * kBN : kBN;
  const int64_t NBLK = (p.N + unit_n - 1) / unit_n;
  const int64_t ntiles = p.dense_rows > 0 ? (p.dense_rows + kBM - 1) / kBM : *p.num_tiles;
  // Units are dealt round-robin: at any moment the CTAs work on consecutive units, so
  // the channel blocks of one activation tile (and the tiles of one expert) run
  // concurrently and share their operands through L2.
  const int64_t units = ntiles * NBLK;
  const int64_t u_begin = blockIdx.x, u_step = gridDim.x;
  const int64_t u_end = units;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_a);
      uint32_t it = 0, sbit = 0, pbit = 0;
      bool ab = false;
      for (int64_t u = u_begin; u < u_end && !ab; u += u_step) {
        const Tile tl = tc_tile(p, u / NBLK);
        const int64_t n0 = (u % NBLK) * unit_n;
        const int64_t wrow = static_cast<int64_t>(tl.expert) * p.N + n0;
        for (int64_t ks = 0; ks < KS; ++ks) {
          if (*abort_flag) { ab = true; break; }
          if constexpr (C::WBF16) {
            // bf16 weight tiles, 128 rows x 64 k per stack, straight into the weight ring
            const uint32_t s2 = it % kS2;
            if (!mbar_wait<false>(&empty2[s2], ((it / kS2) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
            mbar_arrive_expect_tx(&full2[s2], C::B_BYTES);
#pragma unroll
            for (int m = 0; m < 2; ++m)
              tma_load_2d(smem + C::OFF_B + s2 * C::B_BYTES + m * kBN * kBK * 2, &p.tm_w[m],
                          &full2[s2], static_cast<int32_t>(ks * kBK),
                          static_cast<int32_t>(wrow + (p.pair ? kBN * m : 0)));
          } else {
            if (sb_first(ks)) {
              const uint32_t e = sbit & 1;
              if (!mbar_wait<false>(&empty_sb[e], ((sbit >> 1) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
              if constexpr (SB_WHOLE) {
                // rows wrow.. of one stack are contiguous: [128 rows][sb_groups] per array
                const uint32_t bytes = kBM * p.sb_groups * 2;
                mbar_arrive_expect_tx(&full_sb[e], 4 * bytes);
  #pragma unroll
                for (int m = 0; m < 2; ++m) {
                  const int64_t r0 = wrow + (p.pair ? kBN * m : 0);
  #pragma unroll
                  for (int arr = 0; arr < 2; ++arr)
                    bulk_load(smem + C::OFF_SB + e * C::SB_BYTES + (m * 2 + arr) * kBM * kSbGroups * 2,
                              (arr ? p.biases[m] : p.scales[m]) + r0 * p.sb_groups, bytes, &full_sb[e]);
                }
              } else {
                mbar_arrive_expect_tx(&full_sb[e], C::SB_BYTES);
                const int32_t gx = static_cast<int32_t>(ks * kBK / GS);
  #pragma unroll
                for (int m = 0; m < 2; ++m)
  #pragma unroll
                  for (int arr = 0; arr < 2; ++arr)
                    tma_load_2d(smem + C::OFF_SB + e * C::SB_BYTES + (m * 2 + arr) * kBM * kSbGroups * 2,
                                &p.tm_sb[m][arr], &full_sb[e], gx,
                                static_cast<int32_t>(wrow + (p.pair ? kBN * m : 0)));
              }
              ++sbit;
            }
            if (ks % C::PK == 0) {
              // packed codes of the next PK stages: 128 bytes of each row, 128B-swizzled
              const uint32_t ps = pbit % C::SP;
              if (!mbar_wait<false>(&emptyP[ps], ((pbit / C::SP) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
              mbar_arrive_expect_tx(&fullP[ps], C::P_SLOT);
  #pragma unroll
              for (int m = 0; m < 2; ++m)
                tma_load_2d(smem + C::OFF_P + ps * C::P_SLOT + m * kBM * 128, &p.tm_w[m], &fullP[ps],
                            static_cast<int32_t>(ks * kBK * BITS / 32),
                            static_cast<int32_t>(wrow + (p.pair ? kBN * m : 0)));
              ++pbit;
            }
          }
          const uint32_t s1 = it % kS1;
          if (!mbar_wait<false>(&empty1[s1], ((it / kS1) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
          mbar_arrive_expect_tx(&full1[s1], C::A_BYTES);
          tma_load_2d(smem + C::OFF_A + s1 * C::A_BYTES, &p.tm_a, &full1[s1],
                      static_cast<int32_t>(ks * kBK), static_cast<int32_t>(tl.row_start));
          ++it;
        }
      }
      if (ab) {
        // let the copies already issued land before the CTA can exit
        const uint32_t first = it > static_cast<uint32_t>(kS1) ? it - kS1 : 0u;
        for (uint32_t k = first; k < it; ++k) mbar_wait<false>(&full1[k % kS1], (k / kS1) & 1, nullptr);
        const uint32_t sfirst = sbit > 2u ? sbit - 2 : 0u;
        for (uint32_t k = sfirst; k < sbit; ++k) mbar_wait<false>(&full_sb[k & 1], (k >> 1) & 1, nullptr);
        if constexpr (C::WBF16) {
          const uint32_t bfirst = it > static_cast<uint32_t>(kS2) ? it - kS2 : 0u;
          for (uint32_t k = bfirst; k < it; ++k) mbar_wait<false>(&full2[k % kS2], (k / kS2) & 1, nullptr);
        } else {
          const uint32_t pfirst = pbit > static_cast<uint32_t>(C::SP) ? pbit - C::SP : 0u;
          for (uint32_t k = pfirst; k < pbit; ++k)
            mbar_wait<false>(&fullP[k % C::SP], (k / C::SP) & 1, nullptr);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp walks the loop, so that addresses and descriptors stay
    // warp-uniform; lane 0 waits and one elected lane (the same one throughout)
    // issues the MMAs and the commits that track them.
    uint32_t it = 0, tc = 0;
    bool issued = false;
    int ok = 1;
    for (int64_t u = u_begin; u < u_end; u += u_step, ++tc) {
      const uint32_t buf = tc & 1;
      if (lane == 0) ok = !*abort_flag && mbar_wait<false>(&tempty[buf], ((tc >> 1) & 1) ^ 1, p.d_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d0 = tmem_base + buf * (2 * kBN);
      for (int64_t ks = 0; ks < KS; ++ks, ++it) {
        const uint32_t s1 = it % kS1, s2 = it % kS2;
        if (lane == 0)
          ok = mbar_wait<false>(&full1[s1], (it / kS1) & 1, p.d_status) &&
               mbar_wait<false>(&full2[s2], (it / kS2) & 1, p.d_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = sw128_desc(smem + C::OFF_A + s1 * C::A_BYTES);
        const uint64_t b0 = sw128_desc(smem + C::OFF_B + s2 * C::B_BYTES);  // both stacks' tiles
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)  // +32 bytes along k per step
            tc_mma(d0, a0 + 2 * kk, b0 + 2 * kk, kIdesc, (ks | kk) != 0 ? 1u : 0u);
          tc_commit(&empty1[s1]);
          tc_commit(&empty2[s2]);
        }
        __syncwarp();
        issued = true;
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&tfull[buf]);
      __syncwarp();
    }
    __syncwarp();
    const bool leader = elect_one();
    if (leader && issued && *abort_flag) {
      tc_commit(drain);  // completes when every MMA issued so far has finished
      mbar_wait<false>(drain, 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0) {
    if constexpr (!C::WBF16) {  // bf16 weights arrive by TMA: nothing to dequantise
      // ------------------------------------------------------------------- dequant
      // Thread dq handles half-rows hr = dq and dq + 256 of the 512 (stack, row, half)
      // half-rows of a stage: consecutive lanes read consecutive 16-byte pieces of the
      // packed tile and write distinct swizzled 16-byte chunks (no bank conflicts).
      const int dq = threadIdx.x - kDqWarp0 * 32;  // 0..255
      constexpr int HALF = C::P_ROW / 2;           // packed bytes per half-row: 16 or 32
      uint32_t it = 0, sbit = 0, pbit = 0;
      for (int64_t u = u_begin; u < u_end; u += u_step) {
        for (int64_t ks = 0; ks < KS; ++ks, ++it) {
          if (*abort_flag) break;
          const uint32_t e = sbit & 1;
          if (sb_first(ks) &&
              !mbar_wait<false>(&full_sb[e], (sbit >> 1) & 1, p.d_status)) { *abort_flag = 1; break; }
          const uint32_t ps = pbit % C::SP, s2 = it % kS2;
          if (ks % C::PK == 0 &&
              !mbar_wait<false>(&fullP[ps], (pbit / C::SP) & 1, p.d_status)) { *abort_flag = 1; break; }
          if (!mbar_wait<false>(&empty2[s2], ((it / kS2) & 1) ^ 1, p.d_status)) { *abort_flag = 1; break; }
          const int pj = static_cast<int>(ks % C::PK);  // stage inside the packed rows
          const int gin = sb_whole ? static_cast<int>(ks * kBK / GS)
                                   : static_cast<int>((ks * kBK / GS) % kSbGroups);
#pragma unroll
          for (int rep = 0; rep < 2; ++rep) {
            const int hr = dq + 256 * rep;          // (stack, row, half)
            const int m = hr / (2 * kBM), row = (hr / 2) % kBM, half = hr & 1;
            const uint16_t* sbp = reinterpret_cast<const uint16_t*>(smem + C::OFF_SB + e * C::SB_BYTES) +
                                  (m * 2) * kBM * kSbGroups + row * sb_stride;
            const uint16_t* bbp = sbp + kBM * kSbGroups;
            // packed row: 128 bytes, 16-byte chunk c stored at chunk c ^ (row & 7)
            const uint8_t* prow = smem + C::OFF_P + ps * C::P_SLOT + (m * kBM + row) * 128;
            const int pc = (pj * C::P_ROW + half * HALF) / 16;  // first chunk of this half-row
            uint8_t* brow = smem + C::OFF_B + s2 * C::B_BYTES + (m * kBN + row) * (kBK * 2);
            // codes 32*half .. 32*half+31 of this row's 64
            const int gj = gin + (GS == 32 ? half : 0);
            if constexpr (BITS == 4) {
              const uint4 pw = *reinterpret_cast<const uint4*>(prow + ((pc ^ (row & 7)) << 4));
              const uint32_t w[4] = {pw.x, pw.y, pw.z, pw.w};
              const uint16_t sv = sbp[gj], bv = bbp[gj];
              const __nv_bfloat162 s2v = __halves2bfloat162(__ushort_as_bfloat16(sv), __ushort_as_bfloat16(sv));
              const __nv_bfloat162 b2v = __halves2bfloat162(__ushort_as_bfloat16(bv), __ushort_as_bfloat16(bv));
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int c = 4 * half + j;             // 16-byte chunk = codes 8c .. 8c+7
                *reinterpret_cast<uint4*>(brow + ((c ^ (row & 7)) << 4)) = dequant_word4(w[j], s2v, b2v);
              }
            } else {
              const uint4 pa = *reinterpret_cast<const uint4*>(prow + ((pc ^ (row & 7)) << 4));
              const uint4 pb = *reinterpret_cast<const uint4*>(prow + (((pc + 1) ^ (row & 7)) << 4));
              const uint32_t w[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
              const float sv = bf16_to_f32(sbp[gj]), bv = bf16_to_f32(bbp[gj]);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int c = 4 * half + j;             // two 8-bit words per chunk
                const uint2 a = dequant_word8(w[2 * j], sv, bv);
                const uint2 b = dequant_word8(w[2 * j + 1], sv, bv);
                *reinterpret_cast<uint4*>(brow + ((c ^ (row & 7)) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
              }
            }
          }
          fence_proxy_async_smem();  // make the generic-proxy writes visible to the MMA
          __syncwarp();
          const bool p_done = ks % C::PK == C::PK - 1 || ks == KS - 1;
          if (lane == 0) {
            mbar_arrive(&full2[s2]);
            if (p_done) mbar_arrive(&emptyP[ps]);
            if (sb_last(ks)) mbar_arrive(&empty_sb[e]);
          }
          if (p_done) ++pbit;
          if (sb_last(ks)) ++sbit;
        }
        if (*abort_flag) break;
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    const int row = warp * 32 + lane;  // TMEM lane
    uint32_t tc = 0;
    for (int64_t u = u_begin; u < u_end; u += u_step, ++tc) {
      if (*abort_flag) break;
      const uint32_t buf = tc & 1;
      if (!mbar_wait<false>(&tfull[buf], (tc >> 1) & 1, p.d_status)) { *abort_flag = 1; break; }
      tc_fence_after();
      const Tile tl = tc_tile(p, u / NBLK);
      const int64_t n0 = (u % NBLK) * unit_n;
      const bool valid = static_cast<uint32_t>(row) < tl.valid;
      uint16_t* yrow = nullptr;
      if (valid) {
        const uint32_t pos = tl.row_start + row;
        const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
        yrow = p.y + static_cast<int64_t>(dr) * p.N;
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + buf * (2 * kBN);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        float v0[32], v1[32];
        tmem_ld32(tbase + c * 32, v0);
        tmem_ld32(tbase + kBN + c * 32, v1);
        if (!valid) continue;
        if (p.pair) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int64_t nb = n0 + half * kBN + c * 32;
            const float* v = half ? v1 : v0;
            if (nb + 32 <= p.N && (p.N & 7) == 0) {  // 16-byte aligned row segments
              uint4* dst = reinterpret_cast<uint4*>(yrow + nb);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(bf16x2_of(v[8 * q], v[8 * q + 1]), bf16x2_of(v[8 * q + 2], v[8 * q + 3]),
                                    bf16x2_of(v[8 * q + 4], v[8 * q + 5]), bf16x2_of(v[8 * q + 6], v[8 * q + 7]));
            } else {
              for (int i = 0; i < 32 && nb + i < p.N; ++i) yrow[nb + i] = f32_to_bf16(v[i]);
            }
          }
        } else {
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = v0[i] * v1[i] * __frcp_rn(1.0f + __expf(-v1[i]));  // up * silu(gate)
          const int64_t nb = n0 + c * 32;
          if (nb + 32 <= p.N && (p.N & 7) == 0) {  // 16-byte aligned row segments
            uint4* dst = reinterpret_cast<uint4*>(yrow + nb);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(bf16x2_of(h[8 * q], h[8 * q + 1]), bf16x2_of(h[8 * q + 2], h[8 * q + 3]),
                                  bf16x2_of(h[8 * q + 4], h[8 * q + 5]), bf16x2_of(h[8 * q + 6], h[8 * q + 7]));
          } else {
            for (int i = 0; i < 32 && nb + i < p.N; ++i) yrow[nb + i] = f32_to_bf16(h[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }

  // ------------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) prof_end(p.prof);
}

template <int BITS, int GS, bool SB_WHOLE>
cudaError_t launch_tc_sb(TcParams prm, cudaStream_t stream) {
  using C = TcCfg<BITS>;
  auto kern = qmm_tc_kernel<BITS, GS, SB_WHOLE>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchTimer timer(prm.pair ? "tc" : "tc_glu", stream);
  prm.prof = timer.slot();
  cudaError_t le = launch_pdl(kern, dim3(sm_count()), dim3(kThreads), C::SMEM + 1024, stream, prm);
  if (le != cudaSuccess) return le;
  count_launch();
  return cudaGetLastError();
}

template <int BITS, int GS>
cudaError_t launch_tc(const TcParams& prm, cudaStream_t stream) {
  return prm.sb_groups > 0 ? launch_tc_sb<BITS, GS, true>(prm, stream)
                           : launch_tc_sb<BITS, GS, false>(prm, stream);
}

}  // namespace

bool qmm_tc_supported(const GemmArgs& a) {
  if (a.bits == 16) return a.K % kBK == 0 && a.x_rows > 0;  // unquantized bf16 weights
  if (a.bits != 4 && a.bits != 8) return false;
  if (a.K % kBK != 0) return false;
  const int64_t gpr = a.K / a.group;
  // scale/bias rows: a 16-byte pitch for the 2-D boxes, or fewer than 8 groups with
  // whole units (128 channels of each of two stacks, or 256 of one), so that every
  // bulk copy of a unit's 128-row blocks stays inside the arrays
  const int64_t unit_n = a.nmat == 2 ? kBN : 2 * kBN;
  if (gpr % kSbGroups != 0 && !(gpr < kSbGroups && a.N % unit_n == 0)) return false;
  if (a.x_rows <= 0) return false;
  return true;
}

cudaError_t launch_qmm_tc(const GemmArgs& a, cudaStream_t stream) {
  if (!qmm_tc_supported(a)) return cudaErrorNotSupported;
  TcParams prm{};
  cudaError_t e = make_tmap_2d_bf16(&prm.tm_a, a.x, a.K, a.x_rows, kBK, kBM, /*swizzle128=*/true);
  if (e != cudaSuccess) return e;
  prm.pair = a.nmat == 2 ? 0 : 1;
  if (a.bits == 16) {
    // bf16 weights [E*N, K]: 128 rows x 64 k per box, 128B-swizzled like the
    // dequantised tiles
    for (int m = 0; m < 2; ++m) {
      const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
      e = make_tmap_2d_bf16(&prm.tm_w[m], wm.codes, a.K, a.E * a.N, kBK, kBM, /*swizzle128=*/true);
      if (e != cudaSuccess) return e;
    }
    prm.y = a.y;
    prm.dst_row = a.dst_row;
    prm.tiles = a.tiles;
    prm.num_tiles = a.num_tiles;
    prm.dense_rows = a.dense_rows;
    prm.N = a.N;
    prm.K = a.K;
    prm.d_status = a.d_status;
    return launch_tc_sb<16, 64, false>(prm, stream);
  }
  const int64_t words = a.K * a.bits / 32;
  const int64_t gpr = a.K / a.group;
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
    // 128 bytes of each row (several k stages) per copy, 128B-swizzled
    e = make_tmap_2d_u32(&prm.tm_w[m], wm.codes, words, a.E * a.N, 32, kBM,
                         /*swizzle128=*/true);
    if (e != cudaSuccess) return e;
    prm.scales[m] = wm.scales;
    prm.biases[m] = wm.biases;
    if (gpr % kSbGroups == 0) {
      e = make_tmap_2d_bf16(&prm.tm_sb[m][0], wm.scales, gpr, a.E * a.N, kSbGroups, kBM, false);
      if (e != cudaSuccess) return e;
      e = make_tmap_2d_bf16(&prm.tm_sb[m][1], wm.biases, gpr, a.E * a.N, kSbGroups, kBM, false);
      if (e != cudaSuccess) return e;
    }
  }
  prm.sb_groups = gpr % kSbGroups == 0 ? 0 : static_cast<int>(gpr);
  prm.y = a.y;
  prm.dst_row = a.dst_row;
  prm.tiles = a.tiles;
  prm.num_tiles = a.num_tiles;
  prm.dense_rows = a.dense_rows;
  prm.N = a.N;
  prm.K = a.K;
  prm.d_status = a.d_status;
  if (a.bits == 4) {
    if (a.group == 32) return launch_tc<4, 32>(prm, stream);
    if (a.group == 64) return launch_tc<4, 64>(prm, stream);
    return launch_tc<4, 128>(prm, stream);
  }
  if (a.group == 32) return launch_tc<8, 32>(prm, stream);
  if (a.group == 64) return launch_tc<8, 64>(prm, stream);
  return launch_tc<8, 128>(prm, stream);
}

}  // namespace qmoe
