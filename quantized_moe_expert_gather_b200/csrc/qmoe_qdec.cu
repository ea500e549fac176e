// Tensor-core streaming gathered quantised matmul for few rows per expert (decode).
//
// The product of the mma.sync streaming kernel (qmoe_qmv.cu) -- for every expert-aligned
// tile of <= 16 routed rows (MLX PR #4567 "[Metal] Gather mm improvement", Proposed
// changes) and every block of output channels, y[row, n] = x[row] . dequantize(W[e])[n]^T
// (nuvec-core 0.4.0 tests/quantized.rs, gather_qmm_selects_batches), with the SwitchGLU
// epilogue h = silu(gate) * up for two weight stacks (MLX issue #4509 repro script, `moe`)
// -- computed with the roles of the tensor-core prefill kernel swapped: the weights are
// the 128-row A operand, dequantised to bf16 (q*s + b, one rounding) straight into tensor
// memory, and the tile's (up to) 16 activation rows are the N = 16 B operand.  The
// compute warps then run independent streams of code unpacking and bf16x2 FMAs; the MMAs
// and their accumulation are the tensor core's.
//
// One persistent CTA per SM walks a contiguous range of units.  A unit is 128 weight rows:
// 64 channels of both stacks (rows 0..63 of the first, 64..127 of the second) or 128
// channels of one stack.  Warps:
//   0-3   epilogue: tcgen05.ld of the unit's 128 x 16 fp32 accumulator (one TMEM lane per
//         weight row), silu*mul through shared memory, bf16 stores of the valid rows;
//   4     producer: per 256-k stage, TMA of the packed codes (two boxes of 64 rows x 128 B,
//         128B-swizzled) and of the activation tile (four boxes of 16 rows x 64 k,
//         128B-swizzled, the K-major layout the MMA reads); scale/bias boxes (64 rows x 8
//         groups per stack) every 8 groups;
//   5     MMA issuer: tcgen05.mma kind::f16, A from tensor memory, M=128 N=16 K=16;
//   6-13  dequant: warp w owns the weight rows of TMEM lane quarter w%4 and one slice of
//         each stage's k (half of it with 8 dequant warps, a quarter with 16); one weight
//         row per thread.
//
// Measured on B200 (decode layer, hidden 4096, intermediate 2048, 288 experts, top-8):
// 2.5 TB/s for the fused up/gate launch against 3.1 TB/s for the mma.sync kernel, which
// therefore stays the default; this kernel is selected with QMOE_DECODE=qdec.  The limit
// is the exact bf16 dequantisation (9 integer and 8 bf16x2 operations per packed word),
// which the compute warps all run at once after each stage lands, saturating the integer
// pipe in bursts.  The mma.sync kernel instead scales each group in fp32 after its MMAs
// and spends 7 integer operations per word.
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

constexpr int kM = 128;                    // weight rows per unit = TMEM lanes = MMA M
constexpr int kNt = 16;                    // routed rows per tile = MMA N
constexpr int kKC = 256;                   // k per stage
constexpr int kRowBytes = kKC / 2;         // packed 4-bit bytes of one row per stage
constexpr int kCodeBytes = kM * kRowBytes;               // 16 KB: two 64-row boxes
constexpr int kXBytes = kNt * kKC * 2;                   // 8 KB: four 16-row x 64-k slabs
constexpr int kStageBytes = kCodeBytes + kXBytes;        // 24 KB
#ifndef QDEC_STAGES
#define QDEC_STAGES 6
#endif
#ifndef QDEC_SB_SLOTS
#define QDEC_SB_SLOTS 4
#endif
constexpr int kStages = QDEC_STAGES;
constexpr int kSbGroups = 8;                             // groups per scale/bias box
constexpr int kSbBytes = 2 * 2 * 64 * kSbGroups * 2;     // [box][s|b][64 rows][8] bf16
constexpr int kSbSlots = QDEC_SB_SLOTS;                  // scale/bias windows in flight
constexpr int kASlots = 3;                               // dequantised A tiles in TMEM
constexpr int kACols = kKC / 2;                          // TMEM columns per A tile
constexpr int kDCol0 = kASlots * kACols;                 // accumulators after the A tiles
constexpr int kTmemCols = 512;
#ifndef QDEC_DQ_WARPS
#define QDEC_DQ_WARPS 8
#endif
constexpr int kEpiWarps = 4, kProdWarp = 4, kMmaWarp = 5, kDqWarp0 = 6;
constexpr int kDqWarps = QDEC_DQ_WARPS;                  // 8 or 16
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kParts = kDqWarps / 4;                     // k slices of a stage, one per warp
constexpr int kPartK = kKC / kParts;                     // k per dequant thread and stage
constexpr int kPartWords = kPartK / 8;                   // packed words per thread and stage
static_assert(kDqWarps == 8 || kDqWarps == 16, "dequant warps");
constexpr int kOffSb = kStages * kStageBytes;            // 144 KB
constexpr int kOffXchg = kOffSb + kSbSlots * kSbBytes;          // second-stack values: [64][17] f32
constexpr int kXchgStride = kNt + 1;                     // padded: conflict-free columns
constexpr int kOffBar = kOffXchg + 64 * kXchgStride * 4;
constexpr int kSmem = kOffBar + 512;
static_assert(kDCol0 + 2 * kNt <= kTmemCols, "tensor memory budget");
static_assert(kSmem + 1024 <= 227 * 1024, "shared memory budget");
static_assert(kStageBytes % 1024 == 0 && kOffSb % 1024 == 0, "128B-swizzle boxes need 1 KB alignment");

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, M=128, N=16.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kNt >> 3) << 17) |
                            (uint32_t(kM >> 4) << 24);

struct alignas(64) QdecParams {
  CUtensorMap tm_w[2];      // packed codes [E*N, K/8] u32, box {32 words, 64 rows}, 128B swizzle
  CUtensorMap tm_sb[2][2];  // [box][scales|biases] [E*N, K/group] bf16, box {8, 64}
  CUtensorMap tm_x;         // activation rows [x_rows, K] bf16, box {64, 16}, 128B swizzle
  uint16_t* y;
  const uint32_t* dst_row;
  const uint32_t* tiles;
  const uint32_t* num_tiles;
  int64_t dense_rows;
  int64_t N, K;
  int pair;                 // 1: one stack, a unit is 128 of its channels
  int* d_status;
  ProfSlot* prof;
};

struct QTile {
  uint32_t row_start, expert, valid;
};

__device__ __forceinline__ QTile qdec_tile(const QdecParams& p, int64_t j) {
  QTile t;
  if (p.dense_rows > 0) {
    t.row_start = static_cast<uint32_t>(j * kNt);
    t.expert = 0;
    t.valid = static_cast<uint32_t>(imin64(kNt, p.dense_rows - j * kNt));
  } else {
    t.row_start = p.tiles[3 * j];
    t.expert = p.tiles[3 * j + 1];
    t.valid = min(p.tiles[3 * j + 2], static_cast<uint32_t>(kNt));
  }
  return t;
}

template <int GS>
__global__ void __launch_bounds__(kThreads, 1) qdec_kernel(const __grid_constant__ QdecParams p) {
  constexpr int KS_SB = kSbGroups * GS / kKC;  // stages per scale/bias window
  static_assert(KS_SB >= 1 && (kSbGroups * GS) % kKC == 0, "group size");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                    // [kStages] TMA tx (codes + activations)
  uint64_t* empty = full + kStages;         // [kStages] MMA commit + dequant warps
  uint64_t* full_sb = empty + kStages;      // [kSbSlots] TMA tx
  uint64_t* empty_sb = full_sb + kSbSlots;  // [kSbSlots] dequant warps
  uint64_t* a_full = empty_sb + kSbSlots;   // [kASlots] dequant warps: A tile written
  uint64_t* a_empty = a_full + kASlots;     // [kASlots] MMA commit: A tile read
  uint64_t* d_full = a_empty + kASlots;     // [2] MMA commit: accumulator ready
  uint64_t* d_empty = d_full + 2;           // [2] epilogue warps: accumulator drained
  uint64_t* drain = d_empty + 2;            // [1] final MMA commit on the abort path
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sh + 1);
  float* xchg = reinterpret_cast<float*>(smem + kOffXchg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kDqWarps);
    }
    for (int s = 0; s < kSbSlots; ++s) {
      mbar_init(&full_sb[s], 1);
      mbar_init(&empty_sb[s], kDqWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], kEpiWarps);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(&a_full[s], kDqWarps);
      mbar_init(&a_empty[s], 1);
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

  const int64_t KS = (p.K + kKC - 1) / kKC;  // stages per unit
  const int unit_n = p.pair ? kM : kM / 2;   // output channels per unit
  const int64_t NB = (p.N + unit_n - 1) / unit_n;
  const int64_t ntiles = p.dense_rows > 0 ? (p.dense_rows + kNt - 1) / kNt : *p.num_tiles;
  const int64_t units = ntiles * NB;
  const int64_t u_begin = units * blockIdx.x / gridDim.x;
  const int64_t u_end = units * (blockIdx.x + 1) / gridDim.x;
  // first weight row of box m (rows 0..63 and 64..127 of the unit)
  auto box_row = [&](const QTile& t, int64_t u, int m) -> int64_t {
    const int64_t n0 = (u % NB) * unit_n;
    return static_cast<int64_t>(t.expert) * p.N + n0 + (p.pair ? 64 * m : 0);
  };

  if (warp == kProdWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_x);
      tma_prefetch_desc(&p.tm_w[0]);
      tma_prefetch_desc(&p.tm_w[1]);
      uint32_t it = 0, sbit = 0;
      bool ab = false;
      int64_t cur = -1;
      QTile tl{};
      for (int64_t u = u_begin; u < u_end && !ab; ++u) {
        if (u / NB != cur) {
          cur = u / NB;
          tl = qdec_tile(p, cur);
        }
        const int64_t r0 = box_row(tl, u, 0), r1 = box_row(tl, u, 1);
        for (int64_t ks = 0; ks < KS; ++ks, ++it) {
          if (*abort_flag) { ab = true; break; }
          if (ks % KS_SB == 0) {
            const uint32_t e = sbit % kSbSlots;
            if (!mbar_wait(&empty_sb[e], ((sbit / kSbSlots) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
            mbar_arrive_expect_tx(&full_sb[e], kSbBytes);
            const int32_t gx = static_cast<int32_t>(ks * kKC / GS);
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
              for (int arr = 0; arr < 2; ++arr)
                tma_load_2d(smem + kOffSb + e * kSbBytes + (m * 2 + arr) * 64 * kSbGroups * 2,
                            &p.tm_sb[m][arr], &full_sb[e], gx,
                            static_cast<int32_t>(m ? r1 : r0));
            ++sbit;
          }
          const int st = static_cast<int>(it % kStages);
          if (!mbar_wait(&empty[st], ((it / kStages) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          uint8_t* sp = smem + st * kStageBytes;
#pragma unroll
          for (int m = 0; m < 2; ++m)
            tma_load_2d(sp + m * 64 * kRowBytes, &p.tm_w[m], &full[st],
                        static_cast<int32_t>(ks * kKC / 8), static_cast<int32_t>(m ? r1 : r0));
#pragma unroll
          for (int j = 0; j < kKC / 64; ++j)
            tma_load_2d(sp + kCodeBytes + j * kNt * 128, &p.tm_x, &full[st],
                        static_cast<int32_t>(ks * kKC + 64 * j), static_cast<int32_t>(tl.row_start));
        }
      }
      if (ab) {
        // let the copies already issued land before the CTA can exit
        const uint32_t first = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u;
        for (uint32_t k = first; k < it; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, nullptr);
        const uint32_t sfirst = sbit > static_cast<uint32_t>(kSbSlots) ? sbit - kSbSlots : 0u;
        for (uint32_t k = sfirst; k < sbit; ++k) mbar_wait(&full_sb[k % kSbSlots], (k / kSbSlots) & 1, nullptr);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp walks the loop, so that addresses and descriptors stay
    // warp-uniform; lane 0 waits and one elected lane (the same one throughout)
    // issues the MMAs and the commits that track them.
    uint32_t it = 0, tc = 0;
    bool issued = false;
    for (int64_t u = u_begin; u < u_end; ++u, ++tc) {
      const uint32_t buf = tc & 1;
      int ok = 0;
      if (lane == 0) ok = !*abort_flag && mbar_wait(&d_empty[buf], ((tc >> 1) & 1) ^ 1, p.d_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + kDCol0 + buf * kNt;
      for (int64_t ks = 0; ks < KS; ++ks, ++it) {
        const int st = static_cast<int>(it % kStages);
        const uint32_t as = it % kASlots;
        if (lane == 0)
          ok = mbar_wait(&full[st], (it / kStages) & 1, p.d_status) &&
               mbar_wait(&a_full[as], (it / kASlots) & 1, p.d_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t b0 = sw128_desc(smem + st * kStageBytes + kCodeBytes);
        const uint32_t a0 = tmem_base + as * kACols;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk) {
            // activation slab kk/4 (16 rows x 128 B), 32-byte k step inside the swizzle atom
            const uint64_t bdesc = b0 + (((kk / 4) * kNt * 128) >> 4) + 2 * (kk % 4);
            tc_mma_ts(d, a0 + kk * 8, bdesc, kIdesc, (ks | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[st]);
          tc_commit(&a_empty[as]);
        }
        __syncwarp();
        issued = true;
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&d_full[buf]);
      __syncwarp();
    }
    __syncwarp();
    const bool leader = elect_one();
    if (leader && issued && *abort_flag) {
      tc_commit(drain);  // completes when every MMA issued so far has finished
      mbar_wait(drain, 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------------- dequant
    // Warp w may only reach TMEM lanes 32*(w%4)..+31: it owns those weight rows, and
    // slice `part` of each stage's 256 k.
    const int quarter = warp % 4, part = (warp - kDqWarp0) / 4;
    const int r = quarter * 32 + lane;   // weight row of the unit = TMEM lane
    const int m = r / 64, rr = r % 64;   // code box and row inside it
    uint32_t it = 0, sbit = 0;
    for (int64_t u = u_begin; u < u_end; ++u) {
      for (int64_t ks = 0; ks < KS; ++ks, ++it) {
        if (*abort_flag) break;
        const uint32_t e = sbit % kSbSlots;
        if (ks % KS_SB == 0 &&
            !mbar_wait(&full_sb[e], (sbit / kSbSlots) & 1, p.d_status)) { *abort_flag = 1; break; }
        const int st = static_cast<int>(it % kStages);
        const uint32_t as = it % kASlots;
        if (!mbar_wait(&full[st], (it / kStages) & 1, p.d_status) ||
            !mbar_wait(&a_empty[as], ((it / kASlots) & 1) ^ 1, p.d_status)) { *abort_flag = 1; break; }
        tc_fence_after();
        // this row's 128 packed bytes of the stage; 16-byte chunk c sits at c ^ (rr & 7)
        const uint8_t* rowp = smem + st * kStageBytes + m * 64 * kRowBytes + rr * kRowBytes;
        const uint16_t* srow = reinterpret_cast<const uint16_t*>(smem + kOffSb + e * kSbBytes) +
                               (m * 2 * 64 + rr) * kSbGroups;
        const uint16_t* brow = srow + 64 * kSbGroups;
        // the slice's k fall in GPP groups (one when a group is wider than the slice),
        // the first at g0 of the scale window
        constexpr int GPP = kPartK >= GS ? kPartK / GS : 1;
        const int g0 = (static_cast<int>((ks * kKC) % (kSbGroups * GS)) + part * kPartK) / GS;
        __nv_bfloat162 s2[GPP], b2[GPP];
        load_group_pairs<GPP>(srow + g0, s2);
        load_group_pairs<GPP>(brow + g0, b2);
        uint32_t out[kPartWords * 4];
#pragma unroll
        for (int c = 0; c < kPartWords / 4; ++c) {
          const int chunk = (kPartWords / 4) * part + c;
          const uint4 pw = *reinterpret_cast<const uint4*>(rowp + ((chunk ^ (rr & 7)) << 4));
          const uint32_t w4[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            constexpr int kWordsPerGroup = GS / 8;
            const int gi = (4 * c + j) / kWordsPerGroup;
            const uint4 v = dequant_word4(w4[j], s2[gi], b2[gi]);
            out[(4 * c + j) * 4 + 0] = v.x;
            out[(4 * c + j) * 4 + 1] = v.y;
            out[(4 * c + j) * 4 + 2] = v.z;
            out[(4 * c + j) * 4 + 3] = v.w;
          }
        }
        // A tile: lane r, columns part*kPartK/2.. (two bf16 of consecutive k per column)
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               as * kACols + part * (kPartK / 2);
#pragma unroll
        for (int h = 0; h < kPartWords / 8; ++h) {
          uint32_t cols[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) cols[i] = out[32 * h + i];
          tmem_st32(taddr + 32 * h, cols);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        const bool sb_done = ks % KS_SB == KS_SB - 1 || ks == KS - 1;
        if (lane == 0) {
          mbar_arrive(&a_full[as]);
          mbar_arrive(&empty[st]);
          if (sb_done) mbar_arrive(&empty_sb[e]);
        }
        if (sb_done) ++sbit;
      }
      if (*abort_flag) break;
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    const int r = warp * 32 + lane;  // TMEM lane = weight row of the unit
    uint32_t tc = 0;
    int64_t cur = -1;
    QTile tl{};
    for (int64_t u = u_begin; u < u_end; ++u, ++tc) {
      const uint32_t buf = tc & 1;
      bool stop = *abort_flag || !mbar_wait(&d_full[buf], (tc >> 1) & 1, p.d_status);
      // the SwitchGLU path meets at a named barrier below: its warps stop together
      if (!p.pair) stop = named_bar_any<1>(kEpiWarps * 32, stop);
      if (stop) { *abort_flag = 1; break; }
      tc_fence_after();
      float v[kNt];
      tmem_ld16(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + kDCol0 + buf * kNt, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[buf]);  // the accumulator is in registers now
      if (u / NB != cur) {
        cur = u / NB;
        tl = qdec_tile(p, cur);
      }
      const int64_t n0 = (u % NB) * unit_n;
      if (!p.pair) {
        // rows 64..127 hold the second stack (gate): hand them to rows 0..63 (up)
        if (r >= 64) {
#pragma unroll
          for (int t = 0; t < kNt; ++t) xchg[(r - 64) * kXchgStride + t] = v[t];
        }
        named_bar_sync<1>(kEpiWarps * 32);
        if (r < 64 && n0 + r < p.N) {
#pragma unroll
          for (int t = 0; t < kNt; ++t) {
            if (static_cast<uint32_t>(t) < tl.valid) {
              const float gte = xchg[r * kXchgStride + t];
              const uint32_t pos = tl.row_start + t;
              const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
              p.y[static_cast<int64_t>(dr) * p.N + n0 + r] =
                  f32_to_bf16(v[t] * (gte / (1.0f + expf(-gte))));
            }
          }
        }
        named_bar_sync<1>(kEpiWarps * 32);  // before the next unit overwrites xchg
      } else if (n0 + r < p.N) {
#pragma unroll
        for (int t = 0; t < kNt; ++t) {
          if (static_cast<uint32_t>(t) < tl.valid) {
            const uint32_t pos = tl.row_start + t;
            const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
            p.y[static_cast<int64_t>(dr) * p.N + n0 + r] = f32_to_bf16(v[t]);
          }
        }
      }
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

template <int GS>
cudaError_t launch_qdec_gs(const QdecParams& prm, cudaStream_t stream) {
  auto kern = qdec_kernel<GS>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchTimer timer(prm.pair ? "qdec" : "qdec_glu", stream);
  QdecParams p = prm;
  p.prof = timer.slot();
  const cudaError_t e = launch_pdl(kern, dim3(sm_count()), dim3(kThreads), kSmem + 1024, stream, p);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool qdec_supported(const GemmArgs& a) {
  if (a.bits != 4 || (a.group != 32 && a.group != 64 && a.group != 128)) return false;
  if (a.K % 64 != 0) return false;                    // whole 64-k activation boxes
  if ((a.K / a.group) % kSbGroups != 0) return false;  // scale/bias rows: 16-byte pitch
  if (a.x_rows <= 0 || a.src_row != nullptr) return false;  // activations in tile order
  return true;
}

cudaError_t launch_qdec(const GemmArgs& a, cudaStream_t stream) {
  if (!qdec_supported(a)) return cudaErrorNotSupported;
  QdecParams prm{};
  cudaError_t e = make_tmap_2d_bf16(&prm.tm_x, a.x, a.K, a.x_rows, 64, kNt, /*swizzle128=*/true);
  if (e != cudaSuccess) return e;
  const int64_t words = a.K / 8;
  const int64_t gpr = a.K / a.group;
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
    e = make_tmap_2d_u32(&prm.tm_w[m], wm.codes, words, a.E * a.N, 32, 64, /*swizzle128=*/true);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d_bf16(&prm.tm_sb[m][0], wm.scales, gpr, a.E * a.N, kSbGroups, 64, false);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d_bf16(&prm.tm_sb[m][1], wm.biases, gpr, a.E * a.N, kSbGroups, 64, false);
    if (e != cudaSuccess) return e;
  }
  prm.y = a.y;
  prm.dst_row = a.dst_row;
  prm.tiles = a.tiles;
  prm.num_tiles = a.num_tiles;
  prm.dense_rows = a.dense_rows;
  prm.N = a.N;
  prm.K = a.K;
  prm.pair = a.nmat == 2 ? 0 : 1;
  prm.d_status = a.d_status;
  if (a.group == 32) return launch_qdec_gs<32>(prm, stream);
  if (a.group == 64) return launch_qdec_gs<64>(prm, stream);
  return launch_qdec_gs<128>(prm, stream);
}

}  // namespace qmoe
