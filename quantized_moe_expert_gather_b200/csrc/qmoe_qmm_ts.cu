// Tensor-core gathered quantised matmul for many rows per expert (prefill), with the
// dequantised weights as the MMA's A operand in tensor memory.
//
// The product of the other two kernels -- for every expert-aligned tile of routed rows
// (MLX PR #4567 "[Metal] Gather mm improvement", Proposed changes) and every block of
// output channels, y[row, n] = x[row] . dequantize(W[e])[n]^T (nuvec-core 0.4.0
// tests/quantized.rs, gather_qmm_selects_batches), with the SwitchGLU epilogue
// h = silu(gate) * up for two weight stacks (MLX issue #4509 repro script, `moe`).
//
// Roles are those of a weight-stationary tile: a unit is 128 weight rows (64 channels of
// both stacks, or 128 channels of one) against one tile of up to 192 routed rows of one
// expert.  The weight rows are dequantised (q*s + b, one bf16 rounding; 4- or 8-bit codes)
// straight into tensor memory as the M = 128 A operand; the tile's rows are the N operand, read by the
// MMA from 128B-swizzled shared memory; N is the tile's valid row count rounded up to
// 16, so a sparsely routed expert costs MMA work in proportion to its rows.  Against a
// kernel that stages dequantised weights in shared memory, this halves the
// dequantisation per flop (128 weight rows per 192 routed rows instead of 256 per 128)
// and takes the weight tiles out of shared memory, whose bandwidth the MMAs' operand
// reads, the activation copies and the weight stores otherwise exceed.
//
// One persistent CTA per SM takes every gridDim-th unit.  Warps:
//   0-3, 15-18  epilogue, two groups taking alternate pieces: tcgen05.ld of the unit's
//         128 x N fp32 accumulator in 32-column pieces (one TMEM lane per weight row),
//         transposed through shared memory; a full piece of one stack in tile order leaves
//         by one TMA tensor store, others by 16-byte stores of 8 output channels (after
//         silu*mul for two stacks) per valid routed row;
//   4     activation producer: TMA of the activation slab of each 128-k step (per 64-k
//         swizzle atom one box of as many 32-row blocks as the tile's MMA N reads);
//   5     MMA issuer: tcgen05.mma kind::f16, A from tensor memory, M=128, N <= 192, K=16;
//   6-13  dequant: warp w owns the weight rows of TMEM lane quarter w%4 and one half of
//         each step's 128 k (64 codes per thread and step);
//   14    weight producer: TMA of the packed codes per 128 bytes of each row (two boxes of
//         64 rows x 128 B: 256 k of 4-bit, 128 k of 8-bit codes) and of the scales and
//         biases every 8 groups -- or, when a row has fewer than 8 groups, the unit's
//         whole [64 rows][groups] blocks by 1-D bulk copies.  With a tile table written
//         before the previous kernel (the down projection), the weight producer and the
//         dequant warps start before that kernel completes.
// Tensor memory: two 128-k A slots (128 columns) and two 192-column accumulators.  Steps
// of 128 k rather than 64 halve the mbarrier hand-offs between the roles per flop, which
// bound the kernel (64-k steps: T=16384 up/gate 684 TFLOP/s; 128-k steps: 885).
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

constexpr int kM = 128;                          // weight rows per unit = TMEM lanes = MMA M
constexpr int kNMax = kTsTileRows;               // routed rows per tile: MMA N at most
#ifndef QTS_KC
#define QTS_KC 128
#endif
constexpr int kAtomK = 64;                       // k per 128-byte swizzle atom of bf16
constexpr int kKC = QTS_KC;                      // k per step
constexpr int kAtoms = kKC / kAtomK;             // activation atoms per step
constexpr int kXBoxRows = 32;                    // activation box heights: multiples of 32 rows
constexpr int kNXMaps = kNMax / kXBoxRows;       // one tensor map per box height
constexpr int kXBoxBytes = kXBoxRows * kAtomK * 2;  // 4 KB: 32 rows of one atom
constexpr int kXAtomBytes = kNMax * kAtomK * 2;     // 24 KB: one atom of a full tile
constexpr int kXBytes = kAtoms * kXAtomBytes;       // per activation stage
static_assert(kKC == 64 || kKC == 128, "step");
#ifndef QTS_S1
#define QTS_S1 (6 / (QTS_KC / 64))
#endif
#ifndef QTS_SP
#define QTS_SP 2
#endif
#ifndef QTS_EPI_COLS
#define QTS_EPI_COLS 32
#endif
constexpr int kS1 = QTS_S1;                      // activation stages
// steps per packed-code slot (128 bytes of each row: 256 k of 4-bit, 128 k of 8-bit codes)
template <int BITS>
__host__ __device__ constexpr int steps_per_slot() { return (1024 / BITS) / kKC; }
constexpr int kPBytes = kM * 128;                // 16 KB: two boxes of 64 rows x 128 B
constexpr int kSP = QTS_SP;                      // packed-code slots
constexpr int kSbGroups = 8;                     // groups per scale/bias box
constexpr int kSbBytes = 2 * 2 * 64 * kSbGroups * 2;  // [box][s|b][64 rows][8] bf16
constexpr int kSbSlots = 2;
constexpr int kACols = kKC / 2;                  // TMEM columns per A tile (bf16 pairs)
#ifndef QTS_ASLOTS
#define QTS_ASLOTS (128 / (QTS_KC / 2))
#endif
constexpr int kASlots = QTS_ASLOTS;              // dequantised A tiles in tensor memory
#ifndef QTS_DQ_WARPS
#define QTS_DQ_WARPS 8
#endif
constexpr int kDqWarps = QTS_DQ_WARPS;           // 8 or 16
constexpr int kDqParts = kDqWarps / 4;           // k slices of a step, one per warp of a quarter
constexpr int kKT = kKC / kDqParts;              // k per dequant thread and step
// packed words per dequant thread and step
template <int BITS>
__host__ __device__ constexpr int thread_words() { return kKT * BITS / 32; }
static_assert((kDqWarps == 8 || kDqWarps == 16) && thread_words<4>() % 4 == 0, "dequant split");
constexpr int kDCol0 = kASlots * kACols;         // accumulators after the A tiles
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 4, kProdWarp = 4, kMmaWarp = 5, kDqWarp0 = 6;
constexpr int kProdWWarp = kDqWarp0 + kDqWarps;       // 14: packed codes, scales, biases
constexpr int kEpi2Warp0 = kProdWWarp + 1;            // 15-18: second epilogue group
constexpr int kThreads = (kEpi2Warp0 + kEpiWarps) * 32;  // 608
constexpr int kEpiCols = QTS_EPI_COLS;           // accumulator columns (routed rows) per piece
static_assert(kEpiCols == 16 || kEpiCols == 32, "epilogue piece");
constexpr int kOffP = kS1 * kXBytes;
constexpr int kOffSb = kOffP + kSP * kPBytes;
constexpr int kStageBytes = kEpiCols * kM * 4;           // epilogue transpose: [rows][128] f32
constexpr int kOffStage = kOffSb + kSbSlots * kSbBytes;  // one per epilogue group
constexpr int kOffBar = kOffStage + 2 * kStageBytes;
constexpr int kSmem = kOffBar + 512;
static_assert(kDCol0 + 2 * kNMax <= kTmemCols, "tensor memory budget");
static_assert(kSmem + 1024 <= 227 * 1024, "shared memory budget");
static_assert(kXBytes % 1024 == 0 && kOffP % 1024 == 0 && kOffSb % 1024 == 0,
              "128B-swizzled boxes need 1 KB alignment");
static_assert(kNMax % kXBoxRows == 0 && kNMax % 16 == 0 && kNMax <= 256, "tile rows");

// Instruction descriptor without N: fp32 accumulator, bf16 A and B, both K-major, M=128.
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kM >> 4) << 24);

struct alignas(64) TsParams {
  CUtensorMap tm_w[2];      // packed codes [E*N, K/8] u32, box {32 words, 64 rows}, 128B swizzle
  CUtensorMap tm_sb[2][2];  // [stack][scales|biases] [E*N, K/group] bf16, box {8, 64}
  CUtensorMap tm_x[kNXMaps];  // activation rows [x_rows, K] bf16, box {64, 32*(i+1)}, 128B swizzle
  CUtensorMap tm_y;         // output rows [x_rows, N] bf16, box {128, kEpiCols} (tma_store only)
  uint16_t* y;
  const uint32_t* dst_row;
  const uint32_t* tiles;
  const uint32_t* num_tiles;
  int64_t dense_rows;
  int64_t N, K;
  int pair;                 // 1: one stack, a unit is 128 of its channels
  int sb_groups;            // > 0: a row has fewer than 8 groups; each unit's scales and
                            // biases ([64 rows][sb_groups] per half) come by 1-D bulk copies
  const uint16_t* scales[2];
  const uint16_t* biases[2];
  int vec_store;            // y rows start 16-byte aligned: 8 channels per store
  int tma_store;            // one stack, rows in tile order (no dst_row), vec_store: full
                            // epilogue pieces leave by TMA tensor stores
  int early_weights;        // tile table older than the previous kernel (or none)
  int* d_status;
  ProfSlot* prof;
};

struct TsTile {
  uint32_t row_start, expert, valid;
};

__device__ __forceinline__ TsTile ts_tile(const TsParams& p, int64_t j) {
  TsTile t;
  if (p.dense_rows > 0) {
    t.row_start = static_cast<uint32_t>(j * kNMax);
    t.expert = 0;
    t.valid = static_cast<uint32_t>(imin64(kNMax, p.dense_rows - j * kNMax));
  } else {
    t.row_start = p.tiles[3 * j];
    t.expert = p.tiles[3 * j + 1];
    t.valid = min(p.tiles[3 * j + 2], static_cast<uint32_t>(kNMax));
  }
  return t;
}

// MMA N for a tile: its valid rows rounded up to 16 (at least 16).
__device__ __forceinline__ uint32_t ts_mma_n(uint32_t valid) {
  return max(16u, (valid + 15u) & ~15u);
}


// 4 packed 8-bit codes -> 4 bf16 of q*s + b (the fp32 fma is exact for a <=8-bit code
// times a bf16 scale plus a bf16 bias; one rounding to bf16).
__device__ __forceinline__ uint2 ts_dequant_word8(uint32_t w, float s, float b) {
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t f = prmt(w, 0x4B000000u, k | (4 << 4) | (4 << 8) | (7 << 12));  // 2^23 + q
    v[k] = fmaf(__uint_as_float(f) - 8388608.0f, s, b);
  }
  return make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

template <int BITS, int GS, bool SB_WHOLE>
__global__ void __launch_bounds__(kThreads, 1) qmm_ts_kernel(const __grid_constant__ TsParams p) {
  constexpr int kPK = steps_per_slot<BITS>();
  constexpr int kTW = thread_words<BITS>();
  static_assert(kPK >= 1 && kTW % 4 == 0, "code slots");
  // steps per scale/bias window: 8 groups by TMA, or the whole unit's groups
  constexpr int KS_SB_BOX = kSbGroups * GS / kKC;
  static_assert((kSbGroups * GS) % kKC == 0 && KS_SB_BOX >= 1, "group size");
  constexpr int GPT = kKT >= GS ? kKT / GS : 1;  // groups of a thread's k per step
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full1 = bars;                   // [kS1] TMA tx: activation slab
  uint64_t* empty1 = full1 + kS1;           // [kS1] MMA commit
  uint64_t* fullP = empty1 + kS1;           // [kSP] TMA tx: packed codes
  uint64_t* emptyP = fullP + kSP;           // [kSP] dequant warps
  uint64_t* full_sb = emptyP + kSP;         // [kSbSlots] TMA tx
  uint64_t* empty_sb = full_sb + kSbSlots;  // [kSbSlots] dequant warps
  uint64_t* a_full = empty_sb + kSbSlots;   // [kASlots] dequant warps: A tile written
  uint64_t* a_empty = a_full + kASlots;     // [kASlots] MMA commit: A tile read
  uint64_t* d_full = a_empty + kASlots;     // [2] MMA commit: accumulator ready
  uint64_t* d_empty = d_full + 2;           // [2] epilogue warps: accumulator drained
  uint64_t* drain = d_empty + 2;            // [1] final MMA commit on the abort path
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS1; ++s) {
      mbar_init(&full1[s], 1);
      mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < kSP; ++s) {
      mbar_init(&fullP[s], 1);
      mbar_init(&emptyP[s], kDqWarps);
    }
    for (int s = 0; s < kSbSlots; ++s) {
      mbar_init(&full_sb[s], 1);
      mbar_init(&empty_sb[s], kDqWarps);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(&a_full[s], kDqWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], 2 * kEpiWarps);
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
  // Inputs (tile table, activations) may come from the kernel before this one.  When the
  // tile table is older (or there is none), the weight producer and the dequant warps --
  // which read only the table and the weights, never written by the kernel just before --
  // start at once, overlapping the tail of that kernel.
  if (!(p.early_weights && (warp == kProdWWarp || (warp >= kDqWarp0 && warp < kDqWarp0 + kDqWarps))))
    griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(p.prof);

  const int64_t KS = p.K / kKC;               // steps per unit
  const int64_t KS_SB = SB_WHOLE ? KS : KS_SB_BOX;
  const int unit_n = p.pair ? kM : kM / 2;    // output channels per unit
  const int64_t NB = (p.N + unit_n - 1) / unit_n;
  const int64_t ntiles = p.dense_rows > 0 ? (p.dense_rows + kNMax - 1) / kNMax : *p.num_tiles;
  const int64_t units = ntiles * NB;
  // Units are dealt round-robin: the CTAs working on one tile's channel blocks at the same
  // time share its activation rows through L2 (a tile is re-read once per channel block).
  const int64_t u_begin = blockIdx.x, u_step = gridDim.x, u_end = units;
  // first weight row of code box m (rows 0..63 and 64..127 of the unit)
  auto box_row = [&](const TsTile& t, int64_t u, int m) -> int64_t {
    const int64_t n0 = (u % NB) * unit_n;
    return static_cast<int64_t>(t.expert) * p.N + n0 + (p.pair ? 64 * m : 0);
  };

  if (warp == kProdWarp) {
    // ------------------------------------------------------- activation producer
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kNXMaps; ++i) tma_prefetch_desc(&p.tm_x[i]);
      uint32_t it = 0;
      bool ab = false;
      int64_t cur = -1;
      TsTile tl{};
      int nbox = 1;
      for (int64_t u = u_begin; u < u_end && !ab; u += u_step) {
        if (u / NB != cur) {
          cur = u / NB;
          tl = ts_tile(p, cur);
          nbox = static_cast<int>((ts_mma_n(tl.valid) + kXBoxRows - 1) / kXBoxRows);
        }
        for (int64_t ks = 0; ks < KS; ++ks, ++it) {
          if (*abort_flag) { ab = true; break; }
          const uint32_t s1 = it % kS1;
          if (!mbar_wait(&empty1[s1], ((it / kS1) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
          // per atom one box of as many 32-row blocks as the tile's MMA N reads
          mbar_arrive_expect_tx(&full1[s1], static_cast<uint32_t>(kAtoms * nbox * kXBoxBytes));
#pragma unroll
          for (int a = 0; a < kAtoms; ++a)
            tma_load_2d(smem + s1 * kXBytes + a * kXAtomBytes, &p.tm_x[nbox - 1], &full1[s1],
                        static_cast<int32_t>(ks * kKC + a * kAtomK), static_cast<int32_t>(tl.row_start));
        }
      }
      if (ab) {
        // let the copies already issued land before the CTA can exit
        const uint32_t f1 = it > static_cast<uint32_t>(kS1) ? it - kS1 : 0u;
        for (uint32_t k = f1; k < it; ++k) mbar_wait(&full1[k % kS1], (k / kS1) & 1, nullptr);
      }
    }
  } else if (warp == kProdWWarp) {
    // ----------------------------------------------------------- weight producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_w[0]);
      tma_prefetch_desc(&p.tm_w[1]);
      uint32_t pbit = 0, sbit = 0;
      bool ab = false;
      int64_t cur = -1;
      TsTile tl{};
      for (int64_t u = u_begin; u < u_end && !ab; u += u_step) {
        if (u / NB != cur) {
          cur = u / NB;
          tl = ts_tile(p, cur);
        }
        const int64_t r0 = box_row(tl, u, 0), r1 = box_row(tl, u, 1);
        for (int64_t ks = 0; ks < KS; ++ks) {
          if (*abort_flag) { ab = true; break; }
          if (ks % kPK == 0) {
            const uint32_t sp = pbit % kSP;
            if (!mbar_wait(&emptyP[sp], ((pbit / kSP) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
            mbar_arrive_expect_tx(&fullP[sp], kPBytes);
#pragma unroll
            for (int m = 0; m < 2; ++m)
              tma_load_2d(smem + kOffP + sp * kPBytes + m * 64 * 128, &p.tm_w[m], &fullP[sp],
                          static_cast<int32_t>((ks / kPK) * 32), static_cast<int32_t>(m ? r1 : r0));
            ++pbit;
          }
          if (ks % KS_SB == 0) {
            const uint32_t e = sbit % kSbSlots;
            if (!mbar_wait(&empty_sb[e], ((sbit / kSbSlots) & 1) ^ 1, p.d_status)) { *abort_flag = 1; ab = true; break; }
            if constexpr (SB_WHOLE) {
              // [64 rows][sb_groups] of each half is contiguous: one bulk copy per array
              const uint32_t bytes = static_cast<uint32_t>(64 * p.sb_groups * 2);
              mbar_arrive_expect_tx(&full_sb[e], 4 * bytes);
#pragma unroll
              for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int arr = 0; arr < 2; ++arr) {
                  const uint16_t* src = (arr ? p.biases[p.pair ? 0 : m] : p.scales[p.pair ? 0 : m]) +
                                        (m ? r1 : r0) * p.sb_groups;
                  bulk_load(smem + kOffSb + e * kSbBytes + (m * 2 + arr) * 64 * kSbGroups * 2, src,
                            bytes, &full_sb[e]);
                }
            } else {
              mbar_arrive_expect_tx(&full_sb[e], kSbBytes);
              const int32_t gx = static_cast<int32_t>(ks * kKC / GS);
#pragma unroll
              for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int arr = 0; arr < 2; ++arr)
                  tma_load_2d(smem + kOffSb + e * kSbBytes + (m * 2 + arr) * 64 * kSbGroups * 2,
                              &p.tm_sb[m][arr], &full_sb[e], gx, static_cast<int32_t>(m ? r1 : r0));
            }
            ++sbit;
          }
        }
      }
      if (ab) {
        const uint32_t fp = pbit > static_cast<uint32_t>(kSP) ? pbit - kSP : 0u;
        for (uint32_t k = fp; k < pbit; ++k) mbar_wait(&fullP[k % kSP], (k / kSP) & 1, nullptr);
        const uint32_t fs = sbit > static_cast<uint32_t>(kSbSlots) ? sbit - kSbSlots : 0u;
        for (uint32_t k = fs; k < sbit; ++k) mbar_wait(&full_sb[k % kSbSlots], (k / kSbSlots) & 1, nullptr);
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
    int64_t cur = -1;
    uint32_t idesc = 0;
    for (int64_t u = u_begin; u < u_end; u += u_step, ++tc) {
      if (u / NB != cur) {
        cur = u / NB;
        idesc = kIdescBase | ((ts_mma_n(ts_tile(p, cur).valid) >> 3) << 17);
      }
      const uint32_t buf = tc & 1;
      if (lane == 0) ok = !*abort_flag && mbar_wait(&d_empty[buf], ((tc >> 1) & 1) ^ 1, p.d_status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + kDCol0 + buf * kNMax;
      for (int64_t ks = 0; ks < KS; ++ks, ++it) {
        const uint32_t s1 = it % kS1, as = it % kASlots;
        if (lane == 0)
          ok = mbar_wait(&full1[s1], (it / kS1) & 1, p.d_status) &&
               mbar_wait(&a_full[as], (it / kASlots) & 1, p.d_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t b0 = sw128_desc(smem + s1 * kXBytes);
        const uint32_t a0 = tmem_base + as * kACols;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk)  // atom kk/4, 32 bytes along k inside it
            tc_mma_ts(d, a0 + kk * 8, b0 + ((kk / 4) * kXAtomBytes >> 4) + 2 * (kk % 4), idesc,
                      (ks | kk) != 0 ? 1u : 0u);
          tc_commit(&empty1[s1]);
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
  } else if (warp >= kDqWarp0 && warp < kDqWarp0 + kDqWarps) {
    // ------------------------------------------------------------------- dequant
    // Warp w may only reach TMEM lanes 32*(w%4)..+31: it owns those weight rows, and
    // half `part` of each step's k (kTW packed words).
    const int quarter = warp % 4, part = (warp - kDqWarp0) / 4;
    const int r = quarter * 32 + lane;   // weight row of the unit = TMEM lane
    const int m = r / 64, rr = r % 64;   // code box and row inside it
    uint32_t it = 0, pbit = 0, sbit = 0;
    for (int64_t u = u_begin; u < u_end; u += u_step) {
      for (int64_t ks = 0; ks < KS; ++ks, ++it) {
        if (*abort_flag) break;
        const uint32_t sp = pbit % kSP, e = sbit % kSbSlots, as = it % kASlots;
        if (ks % kPK == 0 && !mbar_wait(&fullP[sp], (pbit / kSP) & 1, p.d_status)) { *abort_flag = 1; break; }
        if (ks % KS_SB == 0 &&
            !mbar_wait(&full_sb[e], (sbit / kSbSlots) & 1, p.d_status)) { *abort_flag = 1; break; }
        if (!mbar_wait(&a_empty[as], ((it / kASlots) & 1) ^ 1, p.d_status)) { *abort_flag = 1; break; }
        tc_fence_after();
        // this thread's kTW words of the row: 16-byte pieces of the slot's 128-byte row,
        // piece c at c ^ (rr & 7)
        const uint8_t* rowp = smem + kOffP + sp * kPBytes + m * 64 * 128 + rr * 128;
        // the thread's k lie in GPT groups, the first at g0 of the scale window (row
        // stride: 8 groups per TMA window, or the row's sb_groups for whole-unit copies)
        const int sbs = SB_WHOLE ? p.sb_groups : kSbGroups;
        const int g0 = SB_WHOLE
                           ? static_cast<int>((ks * kKC + part * kKT) / GS)
                           : (static_cast<int>((ks * kKC) % (kSbGroups * GS)) + part * kKT) / GS;
        const uint16_t* sbw = reinterpret_cast<const uint16_t*>(smem + kOffSb + e * kSbBytes);
        // the four [64 rows][sbs] arrays sit 64 x 8 elements apart
        const uint16_t* srow = sbw + (m * 2) * 64 * kSbGroups + rr * sbs + g0;
        const uint16_t* brow = sbw + (m * 2 + 1) * 64 * kSbGroups + rr * sbs + g0;
        constexpr int kPieceStep = kKC * BITS / 128;  // 16-byte pieces of a row per step
        uint32_t out[kKT / 2];                         // two bf16 of consecutive k per column
        if constexpr (BITS == 4) {
          __nv_bfloat162 s2[GPT], b2[GPT];
          load_group_pairs<GPT>(srow, s2);
          load_group_pairs<GPT>(brow, b2);
#pragma unroll
          for (int q = 0; q < kTW / 4; ++q) {
            const int piece = static_cast<int>(ks % kPK) * kPieceStep + part * (kTW / 4) + q;
            const uint4 pw = *reinterpret_cast<const uint4*>(rowp + ((piece ^ (rr & 7)) << 4));
            const uint32_t w4[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int gi = ((4 * q + j) * 8) / GS;  // the word's group among the thread's
              const uint4 v = dequant_word4(w4[j], s2[gi], b2[gi]);
              out[(4 * q + j) * 4 + 0] = v.x;
              out[(4 * q + j) * 4 + 1] = v.y;
              out[(4 * q + j) * 4 + 2] = v.z;
              out[(4 * q + j) * 4 + 3] = v.w;
            }
          }
        } else {
          float sf[GPT], bf[GPT];
#pragma unroll
          for (int i = 0; i < GPT; ++i) {
            sf[i] = bf16_to_f32(srow[i]);
            bf[i] = bf16_to_f32(brow[i]);
          }
#pragma unroll
          for (int q = 0; q < kTW / 4; ++q) {
            const int piece = static_cast<int>(ks % kPK) * kPieceStep + part * (kTW / 4) + q;
            const uint4 pw = *reinterpret_cast<const uint4*>(rowp + ((piece ^ (rr & 7)) << 4));
            const uint32_t w4[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int gi = ((4 * q + j) * 4) / GS;  // 4 codes per 8-bit word
              const uint2 v = ts_dequant_word8(w4[j], sf[gi], bf[gi]);
              out[(4 * q + j) * 2 + 0] = v.x;
              out[(4 * q + j) * 2 + 1] = v.y;
            }
          }
        }
        // A tile: lane r, columns part*kKT/2.. (two bf16 of consecutive k per column)
        tmem_st_cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + as * kACols +
                         part * (kKT / 2), out);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        const bool p_done = ks % kPK == kPK - 1 || ks == KS - 1;
        const bool sb_done = ks % KS_SB == KS_SB - 1 || ks == KS - 1;
        if (lane == 0) {
          mbar_arrive(&a_full[as]);
          if (p_done) mbar_arrive(&emptyP[sp]);
          if (sb_done) mbar_arrive(&empty_sb[e]);
        }
        if (p_done) ++pbit;
        if (sb_done) ++sbit;
      }
      if (*abort_flag) break;
    }
  } else if (warp < kEpiWarps || warp >= kEpi2Warp0) {
    // ------------------------------------------------------------------ epilogue
    // Two groups of four warps take alternate pieces of 32 routed rows.  Per piece, each
    // thread moves its TMEM lane (one weight row) into its group's [row][weight row] fp32
    // stage; then the group's 128 threads take (routed row, 8 output channels) items,
    // apply silu(gate)*up for two stacks (gate rows sit 64 after their up rows) and write
    // 8 bf16 with one 16-byte store along the output row.
    const int grp = warp < kEpiWarps ? 0 : 1;
    const int quarter = warp % 4;        // a warp reaches TMEM lanes 32*(warp%4)..+31
    const int r = quarter * 32 + lane;   // TMEM lane = weight row of the unit
    // named barriers 1 and 2 (0 is __syncthreads), ids fixed at compile time
    auto group_sync = [&]() {
      if (grp == 0) named_bar_sync<1>(kEpiWarps * 32);
      else named_bar_sync<2>(kEpiWarps * 32);
    };
    auto group_any = [&](bool pred) -> bool {
      return grp == 0 ? named_bar_any<1>(kEpiWarps * 32, pred) : named_bar_any<2>(kEpiWarps * 32, pred);
    };
    float* stage = reinterpret_cast<float*>(smem + kOffStage + grp * kStageBytes);
    const int nch = p.pair ? kM : kM / 2;  // output channels of a unit
    const int groups = nch / 8;
    uint32_t tc = 0;
    int64_t cur = -1;
    TsTile tl{};
    for (int64_t u = u_begin; u < u_end; u += u_step, ++tc) {
      const uint32_t buf = tc & 1;
      bool stop = *abort_flag || !mbar_wait(&d_full[buf], (tc >> 1) & 1, p.d_status);
      stop = group_any(stop);  // the group meets at named barriers below
      if (stop) { *abort_flag = 1; break; }
      tc_fence_after();
      if (u / NB != cur) {
        cur = u / NB;
        tl = ts_tile(p, cur);
      }
      const int64_t n0 = (u % NB) * unit_n;
      const int pieces = static_cast<int>((ts_mma_n(tl.valid) + kEpiCols - 1) / kEpiCols);
      if (grp >= pieces) {  // nothing for this group in this unit
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[buf]);
        continue;
      }
      for (int pc = grp; pc < pieces; pc += 2) {
        float v[kEpiCols];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + kDCol0 +
                               buf * kNMax + pc * kEpiCols;
        tmem_ld_piece(taddr, v);
        if (pc + 2 >= pieces) {  // this group's last piece: its share of the accumulator is read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&d_empty[buf]);
        }
        const int t0 = pc * kEpiCols;
        // the stage is free once this group's previous tensor store has read it
        if (r == 0 && p.tma_store) bulk_wait_read_all();
        group_sync();
        if (p.tma_store && static_cast<uint32_t>(t0 + kEpiCols) <= tl.valid) {
          // a full piece of one stack in tile order: bf16 [rows][128 channels], one TMA store
          uint16_t* sb16 = reinterpret_cast<uint16_t*>(stage);
#pragma unroll
          for (int j = 0; j < kEpiCols; ++j) sb16[j * kM + r] = f32_to_bf16(v[j]);
          fence_proxy_async_smem();
          group_sync();
          if (r == 0) {
            tma_store_2d(&p.tm_y, stage, static_cast<int32_t>(n0),
                         static_cast<int32_t>(tl.row_start + t0));
            bulk_commit_group();
          }
          continue;
        }
#pragma unroll
        for (int j = 0; j < kEpiCols; ++j) stage[j * kM + r] = v[j];
        group_sync();
        for (int item = r; item < kEpiCols * groups; item += kEpiWarps * 32) {
          const int t = item / groups, c0 = (item % groups) * 8;
          if (static_cast<uint32_t>(t0 + t) >= tl.valid) continue;
          const float* srow = stage + t * kM;
          float o[8];
          const float4 a = *reinterpret_cast<const float4*>(srow + c0);
          const float4 b = *reinterpret_cast<const float4*>(srow + c0 + 4);
          o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
          o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
          if (!p.pair) {
            const float4 ga = *reinterpret_cast<const float4*>(srow + 64 + c0);
            const float4 gb = *reinterpret_cast<const float4*>(srow + 64 + c0 + 4);
            const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] *= g[i] / (1.0f + expf(-g[i]));
          }
          const uint32_t pos = tl.row_start + t0 + t;
          const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
          uint16_t* dst = p.y + static_cast<int64_t>(dr) * p.N + n0 + c0;
          if (p.vec_store && n0 + c0 + 8 <= p.N) {
            const uint4 pk = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                        pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
            *reinterpret_cast<uint4*>(dst) = pk;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (n0 + c0 + i < p.N) dst[i] = f32_to_bf16(o[i]);
          }
        }
      }
    }
    if (r == 0 && p.tma_store) bulk_wait_all();  // the tensor stores have landed
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
cudaError_t launch_ts_gs(const TsParams& prm, cudaStream_t stream) {
  auto kern = qmm_ts_kernel<BITS, GS, SB_WHOLE>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchTimer timer(prm.pair ? "ts" : "ts_glu", stream);
  TsParams p = prm;
  p.prof = timer.slot();
  const cudaError_t e = launch_pdl(kern, dim3(sm_count()), dim3(kThreads), kSmem + 1024, stream, p);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool qmm_ts_supported(const GemmArgs& a) {
  if ((a.bits != 4 && a.bits != 8) || (a.group != 32 && a.group != 64 && a.group != 128))
    return false;
  if (a.K % kKC != 0) return false;                    // whole steps of activation boxes
  const int64_t gpr = a.K / a.group;
  if (gpr % kSbGroups != 0) {
    // Fewer than 8 groups per row: each unit's scale/bias blocks come by 1-D bulk copies
    // of whole 64-row halves, which must stay inside the stack (no bounds check) and
    // start 16-byte aligned.
    if (gpr >= kSbGroups) return false;
    if (a.N % (a.nmat == 2 ? 64 : 128) != 0) return false;
    for (int m = 0; m < a.nmat; ++m)
      if (reinterpret_cast<uintptr_t>(a.w[m].scales) % 16 != 0 ||
          reinterpret_cast<uintptr_t>(a.w[m].biases) % 16 != 0)
        return false;
  }
  if (a.x_rows <= 0 || a.src_row != nullptr) return false;  // activations in tile order
  return true;
}

cudaError_t launch_qmm_ts(const GemmArgs& a, cudaStream_t stream) {
  if (!qmm_ts_supported(a)) return cudaErrorNotSupported;
  if (a.dense_rows <= 0 && a.bm != kNMax) return cudaErrorInvalidValue;  // tile table of kNMax rows
  TsParams prm{};
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < kNXMaps; ++i) {
    e = make_tmap_2d_bf16(&prm.tm_x[i], a.x, a.K, a.x_rows, kAtomK, kXBoxRows * (i + 1),
                          /*swizzle128=*/true);
    if (e != cudaSuccess) return e;
  }
  const int64_t words = a.K * a.bits / 32;
  const int64_t gpr = a.K / a.group;
  const bool whole = gpr % kSbGroups != 0;  // scales/biases by bulk copies (no tensor map)
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
    e = make_tmap_2d_u32(&prm.tm_w[m], wm.codes, words, a.E * a.N, 32, 64, /*swizzle128=*/true);
    if (e != cudaSuccess) return e;
    if (whole) continue;
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
  prm.early_weights = (a.dense_rows > 0 || a.tiles_ready) ? 1 : 0;
  prm.vec_store = (a.N % 8 == 0 && reinterpret_cast<uintptr_t>(a.y) % 16 == 0) ? 1 : 0;
  prm.tma_store = (a.nmat == 1 && a.dst_row == nullptr && prm.vec_store) ? 1 : 0;
  if (prm.tma_store) {
    e = make_tmap_2d_bf16(&prm.tm_y, a.y, a.N, a.x_rows, kM, kEpiCols, /*swizzle128=*/false);
    if (e != cudaSuccess) return e;
  }
  prm.d_status = a.d_status;
  prm.sb_groups = whole ? static_cast<int>(gpr) : 0;
  for (int m = 0; m < 2; ++m) {
    prm.scales[m] = a.w[a.nmat == 2 ? m : 0].scales;
    prm.biases[m] = a.w[a.nmat == 2 ? m : 0].biases;
  }
  if (a.bits == 4) {
    if (a.group == 32) return whole ? launch_ts_gs<4, 32, true>(prm, stream) : launch_ts_gs<4, 32, false>(prm, stream);
    if (a.group == 64) return whole ? launch_ts_gs<4, 64, true>(prm, stream) : launch_ts_gs<4, 64, false>(prm, stream);
    return whole ? launch_ts_gs<4, 128, true>(prm, stream) : launch_ts_gs<4, 128, false>(prm, stream);
  }
  if (a.group == 32) return whole ? launch_ts_gs<8, 32, true>(prm, stream) : launch_ts_gs<8, 32, false>(prm, stream);
  if (a.group == 64) return whole ? launch_ts_gs<8, 64, true>(prm, stream) : launch_ts_gs<8, 64, false>(prm, stream);
  return whole ? launch_ts_gs<8, 128, true>(prm, stream) : launch_ts_gs<8, 128, false>(prm, stream);
}

}  // namespace qmoe
