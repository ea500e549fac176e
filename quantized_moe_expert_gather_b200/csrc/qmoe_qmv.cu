// Streaming gathered quantised matmul for few rows per expert (decode, small M).
//
// Computes, for every expert-aligned tile of <= 8*NT routed rows (MLX PR #4567
// "[Metal] Gather mm improvement", Proposed changes) and every block of 16 output
// channels, y[row, n] = x[row] . dequantize(W[e])[n]^T (nuvec-core 0.4.0
// tests/quantized.rs, gather_qmm_selects_batches), and with two weight stacks the
// SwitchGLU epilogue h = silu(gate) * up (MLX issue #4509 repro script, `moe`).
//
// The tile table makes every touched expert's packed weights stream from HBM once
// per tile (MLX issue #4509: M=1 decode must still reach full bandwidth).
//
// Structure (one persistent CTA per SM, 8 consumer warps + 1 producer warp + 1
// epilogue warp):
//   * the producer warp walks the CTA's contiguous range of units (a tile of routed rows
//     and NMAT 16-row weight blocks: of the one stack, or half of each of two) and, per
//     K-chunk of 1 KB of each row (512 B with two token sets or four blocks), loads each
//     16-row block's packed codes with one 3-D TMA box (16 rows x 8 (or 4) column blocks
//     of 128 B, 128B-swizzled so that the consumers' row-strided reads are free of bank
//     conflicts; one 2-D box of 128 B x 16 rows per column block when a row is not a
//     whole number of column blocks) and the
//     matching scales/biases with 2-D TMA boxes (cp.async when their row pitch is not
//     a multiple of 16 bytes), into a ring of stages guarded by full/empty mbarriers.
//     Few large copies per stage matter: the TMA issue and mbarrier round trip of
//     each copy, not DRAM, bounded the stream when every 2 KB box was its own copy;
//   * warps 0..CW-1 (consumers) split each chunk's groups.  Each lane prefetches the
//     activation values its MMA fragments need one chunk ahead into registers (the
//     loads of chunk c+1 are in flight while chunk c is computed; two register buffers
//     alternate between consecutive chunks).  A lane turns its packed
//     codes into bf16 "128 + q" (or "2048 + 16*hi" for the high nibble of 8-bit
//     codes) with one LOP3 per code pair and feeds mma.sync m16n8k16 with W as the
//     16-row A operand and up to 8 routed rows as the B operand.  Each MMA k-step
//     stays inside one quantisation group, so per group
//         sum_k x_k*(q_k*s + b) = s*C + (b - OFFSET*s)*X
//     with C the MMA sum over the magic-offset codes and X = sum_k x_k, obtained
//     from one more MMA with an all-ones A.  Scales and biases stay exact (fp32),
//     accumulation is fp32, and there is one bf16 rounding at the end;
//   * consumers store their partial sums of a unit in per-warp shared-memory slots and
//     move on; a dedicated epilogue warp waits for all slots (mbarrier), adds them in
//     warp order (deterministic, and a row's result does not depend on the other rows
//     of its tile), applies silu*mul and writes bf16.  Two slot buffers alternate, so
//     consumers never wait for each other at unit boundaries.
//
// All waits are bounded (see qmoe_common.cuh).
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "qmoe_common.cuh"
#include "qmoe_internal.h"
#include "qmoe_tma.h"

namespace qmoe {
namespace {

constexpr int kRows = 16;             // output channels per unit (MMA M)
constexpr int kSmemBudget = 225 * 1024;

// Consumer warps: 8.  With the producer and epilogue warps that is 10 warps (three
// per scheduler), which leaves each thread 168 registers: room for two chunks of
// activations and several groups' MMA chains in flight per warp.  More warps cap the
// registers at 96 (five warps on some schedulers) and spill.
template <int BITS, int GS, int NT>
constexpr int consumer_warps() {
  return 8;
}

template <int BITS, int GS, int NMAT, int NT>
struct Cfg {
  static constexpr int CW = consumer_warps<BITS, GS, NT>();
  static constexpr int THREADS = (CW + 2) * 32;  // consumers, producer, epilogue
  static constexpr int KB_BYTES = GS * BITS / 8;                 // one group of one row
  // 1 KB of each row per stage (512 B with two token sets, whose doubled register
  // arrays would otherwise spill, and with four 16-row blocks, whose stage it keeps at
  // 32 KB; half that for 2-bit codes, whose activations per code byte are twice as many),
  // at least one group per consumer warp
  static constexpr int CHUNK_ROW_BYTES =
      std::max((NT == 2 || NMAT == 4 ? 512 : 1024) / (BITS == 2 ? 2 : 1), KB_BYTES * CW);
  static constexpr int KB_PER_CHUNK = CHUNK_ROW_BYTES / KB_BYTES;
  static constexpr int KB_PER_WARP = KB_PER_CHUNK / CW;
  static constexpr int BOXES = CHUNK_ROW_BYTES / 128;
  static constexpr int LANE_BYTES = KB_BYTES / 4;                // per row, per lane
  static constexpr int WORDS = LANE_BYTES / 4;
  // activation vectors (16 B of bf16 for 2- and 4-bit codes, 8 B for 8-bit) per code word
  static constexpr int XW = BITS == 2 ? 2 : 1;
  // MMA k-steps per code word: 16 codes (2-bit) -> 4, 8 codes (4-bit) -> 2, 4 codes (8-bit)
  // -> 2 (low and high nibbles of the same activation pairs)
  static constexpr int MPW = BITS == 2 ? 4 : 2;
  static constexpr int CODE_BYTES = NMAT * BOXES * 2048;
  static constexpr int SB_BYTES = NMAT * 2 * kRows * KB_PER_CHUNK * 2;
  static constexpr int STAGE_BYTES = ((CODE_BYTES + SB_BYTES) + 1023) / 1024 * 1024;
  // per-warp partial sums, double-buffered: [2][CW][NMAT][NT][16 rows][8 tokens] fp32
  static constexpr int RED_SLICE = CW * NMAT * NT * kRows * 8;
  static constexpr int RED_BYTES = 2 * RED_SLICE * 4;
  static constexpr int STAGES =
      std::min(8, (kSmemBudget - RED_BYTES - 1024) / STAGE_BYTES);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + RED_BYTES + 2 * STAGES * 8 + 4 * 8 + 64;
  static constexpr uint32_t TMA_BYTES = CODE_BYTES;
  static_assert((kRows * KB_PER_CHUNK * 2) % 128 == 0, "scale/bias TMA boxes must stay 128-byte aligned");
  static constexpr float OFFSET = BITS == 8 ? 2176.0f : 128.0f;
  static_assert(BITS == 2 || BITS == 4 || BITS == 8, "code width");
  static_assert(LANE_BYTES >= 4, "a lane's share of a group must be whole words");
  static_assert(STAGES >= 3, "too few pipeline stages");
  static_assert(KB_PER_WARP >= 1, "chunk smaller than one group per warp");
};

struct alignas(64) QmvParams {
  CUtensorMap tmap[2];          // packed codes of each weight stack, [E*N rows, K*bits/32 words]
  CUtensorMap tmap_sb[2][2];    // [stack][scales|biases], [E*N rows, K/group] bf16
  const uint16_t* scales[2];
  const uint16_t* biases[2];
  const uint16_t* x;
  const uint32_t* src_row;
  const uint32_t* dst_row;
  uint16_t* y;
  const uint32_t* tiles;
  const uint32_t* num_tiles;
  int64_t dense_rows;
  int64_t N, K, E;
  int pair;                     // 1: one weight stack, a unit is NMAT adjacent 16-row blocks
  int code3d;                   // codes by one 3-D box per 16-row block (else one 2-D box per 128 B)
  int sb_tma;                   // scales/biases by TMA (row pitch a multiple of 16 bytes)
  int sb_vec;                   // else: byte width of the copy pieces (2: plain copies)
  int early_weights;            // the producer may stream before the previous kernel ends
  int64_t skip_stage;           // test hook: stage the last CTA leaves unissued (-1: none)
  int* d_status;
  ProfSlot* prof;
};

struct TileInfo {
  uint32_t row_start, expert, valid;
};

template <int NT>
__device__ __forceinline__ TileInfo tile_info(const QmvParams& p, int64_t j) {
  TileInfo t;
  if (p.dense_rows > 0) {
    t.row_start = static_cast<uint32_t>(j * 8 * NT);
    t.expert = 0;
    t.valid = static_cast<uint32_t>(imin64(8 * NT, p.dense_rows - j * 8 * NT));
  } else {
    t.row_start = p.tiles[3 * j];
    t.expert = p.tiles[3 * j + 1];
    t.valid = min(p.tiles[3 * j + 2], static_cast<uint32_t>(8 * NT));
  }
  return t;
}

template <int NT>
__device__ __forceinline__ int64_t num_tiles(const QmvParams& p) {
  if (p.dense_rows > 0) return (p.dense_rows + 8 * NT - 1) / (8 * NT);
  return *p.num_tiles;
}

// Byte offset of (row, byte c of the chunk row) inside one weight stack's part of a
// stage: boxes of 16 rows x 128 B, 16-byte chunks XOR-swizzled by (row & 7).
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return (c >> 7) * 2048 + row * 128 + ((((c >> 4) & 7) ^ (row & 7)) << 4) + (c & 15);
}

template <int BITS, int GS, int NMAT, int NT>
__global__ void __launch_bounds__(Cfg<BITS, GS, NMAT, NT>::THREADS, 1)
    qmv_kernel(const __grid_constant__ QmvParams p) {
  using C = Cfg<BITS, GS, NMAT, NT>;
  constexpr int kConsumerWarps = C::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::RED_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* red_full = empty + C::STAGES;   // [2] every consumer lane has stored its partials
  uint64_t* red_empty = red_full + 2;       // [2] the epilogue warp has read the buffer
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // producer's expect_tx (+ 32 per-lane arrivals when scales/biases are copied by lanes)
      mbar_init(&full[s], p.sb_tma ? 1 : 1 + 32);
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&red_full[b], kConsumerWarps * 32);
      mbar_init(&red_empty[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Inputs (tile table, activations) may come from the kernel before this one.  When the
  // tile table is older (a dense launch has none; the down projection's was written
  // before the up/gate launch) and the weights are never written by the kernel launched
  // just before it, the producer streams weights at once, overlapping the tail of that
  // kernel, and only the roles that read activations or write y wait.
  if (!(p.early_weights && warp == kConsumerWarps)) griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) prof_start(p.prof);

  const int64_t KB_TOTAL = p.K / GS;
  const int64_t NCH = (KB_TOTAL + C::KB_PER_CHUNK - 1) / C::KB_PER_CHUNK;
  // A unit's 16-row blocks: NMAT of one stack (pair), or NMAT/2 of each of two stacks (block
  // m of the up stack for m < NMAT/2, of the gate stack for the rest).
  constexpr int kHalf = NMAT / 2;
  const int unit_rows = p.pair ? NMAT * kRows : kHalf * kRows;  // output channels per unit
  auto blk_stack = [&](int m) { return p.pair ? 0 : m / kHalf; };
  auto blk_row = [&](int m) { return kRows * (p.pair ? m : m % kHalf); };
  const int64_t NB = (p.N + unit_rows - 1) / unit_rows;
  const int64_t units = num_tiles<NT>(p) * NB;
  const int64_t u_begin = units * blockIdx.x / gridDim.x;
  const int64_t u_end = units * (blockIdx.x + 1) / gridDim.x;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        tma_prefetch_desc(&p.tmap[m]);
        if (p.sb_tma) {
          tma_prefetch_desc(&p.tmap_sb[m][0]);
          tma_prefetch_desc(&p.tmap_sb[m][1]);
        }
      }
    }
    uint32_t it = 0;
    bool aborted = false;
    int64_t cur_tile = -1;
    TileInfo ti{};
    for (int64_t u = u_begin; u < u_end && !aborted; ++u) {
      if (u / NB != cur_tile) {  // the tile table is read once per tile
        cur_tile = u / NB;
        ti = tile_info<NT>(p, cur_tile);
      }
      const int64_t n0 = (u % NB) * unit_rows;
      const int64_t row0 = static_cast<int64_t>(ti.expert) * p.N + n0;
      for (int64_t ch = 0; ch < NCH; ++ch, ++it) {
        const int stage = it % C::STAGES;
        const uint32_t round = it / C::STAGES;
        if (round > 0 && !mbar_wait(&empty[stage], (round - 1) & 1, p.d_status)) {
          *abort_flag = 1;
        }
        if (*abort_flag) {
          aborted = true;
          break;
        }
        // test hook of the bounded waits: nothing lands in this stage, so its waits run out
        if (blockIdx.x == gridDim.x - 1 && static_cast<int64_t>(it) == p.skip_stage) continue;
        uint8_t* st = smem + stage * C::STAGE_BYTES;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], C::TMA_BYTES + (p.sb_tma ? C::SB_BYTES : 0u));
          if (p.code3d) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              tma_load_3d(st + m * C::BOXES * 2048, &p.tmap[blk_stack(m)], &full[stage], 0,
                          static_cast<int32_t>(row0 + blk_row(m)),
                          static_cast<int32_t>(ch * C::BOXES));
          } else {
            const int32_t xw = static_cast<int32_t>(ch * (C::CHUNK_ROW_BYTES / 4));
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
              for (int bx = 0; bx < C::BOXES; ++bx)
                tma_load_2d(st + (m * C::BOXES + bx) * 2048, &p.tmap[blk_stack(m)], &full[stage],
                            xw + bx * 32, static_cast<int32_t>(row0 + blk_row(m)));
          }
          if (p.sb_tma) {
            const int32_t xg = static_cast<int32_t>(ch * C::KB_PER_CHUNK);
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
              for (int arr = 0; arr < 2; ++arr)
                tma_load_2d(st + C::CODE_BYTES + (m * 2 + arr) * kRows * C::KB_PER_CHUNK * 2,
                            &p.tmap_sb[blk_stack(m)][arr], &full[stage], xg,
                            static_cast<int32_t>(row0 + blk_row(m)));
          }
        }
        if (p.sb_tma) continue;
        // scales and biases: [mat][s|b][16 rows][KB_PER_CHUNK] bf16
        const int64_t kb0 = ch * C::KB_PER_CHUNK;
        const int ngroups = static_cast<int>(imin64(C::KB_PER_CHUNK, KB_TOTAL - kb0));
        const int pieces = ngroups * 2 / p.sb_vec;
        // rows of each 16-row block inside [0, N): a unit's tail blocks may be short
        const int nrows = static_cast<int>(imin64(unit_rows, p.N - n0));
        const int tasks = NMAT * 2 * kRows * pieces;
        uint16_t* sb = reinterpret_cast<uint16_t*>(st + C::CODE_BYTES);
        for (int tk = lane; tk < tasks; tk += 32) {
          const int piece = tk % pieces;
          const int rr = (tk / pieces) % kRows;
          const int arr = (tk / (pieces * kRows)) % 2;
          const int m = tk / (pieces * kRows * 2);
          const int mrow = blk_row(m) + rr;  // row inside the unit (of its stack)
          if (mrow >= nrows) continue;
          const int sm = blk_stack(m);  // the weight stack
          const uint16_t* src = (arr ? p.biases[sm] : p.scales[sm]) + (row0 + mrow) * KB_TOTAL + kb0;
          uint16_t* dst = sb + ((m * 2 + arr) * kRows + rr) * C::KB_PER_CHUNK;
          const int off = piece * (p.sb_vec / 2);
          if (p.sb_vec == 16)
            cp_async<16>(dst + off, src + off);
          else if (p.sb_vec == 8)
            cp_async<8>(dst + off, src + off);
          else if (p.sb_vec == 4)
            cp_async<4>(dst + off, src + off);
          else
            dst[off] = src[off];  // odd group count: 2-byte pieces, plain copy
        }
        if (p.sb_vec == 2)
          mbar_arrive(&full[stage]);  // release: orders this lane's plain stores
        else
          cp_async_arrive_noinc(&full[stage]);
      }
    }
    if (aborted) {
      // Let every copy this CTA issued land before the CTA can exit.
      const uint32_t first = it > static_cast<uint32_t>(C::STAGES) ? it - C::STAGES : 0u;
      for (uint32_t k = first; k < it; ++k)
        mbar_wait(&full[k % C::STAGES], (k / C::STAGES) & 1, nullptr);
    }
    return;
  }

  if (warp == kConsumerWarps + 1) {
    // -------------------------------------------------------------- epilogue warp
    for (int64_t u = u_begin; u < u_end; ++u) {
      const uint32_t ui = static_cast<uint32_t>(u - u_begin), b = ui & 1;
      if (*abort_flag) break;
      if (!mbar_wait(&red_full[b], (ui >> 1) & 1, p.d_status)) {
        *abort_flag = 1;
        break;
      }
      const TileInfo ti = tile_info<NT>(p, u / NB);
      const int64_t n0 = (u % NB) * unit_rows;
      const float* ub = red + b * C::RED_SLICE;
      // one (token slot, row) entry per lane and pass; only the tile's valid rows
      for (int e = lane; e < static_cast<int>(ti.valid) * kRows; e += 32) {
        const int slot = e / kRows, row = e % kRows, nt = slot / 8, tok = slot % 8;
        float v[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          float sum = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w)
            sum += ub[(((w * NMAT + m) * NT + nt) * kRows + row) * 8 + tok];
          v[m] = sum;
        }
        const uint32_t pos = ti.row_start + slot;
        const uint32_t dr = p.dst_row ? p.dst_row[pos] : pos;
        uint16_t* yrow = p.y + static_cast<int64_t>(dr) * p.N;
        if (p.pair) {
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const int64_t n = n0 + kRows * m + row;
            if (n < p.N) yrow[n] = f32_to_bf16(v[m]);
          }
        } else {
#pragma unroll
          for (int h = 0; h < kHalf; ++h) {  // up block h and gate block kHalf + h
            const int64_t n = n0 + kRows * h + row;
            if (n < p.N) {
              const float gte = v[kHalf + h];
              yrow[n] = f32_to_bf16(v[h] * (gte / (1.0f + expf(-gte))));
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[b]);
    }
    if (lane == 0) prof_end(p.prof);  // the epilogue warp finishes the CTA's work
    return;
  }

  // ----------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const uint32_t ONES = 0x3F803F80u;  // bf16x2 (1, 1)
  // Activation values of one chunk for this lane: [k-block][token set][word]; 16 B per
  // 4-bit word (8 codes), 8 B per 8-bit word (4 codes).  Two buffers alternate: one is
  // consumed while the loads of the next chunk land in the other.
  using XV = typename std::conditional<BITS == 8, uint2, uint4>::type;
  using XBuf = XV[C::KB_PER_WARP][NT][C::WORDS * C::XW];
  XBuf xa, xb;

  // Shared-memory offsets of this lane, fixed for the kernel.  The warp's group i sits
  // CW*KB_BYTES bytes further along the chunk row: whole 128-byte column blocks, so
  // GROUP_STEP bytes further in the stage with the same swizzle phase.  Row g+8 sits
  // 1024 bytes after row g (same phase: the swizzle uses the row's low three bits).
  constexpr int GROUP_STRIDE = C::CW * C::KB_BYTES;
  static_assert(GROUP_STRIDE % 128 == 0, "a warp's groups must lie whole column blocks apart");
  constexpr uint32_t GROUP_STEP = GROUP_STRIDE / 128 * 2048;
  constexpr int PIECES = C::LANE_BYTES >= 16 ? C::LANE_BYTES / 16 : 1;
  uint32_t code_off[PIECES];
#pragma unroll
  for (int q = 0; q < PIECES; ++q)
    code_off[q] = swz(g, warp * C::KB_BYTES + t * C::LANE_BYTES + 16 * q);
  const int sb_off = g * C::KB_PER_CHUNK + warp;  // into each [16 rows][KB_PER_CHUNK] array
  const int x_off = warp * GS + t * (GS / 4);     // the lane's first activation of a chunk
  constexpr int64_t CHUNK_ELEMS = static_cast<int64_t>(C::KB_PER_CHUNK) * GS;

  // groups of chunk ch that lie inside [0, K/GS)
  auto chunk_groups = [&](int64_t ch) -> int {
    return static_cast<int>(imin64(C::KB_PER_CHUNK, KB_TOTAL - ch * C::KB_PER_CHUNK));
  };
  // This lane's activation pointers for unit u.  A token slot past the tile's valid rows
  // reads the tile's first row: its MMA column is never stored, so any finite values
  // serve, and the loads need no branch.
  auto tile_rows = [&](int64_t u, TileInfo& ti, const uint16_t* (&rows)[NT]) {
    ti = tile_info<NT>(p, u / NB);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t slot = g + 8 * nt;
      const uint32_t pos = ti.row_start + (slot < ti.valid ? slot : 0u);
      const uint32_t sr = p.src_row ? p.src_row[pos] : pos;
      rows[nt] = p.x + static_cast<int64_t>(sr) * p.K;
    }
  };
  // Issues the loads of chunk `ch` for the given rows into `dst`; a group past the chunk's
  // last one (never computed) reads the row's first activations, always in bounds.
  auto load_x = [&](const uint16_t* const (&rows)[NT], int64_t ch, XBuf& dst) {
    const int nkb = chunk_groups(ch);
#pragma unroll
    for (int i = 0; i < C::KB_PER_WARP; ++i) {
      const int64_t off = warp + C::CW * i < nkb ? ch * CHUNK_ELEMS + x_off + i * C::CW * GS : 0;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < C::WORDS * C::XW; ++j) {
          if constexpr (BITS != 8)  // 8 activations per vector, XW vectors per code word
            dst[i][nt][j] = ldg_nc_v4(rows[nt] + off + 8 * j);
          else
            dst[i][nt][j] = ldg_nc_v2(rows[nt] + off + 4 * j);
        }
    }
  };

  int64_t u = u_begin, ch = 0;
  uint32_t it = 0;
  TileInfo ti{}, ti_next{};
  const uint16_t* rows[NT];
  const uint16_t* rows_next[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) rows[nt] = rows_next[nt] = nullptr;
  float acc[NMAT][NT][4];
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[m][nt][i] = 0.f;
  if (u_begin < u_end) {
    tile_rows(u_begin, ti, rows);
    if (u_begin + 1 < u_end) tile_rows(u_begin + 1, ti_next, rows_next);
    load_x(rows, 0, xa);
  }

  // Hands the partial sums of unit u to the epilogue warp (valid token columns only).
  auto finish_unit = [&]() {
    const uint32_t ui = static_cast<uint32_t>(u - u_begin), b = ui & 1;
    if (ui >= 2 && !*abort_flag && !mbar_wait(&red_empty[b], ((ui >> 1) - 1) & 1, p.d_status))
      *abort_flag = 1;
    float* ub = red + b * C::RED_SLICE;
    if (!*abort_flag) {
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float* r = ub + (((warp * NMAT + m) * NT + nt) * kRows) * 8;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (static_cast<uint32_t>(nt * 8 + 2 * t + j) < ti.valid) {
              r[g * 8 + 2 * t + j] = acc[m][nt][j];
              r[(g + 8) * 8 + 2 * t + j] = acc[m][nt][2 + j];
            }
          }
        }
    }
    mbar_arrive(&red_full[b]);  // release: orders this lane's stores
#pragma unroll
    for (int m = 0; m < NMAT; ++m)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][nt][i] = 0.f;
  };

  // One chunk: its activations are in xc; the next chunk's loads go to xn.
  auto step = [&](XBuf& xc, XBuf& xn) {
    if (ch + 1 < NCH)
      load_x(rows, ch + 1, xn);
    else if (u + 1 < u_end)
      load_x(rows_next, 0, xn);
    const int nkb = chunk_groups(ch);
    const int stage = it % C::STAGES;
    bool ok = false;
    if (!*abort_flag) {
      ok = mbar_wait(&full[stage], (it / C::STAGES) & 1, p.d_status);
      if (!ok) *abort_flag = 1;
    }
    if (ok) {
      const uint8_t* st = smem + stage * C::STAGE_BYTES;
      const uint16_t* sb = reinterpret_cast<const uint16_t*>(st + C::CODE_BYTES) + sb_off;
#pragma unroll
      for (int i = 0; i < C::KB_PER_WARP; ++i) {
        if (warp + C::CW * i >= nkb) break;
        // ---- B operand: x values of this lane's codes, permuted to the MMA k order
        uint32_t bfr[NT][C::WORDS][C::MPW][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int j = 0; j < C::WORDS; ++j) {
            if constexpr (BITS == 2) {
              // 16 activations of a 16-code word: MMA m pairs codes (2m, 2m+8) and
              // (2m+1, 2m+9), the halves of component m of the two vectors
              const uint4 v0 = xc[i][nt][2 * j], v1 = xc[i][nt][2 * j + 1];
              const uint32_t c0[4] = {v0.x, v0.y, v0.z, v0.w}, c1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
              for (int mm = 0; mm < 4; ++mm) {
                bfr[nt][j][mm][0] = prmt(c0[mm], c1[mm], 0x5410);
                bfr[nt][j][mm][1] = prmt(c0[mm], c1[mm], 0x7632);
              }
            } else if constexpr (BITS == 4) {
              const uint4 v = xc[i][nt][j];
              bfr[nt][j][0][0] = prmt(v.x, v.z, 0x5410);
              bfr[nt][j][0][1] = prmt(v.x, v.z, 0x7632);
              bfr[nt][j][1][0] = prmt(v.y, v.w, 0x5410);
              bfr[nt][j][1][1] = prmt(v.y, v.w, 0x7632);
            } else {
              const uint2 v = xc[i][nt][j];
              bfr[nt][j][0][0] = prmt(v.x, v.y, 0x5410);
              bfr[nt][j][0][1] = prmt(v.x, v.y, 0x7632);
              bfr[nt][j][1][0] = bfr[nt][j][0][0];
              bfr[nt][j][1][1] = bfr[nt][j][0][1];
            }
          }
        }
        // ---- X = sum of x over the group (all-ones A operand)
        float cx[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int i2 = 0; i2 < 4; ++i2) cx[nt][i2] = 0.f;
          const uint32_t ones[4] = {ONES, ONES, ONES, ONES};
#pragma unroll
          for (int j = 0; j < C::WORDS; ++j) {
            // 8-bit codes reuse one activation pair for both nibbles: count it once
#pragma unroll
            for (int mm = 0; mm < (BITS == 8 ? 1 : C::MPW); ++mm)
              mma_bf16_16816(cx[nt], ones, bfr[nt][j][mm][0], bfr[nt][j][mm][1]);
          }
        }
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const uint8_t* cm = st + m * C::BOXES * 2048 + i * GROUP_STEP;
          uint32_t wg[C::WORDS], wg8[C::WORDS];
          if constexpr (C::LANE_BYTES == 4) {
            wg[0] = *reinterpret_cast<const uint32_t*>(cm + code_off[0]);
            wg8[0] = *reinterpret_cast<const uint32_t*>(cm + code_off[0] + 1024);
          } else if constexpr (C::LANE_BYTES == 8) {
            const uint2 a = *reinterpret_cast<const uint2*>(cm + code_off[0]);
            const uint2 b = *reinterpret_cast<const uint2*>(cm + code_off[0] + 1024);
            wg[0] = a.x; wg[1] = a.y; wg8[0] = b.x; wg8[1] = b.y;
          } else {
#pragma unroll
            for (int q = 0; q < PIECES; ++q) {
              const uint4 a = *reinterpret_cast<const uint4*>(cm + code_off[q]);
              const uint4 b = *reinterpret_cast<const uint4*>(cm + code_off[q] + 1024);
              wg[4 * q + 0] = a.x; wg[4 * q + 1] = a.y; wg[4 * q + 2] = a.z; wg[4 * q + 3] = a.w;
              wg8[4 * q + 0] = b.x; wg8[4 * q + 1] = b.y; wg8[4 * q + 2] = b.z; wg8[4 * q + 3] = b.w;
            }
          }
          float cacc[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2) cacc[nt][i2] = 0.f;
#pragma unroll
          for (int j = 0; j < C::WORDS; ++j) {
            uint32_t a[C::MPW][4];
            if constexpr (BITS == 2) {
              // pair i = (code i, code i+8) from the word shifted by 2i, as bf16 128 + q
              const uint32_t M2 = 0x00030003u, MAG = 0x43004300u;
#pragma unroll
              for (int mm = 0; mm < 4; ++mm) {
                a[mm][0] = and_or(wg[j] >> (4 * mm), M2, MAG);
                a[mm][1] = and_or(wg8[j] >> (4 * mm), M2, MAG);
                a[mm][2] = and_or(wg[j] >> (4 * mm + 2), M2, MAG);
                a[mm][3] = and_or(wg8[j] >> (4 * mm + 2), M2, MAG);
              }
            } else if constexpr (BITS == 4) {
              const uint32_t M4 = 0x000F000Fu, MAG = 0x43004300u;
              a[0][0] = and_or(wg[j], M4, MAG);
              a[0][1] = and_or(wg8[j], M4, MAG);
              a[0][2] = and_or(wg[j] >> 4, M4, MAG);
              a[0][3] = and_or(wg8[j] >> 4, M4, MAG);
              a[1][0] = and_or(wg[j] >> 8, M4, MAG);
              a[1][1] = and_or(wg8[j] >> 8, M4, MAG);
              a[1][2] = and_or(wg[j] >> 12, M4, MAG);
              a[1][3] = and_or(wg8[j] >> 12, M4, MAG);
            } else {
              const uint32_t M4 = 0x000F000Fu, LO = 0x43004300u, HI = 0x45004500u;
              a[0][0] = and_or(wg[j], M4, LO);
              a[0][1] = and_or(wg8[j], M4, LO);
              a[0][2] = and_or(wg[j] >> 8, M4, LO);
              a[0][3] = and_or(wg8[j] >> 8, M4, LO);
              a[1][0] = and_or(wg[j] >> 4, M4, HI);
              a[1][1] = and_or(wg8[j] >> 4, M4, HI);
              a[1][2] = and_or(wg[j] >> 12, M4, HI);
              a[1][3] = and_or(wg8[j] >> 12, M4, HI);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int mm = 0; mm < C::MPW; ++mm)
                mma_bf16_16816(cacc[nt], a[mm], bfr[nt][j][mm][0], bfr[nt][j][mm][1]);
          }
          // scales and biases of rows g and g+8 for this group
          const uint16_t* sm = sb + (m * 2) * kRows * C::KB_PER_CHUNK + C::CW * i;
          const uint16_t* bm = sm + kRows * C::KB_PER_CHUNK;
          const float s0 = bf16_to_f32(sm[0]);
          const float s1 = bf16_to_f32(sm[8 * C::KB_PER_CHUNK]);
          const float c0 = fmaf(-C::OFFSET, s0, bf16_to_f32(bm[0]));
          const float c1 = fmaf(-C::OFFSET, s1, bf16_to_f32(bm[8 * C::KB_PER_CHUNK]));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[m][nt][0] = fmaf(s0, cacc[nt][0], fmaf(c0, cx[nt][0], acc[m][nt][0]));
            acc[m][nt][1] = fmaf(s0, cacc[nt][1], fmaf(c0, cx[nt][1], acc[m][nt][1]));
            acc[m][nt][2] = fmaf(s1, cacc[nt][2], fmaf(c1, cx[nt][2], acc[m][nt][2]));
            acc[m][nt][3] = fmaf(s1, cacc[nt][3], fmaf(c1, cx[nt][3], acc[m][nt][3]));
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    ++it;
    if (++ch == NCH) {
      finish_unit();
      ch = 0;
      ++u;
      ti = ti_next;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) rows[nt] = rows_next[nt];
      if (u + 1 < u_end) tile_rows(u + 1, ti_next, rows_next);
    }
  };

  const int64_t steps = (u_end - u_begin) * NCH;
  // Two token sets with wide lanes hold too many live values for two inlined copies of
  // the step: there the next chunk's activations are moved into place instead.
  constexpr bool kAlternate = !(NT == 2 && C::LANE_BYTES >= 16);
  if constexpr (kAlternate) {
    for (int64_t k = 0; k < steps; k += 2) {
      step(xa, xb);
      if (k + 1 < steps) step(xb, xa);
    }
  } else {
    for (int64_t k = 0; k < steps; ++k) {
      step(xa, xb);
#pragma unroll
      for (int i = 0; i < C::KB_PER_WARP; ++i)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < C::WORDS; ++j) xa[i][nt][j] = xb[i][nt][j];
    }
  }
}

template <int BITS, int GS, int NMAT, int NT>
cudaError_t launch_cfg(QmvParams prm, const GemmArgs& a, cudaStream_t stream) {
  using C = Cfg<BITS, GS, NMAT, NT>;
  // Codes: one 3-D box (16 rows x BOXES column blocks of 128 B) per 16-row block when
  // the row is a whole number of column blocks, else BOXES 2-D boxes of 128 B x 16 rows.
  const int64_t words = a.K * a.bits / 32;
  prm.code3d = (words % 32 == 0) ? 1 : 0;
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
    cudaError_t e = prm.code3d
                        ? make_tmap_3d_u32_colblocks(&prm.tmap[m], wm.codes, words, a.E * a.N,
                                                     kRows, C::BOXES)
                        : make_tmap_2d_u32(&prm.tmap[m], wm.codes, words, a.E * a.N, 32, kRows,
                                           /*swizzle128=*/true);
    if (e != cudaSuccess) return e;
  }
  const int64_t gpr = a.K / GS;
  prm.sb_tma = (gpr % 8 == 0) ? 1 : 0;
  if (prm.sb_tma) {
    for (int m = 0; m < 2; ++m) {
      const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
      const uint16_t* arrs[2] = {wm.scales, wm.biases};
      for (int arr = 0; arr < 2; ++arr) {
        cudaError_t e = make_tmap_2d_bf16(&prm.tmap_sb[m][arr], arrs[arr], gpr, a.E * a.N,
                                          C::KB_PER_CHUNK, kRows, /*swizzle128=*/false);
        if (e != cudaSuccess) return e;
      }
    }
  }
  auto kern = qmv_kernel<BITS, GS, NMAT, NT>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM_BYTES + 1024);
  });
  if (attr_err != cudaSuccess) return attr_err;
  LaunchTimer timer(prm.pair ? "qmv" : "qmv_glu", stream);
  prm.prof = timer.slot();
  cudaError_t le = launch_pdl(kern, dim3(sm_count()), dim3(C::THREADS), C::SMEM_BYTES + 1024,
                              stream, prm);
  if (le != cudaSuccess) return le;
  count_launch();
  return cudaGetLastError();
}

template <int BITS, int GS>
cudaError_t launch_bits_gs(const QmvParams& prm, const GemmArgs& a, int nt, cudaStream_t stream) {
  // A unit is four 16-row blocks (four of one stack, or two of each of up and gate) for
  // routed tiles of one token set when the tile table's bound gives at least eight such
  // units per SM, else two (one of each stack, or two of one).  Four blocks spread each
  // unit's fixed work -- the partial-sum hand-off, the next tile's row pointers, the
  // activation fragments and group sums shared by the blocks -- over twice the weight
  // bytes; fewer, larger units would leave the SMs unevenly loaded at small batches, and
  // dense products need more units to fill the SMs.
  // (4-bit codes in groups of 64, the decode codec measured and tested with four blocks;
  // the other codecs keep two)
  constexpr bool kWide = BITS == 4 && GS == 64;
  if constexpr (kWide) {
    const int wide_rows = prm.pair ? 4 * kRows : 2 * kRows;  // channels of a four-block unit
    const int64_t wide_units = a.max_tiles * ((a.N + wide_rows - 1) / wide_rows);
    if (nt == 1 && a.dense_rows == 0 && wide_units >= 8 * sm_count())
      return launch_cfg<BITS, GS, 4, 1>(prm, a, stream);
  }
  return nt == 2 ? launch_cfg<BITS, GS, 2, 2>(prm, a, stream)
                 : launch_cfg<BITS, GS, 2, 1>(prm, a, stream);
}

}  // namespace

namespace {
std::atomic<int64_t> g_skip_stage{-1};
}  // namespace

int64_t take_skip_stage() { return g_skip_stage.exchange(-1); }

cudaError_t launch_qmv(const GemmArgs& a, cudaStream_t stream) {
  QmvParams prm{};
  prm.pair = a.nmat == 2 ? 0 : 1;
  for (int m = 0; m < 2; ++m) {
    const QWeight& wm = a.w[a.nmat == 2 ? m : 0];
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
  prm.early_weights = (a.dense_rows > 0 || a.tiles_ready) ? 1 : 0;
  prm.skip_stage = take_skip_stage();
  prm.N = a.N;
  prm.K = a.K;
  prm.E = a.E;
  const int64_t gpr = a.K / a.group;
  prm.sb_vec = (gpr % 8 == 0) ? 16 : (gpr % 4 == 0) ? 8 : (gpr % 2 == 0) ? 4 : 2;
  prm.d_status = a.d_status;
  const int nt = a.bm > 8 ? 2 : 1;
  if (a.bits == 2) {  // groups of 64 or 128 (a lane's share of a group is whole words)
    if (a.group == 64) return launch_bits_gs<2, 64>(prm, a, nt, stream);
    return launch_bits_gs<2, 128>(prm, a, nt, stream);
  }
  if (a.bits == 4) {
    if (a.group == 32) return launch_bits_gs<4, 32>(prm, a, nt, stream);
    if (a.group == 64) return launch_bits_gs<4, 64>(prm, a, nt, stream);
    return launch_bits_gs<4, 128>(prm, a, nt, stream);
  }
  if (a.group == 32) return launch_bits_gs<8, 32>(prm, a, nt, stream);
  if (a.group == 64) return launch_bits_gs<8, 64>(prm, a, nt, stream);
  return launch_bits_gs<8, 128>(prm, a, nt, stream);
}

}  // namespace qmoe

extern "C" int qmoe_debug_skip_stage(int64_t stage) {
  qmoe::g_skip_stage.store(stage < 0 ? -1 : stage);
  return QMOE_OK;
}
