// Host helpers that encode TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so the library needs no -lcuda).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace qmoe {

// Row-major 2-D tensor of uint32 words: `inner` words per row, `rows` rows, row
// pitch inner*4 bytes.  Box = box_inner words x box_rows rows; 128-byte swizzle
// when `swizzle128` (box_inner*4 must then be 128).  Out-of-range boxes read zeros.
cudaError_t make_tmap_2d_u32(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                             int box_inner, int box_rows, bool swizzle128);
// Same for bf16 elements (box_inner*2 must be 128 with the swizzle).
cudaError_t make_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                              int box_inner, int box_rows, bool swizzle128);
// The same row-major uint32 matrix ([rows, words] words, row pitch words*4 bytes,
// words a multiple of 32) seen as 3-D: (word within a 128-byte column block,
// row, column block).  A box of box_rows rows x box_blocks column blocks lands in
// shared memory as [block][row][128 bytes], each 128-byte line swizzled by the
// row's low three bits, i.e. the layout of box_blocks separate 2-D boxes of
// 32 words x box_rows rows placed one after another; column blocks past the last
// one read zeros.
cudaError_t make_tmap_3d_u32_colblocks(CUtensorMap* map, const void* base, int64_t words,
                                       int64_t rows, int box_rows, int box_blocks);

}  // namespace qmoe
