// pages.h -- the paged bit-plane layout the CUDA library reads.
//
// PagedWeight (arxivlens abstract; legiblepapers "Summary & Methodology
// Analysis"): the Any-Precision bit-planes of a linear-block are GPU-resident
// pages that the kernel reads directly and that move one plane at a time.
// The pages fix no memory layout.  This library tiles a block's n_max planes
// so that the b active planes of one (128 rows x 256 columns) piece are one
// contiguous run of b * 4 KB, which the tensor-core kernel stages with a
// single bulk copy (copies below ~16 KB are limited by the copy engine's
// per-operation cost, not by bytes):
//
//   a rows x cols block (words = ceil(cols / 32)) has n_rt * n_kt tile
//   groups, n_rt = ceil(rows / 128), n_kt = ceil(words / 8); group (rt, kt)
//   holds n_max tiles of 4096 bytes, plane k's tile at byte
//   ((rt * n_kt + kt) * n_max + k) * 4096.  A tile holds rows 128 rt + r
//   (r < 128) and words 8 kt + j (j < 8) of its plane, zero past the block;
//   word j of row r sits at byte 32 r + 16 * (h ^ ((r >> 2) & 1)) +
//   4 * (j & 3), h = j >> 2 (the two 16-byte halves of a row swap on rows
//   with bit 2 set, so 32 threads reading one row each hit distinct
//   shared-memory banks).
//
// A b-bit view reads planes 0..b-1: the first b tiles of every group.  Plane
// k (one page) is the k-th tile of every group: a strided run that one 2-D
// copy moves.  Within a word, bit (i % 32) is column i and plane 0 is the
// most significant code bit, as in the row-major layout [plane][rows][words]
// that pw_repack_planes converts from.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define PW_PG_HD __host__ __device__ __forceinline__
#else
#define PW_PG_HD inline
#endif

namespace pw {
namespace pages {

constexpr int kTileRows = 128;
constexpr int kTileWords = 8;
constexpr int kTileBytes = kTileRows * kTileWords * 4;

PW_PG_HD int words_of(int cols) { return (cols + 31) >> 5; }
PW_PG_HD int row_tiles(int rows) { return (rows + kTileRows - 1) / kTileRows; }
PW_PG_HD int k_tiles(int cols) { return (words_of(cols) + kTileWords - 1) / kTileWords; }
// tile groups of a block (each n_max tiles)
PW_PG_HD int64_t groups_of(int rows, int cols) {
  return static_cast<int64_t>(row_tiles(rows)) * k_tiles(cols);
}
// uint32 words of one plane (one page): one tile per group
PW_PG_HD int64_t plane_words(int rows, int cols) {
  return groups_of(rows, cols) * (kTileBytes / 4);
}
// uint32 index of word w of row o of plane k
PW_PG_HD int64_t word_index(int k, int o, int w, int rows, int cols, int n_max) {
  const int rt = o / kTileRows, r = o % kTileRows;
  const int kt = w / kTileWords, j = w % kTileWords;
  const int64_t tile = (static_cast<int64_t>(rt) * k_tiles(cols) + kt) * n_max + k;
  const int h = (j >> 2) ^ ((r >> 2) & 1);
  return tile * (kTileBytes / 4) + r * 8 + h * 4 + (j & 3);
}

}  // namespace pages
}  // namespace pw
