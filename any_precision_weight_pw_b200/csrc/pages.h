// pages.h -- the paged bit-plane layout the CUDA library reads.
//
// PagedWeight (arxivlens abstract; legiblepapers "Summary & Methodology
// Analysis"): the Any-Precision bit-planes of a linear-block are GPU-resident
// pages that the kernel reads directly and that are moved one plane at a time.
// The pages fix no memory layout.  This library stores each plane as a page
// of 4 KB tiles so that every (plane, 128 rows, 256 columns) piece the
// tensor-core kernel stages is one contiguous 4 KB copy:
//
//   plane k of a rows x cols block (words = ceil(cols / 32)) is a page of
//   n_rt * n_kt tiles, n_rt = ceil(rows / 128), n_kt = ceil(words / 8);
//   tile (rt, kt) starts at byte ((k * n_rt + rt) * n_kt + kt) * 4096 and
//   holds rows 128 rt + r (r < 128) and words 8 kt + j (j < 8), zero past the
//   block; word j of row r sits at byte 32 r + 16 * (h ^ ((r >> 2) & 1)) +
//   4 * (j & 3), h = j >> 2 (the two 16-byte halves of a row are swapped on
//   rows with bit 2 set, so that 32 threads reading one row each hit distinct
//   shared-memory banks).
//
// Within a word, bit (i % 32) is column i and plane 0 is the most
// significant code bit, exactly as in the row-major layout [plane][rows][words]
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
// uint32 words in one plane page
PW_PG_HD int64_t plane_words(int rows, int cols) {
  return static_cast<int64_t>(row_tiles(rows)) * k_tiles(cols) * (kTileBytes / 4);
}
// uint32 index of word w of row o of plane k
PW_PG_HD int64_t word_index(int k, int o, int w, int rows, int cols) {
  const int rt = o / kTileRows, r = o % kTileRows;
  const int kt = w / kTileWords, j = w % kTileWords;
  const int64_t tile = (static_cast<int64_t>(k) * row_tiles(rows) + rt) * k_tiles(cols) + kt;
  const int h = (j >> 2) ^ ((r >> 2) & 1);
  return tile * (kTileBytes / 4) + r * 8 + h * 4 + (j & 3);
}

}  // namespace pages
}  // namespace pw
