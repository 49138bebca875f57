// repack.cu -- convert row-major bit-planes [n_max][rows][words] into the
// paged layout of pages.h (one thread per destination word, pads zero).
#include "pages.h"
#include "pw_internal.h"

namespace pw {
namespace {

__global__ void repack_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                              int rows, int cols, int n_planes) {
  // destination word i: group g = i / (n_planes * 1024), plane k, tile word
  const int words = pages::words_of(cols);
  const int n_rt = pages::row_tiles(rows), n_kt = pages::k_tiles(cols);
  const int64_t total = static_cast<int64_t>(n_planes) * n_rt * n_kt * (pages::kTileBytes / 4);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = i / (pages::kTileBytes / 4);  // (group, plane)
    const int within = static_cast<int>(i % (pages::kTileBytes / 4));
    const int r = within >> 3, slot = within & 7;
    const int h = (slot >> 2) ^ ((r >> 2) & 1);
    const int j = 4 * h + (slot & 3);
    const int k = static_cast<int>(tile % n_planes);
    const int64_t grp = tile / n_planes;
    const int kt = static_cast<int>(grp % n_kt);
    const int rt = static_cast<int>(grp / n_kt);
    const int o = rt * pages::kTileRows + r, w = kt * pages::kTileWords + j;
    dst[i] = (o < rows && w < words)
                 ? src[(static_cast<int64_t>(k) * rows + o) * words + w]
                 : 0u;
  }
}

}  // namespace

cudaError_t launch_repack(const uint32_t* src, uint32_t* dst, int rows, int cols, int n_planes,
                          cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(n_planes) * pages::plane_words(rows, cols);
  int grid = static_cast<int>((total + 255) / 256);
  if (grid > 65535) grid = 65535;
  if (grid < 1) grid = 1;
  repack_kernel<<<grid, 256, 0, s>>>(src, dst, rows, cols, n_planes);
  return cudaGetLastError();
}

}  // namespace pw
