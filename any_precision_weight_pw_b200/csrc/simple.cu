// simple.cu -- CUDA-core dequant-GEMV for any block shape.
//
// One warp per output row: the lanes split the row's 32-column words, unpack
// the b-bit codes from the top b bit-planes, gather the row's LUT entries and
// accumulate in fp32 for up to 8 tokens at a time, then reduce across the
// warp.  This path handles every shape (the tensor-core path needs widths
// that are multiples of 128) and serves as a second GPU implementation in the
// tests.
//
// PagedWeight (legiblepapers summary, FAQ Q5): the kernel reads bit-planes
// and lookup tables directly, with a different bitwidth per linear-block.
#include <cuda_fp16.h>

#include "pages.h"
#include "pw_internal.h"

namespace pw {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;
constexpr int kTok = 8;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float bf16f(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float half_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Input value of "token" position n at column c for the three modes.
struct InputRow {
  const uint16_t* xb;  // bf16 row (modes 0, 2)
  const float* g;      // gate row (mode 1)
  const float* u;      // up row (mode 1)
  __device__ __forceinline__ float at(int c) const {
    if (xb) return bf16f(xb[c]);
    const float gv = g[c];
    return gv / (1.0f + expf(-gv)) * u[c];  // SwiGLU activation of the expert
  }
};

__global__ void __launch_bounds__(kWarps * 32) simple_kernel(const SimpleParams p) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int mode = p.mode;

  // Which block, rows, cols and token range this CTA serves.
  int blk = 0, rows, cols, bits, pos0, n_tok, n_max;
  const uint32_t* planes;
  const uint16_t* lut;
  int group = 0, proj = 0;
  if (mode == 2) {
    rows = p.lin_rows;
    cols = p.lin_cols;
    bits = p.lin_bits;
    n_max = p.lin_n_max;
    planes = p.lin_planes;
    lut = p.lin_lut;
    pos0 = 0;
    n_tok = p.T;
  } else {
    group = (mode == 0) ? (blockIdx.y >> 1) : blockIdx.y;
    proj = (mode == 0) ? (blockIdx.y & 1) : 2;
    blk = 3 * group + proj;
    const int Fg = (group == p.E) ? p.S : p.F;
    rows = (proj < 2) ? Fg : p.H;
    cols = (proj < 2) ? p.H : Fg;
    bits = p.pt.bits[blk];
    n_max = p.pt.stride[blk];
    planes = p.pt.blk[blk].planes;
    lut = p.pt.blk[blk].lut;
    pos0 = p.offsets[group];
    n_tok = p.offsets[group + 1] - pos0;
  }
  const int row0 = blockIdx.x * kRowsPerCta;
  if (row0 >= rows || n_tok <= 0) return;
  const int words = (cols + 31) >> 5;
  const int Fg = (mode == 1) ? cols : rows;

  for (int tb = 0; tb < n_tok; tb += kTok) {
    const int nt = min(kTok, n_tok - tb);
    InputRow in[kTok];
#pragma unroll
    for (int j = 0; j < kTok; ++j) {
      const int pos = pos0 + tb + min(j, nt - 1);
      if (mode == 2) {
        in[j] = {p.x + static_cast<size_t>(tb + min(j, nt - 1)) * cols, nullptr, nullptr};
      } else if (mode == 0) {
        in[j] = {p.x + static_cast<size_t>(p.slot_token[pos]) * p.H, nullptr, nullptr};
      } else {
        const float* gr = p.gu + static_cast<size_t>(pos) * p.gu_stride;
        in[j] = {nullptr, gr, gr + Fg};
      }
    }
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int o = row0 + warp * kRowsPerWarp + rr;
      if (o >= rows) break;
      float acc[kTok];
#pragma unroll
      for (int j = 0; j < kTok; ++j) acc[j] = 0.0f;
      const uint16_t* lrow = lut + (static_cast<size_t>(o) << bits);
      for (int w = lane; w < words; w += 32) {
        uint32_t pw_[PW_MAX_BITS];
        for (int k = 0; k < bits; ++k)
          pw_[k] = planes[pages::word_index(k, o, w, rows, cols, n_max)];
        const int cmax = min(32, cols - 32 * w);
        for (int c = 0; c < cmax; ++c) {
          int code = 0;
          for (int k = 0; k < bits; ++k) code = (code << 1) | ((pw_[k] >> c) & 1u);
          const float wv = half_bits_to_f32(lrow[code]);
          const int col = 32 * w + c;
#pragma unroll
          for (int j = 0; j < kTok; ++j)
            if (j < nt) acc[j] = fmaf(wv, in[j].at(col), acc[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < kTok; ++j) {
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc[j] += __shfl_xor_sync(kFull, acc[j], m);
      }
      if (lane == 0) {
        for (int j = 0; j < nt; ++j) {
          const int pos = pos0 + tb + j;
          if (mode == 0) {
            p.gu[static_cast<size_t>(pos) * p.gu_stride + proj * rows + o] = acc[j];
          } else if (mode == 1) {
            p.ysorted[static_cast<size_t>(pos) * p.H + o] = p.slot_w[pos] * acc[j];
          } else {
            p.y[static_cast<size_t>(tb + j) * rows + o] = acc[j];
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_simple(const SimpleParams& p, int grid_rows, cudaStream_t s) {
  dim3 grid((grid_rows + kRowsPerCta - 1) / kRowsPerCta,
            p.mode == 0 ? 2 * p.n_groups : (p.mode == 1 ? p.n_groups : 1));
  simple_kernel<<<grid, kWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace pw
