// gv.cu -- CUDA-core dequant-GEMV passes for decode batches with few tokens
// per expert.
//
// PagedWeight (legiblepapers summary, FAQ Q5; arxivlens abstract): the fused
// MoE kernel reads the bit-planes and per-row LUTs of the resident pages
// directly, at a separate bitwidth per linear-block, with the expert
// activation and the routing-weighted output fused in.  With one or two
// tokens per expert a tensor-core tile carries almost no useful columns and
// a persistent one-CTA-per-SM pipeline has too few items to fill the GPU, so
// small batches take these passes instead: many small CTAs stream the plane
// pages straight into registers, dequantise on the CUDA cores through LUT
// tables in shared memory, and accumulate in fp32 (packed two-lane fp32
// fused multiply-adds).
//
//   gather   x_gv[pos] = the token's activations in fp32, each 32-column
//            group in the dequantiser's K order, zero past H.
//   gate/up  one item = 32 rows of one group's gate and up blocks x up to 4
//            of its tokens: warps 0-3 take the gate rows, warps 4-7 the up
//            rows, lane = row, the four warps of a projection splitting the
//            256-column tile groups; per-warp sums meet in shared memory in a
//            fixed order, then h = silu(g) u goes to h_gv in the down pass's
//            K order (zero past F).
//   down     one item = 32 rows of a group's down block x one K split x up
//            to 4 tokens; the eight warps split the split's tile groups; the
//            routing-weighted partial goes to ysorted[split] and the combine
//            kernel sums the splits in order.
// Lookup tables (dequant.cuh): pair tables up to b = 4 (one 32-bit load per
// two weights), single tables above, row-interleaved so a warp's 32 rows hit
// 32 banks; entry (code, row) of a 32-row table at code * 128 + 4 row.
// Items are visited with a grid-stride loop; everything each CTA does is
// fixed by the routing, so results are the same on every run.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dequant.cuh"
#include "pages.h"
#include "pw_internal.h"

namespace pw {
namespace {

constexpr int kGvThreads = 256;             // 8 warps
constexpr int kGvRows = 32;                 // output rows per item (lane = row)
constexpr int kGvTok = 4;                   // tokens per item
constexpr uint32_t kGvTab = 32768;          // one projection's tables
constexpr uint32_t kGvRed = 8 * 32 * kGvTok * 4;  // per-warp sums
constexpr uint32_t kGvSmemGateUp = 2 * kGvTab + kGvRed;
constexpr uint32_t kGvSmemDown = kGvTab + kGvRed;

extern __shared__ __align__(16) uint8_t gv_smem[];

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// acc (two fp32 lanes) += w * x, each lane a correctly rounded fused
// multiply-add.
__device__ __forceinline__ void fma2(unsigned long long& acc, unsigned long long w,
                                     unsigned long long x) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(w), "l"(x));
}
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return static_cast<unsigned long long>(__float_as_uint(lo)) |
         (static_cast<unsigned long long>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo_of(unsigned long long v) {
  return __uint_as_float(static_cast<uint32_t>(v));
}
__device__ __forceinline__ float hi_of(unsigned long long v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}

// Items of one pass: per group, row tiles x K splits x token chunks.
struct GvItem {
  int g, rt, split, pos0, nt, rows;
};

// Item prefix over the groups (thread 0 fills pre[0..G]).
__device__ void gv_prefix(const GvParams& p, bool down, int* pre) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int g = 0; g < p.n_groups; ++g) {
      pre[g] = acc;
      const int n = p.offsets[g + 1] - p.offsets[g];
      const int rows = down ? p.H : (g == p.E ? p.S : p.F);
      const int ns = down ? p.n_split : 1;
      acc += ((rows + kGvRows - 1) / kGvRows) * ns * ((n + kGvTok - 1) / kGvTok);
    }
    pre[p.n_groups] = acc;
  }
}

__device__ __forceinline__ GvItem gv_item(const GvParams& p, bool down, const int* pre, int i) {
  int g = 0;
  while (g + 1 < p.n_groups && pre[g + 1] <= i) ++g;
  GvItem it;
  it.g = g;
  const int n = p.offsets[g + 1] - p.offsets[g];
  it.rows = down ? p.H : (g == p.E ? p.S : p.F);
  const int ns = down ? p.n_split : 1;
  const int n_tc = (n + kGvTok - 1) / kGvTok;
  int local = i - pre[g];
  const int tc = local % n_tc;
  local /= n_tc;
  it.split = local % ns;
  it.rt = local / ns;
  it.pos0 = p.offsets[g] + kGvTok * tc;
  it.nt = min(kGvTok, n - kGvTok * tc);
  return it;
}

// One projection's table for rows o0 .. o0 + 31 (lane = row), written by the
// four warps of the projection (part = warp index among them).
template <int B>
__device__ void gv_install(uint32_t tab, const uint16_t* lut, int o, bool live, int part,
                           int lane) {
  if (!live) return;
  const uint16_t* row = lut + (static_cast<size_t>(o) << B);
  if constexpr (B <= dq::pair_max(true)) {
    // pair entry (v1, v2) = LUT[v1] | LUT[v2] << 16 at byte ((v1 << B) | v2)
    uint32_t v[1 << B];
#pragma unroll
    for (int c = 0; c < (1 << B); ++c) v[c] = row[c];
#pragma unroll
    for (int v1 = 0; v1 < (1 << B); ++v1)
#pragma unroll
      for (int v2 = 0; v2 < (1 << B); ++v2) {
        const int byte = (v1 << B) | v2;
        if ((byte & 3) == part)
          *reinterpret_cast<uint32_t*>(gv_smem + tab + byte * 128 + 4 * lane) =
              v[v1] | (v[v2] << 16);
      }
  } else {
    // single entry v in the low half of the 32-bit slot at v * 128 + 4 row
    const uint4* src = reinterpret_cast<const uint4*>(row);
#pragma unroll
    for (int c = 0; c < (1 << B) / 8; ++c) {
      if ((c & 3) != part) continue;
      const uint4 q = src[c];
      const uint32_t e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint16_t*>(gv_smem + tab + (8 * c + u) * 128 + 4 * lane) =
            static_cast<uint16_t>(u & 1 ? e[u >> 1] >> 16 : e[u >> 1]);
    }
  }
}

// Sum over the tile groups kt = kt0, kt0 + step, ... < kt1 of row o's
// dequantised weights times the tokens' activations (x rows of ldx floats
// in the dequantiser's K order); acc[t] holds two partial lanes per token.
// A row's 8 words of a plane are two 16-byte halves (swapped on rows with
// bit 2 set); each half is loaded and consumed in turn.
template <int B>
__device__ void gv_rows(const uint32_t* planes, int stride, int o, int rows, int cols, uint32_t tab,
                        int kt0, int kt1, int step, const float* x, int ldx, int nt,
                        unsigned long long (&acc)[kGvTok], int lane) {
  auto lds32 = [tab](uint32_t a) -> uint32_t {
    return *reinterpret_cast<const uint32_t*>(gv_smem + tab + (a >> 1));
  };
  auto lds16 = [tab](uint32_t a) -> uint32_t {
    return *reinterpret_cast<const uint16_t*>(gv_smem + tab + (a >> 1));
  };
  const int n_kt = pages::k_tiles(cols);
  const int rt = o / pages::kTileRows, rr = o % pages::kTileRows;
  const int sw = (rr >> 2) & 1;
  const bool live = o < rows;
  for (int kt = kt0; kt < kt1; kt += step) {
    const uint8_t* tile = reinterpret_cast<const uint8_t*>(
        planes + (static_cast<int64_t>(rt) * n_kt + kt) * stride * (pages::kTileBytes / 4));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t W[B][4];
#pragma unroll
      for (int k = 0; k < B; ++k) {
        uint4 c = make_uint4(0u, 0u, 0u, 0u);
        if (live)
          c = *reinterpret_cast<const uint4*>(tile + k * pages::kTileBytes + 32 * rr +
                                              16 * (half ^ sw));
        W[k][0] = c.x;
        W[k][1] = c.y;
        W[k][2] = c.z;
        W[k][3] = c.w;
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t P[B];
#pragma unroll
        for (int k = 0; k < B; ++k) P[k] = W[k][jj];
        uint32_t out[16];
        if constexpr (B <= dq::pair_max(true))
          dq::dq_word_pair<B, true>(P, static_cast<uint32_t>(2 * lane), lds32, out);
        else
          dq::dq_word_single<B, true>(P, static_cast<uint32_t>(2 * lane), lds16, out);
        const int col = kt * 256 + 32 * (4 * half + jj);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          // pair registers 2q and 2q + 1 against four activations per token
          const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&out[2 * q]));
          const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&out[2 * q + 1]));
          const unsigned long long wa = pack2(fa.x, fa.y), wb = pack2(fb.x, fb.y);
#pragma unroll
          for (int t = 0; t < kGvTok; ++t) {
            if (t >= nt) break;
            const ulonglong2 xv =
                reinterpret_cast<const ulonglong2*>(x + static_cast<size_t>(t) * ldx + col)[q];
            fma2(acc[t], wa, xv.x);
            fma2(acc[t], wb, xv.y);
          }
        }
      }
    }
  }
}

// Dispatch on the bitwidth (templates up to PW_MAX_BITS).
#define PW_GV_SWITCH(b, CALL) \
  switch (b) {                \
    case 1: CALL(1); break;   \
    case 2: CALL(2); break;   \
    case 3: CALL(3); break;   \
    case 4: CALL(4); break;   \
    case 5: CALL(5); break;   \
    case 6: CALL(6); break;   \
    case 7: CALL(7); break;   \
    default: CALL(8); break;  \
  }

__global__ void gv_gather_kernel(const GvParams p) {
  pdl_wait();
  pdl_trigger();
  const int P = p.offsets[p.n_groups];
  const int wpr = p.H_pad >> 5;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < P * wpr;
       idx += gridDim.x * blockDim.x) {
    const int pos = idx / wpr, w = idx - pos * wpr;
    float4* dst = reinterpret_cast<float4*>(p.x_gv + static_cast<size_t>(pos) * p.H_pad + 32 * w);
    if (32 * w >= p.H) {
      for (int q = 0; q < 8; ++q) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const uint16_t* row = p.x + static_cast<size_t>(p.slot_token[pos]) * p.H + 32 * w;
    float v[32];
    if (32 * w + 32 <= p.H) {
      const uint4* src = reinterpret_cast<const uint4*>(row);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 r = src[q];
        const uint32_t r4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * q + 2 * e] = bf16_to_f32(static_cast<uint16_t>(r4[e] & 0xFFFFu));
          v[8 * q + 2 * e + 1] = bf16_to_f32(static_cast<uint16_t>(r4[e] >> 16));
        }
      }
    } else {
      // the row's last, partial 32-column group: zero past H
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = (32 * w + c < p.H) ? bf16_to_f32(row[c]) : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      dst[q] = make_float4(v[dq::col_of_kpos(4 * q)], v[dq::col_of_kpos(4 * q + 1)],
                           v[dq::col_of_kpos(4 * q + 2)], v[dq::col_of_kpos(4 * q + 3)]);
  }
}

__global__ void __launch_bounds__(kGvThreads, 3) gv_gateup_kernel(const __grid_constant__ GvParams p) {
  __shared__ int pre[kMaxGroups + 2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int proj = warp >> 2, part = warp & 3;
  float* red = reinterpret_cast<float*>(gv_smem + 2 * kGvTab);  // [8][32][kGvTok]
  pdl_wait();
  gv_prefix(p, false, pre);
  __syncthreads();
  const int total = pre[p.n_groups];
  for (int i = blockIdx.x; i < total; i += gridDim.x) {
    const GvItem it = gv_item(p, false, pre, i);
    const int o = kGvRows * it.rt + lane;
    const bool live = o < it.rows;
    const int blk = 3 * it.g + proj;
    const int b = p.pt.bits[blk];
    const uint32_t tab = proj * kGvTab;
    __syncthreads();  // the previous item's tables and sums are no longer read
#define PW_GV_INSTALL(BB) gv_install<BB>(tab, p.pt.blk[blk].lut, o, live, part, lane)
    PW_GV_SWITCH(b, PW_GV_INSTALL)
#undef PW_GV_INSTALL
    __syncthreads();
    unsigned long long acc[kGvTok];
#pragma unroll
    for (int t = 0; t < kGvTok; ++t) acc[t] = 0ull;
    const float* x = p.x_gv + static_cast<size_t>(it.pos0) * p.H_pad;
    const int n_kt = pages::k_tiles(p.H);
#define PW_GV_ROWS(BB)                                                                       \
  gv_rows<BB>(p.pt.blk[blk].planes, p.pt.stride[blk], o, it.rows, p.H, tab, part, n_kt, 4, x, \
              p.H_pad, it.nt, acc, lane)
    PW_GV_SWITCH(b, PW_GV_ROWS)
#undef PW_GV_ROWS
#pragma unroll
    for (int t = 0; t < kGvTok; ++t)
      red[(warp * 32 + lane) * kGvTok + t] = lo_of(acc[t]) + hi_of(acc[t]);
    __syncthreads();
    // h = silu(g) * u per (row, token); gate sums from warps 0-3, up from 4-7,
    // in warp order
    if (threadIdx.x < 32 * kGvTok) {
      const int r = threadIdx.x & 31, t = threadIdx.x >> 5;
      const int orow = kGvRows * it.rt + r;
      if (t < it.nt && orow < it.rows) {
        float g = 0.0f, u = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          g += red[(w * 32 + r) * kGvTok + t];
          u += red[((4 + w) * 32 + r) * kGvTok + t];
        }
        const float h = g / (1.0f + expf(-g)) * u;
        const int col = (orow & ~31) + dq::kpos_of_col(orow & 31);
        p.h_gv[static_cast<size_t>(it.pos0 + t) * p.F_pad + col] = h;
      }
    }
    // the row tile that ends the block also clears the pad columns up to the
    // next 256, which the down pass's last tile group reads
    const int end = (it.rows + 255) & ~255;
    if (kGvRows * (it.rt + 1) >= it.rows)
      for (int j = it.rows + threadIdx.x; j < end; j += kGvThreads)
        for (int t = 0; t < it.nt; ++t)
          p.h_gv[static_cast<size_t>(it.pos0 + t) * p.F_pad + j] = 0.0f;
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(kGvThreads, 3) gv_down_kernel(const __grid_constant__ GvParams p) {
  __shared__ int pre[kMaxGroups + 2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* red = reinterpret_cast<float*>(gv_smem + kGvTab);  // [8][32][kGvTok]
  pdl_wait();
  gv_prefix(p, true, pre);
  __syncthreads();
  const int total = pre[p.n_groups];
  for (int i = blockIdx.x; i < total; i += gridDim.x) {
    const GvItem it = gv_item(p, true, pre, i);
    const int o = kGvRows * it.rt + lane;
    const bool live = o < it.rows;
    const int blk = 3 * it.g + 2;
    const int b = p.pt.bits[blk];
    const int Fg = it.g == p.E ? p.S : p.F;
    const int n_kt = pages::k_tiles(Fg);
    const int kt0 = n_kt * it.split / p.n_split, kt1 = n_kt * (it.split + 1) / p.n_split;
    __syncthreads();
    // warps 0-3 write the table (a quarter of the entries each)
    if (warp < 4) {
#define PW_GV_INSTALL(BB) gv_install<BB>(0u, p.pt.blk[blk].lut, o, live, warp, lane)
      PW_GV_SWITCH(b, PW_GV_INSTALL)
#undef PW_GV_INSTALL
    }
    __syncthreads();
    unsigned long long acc[kGvTok];
#pragma unroll
    for (int t = 0; t < kGvTok; ++t) acc[t] = 0ull;
    const float* x = p.h_gv + static_cast<size_t>(it.pos0) * p.F_pad;
#define PW_GV_ROWS(BB)                                                                        \
  gv_rows<BB>(p.pt.blk[blk].planes, p.pt.stride[blk], o, it.rows, Fg, 0u, kt0 + warp, kt1, 8, x, \
              p.F_pad, it.nt, acc, lane)
    PW_GV_SWITCH(b, PW_GV_ROWS)
#undef PW_GV_ROWS
#pragma unroll
    for (int t = 0; t < kGvTok; ++t)
      red[(warp * 32 + lane) * kGvTok + t] = lo_of(acc[t]) + hi_of(acc[t]);
    __syncthreads();
    if (threadIdx.x < 32 * kGvTok) {
      const int r = threadIdx.x & 31, t = threadIdx.x >> 5;
      const int orow = kGvRows * it.rt + r;
      if (t < it.nt && orow < it.rows) {
        float y = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) y += red[(w * 32 + r) * kGvTok + t];
        const int pos = it.pos0 + t;
        p.ysorted[it.split * p.split_stride + static_cast<size_t>(pos) * p.H + orow] =
            p.slot_w[pos] * y;
      }
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_gv(const GvParams& p, int pass, int max_rows, int n_sm, cudaStream_t s) {
  if (pass == 0) {
    const int threads = 256;
    int grid = (max_rows * (p.H_pad >> 5) + threads - 1) / threads;
    if (grid > 4 * n_sm) grid = 4 * n_sm;
    if (grid < 1) grid = 1;
    return launch_pdl(gv_gather_kernel, dim3(grid), dim3(threads), 0, s, p);
  }
  // the dynamic shared memory attribute is set on every launch (a cheap host
  // call that keeps no per-device state)
  if (pass == 1) {
    cudaError_t e = cudaFuncSetAttribute(gv_gateup_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGvSmemGateUp));
    if (e != cudaSuccess) return e;
    return launch_pdl(gv_gateup_kernel, dim3(3 * n_sm), dim3(kGvThreads), kGvSmemGateUp, s, p);
  }
  cudaError_t e = cudaFuncSetAttribute(gv_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGvSmemDown));
  if (e != cudaSuccess) return e;
  return launch_pdl(gv_down_kernel, dim3(3 * n_sm), dim3(kGvThreads), kGvSmemDown, s, p);
}

}  // namespace pw
