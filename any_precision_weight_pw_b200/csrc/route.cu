// route.cu -- router GEMV, softmax/top-k and token->expert bucketing in one
// launch, and the final combine.
//
// PagedWeight (legiblepapers summary, FAQ Q5): routing and output
// accumulation are fused into the MoE kernel.  The pages give no routing
// formula; the library's reading is the one stated in pw.h (logits in fp32
// with the lane-butterfly order, ranking by logit with ties to the lower
// expert, softmax over all experts, optional renormalisation).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dequant.cuh"
#include "pw_internal.h"

namespace pw {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRouteThreads = 256;
constexpr int kStageSel = 16384;    // selections kept in shared memory (one byte each)
constexpr int kStageW = 2048;       // routing weights kept in shared memory (8 KB)

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Top-k and softmax of token t by one warp, once all E logits of t are in
// global memory: lane i holds experts i + 32 q (q < 4); each of the k rounds
// is an argmax over the warp under the ranking order (logit descending,
// index ascending); the softmax denominator is a lane-wise sum met in a xor
// butterfly.  Lane 0 writes the selections and their weights.
__device__ void topk_token(const RouteParams& p, int t, int lane) {
  const int E = p.E, k = p.k;
  const float* l = p.ws.logits + static_cast<size_t>(t) * E;
  float v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = lane + 32 * q;
    v[q] = e < E ? __ldcg(l + e) : 0.0f;
  }
  uint32_t taken = 0u;  // bit q: expert lane + 32 q already selected
  int sel[PW_MAX_TOPK];
  float lsel[PW_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < PW_MAX_TOPK; ++j) {
    if (j >= k) break;
    float bv = 0.0f;
    int bi = -1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = lane + 32 * q;
      if (e < E && !((taken >> q) & 1u) && (bi < 0 || v[q] > bv)) {
        bv = v[q];
        bi = e;
      }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, m);
      const int oi = __shfl_xor_sync(kFull, bi, m);
      if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= 0 && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel[j] = bi;
    lsel[j] = bv;
  }
  const float mx = lsel[0];
  float z = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (lane + 32 * q < E) z += expf(v[q] - mx);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) z += __shfl_xor_sync(kFull, z, m);
  if (lane == 0) {
    float psel[PW_MAX_TOPK];
    float ssum = 0.0f;
#pragma unroll
    for (int j = 0; j < PW_MAX_TOPK; ++j) {
      if (j >= k) break;
      psel[j] = expf(lsel[j] - mx) / z;
      ssum += psel[j];
    }
#pragma unroll
    for (int j = 0; j < PW_MAX_TOPK; ++j) {
      if (j >= k) break;
      p.ws.topk_idx[t * k + j] = sel[j];
      p.ws.topk_w[t * k + j] = p.renorm ? psel[j] / ssum : psel[j];
    }
  }
}

// One launch.  Phase 1: every warp computes router logits for (token,
// expert) pairs; lane j owns columns j, j+32, ... and fuses them in
// ascending order, then the 32 partial sums meet in a xor butterfly
// (16, 8, 4, 2, 1), so every lane ends with the same value.  A per-token
// counter finds the warp that writes a token's last logit; that warp takes
// the token's top-k and softmax at once (topk_token), so the selections of
// all tokens are made in parallel.  Phase 2 runs in the block that finishes
// last (a ticket counter, no waiting): per-expert counts from warp ballots
// over the staged selections, one warp-wide scan over the experts, and
// per-expert token lists ordered by token; it also puts the counters back
// to zero for the next launch.
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteParams p) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int warps_per_block = kRouteThreads / 32;
  const int E = p.E, H = p.H, T = p.T, k = p.k;
  const RouteWorkspace& ws = p.ws;
  // the previous kernel on the stream may produce x and still read the
  // workspace; the gather kernel may be scheduled from here on
  pdl_wait();
  pdl_trigger();

  const int total_pairs = T * E;
  for (int pair = blockIdx.x * warps_per_block + warp; pair < total_pairs;
       pair += gridDim.x * warps_per_block) {
    const int t = pair / E;
    const int e = pair - t * E;
    const uint16_t* xr = p.x + static_cast<size_t>(t) * H;
    const float* wr = p.wr + static_cast<size_t>(e) * H;
    // loads in batches of 32 per lane (independent of the sum, so their
    // latencies overlap), the next batch issued before the current one is
    // summed; the fused multiply-adds stay in ascending i
    float s = 0.0f;
    int i0 = lane;
    float xv[32], wv[32];
    bool have = i0 + 32 * 31 < H;
    if (have) {
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        xv[u] = bf16_bits_to_f32(xr[i0 + 32 * u]);
        wv[u] = wr[i0 + 32 * u];
      }
    }
    while (have) {
      const int i1 = i0 + 32 * 32;
      const bool more = i1 + 32 * 31 < H;
      float xn[32], wn[32];
      if (more) {
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          xn[u] = bf16_bits_to_f32(xr[i1 + 32 * u]);
          wn[u] = wr[i1 + 32 * u];
        }
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) s = __fmaf_rn(xv[u], wv[u], s);
      i0 = i1;
      have = more;
      if (more) {
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          xv[u] = xn[u];
          wv[u] = wn[u];
        }
      }
    }
    for (int i = i0; i < H; i += 32) s = __fmaf_rn(bf16_bits_to_f32(xr[i]), wr[i], s);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s = s + __shfl_xor_sync(kFull, s, m);
    int last = 0;
    if (lane == 0) {
      ws.logits[pair] = p.bias ? s + p.bias[e] : s;
      __threadfence();
      last = atomicAdd(ws.tok_ctr + t, 1u) == static_cast<unsigned>(E - 1);
    }
    if (__shfl_sync(kFull, last, 0)) {
      __threadfence();
      topk_token(p, t, lane);
    }
  }

  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(ws.ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- phase 2 (one block): bucketing ------------------------------------
  // Every token's selections are in global memory; they are staged in shared
  // memory (one byte each) with coalesced loads, with the weights when they
  // fit, and the token counters go back to zero for the next launch.
  __shared__ uint8_t s_idx[kStageSel];
  __shared__ float s_w[kStageW];
  const bool sel_staged = T * k <= kStageSel;
  const bool w_staged = T * k <= kStageW;
  for (int j = threadIdx.x; j < T * k; j += kRouteThreads) {
    if (sel_staged) s_idx[j] = static_cast<uint8_t>(__ldcg(ws.topk_idx + j));
    if (w_staged) s_w[j] = __ldcg(ws.topk_w + j);
  }
  for (int t = threadIdx.x; t < T; t += kRouteThreads) ws.tok_ctr[t] = 0u;
  __syncthreads();
  auto sel_of = [&](int t, int j) -> int {
    return sel_staged ? static_cast<int>(s_idx[t * k + j]) : __ldcg(ws.topk_idx + t * k + j);
  };

  // ---- bucketing: counts per expert with warp ballots ---------------------
  __shared__ int s_cnt[kMaxGroups + 1];
  __shared__ int s_off[kMaxGroups + 2];
  for (int e = warp; e < E; e += warps_per_block) {
    int cnt = 0;
    for (int base = 0; base < T; base += 32) {
      const int t = base + lane;
      bool hit = false;
      if (t < T)
        for (int j = 0; j < k; ++j) hit |= (sel_of(t, j) == e);
      cnt += __popc(__ballot_sync(kFull, hit));
    }
    if (lane == 0) s_cnt[e] = cnt;
  }
  __syncthreads();
  const int G = E + (p.has_shared ? 1 : 0);
  if (warp == 0) {
    // exclusive scan over the experts: lane holds experts 4 lane .. 4 lane + 3
    int c4[4], run = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = 4 * lane + q;
      c4[q] = e < E ? s_cnt[e] : 0;
      run += c4[q];
    }
    int incl = run;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int o = __shfl_up_sync(kFull, incl, m);
      if (lane >= m) incl += o;
    }
    int base = incl - run;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = 4 * lane + q;
      if (e < E) s_off[e] = base;
      base += c4[q];
    }
    const int routed = __shfl_sync(kFull, incl, 31);
    if (lane == 0) {
      s_off[E] = routed;
      if (p.has_shared) {
        s_cnt[E] = T;
        s_off[E + 1] = routed + T;
      }
      *ws.ticket = 0u;  // ready for the next forward (kernels on a stream do not overlap)
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g <= G; g += kRouteThreads) ws.offsets[g] = s_off[g];
  for (int j = threadIdx.x; j < p.n_zero; j += kRouteThreads) p.zero_words[j] = 0;

  // ---- bucketing: lists ordered by token ----------------------------------
  // With routing statistics on, the warp of expert e also sums the weights of
  // e's slots (in double: per 32-token block a xor butterfly, blocks in token
  // order) and adds its count and weight sum to the handle's counters; one
  // warp owns each expert, so the counters need no atomics.
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int e = warp; e < E; e += warps_per_block) {
    int run = s_off[e];
    double mass = 0.0;
    for (int base = 0; base < T; base += 32) {
      const int t = base + lane;
      int slot = -1;
      if (t < T)
        for (int j = 0; j < k; ++j)
          if (sel_of(t, j) == e) slot = j;
      const unsigned m = __ballot_sync(kFull, slot >= 0);
      double wm = 0.0;
      if (slot >= 0) {
        const int pos = run + __popc(m & lt_mask);
        ws.slot_token[pos] = t;
        ws.token_pos[t * k + slot] = pos;
        const float w = w_staged       ? s_w[t * k + slot]
                        : p.stat_count ? __ldcg(ws.topk_w + t * k + slot)
                                       : 0.0f;
        if (w_staged) ws.slot_w[pos] = w;
        wm = static_cast<double>(w);
      }
      if (p.stat_count) {
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) wm += __shfl_xor_sync(kFull, wm, sh);
        mass += wm;
      }
      run += __popc(m);
    }
    if (p.stat_count && lane == 0) {
      p.stat_count[e] += static_cast<unsigned long long>(s_off[e + 1] - s_off[e]);
      p.stat_mass[e] += mass;
    }
  }
  if (p.has_shared) {
    for (int t = threadIdx.x; t < T; t += kRouteThreads) {
      const int pos = s_off[E] + t;
      ws.slot_token[pos] = t;
      ws.slot_w[pos] = 1.0f;
      ws.token_pos[T * k + t] = pos;
    }
  }
  if (!w_staged) {
    // routing weight of every routed position (independent loads, all threads)
    __syncthreads();
    for (int j = threadIdx.x; j < T * k; j += kRouteThreads)
      ws.slot_w[__ldcg(ws.token_pos + j)] = __ldcg(ws.topk_w + j);
  }
}

// x_sorted row pos = the activations of token slot_token[pos] as fp16, each
// 32-column group permuted into the tensor-core kernel's K order; rows are the
// sorted positions of all groups, so every expert's token tile is contiguous.
// Stored atom-major, [ld / 64][rows][64], so one 3-D copy fetches a stage.
// One 32-column group per thread.
__global__ void gather_kernel(const GatherParams p) {
  pdl_wait();
  pdl_trigger();  // the tensor-core kernel may be scheduled (it waits for this grid)
  const int P = p.offsets[p.n_groups];
  const int wpr = p.H >> 5;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < P * wpr;
       idx += gridDim.x * blockDim.x) {
    const int pos = idx / wpr, w = idx - pos * wpr;
    const uint4* src = reinterpret_cast<const uint4*>(
        p.x + static_cast<size_t>(p.slot_token[pos]) * p.H + 32 * w);
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 r = src[q];
      const uint32_t r4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * q + 2 * e] = bf16_bits_to_f32(static_cast<uint16_t>(r4[e] & 0xFFFFu));
        v[8 * q + 2 * e + 1] = bf16_bits_to_f32(static_cast<uint16_t>(r4[e] >> 16));
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(
        p.x_sorted + (static_cast<size_t>(w >> 1) * p.rows + pos) * 64 + 32 * (w & 1));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 h2 = __floats2half2_rn(v[dq::col_of_kpos(8 * q + 2 * e)],
                                             v[dq::col_of_kpos(8 * q + 2 * e + 1)]);
        o[e] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// out[t] = sum_j ysorted[pos(t, j)] (+ shared) in slot order, summing the
// split-K partials of each position in split order; fp32, rounded to bf16.
__global__ void combine_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (c >= p.H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int nslots = p.k + (p.has_shared ? 1 : 0);
  for (int j = 0; j < nslots; ++j) {
    const int pos = (j < p.k) ? p.token_pos[t * p.k + j] : p.token_pos[p.T * p.k + t];
    for (int s = 0; s < p.n_split; ++s) {
      const float4 v = *reinterpret_cast<const float4*>(
          p.ysorted + s * p.split_stride + static_cast<size_t>(pos) * p.H + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 out;
  out.x = *reinterpret_cast<uint32_t*>(&lo);
  out.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p.y + static_cast<size_t>(t) * p.H + c) = out;
}

}  // namespace

cudaError_t launch_route(const RouteParams& p, int n_sm, cudaStream_t s) {
  const int pairs = p.T * p.E;
  const int warps = kRouteThreads / 32;
  int grid = (pairs + warps - 1) / warps;
  if (grid > 4 * n_sm) grid = 4 * n_sm;
  if (grid < 1) grid = 1;
  return launch_pdl(route_kernel, dim3(grid), dim3(kRouteThreads), 0, s, p);
}

cudaError_t launch_gather(const GatherParams& p, int max_rows, int n_sm, cudaStream_t s) {
  const int threads = 256;
  int grid = (max_rows * (p.H >> 5) + threads - 1) / threads;
  if (grid > 4 * n_sm) grid = 4 * n_sm;
  if (grid < 1) grid = 1;
  return launch_pdl(gather_kernel, dim3(grid), dim3(threads), 0, s, p);
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  const int threads = 128;
  dim3 grid((p.H / 4 + threads - 1) / threads, p.T);
  return launch_pdl(combine_kernel, grid, dim3(threads), 0, s, p);
}

}  // namespace pw
