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

#include <mutex>

#include "dequant.cuh"
#include "pw_internal.h"

namespace pw {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---- cluster and asynchronous-copy primitives ------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// store v to the shared-memory word at local address a in cluster block 0
__device__ __forceinline__ void st_leader(uint32_t a, float v) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(a));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(r), "f"(v) : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- the lane butterfly, for N accumulators at once ------------------------
// Every lane holds N partial sums (N a power of two <= 32).  The logit order
// adds, at levels m = 16, 8, 4, 2, 1, each lane's value to that of lane ^ m.
// Here each level also halves the live values: the lane with bit m set keeps
// the upper half, receives its partner's copy of that half and adds it to its
// own, the other lane keeps the lower half.  Every sum is the one the plain
// butterfly forms (own value + partner's, the same operands), so the result
// is bit-identical.  Afterwards lane l holds accumulator l >> (5 - log2 N);
// the levels past log2 N are plain butterfly levels.
template <int N>
__device__ __forceinline__ float tree_sum(float (&a)[N], int lane) {
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int m = 16 >> lvl;
    constexpr int kN = N;
    const int n = kN >> lvl;  // live values before this level
    if (n > 1) {
      const bool hi = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float send = hi ? a[i] : a[i + n / 2];
        const float keep = hi ? a[i + n / 2] : a[i];
        a[i] = keep + __shfl_xor_sync(kFull, send, m);
      }
    } else {
      a[0] = a[0] + __shfl_xor_sync(kFull, a[0], m);
    }
  }
  return a[0];
}
template <int N>
struct Log2 {
  static constexpr int value = N <= 1 ? 0 : 1 + Log2<(N > 1 ? N / 2 : 1)>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

// Top-k and softmax of one token by a group of L lanes (L a power of two,
// 4 L >= E) from its E logits in shared memory: lane i of the group holds
// experts i + L q (q < 4); each of the k rounds is an argmax over the group
// under the ranking order (logit descending, index ascending), met in xor
// shuffles within the group, so every lane of the group ends with the same
// selection; the softmax denominator is a group-wise xor sum.  Every lane of
// the warp calls this (the shuffles take the whole warp); `active` is false
// for groups without a token.  Lane 0 of a group writes the selections and
// their weights to global memory and, when sel is non-null, to the shared-
// memory staging arrays.
__device__ __forceinline__ void topk_group(const RouteParams& p, const float* l, int t,
                                           bool active, int gl, int L, uint8_t* sel,
                                           float* selw) {
  const int E = p.E, k = p.k;
  float v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = gl + L * q;
    v[q] = (active && e < E) ? l[e] : 0.0f;
  }
  uint32_t taken = 0u;  // bit q: expert gl + L q already selected
  int sidx[PW_MAX_TOPK];
  float lsel[PW_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < PW_MAX_TOPK; ++j) {
    if (j >= k) break;
    float bv = 0.0f;
    int bi = -1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = gl + L * q;
      if (active && e < E && !((taken >> q) & 1u) && (bi < 0 || v[q] > bv)) {
        bv = v[q];
        bi = e;
      }
    }
    for (int m = L >> 1; m >= 1; m >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, m);
      const int oi = __shfl_xor_sync(kFull, bi, m);
      if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= 0 && (bi & (L - 1)) == gl) taken |= 1u << (bi / L);
    sidx[j] = bi;
    lsel[j] = bv;
  }
  const float mx = lsel[0];
  float z = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (active && gl + L * q < E) z += expf(v[q] - mx);
  for (int m = L >> 1; m >= 1; m >>= 1) z += __shfl_xor_sync(kFull, z, m);
  if (active && gl == 0) {
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
      const float w = p.renorm ? psel[j] / ssum : psel[j];
      p.ws.topk_idx[t * k + j] = sidx[j];
      p.ws.topk_w[t * k + j] = w;
      if (sel) {
        sel[t * k + j] = static_cast<uint8_t>(sidx[j]);
        selw[t * k + j] = w;
      }
    }
  }
}

// One launch, in clusters of p.cb = (token groups) x p.ce (expert groups)
// blocks.  Cluster c owns tokens [c tb, c tb + tb); its block r owns the
// p.tbb tokens of token group r / ce and the p.eb experts of expert group
// r % ce.
//
// Phase 1 (every block): the block's token rows and router rows are copied
// into shared memory in column chunks (16-byte asynchronous copies, two
// buffers), and each warp computes the logits of a TT x TE tile of (token,
// expert) pairs: lane j owns columns j, j + 32, ... and fuses them in
// ascending order into TT x TE accumulators, which meet in the lane butterfly
// (tree_sum).  The logits go to the shared memory of the cluster's block 0
// (distributed shared memory), and a cluster barrier hands them over.
//
// Phase 2 (block 0 of each cluster): a group of lanes per token takes its
// top-k and softmax from the logits in shared memory.
//
// Phase 3 (bucketing, one block): with one cluster, its block 0 carries on
// from the selections it holds in shared memory; with several, the block 0
// that finishes last (a ticket counter, no waiting) stages every selection
// with coalesced loads.  Per-expert counts come from warp ballots over
// 32-token blocks, offsets from one warp-wide scan, and per-expert token
// lists ordered by token; the ticket goes back to zero for the next launch.
template <int TT, int TE>
__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(const RouteParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int E = p.E, H = p.H, T = p.T, k = p.k;
  const RouteWorkspace& ws = p.ws;
  const int rank = static_cast<int>(cluster_rank());
  const int tc0 = static_cast<int>(blockIdx.x) / p.cb * p.tb;  // the cluster's first token
  const int tl0 = (rank / p.ce) * p.tbb;                         // the block's, within the cluster
  const int t0 = tc0 + tl0;
  const int e0 = (rank - (rank / p.ce) * p.ce) * p.eb;
  const int nt = min(min(p.tbb, p.tb - tl0), T - t0);  // may be <= 0
  const int ne = min(p.eb, E - e0);                    // may be <= 0 (trailing block)
  cluster_arrive_relaxed();  // block 0's shared memory is live once all have arrived
  // the previous kernel on the stream may produce x and still read the
  // workspace; the gather kernel may be scheduled from here on
  pdl_wait();
  pdl_trigger();

  // ---- phase 1: logits ----------------------------------------------------
  const int kc_max = p.kc;
  const size_t xbytes = (static_cast<size_t>(p.tbb) * kc_max * 2 + 15) & ~static_cast<size_t>(15);
  const size_t sbytes = xbytes + static_cast<size_t>(p.eb) * kc_max * 4;
  const int n_chunks = (H + kc_max - 1) / kc_max;
  auto issue = [&](int ci) {
    const int k0 = ci * kc_max;
    const int kc = min(kc_max, H - k0);
    unsigned char* dx = smem + (ci & 1) * sbytes;
    float* dw = reinterpret_cast<float*>(dx + xbytes);
    uint16_t* dxh = reinterpret_cast<uint16_t*>(dx);
    if (p.vec) {
      const int xp = kc >> 3;  // 16-byte pieces of a token row chunk
      for (int r = 0; r < nt; ++r) {
        const uint16_t* src = p.x + static_cast<size_t>(t0 + r) * H + k0;
        for (int q = threadIdx.x; q < xp; q += kRouteThreads)
          cp_async16(dxh + r * kc_max + 8 * q, src + 8 * q);
      }
      const int wp = kc >> 2;
      for (int r = 0; r < ne; ++r) {
        const float* src = p.wr + static_cast<size_t>(e0 + r) * H + k0;
        for (int q = threadIdx.x; q < wp; q += kRouteThreads)
          cp_async16(dw + r * kc_max + 4 * q, src + 4 * q);
      }
    } else {
      for (int r = 0; r < nt; ++r)
        for (int q = threadIdx.x; q < kc; q += kRouteThreads)
          dxh[r * kc_max + q] = p.x[static_cast<size_t>(t0 + r) * H + k0 + q];
      for (int r = 0; r < ne; ++r)
        for (int q = threadIdx.x; q < kc; q += kRouteThreads)
          dw[r * kc_max + q] = p.wr[static_cast<size_t>(e0 + r) * H + k0 + q];
    }
    cp_async_commit();
  };

  constexpr int kN = TT * TE;
  const int tasks_e = (p.eb + TE - 1) / TE;
  const int n_tasks = ((p.tbb + TT - 1) / TT) * tasks_e;  // <= kRouteWarps (host)
  const bool busy = warp < n_tasks;
  const int tt0 = (warp / tasks_e) * TT;
  const int te0 = (warp - (warp / tasks_e) * tasks_e) * TE;
  float acc[kN];
#pragma unroll
  for (int i = 0; i < kN; ++i) acc[i] = 0.0f;

  issue(0);
  if (n_chunks > 1) issue(1);
  for (int ci = 0; ci < n_chunks; ++ci) {
    if (ci + 1 < n_chunks)
      cp_async_wait<1>();
    else
      cp_async_wait<0>();
    __syncthreads();
    if (busy) {
      const int kc = min(kc_max, H - ci * kc_max);
      const unsigned char* base = smem + (ci & 1) * sbytes;
      // a tile's rows past the buffer's tbb token rows or eb router rows
      // read the last row instead; rows past the block's tokens or experts
      // hold stale data; the sums of both are never written
      const uint16_t* xr[TT];
      const float* wrs[TE];
#pragma unroll
      for (int a = 0; a < TT; ++a)
        xr[a] = reinterpret_cast<const uint16_t*>(base) + min(tt0 + a, p.tbb - 1) * kc_max;
#pragma unroll
      for (int b = 0; b < TE; ++b)
        wrs[b] = reinterpret_cast<const float*>(base + xbytes) + min(te0 + b, p.eb - 1) * kc_max;
#pragma unroll 4
      for (int c = lane; c < kc; c += 32) {
        float xv[TT], wv[TE];
#pragma unroll
        for (int a = 0; a < TT; ++a) xv[a] = bf16_bits_to_f32(xr[a][c]);
#pragma unroll
        for (int b = 0; b < TE; ++b) wv[b] = wrs[b][c];
#pragma unroll
        for (int a = 0; a < TT; ++a)
#pragma unroll
          for (int b = 0; b < TE; ++b) acc[a * TE + b] = __fmaf_rn(xv[a], wv[b], acc[a * TE + b]);
      }
    }
    __syncthreads();  // this buffer is free again
    if (ci + 2 < n_chunks) issue(ci + 2);
  }

  float* s_logits = reinterpret_cast<float*>(smem + p.logits_off);  // [tb][E], block 0
  cluster_wait();  // pairs with the arrive at the start
  if (busy) {
    const float v = tree_sum<kN>(acc, lane);
    constexpr int kShift = 5 - Log2<kN>::value;
    const int a = lane >> kShift;
    const int tl = tt0 + a / TE, el = te0 + a % TE;
    if ((lane & ((1 << kShift) - 1)) == 0 && tl < nt && el < ne) {
      const int e = e0 + el;
      st_leader(smem_u32(s_logits + (tl0 + tl) * E + e), p.bias ? v + p.bias[e] : v);
    }
  }
  cluster_arrive_release();
  cluster_wait();
  if (rank != 0) return;

  // ---- phase 2: top-k per token (block 0 of the cluster) -------------------
  // With one cluster the selections also go to shared memory for phase 3;
  // they reuse the staging buffers, which no warp reads any more.
  const bool one = p.n_clusters == 1;
  const bool staged = p.sel_staged != 0;
  uint8_t* s_idx = smem;
  float* s_w = reinterpret_cast<float*>(smem + ((static_cast<size_t>(T) * k + 15) & ~static_cast<size_t>(15)));
  {
    int L = 1;
    while (4 * L < E) L <<= 1;
    const int per_warp = 32 / L;
    const int ntc = min(p.tb, T - tc0);
    const int gl = lane & (L - 1);
    for (int base = warp * per_warp; base < ntc; base += kRouteWarps * per_warp) {
      const int tl = base + lane / L;
      const bool act = tl < ntc;
      topk_group(p, s_logits + (act ? tl : 0) * E, tc0 + tl, act, gl, L,
                 (one && staged) ? s_idx : nullptr, s_w);
    }
  }

  __shared__ int s_last;
  if (!one) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(ws.ticket, 1u) == static_cast<unsigned>(p.n_clusters - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (staged) {
      // every selection, eight independent loads per thread in flight
      const int n = T * k;
      for (int j0 = threadIdx.x; j0 < n; j0 += 8 * kRouteThreads) {
        int iv[8];
        float wv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u * kRouteThreads;
          iv[u] = j < n ? __ldcg(ws.topk_idx + j) : 0;
          wv[u] = j < n ? __ldcg(ws.topk_w + j) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u * kRouteThreads;
          if (j < n) {
            s_idx[j] = static_cast<uint8_t>(iv[u]);
            s_w[j] = wv[u];
          }
        }
      }
    }
  }
  __syncthreads();
  // the slot of token t that selected expert e, or -1
  auto slot_of = [&](int t, int e) -> int {
    int slot = -1;
    if (t < T)
      for (int j = 0; j < k; ++j)
        if ((staged ? static_cast<int>(s_idx[t * k + j]) : __ldcg(ws.topk_idx + t * k + j)) == e)
          slot = j;
    return slot;
  };

  // ---- phase 3: counts per expert with warp ballots -----------------------
  __shared__ int s_cnt[kMaxGroups + 1];
  __shared__ int s_off[kMaxGroups + 2];
  for (int e = warp; e < E; e += kRouteWarps) {
    int cnt = 0;
    for (int base = 0; base < T; base += 32)
      cnt += __popc(__ballot_sync(kFull, slot_of(base + lane, e) >= 0));
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
      if (!one) *ws.ticket = 0u;  // ready for the next forward (kernels on a stream do not overlap)
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g <= G; g += kRouteThreads) ws.offsets[g] = s_off[g];
  for (int j = threadIdx.x; j < p.n_zero; j += kRouteThreads) p.zero_words[j] = 0;

  // ---- phase 3: lists ordered by token ------------------------------------
  // With routing statistics on, the warp of expert e also sums the weights of
  // e's slots (in double: each lane over its tokens in order, then a xor
  // butterfly) and adds its count and weight sum to the handle's counters
  // (reductions whose results are not waited for); one warp owns each
  // expert, so every counter gets one addition per forward.
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int e = warp; e < E; e += kRouteWarps) {
    if (s_off[e + 1] == s_off[e]) continue;  // no token chose e: nothing to list or count
    int run = s_off[e];
    double mass = 0.0;
    for (int base = 0; base < T; base += 32) {
      const int t = base + lane;
      const int slot = slot_of(t, e);
      const unsigned m = __ballot_sync(kFull, slot >= 0);
      if (slot >= 0) {
        const int pos = run + __popc(m & lt_mask);
        const float w = staged ? s_w[t * k + slot] : __ldcg(ws.topk_w + t * k + slot);
        ws.slot_token[pos] = t;
        ws.token_pos[t * k + slot] = pos;
        ws.slot_w[pos] = w;
        mass += static_cast<double>(w);
      }
      run += __popc(m);
    }
    if (p.stat_count) {
#pragma unroll
      for (int sh = 16; sh >= 1; sh >>= 1) mass += __shfl_xor_sync(kFull, mass, sh);
      if (lane == 0) {
        atomicAdd(p.stat_count + e, static_cast<unsigned long long>(s_off[e + 1] - s_off[e]));
        atomicAdd(p.stat_mass + e, mass);
      }
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


// Launch of one router shape: the per-device shared-memory attribute is set
// once (under a lock), then the grid goes out in clusters of p.cb blocks with
// programmatic dependent launch.
constexpr size_t kStageBudget = 96 * 1024;  // bytes of one staging buffer, at most
constexpr size_t kRouteSmemMax = 2 * kStageBudget + 16 * 1024 + 32 * PW_MAX_EXPERTS * 4;

template <int TT, int TE>
cudaError_t launch_route_shape(const RouteParams& p, size_t smem, cudaStream_t s) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(route_kernel<TT, TE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kRouteSmemMax));
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_clusters * p.cb);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.cb;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, route_kernel<TT, TE>, p);
}

}  // namespace

RouteGeometry route_geometry(int T, int E, int H, int k) {
  RouteGeometry g{};
  const bool big = T >= 256;
  if (big) {
    // many clusters: each block covers up to 8 experts of 16-32 tokens
    const int cb0 = (E + 7) / 8 < 8 ? (E + 7) / 8 : 8;
    g.eb = (E + cb0 - 1) / cb0;
    g.ce = (E + g.eb - 1) / g.eb;
    g.cb = g.ce;
    g.tb = g.eb <= 8 ? 32 : 16;
    g.tbb = g.tb;
  } else {
    // one cluster of up to 8 blocks per 16 tokens, split between token and
    // expert groups so each block stages the fewest bytes
    int tb = 1;
    while (tb < T && tb < 16) tb *= 2;
    g.tb = tb;
    const int cb = E * tb < 8 ? E * tb : 8;
    size_t best = ~static_cast<size_t>(0);
    for (int ca = 1; ca <= cb; ca *= 2) {
      if (cb % ca || ca > tb) continue;
      const int ce = cb / ca;
      if (ce > E) continue;
      const int tbb = (tb + ca - 1) / ca, eb = (E + ce - 1) / ce;
      const size_t bytes = static_cast<size_t>(tbb) * H * 2 + static_cast<size_t>(eb) * H * 4;
      if (bytes < best) {
        best = bytes;
        g.ce = (E + eb - 1) / eb;  // expert groups that hold an expert
        g.cb = ca * g.ce;
        g.tbb = tbb;
        g.eb = eb;
      }
    }
  }
  // the smallest register tile that needs at most one task per warp
  static const int kTiles[][2] = {{1, 1}, {2, 1}, {1, 4}, {4, 1}, {2, 4},
                                  {8, 1}, {1, 8}, {4, 4}, {2, 8}, {4, 8}};
  g.tt = 0;
  for (const auto& tl : kTiles) {
    const int tasks = ((g.tbb + tl[0] - 1) / tl[0]) * ((g.eb + tl[1] - 1) / tl[1]);
    if (tasks <= kRouteWarps) {
      g.tt = tl[0];
      g.te = tl[1];
      break;
    }
  }
  const int per_col = 2 * g.tbb + 4 * g.eb;
  int kc = static_cast<int>(kStageBudget / per_col) & ~31;
  if (kc < 32) kc = 32;
  const int h32 = (H + 31) & ~31;
  if (kc > h32) kc = h32;
  g.kc = kc;
  const int n_chunks = (H + kc - 1) / kc;
  const size_t xbytes = (static_cast<size_t>(g.tbb) * kc * 2 + 15) & ~static_cast<size_t>(15);
  const size_t stage = (n_chunks > 1 ? 2 : 1) * (xbytes + static_cast<size_t>(g.eb) * kc * 4);
  const size_t tk = static_cast<size_t>(T) * k;
  const size_t sel = ((tk + 15) & ~static_cast<size_t>(15)) + 4 * tk;
  g.sel_staged = sel <= 2 * kStageBudget;
  size_t region = stage;
  if (g.sel_staged && sel > region) region = sel;
  g.logits_off = (region + 15) & ~static_cast<size_t>(15);
  g.smem = g.logits_off + static_cast<size_t>(g.tb) * E * 4;
  g.n_clusters = T > 0 ? (T + g.tb - 1) / g.tb : 1;
  return g;
}

cudaError_t launch_route(const RouteParams& p_in, int n_sm, cudaStream_t s) {
  (void)n_sm;
  RouteParams p = p_in;
  const RouteGeometry g = route_geometry(p.T, p.E, p.H, p.k);
  if (g.tt == 0 || g.smem > kRouteSmemMax) return cudaErrorInvalidConfiguration;
  p.cb = g.cb;
  p.ce = g.ce;
  p.tb = g.tb;
  p.tbb = g.tbb;
  p.eb = g.eb;
  p.kc = g.kc;
  p.n_clusters = g.n_clusters;
  p.logits_off = static_cast<int>(g.logits_off);
  p.sel_staged = g.sel_staged ? 1 : 0;
  p.vec = (p.H % 8 == 0) && (reinterpret_cast<uintptr_t>(p.x) % 16 == 0) &&
          (reinterpret_cast<uintptr_t>(p.wr) % 16 == 0);
  switch (g.tt * 16 + g.te) {
    case 0x11: return launch_route_shape<1, 1>(p, g.smem, s);
    case 0x21: return launch_route_shape<2, 1>(p, g.smem, s);
    case 0x14: return launch_route_shape<1, 4>(p, g.smem, s);
    case 0x41: return launch_route_shape<4, 1>(p, g.smem, s);
    case 0x24: return launch_route_shape<2, 4>(p, g.smem, s);
    case 0x81: return launch_route_shape<8, 1>(p, g.smem, s);
    case 0x18: return launch_route_shape<1, 8>(p, g.smem, s);
    case 0x44: return launch_route_shape<4, 4>(p, g.smem, s);
    case 0x28: return launch_route_shape<2, 8>(p, g.smem, s);
    case 0x48: return launch_route_shape<4, 8>(p, g.smem, s);
    default: return cudaErrorInvalidConfiguration;
  }
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
