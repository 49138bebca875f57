// pw_internal.h -- shared between the host side (pw_api.cu) and the kernels
// of the B200 fused mixed-precision MoE library.  Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pw.h"

namespace pw {

// Programmatic dependent launch.  The forward's kernels go on the stream with
// the programmatic-serialisation attribute, so each can be scheduled while
// its predecessor drains; every such kernel calls pdl_wait() before it reads
// anything a predecessor wrote (or writes anything a predecessor reads), and
// may call pdl_trigger() to let its own successor be scheduled early.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// cooperative: the grid's CTAs are all resident at once or the launch fails
// (for kernels whose CTAs wait on one another).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_ex(bool cooperative, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                          size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  return launch_pdl_ex(false, kernel, grid, block, smem, s, static_cast<Args&&>(args)...);
}
#endif

constexpr int kMaxBlocks = 3 * (PW_MAX_EXPERTS + 1);
constexpr int kMaxGroups = PW_MAX_EXPERTS + 1;  // routed experts + shared

// Page-table entry of one linear-block as the kernels see it for one forward:
// the plane buffer and the LUT slot that holds LUT_bits.  Passed by value in
// the kernel parameters, so a forward keeps the table it was launched with
// while the host moves on to the next one.
struct BlockRef {
  const uint32_t* planes;  // n_max plane pages (layout: pages.h)
  const uint16_t* lut;     // [rows][2^bits] fp16 bits
};

struct PageTable {
  BlockRef blk[kMaxBlocks];
  uint8_t bits[kMaxBlocks];
  uint8_t stride[kMaxBlocks];  // planes stored per tile group: n_max for caller
                               // storage, the resident count for paged storage
};

// Routing results and per-group token lists, written by the route kernel.
// "Group" g < E is routed expert g; g == E is the shared expert (all tokens).
// Sorted positions: group g owns positions [offsets[g], offsets[g+1]); the
// routed lists are ordered by token, the shared list is tokens 0..T-1.
struct RouteWorkspace {
  int32_t* topk_idx;    // [T][k]
  float* topk_w;        // [T][k]
  int32_t* offsets;     // [G+1]
  int32_t* slot_token;  // [P] token of each sorted position
  float* slot_w;        // [P] routing weight of each sorted position
  int32_t* token_pos;   // [T][k] (+ [T] shared) sorted position of (t, j)
  uint32_t* ticket;     // last-cluster-done counter (self-resetting)
};

struct RouteParams {
  const uint16_t* x;       // bf16 [T][H]
  const float* wr;         // [E][H]
  const float* bias;       // [E] or null
  int T, H, E, k, renorm, has_shared;
  RouteWorkspace ws;
  int* zero_words;         // counters of the launches that follow, set to zero
  int n_zero;              // (may be null / 0)
  unsigned long long* stat_count;  // [E] routing statistics, accumulated over
  double* stat_mass;               // forwards (both null: none kept)
  // launch geometry (launch_route fills these from route_geometry)
  int cb, ce;         // blocks per cluster = token groups x ce expert groups
  int tb, tbb, eb;    // tokens per cluster, tokens per block, experts per block
  int kc;             // columns per staged chunk (a multiple of 32)
  int n_clusters;
  int logits_off;     // shared-memory offset of the cluster's logits [tb][E]
  int sel_staged;     // every selection fits in shared memory for the bucketing
  int vec;            // 16-byte asynchronous copies of x and wr are legal
};

// Router launch geometry for T tokens, E experts, hidden H and top-k (host).
struct RouteGeometry {
  int cb, ce, tb, tbb, eb, kc, n_clusters;
  int tt, te;         // register tile of a warp: tokens x experts (tt = 0: none fits)
  bool sel_staged;
  size_t logits_off, smem;
};
RouteGeometry route_geometry(int T, int E, int H, int k);

struct GatherParams {
  const uint16_t* x;         // bf16 [T][H]
  const int32_t* offsets;    // [n_groups+1]
  const int32_t* slot_token; // [P]
  uint16_t* x_sorted;        // fp16 atom-major [ld/64][rows][64], tensor-core K order
  int H, ld, rows, n_groups;
};

struct CombineParams {
  const float* ysorted;  // [P][H] routing-weighted expert outputs
  const int32_t* token_pos;
  uint16_t* y;           // bf16 [T][H]
  int T, H, k, has_shared;
  int n_split;           // partial sums per position (split-K of the down pass)
  long long split_stride;  // floats between splits
};

// Expert pass over all groups on the CUDA-core (simple) path.
struct SimpleParams {
  PageTable pt;
  int mode;        // 0 = gate/up -> gu, 1 = down -> ysorted, 2 = single linear
  int H, F, S, E, n_groups;
  const int32_t* offsets;
  const int32_t* slot_token;
  const float* slot_w;
  const uint16_t* x;      // bf16 [T][H] (modes 0, 2)
  float* gu;              // [P][2*Fmax] gate | up (mode 0 out, mode 1 in)
  int gu_stride;          // floats per gu row
  float* ysorted;         // [P][H] (mode 1 out)
  float* y;               // [T][rows] (mode 2 out)
  int T;                  // tokens (mode 2)
  int lin_rows, lin_cols, lin_bits, lin_n_max;  // mode 2 block
  int n_max;                         // planes per block (modes 0, 1)
  const uint32_t* lin_planes;
  const uint16_t* lin_lut;
};

// Decode passes on the CUDA cores for few tokens per expert (gv.cu).
struct GvParams {
  PageTable pt;
  int H, F, S, E, n_groups;
  const int32_t* offsets;     // [G+1]
  const int32_t* slot_token;  // [P]
  const float* slot_w;        // [P]
  const uint16_t* x;          // bf16 [T][H]
  float* x_gv;                // [P][H_pad] fp32 activations, dequantiser K order, 0 past H
  float* h_gv;                // [P][F_pad] fp32 silu(g) * u, same order, 0 past F
  int H_pad, F_pad;           // multiples of 256
  float* ysorted;             // [n_split][P][H] routing-weighted partials
  long long split_stride;     // floats between splits
  int n_split;                // K splits of the down pass
};

// Sets the calling thread's pw_last_error() text and returns st (pw_api.cu).
pw_status_t record_error(pw_status_t st, const char* msg);

// Launchers (defined in the .cu files).
cudaError_t launch_route(const RouteParams& p, int n_sm, cudaStream_t s);
cudaError_t launch_repack(const uint32_t* src, uint32_t* dst, int rows, int cols, int n_planes,
                          cudaStream_t s);
cudaError_t launch_gather(const GatherParams& p, int max_rows, int n_sm, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);
cudaError_t launch_simple(const SimpleParams& p, int grid_rows, cudaStream_t s);
// pass 0: gather (max_rows positions at most), 1: gate/up + SwiGLU, 2: down
cudaError_t launch_gv(const GvParams& p, int pass, int max_rows, int n_sm, cudaStream_t s);

}  // namespace pw
