// pw_api.cu -- host side of the C ABI (include/pw.h): argument checks, the
// per-block page table, the asynchronous bitwidth switch, workspace and the
// launch sequence of one forward.
//
// PagedWeight (legiblepapers summary, "Summary & Methodology Analysis"; the
// arxivlens abstract): the bit-plane and LUT buffers are GPU-resident pages
// that move between host and device asynchronously while the layer keeps
// serving.  Here a bitwidth change is a page move on a side stream; a
// forward uses the new width once it finds the move complete, or waits for
// it after a bounded number of forwards (see pw_set_block_bits); with paging
// on, lowering a width also frees the dropped planes' device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "pages.h"
#include "pw_internal.h"
#include "tc.h"

namespace {

// Host-side NVTX ranges around the calls a profiler should see (a forward, a
// page move, paging and compaction); free when no tool is attached, and off
// with PW_NVTX=0.
struct NvtxRange {
  bool on;
  explicit NvtxRange(const char* name) : on(nvtx_on()) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
  static bool nvtx_on() {
    static const bool v = [] {
      const char* e = std::getenv("PW_NVTX");
      return !(e && e[0] == '0');
    }();
    return v;
  }
};

thread_local std::string g_err;

pw_status_t fail(pw_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
pw_status_t fail(pw_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

#define PW_CUDA(call)                                                                  \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(PW_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Error text for calls implemented in other translation units.
pw_status_t pw::record_error(pw_status_t st, const char* msg) { return fail(st, "%s", msg); }

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// The tensor-core path stages planes with 3-D TMA tiles (words x rows x
// plane), whose row pitch must be a multiple of 16 bytes, and permutes
// activations in whole 32-column groups: it takes cols % 128 == 0.
bool tc_shape_ok(int cols) { return cols % 128 == 0; }

// Maps over an atom-major fp16 buffer [ld / 64][rows][64] for the token
// tiles, as {64 columns, rows, atoms}: box i loads 8(i+1) rows x 2 atoms with
// the 128-byte swizzle of the MMA's K-major operand, one copy per 128-column
// B stage.
pw_status_t make_row_maps(CUtensorMap* m, const uint16_t* base, int ld, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PW_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  for (int i = 0; i < 4; ++i) {
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(ld / 64)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(rows) * 128};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(8 * (i + 1)), 2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return fail(PW_ERR_CUDA, "cuTensorMapEncodeTiled (token rows) failed (%d)", (int)r);
  }
  return PW_OK;
}

// Map for the prefill passes: box {64 columns, 256 rows, 1 atom}.
pw_status_t make_chunk_map(CUtensorMap* m, const uint16_t* base, int ld, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PW_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(ld / 64)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(rows) * 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(pw::kTcPfTokens), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(PW_ERR_CUDA, "cuTensorMapEncodeTiled (token chunks) failed (%d)", (int)r);
  return PW_OK;
}

int env_int(const char* name, int dflt) {
  const char* v = getenv(name);
  return v ? atoi(v) : dflt;
}

}  // namespace

// Paged plane storage: one allocation of the handle's pool, shared by the
// blocks placed in it (one block after a page move, every block after
// pw_enable_paging or pw_compact_pages); freed when its last block leaves.
struct PageAlloc {
  void* base;
  int refs;
};

struct pw_moe {
  pw_moe_config_t cfg{};
  int n_blocks = 0, G = 0, device = 0, n_sm = 0;
  struct Blk {
    int rows, cols;
    uint32_t* d_planes;
    uint16_t* d_lut[2];
    const uint32_t* h_planes;
    const uint16_t* h_lut[PW_MAX_BITS + 1];
    int bits, slot;            // active bitwidth and LUT slot
    int stride;                // planes per tile group of d_planes
    PageAlloc* alloc;          // paging: the allocation d_planes lies in (null:
                               // the caller's storage)
    int pend_bits;             // 0 = none
    long long pend_req;        // forwards issued when the change was requested
    uint32_t* pend_planes;     // paging: the storage the pending change fills
    PageAlloc* pend_alloc;
    cudaEvent_t ready;
  };
  std::vector<Blk> blk;
  bool paging = false;               // plane storage owned by the library
  bool compacted = false;            // the next forward waits for pw_compact_pages
  cudaMemPool_t pool = nullptr;      // paging: the plane pages' memory pool
  long long n_forwards = 0;
  int max_lag = 8;                   // forwards a page move may stay pending
  std::vector<int32_t> fwd_bits;     // bitwidths of the most recent forward
  cudaEvent_t fwd_done = nullptr;
  bool any_forward = false;
  // workspace
  pw::RouteWorkspace ws{};
  float* gu = nullptr;          // CUDA-core path: gate | up per sorted position
  uint16_t* x_sorted = nullptr; // tensor-core path: gathered fp16 activations, K-permuted
  uint16_t* h_perm = nullptr;   // tensor-core path: fp16 silu(g) * u, K-permuted
  int x_ld = 0, h_perm_ld = 0;
  CUtensorMap x_maps[4], h_maps[4];  // token-tile maps over x_sorted and h_perm
  CUtensorMap x_pf_map, h_pf_map;    // 256-row chunk maps (prefill passes)
  uint16_t* gbuf = nullptr;          // prefill: gate outputs [P_max][Fmax] fp16
  int* gu_done = nullptr;            // fused decode launch: per-group gate/up counts
  int gbuf_ld = 0;
  bool pf = false;                   // the prefill passes are available
  float* ysorted = nullptr;
  int* err = nullptr;
  unsigned long long* stat_count = nullptr;  // routing statistics [E]
  double* stat_mass = nullptr;               // [E]
  uint16_t* stage_x = nullptr;
  uint16_t* stage_y = nullptr;
  int P_max = 0, gu_stride = 0, last_T = 0;
  size_t ys_floats = 0;   // capacity of the down partials (shared with gbuf)
  int gv_T = 0, gv_H_pad = 0, gv_F_pad = 0;   // CUDA-core decode passes
  float* x_gv = nullptr;
  float* h_gv = nullptr;
  size_t ws_bytes = 0;
  bool tc = false;  // both expert passes on the tensor-core kernel
  void* ws_base = nullptr;
  // per-launch timing (pw_profile_*): 5 events per forward bracket 4 launches
  bool profiling = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<std::vector<cudaEvent_t>> ev_pending;
};

namespace {

int block_rows(const pw_moe_config_t& c, int id) {
  const int e = id / 3, proj = id % 3;
  const int F = (e == c.n_experts) ? c.shared_ffn : c.ffn;
  return proj < 2 ? F : c.hidden;
}
int block_cols(const pw_moe_config_t& c, int id) {
  const int e = id / 3, proj = id % 3;
  const int F = (e == c.n_experts) ? c.shared_ffn : c.ffn;
  return proj < 2 ? c.hidden : F;
}

void free_all(pw_moe* h) {
  if (!h) return;
  for (auto& v : h->ev_pending)
    for (auto e : v) cudaEventDestroy(e);
  for (auto e : h->ev_pool) cudaEventDestroy(e);
  std::vector<PageAlloc*> allocs;
  for (auto& b : h->blk) {
    if (b.ready) cudaEventDestroy(b.ready);
    for (PageAlloc* a : {b.alloc, b.pend_alloc})
      if (a && --a->refs == 0) allocs.push_back(a);
  }
  for (PageAlloc* a : allocs) {
    cudaFree(a->base);
    delete a;
  }
  if (h->pool) cudaMemPoolDestroy(h->pool);
  if (h->fwd_done) cudaEventDestroy(h->fwd_done);
  if (h->ws_base) cudaFree(h->ws_base);
  delete h;
}

constexpr int kMaxSplit = 8;  // K splits of the down pass at most

// K splits of the down items: enough items for `per_sm` rounds of the grid
// (more in the fused launch, where down items also fill the gate/up tail).
int splits_for(const pw_moe_config_t& c, int n_sm, int T, int per_sm) {
  const int row_tiles = (c.hidden + 127) / 128;
  int groups = T * c.top_k < c.n_experts ? T * c.top_k : c.n_experts;
  if (c.shared_ffn > 0) groups += 1;
  const int items = row_tiles * groups;
  int ns = (per_sm * n_sm + items - 1) / items;
  const int stages = ((c.ffn + 31) / 32 + 7) / 8;
  if (ns > stages) ns = stages;
  if (ns > kMaxSplit) ns = kMaxSplit;
  if (ns < 1) ns = 1;
  return ns;
}

// K splits of the CUDA-core down pass (gv.cu): about two rounds of three
// CTAs per SM over (group, 32-row tile, split) items, at most one split per
// 256-column tile group of the narrowest down block and kMaxSplit.
int gv_splits_for(const pw_moe_config_t& c, int n_sm, int T) {
  int groups = T * c.top_k < c.n_experts ? T * c.top_k : c.n_experts;
  if (c.shared_ffn > 0) groups += 1;
  const int row_tiles = (c.hidden + 31) / 32;
  int ns = (6 * n_sm + groups * row_tiles - 1) / (groups * row_tiles);
  const int stages = ((c.ffn + 31) / 32 + 7) / 8;
  if (ns > stages) ns = stages;
  if (ns > kMaxSplit) ns = kMaxSplit;
  return ns < 1 ? 1 : ns;
}

// Largest token count the CUDA-core decode passes take (PW_GV_T, read at
// create; 0, the default, keeps every decode batch on the tensor cores,
// which measured faster at every batch of the benchmark workloads).
int gv_max_tokens(const pw_moe_config_t& c) {
  const int forced = env_int("PW_GV_T", 0);
  if (forced <= 0) return 0;
  return forced < c.max_tokens ? forced : c.max_tokens;
}

// Sorted positions of a forward of T tokens (routed slots + shared rows).
size_t positions(const pw_moe_config_t& c, int T) {
  return static_cast<size_t>(T) * c.top_k + (c.shared_ffn > 0 ? T : 0);
}

// The prefill passes are the default when the routed slots average at least
// 64 tokens per expert.
bool prefill_default(const pw_moe_config_t& c, int T) {
  return static_cast<long long>(T) * c.top_k >= 64ll * c.n_experts;
}

// The workspace of a handle: one allocation, every piece 256-byte aligned.
// The down pass's per-split partials and the prefill gate outputs share one
// region (the gate outputs are dead once the up pass has run, before the
// down pass writes), sized for the larger of: one split of every position
// at max_tokens, the splits the decode passes choose at each token count
// they serve, and the prefill gate outputs.
struct Layout {
  bool tc = false, pf = false;
  int P_max = 0, gu_stride = 0, x_ld = 0, h_perm_ld = 0, gbuf_ld = 0;
  int gv_T = 0, gv_H_pad = 0, gv_F_pad = 0;  // CUDA-core decode passes
  size_t ys_floats = 0;
  size_t o_tki, o_tkw, o_off, o_st, o_sw, o_tp, o_tk, o_err, o_gd, o_sc, o_sm,
      o_gu, o_xp, o_hp, o_xg, o_hg, o_ys, o_sx, o_sy, total;
};

Layout make_layout(const pw_moe_config_t& c, int n_sm) {
  Layout L;
  const int T = c.max_tokens, E = c.n_experts, k = c.top_k, S = c.shared_ffn;
  const int G = E + (S > 0 ? 1 : 0);
  L.P_max = static_cast<int>(positions(c, T));
  const int Fmax = c.ffn > S ? c.ffn : S;
  L.tc = tc_shape_ok(c.hidden) && tc_shape_ok(c.ffn) && (S == 0 || tc_shape_ok(S)) &&
         env_int("PW_FORCE_SIMPLE", 0) == 0;
  L.gu_stride = L.tc ? 0 : 2 * Fmax;
  // rows padded to whole 256-column stages, zero past the end
  L.x_ld = L.tc ? (c.hidden + 255) / 256 * 256 : 0;
  L.h_perm_ld = L.tc ? (Fmax + 255) / 256 * 256 : 0;
  L.pf = L.tc && L.P_max >= pw::kTcPfTokens;
  L.gbuf_ld = L.pf ? Fmax : 0;
  L.gv_T = gv_max_tokens(c);
  L.gv_H_pad = (c.hidden + 255) / 256 * 256;
  L.gv_F_pad = (Fmax + 255) / 256 * 256;
  size_t ys = static_cast<size_t>(L.P_max) * c.hidden;
  for (int t = 1; t <= T; ++t) {
    if (L.pf && prefill_default(c, t)) break;
    int ns = 1;
    if (L.tc) {
      ns = splits_for(c, n_sm, t, 6);
      const int ns4 = splits_for(c, n_sm, t, 4);
      if (ns4 > ns) ns = ns4;
    }
    if (t <= L.gv_T) {
      const int ng = gv_splits_for(c, n_sm, t);
      if (ng > ns) ns = ng;
    }
    const size_t need = ns * positions(c, t) * c.hidden;
    if (need > ys) ys = need;
  }
  const size_t P_gv = positions(c, L.gv_T);
  const size_t gb = (static_cast<size_t>(L.P_max) * L.gbuf_ld + 1) / 2;  // fp16, in floats
  L.ys_floats = ys;
  auto al = [](size_t n) { return (n + 255) & ~size_t(255); };
  size_t off = 0;
  L.o_tki = off; off += al(sizeof(int32_t) * T * k);
  L.o_tkw = off; off += al(sizeof(float) * T * k);
  L.o_off = off; off += al(sizeof(int32_t) * (G + 1));
  L.o_st = off; off += al(sizeof(int32_t) * L.P_max);
  L.o_sw = off; off += al(sizeof(float) * L.P_max);
  L.o_tp = off; off += al(sizeof(int32_t) * (T * k + T));
  L.o_tk = off; off += al(sizeof(uint32_t) * 4);
  L.o_err = off; off += al(sizeof(int) * 4);
  L.o_gd = off; off += al(sizeof(int) * (G + 1));
  L.o_sc = off; off += al(sizeof(unsigned long long) * E);
  L.o_sm = off; off += al(sizeof(double) * E);
  L.o_gu = off; off += al(sizeof(float) * size_t(L.P_max) * L.gu_stride);
  L.o_xp = off; off += al(sizeof(uint16_t) * size_t(L.P_max) * L.x_ld);
  L.o_hp = off; off += al(sizeof(uint16_t) * size_t(L.P_max) * L.h_perm_ld);
  L.o_xg = off; off += al(sizeof(float) * P_gv * L.gv_H_pad);
  L.o_hg = off; off += al(sizeof(float) * P_gv * L.gv_F_pad);
  L.o_ys = off; off += al(sizeof(float) * (ys > gb ? ys : gb));
  L.o_sx = off; off += al(sizeof(uint16_t) * size_t(T) * c.hidden);
  L.o_sy = off; off += al(sizeof(uint16_t) * size_t(T) * c.hidden);
  L.total = off;
  return L;
}

// Splits of the down pass for a forward of T tokens: the automatic choice
// (or PW_DOWN_SPLIT), never more than the partials region holds.  per_sm 0
// selects the CUDA-core pass's choice.
int down_splits(const pw_moe* h, int T, int per_sm) {
  const int forced = env_int("PW_DOWN_SPLIT", 0);
  int ns = forced > 0 ? (forced < kMaxSplit ? forced : kMaxSplit)
           : per_sm > 0 ? splits_for(h->cfg, h->n_sm, T, per_sm)
                        : gv_splits_for(h->cfg, h->n_sm, T);
  const size_t per_split = positions(h->cfg, T) * h->cfg.hidden;
  while (ns > 1 && ns * per_split > h->ys_floats) --ns;
  return ns;
}

// CUDA-core decode passes for T up to the handle's gv_T (PW_GV=0 turns them
// off).
bool use_gv(const pw_moe* h, int T) {
  return h->gv_T > 0 && T <= h->gv_T && env_int("PW_GV", 1) != 0;
}

// Prefill passes (256-token chunks) when the routed slots average at least
// 64 tokens per expert; PW_PREFILL=0/1 forces the choice.
bool use_prefill(const pw_moe* h, int T) {
  if (!h->pf) return false;
  const int forced = env_int("PW_PREFILL", -1);
  if (forced >= 0) return forced != 0;
  return prefill_default(h->cfg, T);
}

}  // namespace

extern "C" {

int32_t pw_abi_version(void) { return PW_ABI_VERSION; }

pw_status_t pw_workspace_bytes(const pw_moe_config_t* cfg, int64_t* bytes) {
  if (!cfg || !bytes) return fail(PW_ERR_INVALID_ARG, "null argument");
  if (cfg->max_tokens < 1 || cfg->hidden < 8 || cfg->n_experts < 1 || cfg->top_k < 1 ||
      cfg->ffn < 1 || cfg->shared_ffn < 0)
    return fail(PW_ERR_INVALID_ARG, "bad config");
  int dev = 0, n_sm = 0;
  PW_CUDA(cudaGetDevice(&dev));
  PW_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  *bytes = static_cast<int64_t>(make_layout(*cfg, n_sm).total);
  return PW_OK;
}
const char* pw_last_error(void) { return g_err.c_str(); }

pw_status_t pw_moe_create(const pw_moe_config_t* cfg, const pw_block_desc_t* blocks,
                          int32_t n_blocks, pw_moe_t** out) {
  if (!cfg || !blocks || !out) return fail(PW_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  const pw_moe_config_t c = *cfg;
  if (c.hidden < 8 || c.hidden % 8) return fail(PW_ERR_INVALID_ARG, "hidden must be a positive multiple of 8");
  if (c.ffn < 1) return fail(PW_ERR_INVALID_ARG, "ffn must be positive");
  if (c.n_experts < 1 || c.n_experts > PW_MAX_EXPERTS)
    return fail(PW_ERR_INVALID_ARG, "n_experts must be in [1, %d]", PW_MAX_EXPERTS);
  if (c.top_k < 1 || c.top_k > c.n_experts || c.top_k > PW_MAX_TOPK)
    return fail(PW_ERR_INVALID_ARG, "top_k must be in [1, min(E, %d)]", PW_MAX_TOPK);
  if (c.shared_ffn < 0) return fail(PW_ERR_INVALID_ARG, "shared_ffn must be >= 0");
  if (c.n_max < 1 || c.n_max > PW_MAX_BITS) return fail(PW_ERR_INVALID_ARG, "n_max must be in [1, 8]");
  if (c.max_tokens < 1) return fail(PW_ERR_INVALID_ARG, "max_tokens must be >= 1");
  const int want_blocks = 3 * (c.n_experts + (c.shared_ffn > 0 ? 1 : 0));
  if (n_blocks != want_blocks)
    return fail(PW_ERR_INVALID_ARG, "expected %d blocks, got %d", want_blocks, n_blocks);
  for (int i = 0; i < n_blocks; ++i) {
    const pw_block_desc_t& b = blocks[i];
    if (!b.d_planes || !b.d_lut[0] || !b.d_lut[1])
      return fail(PW_ERR_INVALID_ARG, "block %d: null device buffer", i);
    if (!aligned16(b.d_planes) || !aligned16(b.d_lut[0]) || !aligned16(b.d_lut[1]))
      return fail(PW_ERR_INVALID_ARG, "block %d: device buffers must be 16-byte aligned", i);
    if (b.bits < 1 || b.bits > c.n_max)
      return fail(PW_ERR_INVALID_ARG, "block %d: bits %d outside [1, n_max]", i, b.bits);
  }

  pw_moe* h = new (std::nothrow) pw_moe();
  if (!h) return fail(PW_ERR_OOM, "host allocation failed");
  h->cfg = c;
  h->n_blocks = n_blocks;
  h->G = c.n_experts + (c.shared_ffn > 0 ? 1 : 0);
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
    free_all(h);
    return fail(PW_ERR_CUDA, "no CUDA device");
  }
  h->blk.resize(n_blocks);
  for (int i = 0; i < n_blocks; ++i) {
    auto& d = h->blk[i];
    const pw_block_desc_t& b = blocks[i];
    d.rows = block_rows(c, i);
    d.cols = block_cols(c, i);
    d.d_planes = b.d_planes;
    d.d_lut[0] = b.d_lut[0];
    d.d_lut[1] = b.d_lut[1];
    d.h_planes = b.h_planes;
    for (int k = 0; k <= PW_MAX_BITS; ++k) d.h_lut[k] = b.h_lut[k];
    d.bits = b.bits;
    d.slot = 0;
    d.stride = c.n_max;
    d.alloc = nullptr;
    d.pend_alloc = nullptr;
    d.pend_bits = 0;
    d.pend_req = 0;
    d.pend_planes = nullptr;
    d.ready = nullptr;
    if (cudaEventCreateWithFlags(&d.ready, cudaEventDisableTiming) != cudaSuccess) {
      free_all(h);
      return fail(PW_ERR_CUDA, "cudaEventCreate failed");
    }
  }
  if (cudaEventCreateWithFlags(&h->fwd_done, cudaEventDisableTiming) != cudaSuccess) {
    free_all(h);
    return fail(PW_ERR_CUDA, "cudaEventCreate failed");
  }

  // workspace, one allocation
  const Layout L = make_layout(c, h->n_sm);
  h->P_max = L.P_max;
  h->tc = L.tc;
  h->pf = L.pf;
  h->gu_stride = L.gu_stride;
  h->x_ld = L.x_ld;
  h->h_perm_ld = L.h_perm_ld;
  h->gbuf_ld = L.gbuf_ld;
  h->ys_floats = L.ys_floats;
  h->gv_T = L.gv_T;
  h->gv_H_pad = L.gv_H_pad;
  h->gv_F_pad = L.gv_F_pad;
  h->ws_bytes = L.total;
  const size_t o_tki = L.o_tki, o_tkw = L.o_tkw, o_off = L.o_off,
               o_st = L.o_st, o_sw = L.o_sw, o_tp = L.o_tp, o_tk = L.o_tk,
               o_err = L.o_err, o_gd = L.o_gd, o_sc = L.o_sc, o_sm = L.o_sm, o_gu = L.o_gu,
               o_xp = L.o_xp, o_hp = L.o_hp, o_ys = L.o_ys, o_sx = L.o_sx, o_sy = L.o_sy,
               o_xg = L.o_xg, o_hg = L.o_hg;
  const size_t off = L.total;
  if (cudaMalloc(&h->ws_base, off) != cudaSuccess) {
    free_all(h);
    return fail(PW_ERR_OOM, "workspace allocation of %zu bytes failed", off);
  }
  char* w = static_cast<char*>(h->ws_base);
  h->ws.topk_idx = reinterpret_cast<int32_t*>(w + o_tki);
  h->ws.topk_w = reinterpret_cast<float*>(w + o_tkw);
  h->ws.offsets = reinterpret_cast<int32_t*>(w + o_off);
  h->ws.slot_token = reinterpret_cast<int32_t*>(w + o_st);
  h->ws.slot_w = reinterpret_cast<float*>(w + o_sw);
  h->ws.token_pos = reinterpret_cast<int32_t*>(w + o_tp);
  h->ws.ticket = reinterpret_cast<uint32_t*>(w + o_tk);
  h->err = reinterpret_cast<int*>(w + o_err);
  h->gu_done = reinterpret_cast<int*>(w + o_gd);
  h->stat_count = reinterpret_cast<unsigned long long*>(w + o_sc);
  h->stat_mass = reinterpret_cast<double*>(w + o_sm);
  h->gu = reinterpret_cast<float*>(w + o_gu);
  h->x_sorted = reinterpret_cast<uint16_t*>(w + o_xp);
  h->h_perm = reinterpret_cast<uint16_t*>(w + o_hp);
  h->ysorted = reinterpret_cast<float*>(w + o_ys);
  h->gbuf = reinterpret_cast<uint16_t*>(w + o_ys);  // shares the partials region
  h->x_gv = reinterpret_cast<float*>(w + o_xg);
  h->h_gv = reinterpret_cast<float*>(w + o_hg);
  h->stage_x = reinterpret_cast<uint16_t*>(w + o_sx);
  h->stage_y = reinterpret_cast<uint16_t*>(w + o_sy);
  if (cudaMemset(w + o_tk, 0, o_gu - o_tk) != cudaSuccess ||
      cudaMemset(w + o_xp, 0, o_sx - o_xp) != cudaSuccess) {
    free_all(h);
    return fail(PW_ERR_CUDA, "cudaMemset failed");
  }
  // token-tile tensor maps for the tensor-core passes
  if (h->tc) {
    pw_status_t st = make_row_maps(h->x_maps, h->x_sorted, h->x_ld, h->P_max);
    if (st == PW_OK) st = make_row_maps(h->h_maps, h->h_perm, h->h_perm_ld, h->P_max);
    if (st == PW_OK && h->pf) st = make_chunk_map(&h->x_pf_map, h->x_sorted, h->x_ld, h->P_max);
    if (st == PW_OK && h->pf) st = make_chunk_map(&h->h_pf_map, h->h_perm, h->h_perm_ld, h->P_max);
    if (st != PW_OK) {
      free_all(h);
      return st;
    }
  }
  *out = h;
  return PW_OK;
}

pw_status_t pw_set_block_bits(pw_moe_t* h, int32_t block_id, int32_t new_bits,
                              pw_stream_t side_stream) {
  const NvtxRange nvtx("pw_set_block_bits (page move)");
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (block_id < 0 || block_id >= h->n_blocks)
    return fail(PW_ERR_INVALID_ARG, "block id %d out of range", block_id);
  auto& b = h->blk[block_id];
  if (new_bits < 1 || new_bits > h->cfg.n_max)
    return fail(PW_ERR_INVALID_ARG, "bits %d outside [1, n_max]", new_bits);
  if (b.pend_bits) return fail(PW_ERR_STATE, "block %d: a change to %d bits is still pending", block_id, b.pend_bits);
  if (new_bits == b.bits) return PW_OK;
  if (!b.h_lut[new_bits])
    return fail(PW_ERR_INVALID_ARG, "block %d: no host LUT for %d bits", block_id, new_bits);
  if (new_bits > b.bits && !b.h_planes)
    return fail(PW_ERR_INVALID_ARG, "block %d: raising bits needs the host planes", block_id);
  cudaStream_t s = static_cast<cudaStream_t>(side_stream);
  if (h->any_forward) PW_CUDA(cudaStreamWaitEvent(s, h->fwd_done, 0));
  if (h->paging) {
    // new storage holding exactly new_bits planes per tile group: the kept
    // planes come from the current storage, raised ones from the host copy;
    // the current storage is freed once the change has taken effect
    const size_t tile = pw::pages::kTileBytes;
    const size_t groups = static_cast<size_t>(pw::pages::groups_of(b.rows, b.cols));
    void* np = nullptr;
    if (cudaMallocFromPoolAsync(&np, static_cast<size_t>(new_bits) * groups * tile, h->pool, s) !=
        cudaSuccess) {
      cudaGetLastError();
      return fail(PW_ERR_OOM, "block %d: no room in the plane-page pool for %d planes", block_id,
                  new_bits);
    }
    uint32_t* dst = static_cast<uint32_t*>(np);
    b.pend_alloc = new PageAlloc{np, 1};
    const int keep = new_bits < b.bits ? new_bits : b.bits;
    PW_CUDA(cudaMemcpy2DAsync(dst, new_bits * tile, b.d_planes, b.stride * tile, keep * tile, groups,
                              cudaMemcpyDeviceToDevice, s));
    if (new_bits > b.bits) {
      const size_t pitch = static_cast<size_t>(h->cfg.n_max) * tile;
      const size_t off = static_cast<size_t>(b.bits) * (tile / 4);
      PW_CUDA(cudaMemcpy2DAsync(dst + off, new_bits * tile, b.h_planes + off, pitch,
                                static_cast<size_t>(new_bits - b.bits) * tile, groups,
                                cudaMemcpyHostToDevice, s));
    }
    b.pend_planes = dst;
  } else if (new_bits > b.bits) {
    // planes b.bits .. new_bits-1 are tiles b.bits.. of every tile group
    const size_t pitch = static_cast<size_t>(h->cfg.n_max) * pw::pages::kTileBytes;
    const size_t groups = static_cast<size_t>(pw::pages::groups_of(b.rows, b.cols));
    const size_t off = static_cast<size_t>(b.bits) * (pw::pages::kTileBytes / 4);
    PW_CUDA(cudaMemcpy2DAsync(b.d_planes + off, pitch, b.h_planes + off, pitch,
                              static_cast<size_t>(new_bits - b.bits) * pw::pages::kTileBytes,
                              groups, cudaMemcpyHostToDevice, s));
  }
  PW_CUDA(cudaMemcpyAsync(b.d_lut[b.slot ^ 1], b.h_lut[new_bits],
                          sizeof(uint16_t) * static_cast<size_t>(b.rows) << new_bits,
                          cudaMemcpyHostToDevice, s));
  PW_CUDA(cudaEventRecord(b.ready, s));
  b.pend_bits = new_bits;
  b.pend_req = h->n_forwards;
  return PW_OK;
}

pw_status_t pw_get_block_bits(const pw_moe_t* h, int32_t block_id, int32_t* bits_active,
                              int32_t* bits_pending) {
  if (!h || !bits_active) return fail(PW_ERR_INVALID_ARG, "null argument");
  if (block_id < 0 || block_id >= h->n_blocks)
    return fail(PW_ERR_INVALID_ARG, "block id %d out of range", block_id);
  const auto& b = h->blk[block_id];
  *bits_active = b.bits;
  if (bits_pending) *bits_pending = b.pend_bits;
  return PW_OK;
}

pw_status_t pw_get_forward_bits(const pw_moe_t* h, int32_t* bits, int32_t n) {
  if (!h || !bits) return fail(PW_ERR_INVALID_ARG, "null argument");
  if (n < h->n_blocks) return fail(PW_ERR_INVALID_ARG, "need room for %d bitwidths", h->n_blocks);
  for (int i = 0; i < h->n_blocks; ++i)
    bits[i] = h->fwd_bits.empty() ? h->blk[i].bits : h->fwd_bits[i];
  return PW_OK;
}

pw_status_t pw_set_switch_lag(pw_moe_t* h, int32_t max_lag) {
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (max_lag < 0) return fail(PW_ERR_INVALID_ARG, "max_lag must be >= 0");
  h->max_lag = max_lag;
  return PW_OK;
}

static pw_status_t forward_impl(pw_moe_t* h, const uint16_t* d_x, int32_t T,
                                const float* d_wr, const float* d_bias, uint16_t* d_y,
                                cudaStream_t s) {
  const NvtxRange nvtx("pw_moe_forward");
  const pw_moe_config_t& c = h->cfg;
  // pending page moves: one whose copy has already completed takes effect
  // now, without any wait; one that has stayed pending for max_lag forwards
  // takes effect now too, and the stream waits for its copy
  for (auto& b : h->blk) {
    if (!b.pend_bits) continue;
    const cudaError_t q = cudaEventQuery(b.ready);
    if (q != cudaSuccess && q != cudaErrorNotReady)
      return fail(PW_ERR_CUDA, "cudaEventQuery (page move) failed: %s", cudaGetErrorString(q));
    const bool landed = q == cudaSuccess;
    if (!landed && h->n_forwards - b.pend_req < h->max_lag) continue;
    if (!landed) PW_CUDA(cudaStreamWaitEvent(s, b.ready, 0));
    if (b.pend_planes) {
      // paging: the forwards issued so far may still read the old storage;
      // this stream-ordered free runs after them and before this forward
      if (b.alloc && --b.alloc->refs == 0) {
        PW_CUDA(cudaFreeAsync(b.alloc->base, s));
        delete b.alloc;
      }
      b.d_planes = b.pend_planes;
      b.stride = b.pend_bits;
      b.alloc = b.pend_alloc;
      b.pend_planes = nullptr;
      b.pend_alloc = nullptr;
    }
    b.bits = b.pend_bits;
    b.slot ^= 1;
    b.pend_bits = 0;
  }
  if (h->compacted) {
    PW_CUDA(cudaStreamWaitEvent(s, h->fwd_done, 0));
    h->compacted = false;
  }
  h->fwd_bits.resize(h->n_blocks);
  for (int i = 0; i < h->n_blocks; ++i) h->fwd_bits[i] = h->blk[i].bits;
  h->n_forwards++;
  h->last_T = T;
  if (T == 0) {
    PW_CUDA(cudaEventRecord(h->fwd_done, s));
    h->any_forward = true;
    return PW_OK;
  }
  pw::PageTable pt;
  for (int i = 0; i < h->n_blocks; ++i) {
    pt.blk[i].planes = h->blk[i].d_planes;
    pt.blk[i].lut = h->blk[i].d_lut[h->blk[i].slot];
    pt.bits[i] = static_cast<uint8_t>(h->blk[i].bits);
    pt.stride[i] = static_cast<uint8_t>(h->blk[i].stride);
  }
  const int has_shared = c.shared_ffn > 0 ? 1 : 0;
  const bool prefill = h->tc && use_prefill(h, T);
  // the down partials of split s start at s * split_stride: this forward's
  // positions times H, so the splits down_splits allows fit the region
  const long long split_stride = static_cast<long long>(positions(c, T)) * c.hidden;
  // few tokens per expert: the CUDA-core passes (gv.cu)
  const bool gv = !prefill && use_gv(h, T);
  // decode on the tensor cores: gate/up and down in one launch (PW_FUSED=0
  // splits them)
  const bool fused = h->tc && !prefill && !gv && env_int("PW_FUSED", 1) != 0;
  pw::GvParams gvp;
  if (gv) {
    std::memset(&gvp, 0, sizeof(gvp));
    gvp.pt = pt;
    gvp.H = c.hidden;
    gvp.F = c.ffn;
    gvp.S = c.shared_ffn;
    gvp.E = c.n_experts;
    gvp.n_groups = h->G;
    gvp.offsets = h->ws.offsets;
    gvp.slot_token = h->ws.slot_token;
    gvp.slot_w = h->ws.slot_w;
    gvp.x = d_x;
    gvp.x_gv = h->x_gv;
    gvp.h_gv = h->h_gv;
    gvp.H_pad = h->gv_H_pad;
    gvp.F_pad = h->gv_F_pad;
    gvp.ysorted = h->ysorted;
    gvp.split_stride = split_stride;
  }
  std::vector<cudaEvent_t> evs;
  if (h->profiling) {
    for (int i = 0; i < 5; ++i) {
      cudaEvent_t e;
      if (!h->ev_pool.empty()) {
        e = h->ev_pool.back();
        h->ev_pool.pop_back();
      } else {
        PW_CUDA(cudaEventCreate(&e));
      }
      evs.push_back(e);
    }
  }
  auto mark = [&](int i) -> cudaError_t {
    return h->profiling ? cudaEventRecord(evs[i], s) : cudaSuccess;
  };
  PW_CUDA(mark(0));

  pw::RouteParams rp{};
  rp.x = d_x;
  rp.wr = d_wr;
  rp.bias = d_bias;
  rp.T = T;
  rp.H = c.hidden;
  rp.E = c.n_experts;
  rp.k = c.top_k;
  rp.renorm = c.renorm_topk;
  rp.has_shared = has_shared;
  rp.ws = h->ws;
  rp.zero_words = fused ? h->gu_done : nullptr;
  rp.n_zero = fused ? h->G : 0;
  rp.stat_count = h->stat_count;
  rp.stat_mass = h->stat_mass;
  PW_CUDA(pw::launch_route(rp, h->n_sm, s));
  PW_CUDA(mark(1));

  // gate/up pass
  if (gv) {
    PW_CUDA(pw::launch_gv(gvp, 0, static_cast<int>(positions(c, T)), h->n_sm, s));
    PW_CUDA(pw::launch_gv(gvp, 1, 0, h->n_sm, s));
  } else if (h->tc) {
    pw::GatherParams gp{};
    gp.x = d_x;
    gp.offsets = h->ws.offsets;
    gp.slot_token = h->ws.slot_token;
    gp.x_sorted = h->x_sorted;
    gp.H = c.hidden;
    gp.ld = h->x_ld;
    gp.rows = h->P_max;
    gp.n_groups = h->G;
    PW_CUDA(pw::launch_gather(gp, T * c.top_k + (c.shared_ffn > 0 ? T : 0), h->n_sm, s));
    pw::TcParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.pt = pt;
    tp.mode = prefill ? pw::kTcPfGate : (fused ? pw::kTcFused : pw::kTcGateUp);
    tp.H = c.hidden;
    tp.F = c.ffn;
    tp.S = c.shared_ffn;
    tp.E = c.n_experts;
    tp.n_groups = h->G;
    tp.n_split = 1;
    tp.offsets = h->ws.offsets;
    tp.slot_token = h->ws.slot_token;
    tp.slot_w = h->ws.slot_w;
    for (int i = 0; i < 4; ++i) tp.b_maps[i] = h->x_maps[i];
    tp.n_max = c.n_max;
    tp.h_perm = h->h_perm;
    tp.h_perm_ld = h->h_perm_ld;
    tp.h_rows = h->P_max;
    tp.err = h->err;
    tp.test_stall_group = -1;
    if (fused) {
      // test switches: a shorter wait limit, and one group's down items
      // waiting for a count that never arrives (failure-detection tests)
      tp.wait_ns = static_cast<unsigned long long>(env_int("PW_TEST_WAIT_US", 0)) * 1000ull;
      tp.test_stall_group = env_int("PW_TEST_STALL_GROUP", -1);
      tp.n_split = down_splits(h, T, 6);
      if (static_cast<size_t>(tp.n_split) * split_stride > h->ys_floats)
        return fail(PW_ERR_STATE, "down partials (%d splits) exceed the workspace", tp.n_split);
      // down items wait on other CTAs' gate/up items, so every CTA must be
      // resident: the launch is cooperative (refused rather than stalled when
      // the grid cannot be co-resident); PW_COOP=0 drops the attribute
      tp.cooperative = env_int("PW_COOP", 1);
      for (int i = 0; i < 4; ++i) tp.h_maps[i] = h->h_maps[i];
      tp.gu_done = h->gu_done;
      tp.ysorted = h->ysorted;
      tp.split_stride = split_stride;
    }
    if (prefill) {
      // gate -> g (fp16), then up -> h = silu(g) * u
      tp.pf_map = h->x_pf_map;
      tp.gbuf = h->gbuf;
      tp.gbuf_ld = h->gbuf_ld;
      PW_CUDA(pw::launch_tc(tp, h->n_sm, s));
      tp.mode = pw::kTcPfUp;
    }
    PW_CUDA(pw::launch_tc(tp, h->n_sm, s));
  } else {
    pw::SimpleParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.pt = pt;
    sp.mode = 0;
    sp.n_max = c.n_max;
    sp.H = c.hidden;
    sp.F = c.ffn;
    sp.S = c.shared_ffn;
    sp.E = c.n_experts;
    sp.n_groups = h->G;
    sp.offsets = h->ws.offsets;
    sp.slot_token = h->ws.slot_token;
    sp.slot_w = h->ws.slot_w;
    sp.x = d_x;
    sp.gu = h->gu;
    sp.gu_stride = h->gu_stride;
    const int rows = c.ffn > c.shared_ffn ? c.ffn : c.shared_ffn;
    PW_CUDA(pw::launch_simple(sp, rows, s));
  }
  PW_CUDA(mark(2));
  // down pass
  int n_split = 1;
  if (gv) {
    n_split = down_splits(h, T, 0);
    if (static_cast<size_t>(n_split) * split_stride > h->ys_floats)
      return fail(PW_ERR_STATE, "down partials (%d splits) exceed the workspace", n_split);
    gvp.n_split = n_split;
    PW_CUDA(pw::launch_gv(gvp, 2, 0, h->n_sm, s));
  } else if (fused) {
    n_split = down_splits(h, T, 6);  // the down items ran in the launch above
  } else if (h->tc) {
    n_split = prefill ? 1 : down_splits(h, T, 4);
    if (static_cast<size_t>(n_split) * split_stride > h->ys_floats)
      return fail(PW_ERR_STATE, "down partials (%d splits) exceed the workspace", n_split);
    pw::TcParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.test_stall_group = -1;
    tp.pt = pt;
    tp.mode = prefill ? pw::kTcPfDown : pw::kTcDown;
    tp.pf_map = h->h_pf_map;
    tp.H = c.hidden;
    tp.F = c.ffn;
    tp.S = c.shared_ffn;
    tp.E = c.n_experts;
    tp.n_groups = h->G;
    tp.n_split = n_split;
    tp.offsets = h->ws.offsets;
    tp.slot_token = h->ws.slot_token;
    tp.slot_w = h->ws.slot_w;
    for (int i = 0; i < 4; ++i) tp.b_maps[i] = h->h_maps[i];
    tp.n_max = c.n_max;
    tp.h_perm = h->h_perm;
    tp.h_perm_ld = h->h_perm_ld;
    tp.ysorted = h->ysorted;
    tp.split_stride = split_stride;
    tp.err = h->err;
    PW_CUDA(pw::launch_tc(tp, h->n_sm, s));
  } else {
    pw::SimpleParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.pt = pt;
    sp.mode = 1;
    sp.n_max = c.n_max;
    sp.H = c.hidden;
    sp.F = c.ffn;
    sp.S = c.shared_ffn;
    sp.E = c.n_experts;
    sp.n_groups = h->G;
    sp.offsets = h->ws.offsets;
    sp.slot_token = h->ws.slot_token;
    sp.slot_w = h->ws.slot_w;
    sp.gu = h->gu;
    sp.gu_stride = h->gu_stride;
    sp.ysorted = h->ysorted;
    PW_CUDA(pw::launch_simple(sp, c.hidden, s));
  }
  PW_CUDA(mark(3));
  pw::CombineParams cp{};
  cp.ysorted = h->ysorted;
  cp.token_pos = h->ws.token_pos;
  cp.y = d_y;
  cp.T = T;
  cp.H = c.hidden;
  cp.k = c.top_k;
  cp.has_shared = has_shared;
  cp.n_split = n_split;
  cp.split_stride = split_stride;
  PW_CUDA(pw::launch_combine(cp, s));
  PW_CUDA(mark(4));
  if (h->profiling) h->ev_pending.push_back(evs);
  PW_CUDA(cudaEventRecord(h->fwd_done, s));
  h->any_forward = true;
  return PW_OK;
}

pw_status_t pw_moe_forward(pw_moe_t* h, const uint16_t* d_x, int32_t T, const float* d_router_w,
                           const float* d_router_bias, uint16_t* d_y, pw_stream_t stream) {
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (T < 0 || T > h->cfg.max_tokens)
    return fail(PW_ERR_INVALID_ARG, "T = %d outside [0, max_tokens = %d]", T, h->cfg.max_tokens);
  if (T > 0 && (!d_x || !d_router_w || !d_y)) return fail(PW_ERR_INVALID_ARG, "null buffer");
  if ((d_x && !aligned16(d_x)) || (d_y && !aligned16(d_y)) ||
      (d_router_w && !aligned16(d_router_w)))
    return fail(PW_ERR_INVALID_ARG, "x, y and router weights must be 16-byte aligned");
  return forward_impl(h, d_x, T, d_router_w, d_router_bias, d_y, static_cast<cudaStream_t>(stream));
}

pw_status_t pw_moe_forward_host(pw_moe_t* h, const uint16_t* x_host, int32_t T,
                                const float* d_router_w, const float* d_router_bias,
                                uint16_t* y_host, pw_stream_t stream) {
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (T < 0 || T > h->cfg.max_tokens)
    return fail(PW_ERR_INVALID_ARG, "T = %d outside [0, max_tokens = %d]", T, h->cfg.max_tokens);
  if (T > 0 && (!x_host || !y_host || !d_router_w)) return fail(PW_ERR_INVALID_ARG, "null buffer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(uint16_t) * static_cast<size_t>(T) * h->cfg.hidden;
  if (T > 0) PW_CUDA(cudaMemcpyAsync(h->stage_x, x_host, bytes, cudaMemcpyHostToDevice, s));
  pw_status_t st = forward_impl(h, h->stage_x, T, d_router_w, d_router_bias, h->stage_y, s);
  if (st != PW_OK) return st;
  if (T > 0) PW_CUDA(cudaMemcpyAsync(y_host, h->stage_y, bytes, cudaMemcpyDeviceToHost, s));
  PW_CUDA(cudaStreamSynchronize(s));
  return PW_OK;
}

pw_status_t pw_linear(const uint32_t* d_planes, const uint16_t* d_lut, int32_t rows, int32_t cols,
                      int32_t n_max, int32_t bits, const uint16_t* d_x, int32_t T, float* d_y,
                      pw_stream_t stream) {
  if (rows < 1 || cols < 1 || T < 0) return fail(PW_ERR_INVALID_ARG, "bad shape");
  if (n_max < 1 || n_max > PW_MAX_BITS || bits < 1 || bits > n_max)
    return fail(PW_ERR_INVALID_ARG, "need 1 <= bits <= n_max <= 8");
  if (!d_planes || !d_lut || (T > 0 && (!d_x || !d_y))) return fail(PW_ERR_INVALID_ARG, "null buffer");
  if (!aligned16(d_planes) || !aligned16(d_lut) || (d_x && !aligned16(d_x)))
    return fail(PW_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  if (T == 0) return PW_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dev = 0, n_sm = 0;
  PW_CUDA(cudaGetDevice(&dev));
  PW_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  if (tc_shape_ok(cols) && env_int("PW_FORCE_SIMPLE", 0) == 0) {
    pw::TcParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.test_stall_group = -1;
    tp.mode = pw::kTcLinear;
    tp.n_groups = 1;
    tp.n_split = 1;
    tp.x = d_x;
    tp.y = d_y;
    tp.T = T;
    tp.lin_rows = rows;
    tp.lin_cols = cols;
    tp.lin_bits = bits;
    tp.lin_lut = d_lut;
    tp.lin_planes = d_planes;
    tp.lin_n_max = n_max;
    tp.err = nullptr;
    PW_CUDA(pw::launch_tc(tp, n_sm, s));
  } else {
    pw::SimpleParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.mode = 2;
    sp.x = d_x;
    sp.y = d_y;
    sp.T = T;
    sp.lin_rows = rows;
    sp.lin_cols = cols;
    sp.lin_bits = bits;
    sp.lin_n_max = n_max;
    sp.lin_planes = d_planes;
    sp.lin_lut = d_lut;
    PW_CUDA(pw::launch_simple(sp, rows, s));
  }
  return PW_OK;
}

int64_t pw_plane_bytes(int32_t rows, int32_t cols) {
  if (rows < 1 || cols < 1) return 0;
  return pw::pages::plane_words(rows, cols) * 4;
}

pw_status_t pw_repack_planes(const uint32_t* d_src, uint32_t* d_dst, int32_t rows, int32_t cols,
                             int32_t n_planes, pw_stream_t stream) {
  if (!d_src || !d_dst || rows < 1 || cols < 1 || n_planes < 1 || n_planes > PW_MAX_BITS)
    return fail(PW_ERR_INVALID_ARG, "bad repack arguments");
  if (!aligned16(d_src) || !aligned16(d_dst))
    return fail(PW_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  PW_CUDA(pw::launch_repack(d_src, d_dst, rows, cols, n_planes, static_cast<cudaStream_t>(stream)));
  return PW_OK;
}

pw_status_t pw_get_routing(const pw_moe_t* h, int32_t* d_idx, float* d_w, pw_stream_t stream) {
  if (!h || !d_idx || !d_w) return fail(PW_ERR_INVALID_ARG, "null argument");
  const size_t n = static_cast<size_t>(h->last_T) * h->cfg.top_k;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n) {
    PW_CUDA(cudaMemcpyAsync(d_idx, h->ws.topk_idx, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
    PW_CUDA(cudaMemcpyAsync(d_w, h->ws.topk_w, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
  }
  return PW_OK;
}

pw_status_t pw_routing_stats(pw_moe_t* h, uint64_t* counts, double* mass, int32_t reset,
                             pw_stream_t stream) {
  if (!h || !counts || !mass) return fail(PW_ERR_INVALID_ARG, "null argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = h->cfg.n_experts;
  static_assert(sizeof(uint64_t) == sizeof(unsigned long long), "64-bit counters");
  PW_CUDA(cudaMemcpyAsync(counts, h->stat_count, sizeof(uint64_t) * E, cudaMemcpyDeviceToHost, s));
  PW_CUDA(cudaMemcpyAsync(mass, h->stat_mass, sizeof(double) * E, cudaMemcpyDeviceToHost, s));
  if (reset) {
    PW_CUDA(cudaMemsetAsync(h->stat_count, 0, sizeof(uint64_t) * E, s));
    PW_CUDA(cudaMemsetAsync(h->stat_mass, 0, sizeof(double) * E, s));
  }
  PW_CUDA(cudaStreamSynchronize(s));
  return PW_OK;
}

pw_status_t pw_enable_paging(pw_moe_t* h, pw_stream_t stream) {
  const NvtxRange nvtx("pw_enable_paging");
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (h->paging) return PW_OK;
  for (int i = 0; i < h->n_blocks; ++i) {
    if (!h->blk[i].h_planes)
      return fail(PW_ERR_INVALID_ARG, "block %d: paging needs the host copy of its planes", i);
    if (h->blk[i].pend_bits)
      return fail(PW_ERR_STATE, "block %d: a bitwidth change is still pending", i);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemPoolProps props = {};
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = h->device;
  PW_CUDA(cudaMemPoolCreate(&h->pool, &props));
  const size_t tile = pw::pages::kTileBytes;
  size_t total = 0;
  for (const auto& b : h->blk)
    total += static_cast<size_t>(b.bits) * pw::pages::groups_of(b.rows, b.cols) * tile;
  void* arena = nullptr;
  if (cudaMallocFromPoolAsync(&arena, total, h->pool, s) != cudaSuccess) {
    cudaGetLastError();
    cudaMemPoolDestroy(h->pool);
    h->pool = nullptr;
    return fail(PW_ERR_OOM, "plane-page pool allocation of %zu bytes failed", total);
  }
  // every block's resident planes, packed one block after another
  size_t off = 0;
  std::vector<uint32_t*> fresh(h->n_blocks, nullptr);
  for (int i = 0; i < h->n_blocks; ++i) {
    auto& b = h->blk[i];
    const size_t groups = static_cast<size_t>(pw::pages::groups_of(b.rows, b.cols));
    fresh[i] = reinterpret_cast<uint32_t*>(static_cast<char*>(arena) + off);
    PW_CUDA(cudaMemcpy2DAsync(fresh[i], b.bits * tile, b.d_planes, b.stride * tile, b.bits * tile,
                              groups, cudaMemcpyDeviceToDevice, s));
    off += static_cast<size_t>(b.bits) * groups * tile;
  }
  // the copies have landed and no forward issued so far still reads the
  // caller's storage
  PW_CUDA(cudaStreamSynchronize(s));
  if (h->any_forward) PW_CUDA(cudaEventSynchronize(h->fwd_done));
  PageAlloc* a = new PageAlloc{arena, h->n_blocks};
  for (int i = 0; i < h->n_blocks; ++i) {
    auto& b = h->blk[i];
    b.d_planes = fresh[i];
    b.stride = b.bits;
    b.alloc = a;
  }
  h->paging = true;
  return PW_OK;
}

pw_status_t pw_compact_pages(pw_moe_t* h, pw_stream_t stream) {
  const NvtxRange nvtx("pw_compact_pages");
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  if (!h->paging) return fail(PW_ERR_STATE, "paging is not enabled");
  for (int i = 0; i < h->n_blocks; ++i)
    if (h->blk[i].pend_bits)
      return fail(PW_ERR_STATE, "block %d: a bitwidth change is still pending", i);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tile = pw::pages::kTileBytes;
  size_t total = 0;
  for (const auto& b : h->blk)
    total += static_cast<size_t>(b.stride) * pw::pages::groups_of(b.rows, b.cols) * tile;
  // after every forward issued so far; the caller's next forwards run on
  // this stream, behind the copies
  if (h->any_forward) PW_CUDA(cudaStreamWaitEvent(s, h->fwd_done, 0));
  void* arena = nullptr;
  if (cudaMallocFromPoolAsync(&arena, total, h->pool, s) != cudaSuccess) {
    cudaGetLastError();
    return fail(PW_ERR_OOM, "plane-page pool allocation of %zu bytes failed", total);
  }
  size_t off = 0;
  PageAlloc* a = new PageAlloc{arena, h->n_blocks};
  for (auto& b : h->blk) {
    const size_t bytes = static_cast<size_t>(b.stride) * pw::pages::groups_of(b.rows, b.cols) * tile;
    uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<char*>(arena) + off);
    PW_CUDA(cudaMemcpyAsync(dst, b.d_planes, bytes, cudaMemcpyDeviceToDevice, s));
    if (b.alloc && --b.alloc->refs == 0) {
      PW_CUDA(cudaFreeAsync(b.alloc->base, s));
      delete b.alloc;
    }
    b.d_planes = dst;
    b.alloc = a;
    off += bytes;
  }
  PW_CUDA(cudaEventRecord(h->fwd_done, s));
  h->any_forward = true;
  h->compacted = true;  // a forward on another stream waits for the copies
  return PW_OK;
}

pw_status_t pw_resident_bytes(pw_moe_t* h, int64_t* plane_bytes, int64_t* pool_reserved) {
  if (!h || !plane_bytes) return fail(PW_ERR_INVALID_ARG, "null argument");
  int64_t total = 0;
  for (const auto& b : h->blk) {
    const int64_t groups = pw::pages::groups_of(b.rows, b.cols);
    const int64_t planes = (b.alloc || !h->paging) ? b.stride : 0;
    total += planes * groups * pw::pages::kTileBytes;
    if (b.pend_planes) total += static_cast<int64_t>(b.pend_bits) * groups * pw::pages::kTileBytes;
  }
  *plane_bytes = total;
  if (pool_reserved) {
    *pool_reserved = 0;
    if (h->pool) {
      // hand memory the pool no longer uses back to the device first
      if (h->fwd_done) PW_CUDA(cudaEventSynchronize(h->fwd_done));
      for (auto& b : h->blk)
        if (b.pend_bits) PW_CUDA(cudaEventSynchronize(b.ready));
      PW_CUDA(cudaMemPoolTrimTo(h->pool, 0));
      cuuint64_t v = 0;
      PW_CUDA(cudaMemPoolGetAttribute(h->pool, cudaMemPoolAttrReservedMemCurrent, &v));
      *pool_reserved = static_cast<int64_t>(v);
    }
  }
  return PW_OK;
}

pw_status_t pw_check_device_error(pw_moe_t* h) {
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  PW_CUDA(cudaDeviceSynchronize());
  int e = 0;
  PW_CUDA(cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (e) {
    PW_CUDA(cudaMemset(h->err, 0, sizeof(int)));
    return fail(static_cast<pw_status_t>(e), "device-side wait gave up (error %d)", e);
  }
  return PW_OK;
}

pw_status_t pw_profile_enable(pw_moe_t* h, int32_t on) {
  if (!h) return fail(PW_ERR_INVALID_ARG, "null handle");
  h->profiling = on != 0;
  return PW_OK;
}

pw_status_t pw_profile_read(pw_moe_t* h, float* ms, int32_t n, int32_t* n_forwards) {
  if (!h || !ms || n < 4) return fail(PW_ERR_INVALID_ARG, "need a handle and room for 4 floats");
  for (int i = 0; i < n; ++i) ms[i] = 0.0f;
  int count = 0;
  for (auto& v : h->ev_pending) {
    PW_CUDA(cudaEventSynchronize(v[4]));
    for (int i = 0; i < 4; ++i) {
      float t = 0.0f;
      PW_CUDA(cudaEventElapsedTime(&t, v[i], v[i + 1]));
      ms[i] += t;
    }
    for (auto e : v) h->ev_pool.push_back(e);
    ++count;
  }
  h->ev_pending.clear();
  if (n_forwards) *n_forwards = count;
  return PW_OK;
}

int32_t pw_forward_launches(const pw_moe_t* h, int32_t T) {
  if (!h) return 0;
  if (T <= 0) return 0;
  if (use_prefill(h, T)) return 6;
  if (use_gv(h, T)) return 5;
  if (!h->tc) return 4;
  return env_int("PW_FUSED", 1) != 0 ? 4 : 5;
}

pw_status_t pw_destroy(pw_moe_t* h) {
  if (!h) return PW_OK;
  pw_status_t st = PW_OK;
  if (h->fwd_done && cudaEventSynchronize(h->fwd_done) != cudaSuccess)
    st = fail(PW_ERR_CUDA, "waiting for the last forward failed");
  for (auto& b : h->blk)
    if (b.ready && cudaEventSynchronize(b.ready) != cudaSuccess)
      st = fail(PW_ERR_CUDA, "waiting for a page move failed");
  free_all(h);
  return st;
}

}  // extern "C"
