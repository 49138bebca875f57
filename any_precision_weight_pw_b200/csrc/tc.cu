// tc.cu -- tensor-core dequant-GEMM over Any-Precision bit-plane pages
// (sm_100a: TMA + tcgen05 + TMEM).
//
// PagedWeight (legiblepapers summary, FAQ Q5; arxivlens abstract): the fused
// mixed-precision MoE kernel reads the AP bit-planes and per-row LUTs of the
// resident pages directly, at a separate bitwidth for every linear-block, and
// fuses the expert activation and the output accumulation.
//
// One persistent CTA per SM walks a list of work items.  A decode item is
// 128 output rows x up to 32 tokens of one expert, in one or two passes over
// K: the gate/up item makes a gate pass and an up pass over the same rows (so
// its epilogue can apply SwiGLU); the down item makes one pass (over one K
// range when the down pass is split); a standalone linear makes one pass.  At
// decode both kinds run in one launch (mode kTcFused): gate/up items first,
// then down items, a down item of group g loading h only after g's gate/up
// epilogues have all counted themselves.  Prefill items (Cfg<true>) are 128
// rows x 256 tokens, one pass each, gate, up and down as three launches.
//   warp 8      producer: streams only the b active bit-planes of the block,
//               128 rows x 256 columns (8 words) per stage: in the paged
//               layout (pages.h) the b tiles are one contiguous b * 4 KB run,
//               moved by ONE bulk copy into a ring of 4 KB slots (stages take
//               b consecutive slots, so the ring holds more stages at low b);
//               the tiles arrive with their rows' halves already swizzled, so
//               the thread-per-row reads below are bank-conflict free.
//   warp 10     token-tile loader: the item's token rows are contiguous in an
//               fp16 buffer already in the A operand's K order (the gathered
//               activations for gate/up, h = silu(g)*u for down), so one lane
//               moves each B stage with ONE 3-D TMA box (decode: 2 atoms of
//               64 columns x 8, 16, 24 or 32 rows, two B stages per plane
//               stage; prefill: 1 atom x 256 rows; 128-byte swizzle = the
//               MMA's K-major B layout).  A standalone linear converts its
//               bf16 rows with all 32 lanes.
//   warps 0-7   dequantisers in two K halves: warps q and q+4 both own rows
//               32q..32q+31 (thread <-> output row <-> TMEM lane); the first
//               group takes columns 0-127 of every stage, the second
//               columns 128-255.  Each thread unpacks its row's codes from the
//               b plane words (a bit-matrix transpose), looks them up in the
//               shared-memory table of the pass (pair table up to b = 4 at
//               decode and b = 3 at prefill, single table above; see
//               dequant.cuh) and writes fp16 weights into a TMEM ring slot
//               (the MMA's A operand).
//   warp 9      MMA issuer: tcgen05.mma kind::f16, M=128, N=16/32 (decode)
//               or 256 (prefill), K=16, fp32 accumulators in TMEM (decode:
//               two buffers, alternating items, gate and up side by side).
//   warps 11-14 epilogue: tcgen05.ld the accumulators; write h = silu(g)*u
//               as fp16 in the down pass's K order (gate/up), the routing-
//               weighted fp32 partials (down), g as fp16 (prefill gate) or
//               the fp32 result (linear).
// The forward's kernels are launched with programmatic dependent launch;
// this kernel waits for its predecessor before it reads anything and
// releases its successor at once: the successor's blocks can only take an
// SM that one of this grid's CTAs has left (all of them are resident by
// then, one per SM, and no other block fits beside one), where they wait
// for this grid to finish, so the successor's launch latency hides behind
// this kernel's tail.
// Every wait is an mbarrier try_wait (the hardware holds the waiting thread
// for a while between tests) bounded by a global-timer deadline; a timeout
// raises the CTA's
// abort flag and the device error word, and every role drains what it has in
// flight before the CTA frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "dequant.cuh"
#include "pages.h"
#include "pw_internal.h"
#include "tc.h"

namespace pw {
namespace {

constexpr int kTileRows = 128;
constexpr int kStageWords = 8;                 // 256 columns per stage
constexpr int kSlotBytes = kTileRows * kStageWords * 4;  // 4 KB: one plane of a stage
constexpr int kNS = 8;                         // plane stages in flight (barrier pairs)
constexpr int kAColsPerSlot = 64;              // TMEM columns of one 128-K A slot
constexpr int kTmemCols = 512;
constexpr int kDqThreads = 256;                // 8 dequantiser warps
constexpr int kWarpProducer = 8, kWarpMma = 9, kWarpLoader = 10;
constexpr int kThreads = 15 * 32;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kOffLut = 0;                // table region (dequant.cuh gives its layout)

// Two configurations of the kernel.
//   decode  token tiles of up to 32 rows (MMA N = 16 or 32); one TMA box per
//           128-column B stage (one per A slot); two accumulator buffers (gate
//           and up side by side) so an item's epilogue overlaps the next
//           item's MMAs; a 128 KB table region, so 4-bit blocks take pair
//           tables too.
//   prefill 256-token chunks (MMA N = 256), so each dequantised weight tile
//           serves 256 tokens; B stages of 64 columns (32 KB); one 256-column
//           accumulator, so gate and up run as separate launches; a 64 KB
//           table region (pair tables up to 3 bits).
// Shared memory offsets are compile-time (from a 1024-byte aligned base) so
// table lookups fold the base into the loads' immediate offsets.
template <bool PF>
struct Cfg {
  static constexpr bool kPrefill = PF;
  static constexpr int kNSlot = 16;            // plane slots
  static constexpr int kNT = PF ? kTcPfTokens : kTcTokens;
  // table layout (dequant.cuh): split (rows own their words, 128 KB) or packed
  static constexpr bool kSplitRows = !PF;
  static constexpr int kPairMax = dq::pair_max(kSplitRows);  // widest pair-table bitwidth
  static constexpr uint32_t kLutBytes = dq::table_bytes(kSplitRows);
  static constexpr int kBStageK = PF ? 64 : 128;
  static constexpr int kBStageBytes = kNT * kBStageK * 2;
  static constexpr int kBPerStage = 256 / kBStageK;
  static constexpr int kNB = PF ? 3 : 4;        // token-tile ring depth (slots of kBStageBytes)
  static constexpr int kNBB = PF ? kNB : 16;    // token-tile barrier pairs (decode: up to 16
                                                // slots when the launch's tiles are small)
  static constexpr int kNA = PF ? 4 : 6;        // TMEM A ring slots (128 K each)
  static constexpr int kNDBuf = PF ? 1 : 2;     // accumulator buffers
  static constexpr int kDColsPerBuf = PF ? 256 : 64;
  static constexpr int kAColBase = kNDBuf * kDColsPerBuf;
  static constexpr uint32_t kOffSlots = kOffLut + kLutBytes;
  static constexpr uint32_t kOffB = kOffSlots + kNSlot * kSlotBytes;
  static constexpr uint32_t kOffBars = kOffB + kNB * kBStageBytes;
  static constexpr uint32_t kNumBars = 2 * kNS + 2 * kNBB + 2 * kNA + 2 * kNDBuf + 1 + 4;
  static constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
  // misc: tmem holder, abort flag, then s_prefix, s_prefix2 and the group
  // offsets (kMaxGroups + 2 ints each)
  static constexpr uint32_t kOffSlotUser = kOffMisc + 16 + 12 * (kMaxGroups + 2);
  static constexpr uint32_t kSmemTotal = kOffSlotUser + 4 * kNSlot;
  static_assert(kSmemTotal <= 232448, "shared memory budget of one CTA");
  static_assert(kAColBase + kNA * kAColsPerSlot <= kTmemCols, "tensor memory budget");
};
using Dec = Cfg<false>;
using Pre = Cfg<true>;

// Plane stages take `bits` consecutive slots of the ring; a stage that would
// run past the end starts again at slot 0.  Producer and dequantisers walk
// the same sequence of stages, so both derive the same placement.
template <class C>
__device__ __forceinline__ uint32_t place_stage(uint32_t& ring_end, int bits) {
  const uint32_t start = (ring_end + bits <= static_cast<uint32_t>(C::kNSlot)) ? ring_end : 0u;
  ring_end = start + bits;
  return start;
}

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
// One arrival for the whole warp, after every lane's earlier accesses (the
// warp barrier orders them before lane 0's release).
__device__ __forceinline__ void mbar_arrive_warp(uint64_t* b) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(b);
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)),
               "r"(bytes)
               : "memory");
}
// Test (and, for a system-dependent time, wait for) completion of a phase.
// No suspend hint: with a 2 or 100 us hint the decode launch measured ~1%
// slower at every width.
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

struct Ctl {
  volatile int* abort;  // shared
  int* err;             // global, may be null
  unsigned long long wait_ns;  // limit of one wait
};

// Wait for the phase with the given parity; false on timeout or abort.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* b, uint32_t parity, const Ctl& c) {
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try(b, parity)) return true;
    if (*c.abort) return false;
    if (global_ns() - t0 > c.wait_ns) {
      *c.abort = 1;
      if (c.err) atomicExch(c.err, PW_ERR_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, const Ctl& c) {
  return mbar_try(b, parity) || mbar_wait_slow(b, parity, c);
}
// The same wait for a whole warp: every lane gets the same answer, so the
// warp-collective tcgen05 instructions that follow never run on a partial warp.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* b, uint32_t parity, const Ctl& c) {
  const bool ok = mbar_wait(b, parity, c);
  return __all_sync(0xffffffffu, ok);
}
// Drain wait: bounded, ignores the abort flag.
__device__ __noinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try(b, parity))
    if (global_ns() - t0 > 200000000ull) return;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
// The same with an L2 policy (the decode configuration streams each plane
// page once per forward: evict-first keeps the L2 for the data and code the
// other kernels of the forward reuse).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_load_hint(uint32_t dst, const void* src, uint32_t bytes,
                                               uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// A fused launch's down item of group g reads h rows that other CTAs' gate/up
// epilogues write: wait (bounded) until all of g's gate/up items are counted,
// then order the TMA reads that follow after those writes.
// (A test switch, p.test_stall_group, makes one group's down items wait for
// one count more than will ever arrive, so the bounded wait runs out.)
__device__ __noinline__ bool wait_gate_up(const TcParams& p, int g, int need, const Ctl& c) {
  if (g == p.test_stall_group) ++need;
  const unsigned long long t0 = global_ns();
  while (ld_acquire_gpu(p.gu_done + g) < need) {
    if (*c.abort) return false;
    if (global_ns() - t0 > c.wait_ns) {
      *c.abort = 1;
      if (c.err) atomicExch(c.err, PW_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(200);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(b))
               : "memory");
}
// One lane of the (converged) warp, the same lane every time.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n.reg .pred P1;\n.reg .b32 r;\nelect.sync r|P1, %1;\nselp.u32 %0, 1, 0, P1;\n}\n"
      : "=r"(pred)
      : "r"(0xffffffffu));
  return pred != 0;
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// UMMA shared-memory descriptor: K-major operand in the 128-byte swizzle
// layout (8-row groups of 1024 B, 16 B leading offset, version 1).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;     // leading byte offset (16 B units)
  d |= static_cast<uint64_t>(64) << 32;    // stride byte offset: 1024 B
  d |= static_cast<uint64_t>(1) << 46;     // descriptor version
  d |= static_cast<uint64_t>(2) << 61;     // 128-byte swizzle
  return d;
}
// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D, M=128.
__device__ __forceinline__ uint32_t mma_idesc(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ float bf16f(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of 16-byte chunk c16 (0..31) of token row n in a B stage of
// `rows` rows (K-major, 128-byte swizzle: 64 columns per 128-byte atom row,
// atoms of `rows` rows one after the other).
__device__ __forceinline__ uint32_t b_chunk_off(int n, int c16, int rows) {
  const int atom = c16 >> 3, c = c16 & 7;
  return atom * (rows * 128) + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4);
}
// Rows of a token tile as loaded: whole 8-row groups covering ntok.
__device__ __forceinline__ int tile_rows(int ntok) { return ((ntok + 7) >> 3) << 3; }

// ---------------------------------------------------------------- work items
struct Pass {
  int blk, bits;
  const uint16_t* lut;
  const uint32_t* planes;  // plane pages (pages.h)
  int stride;              // planes stored per tile group
};
struct Item {
  int g, row0, tok0, ntok, pos0, split, rows, cols, npass, s_begin, s_end;
  int kind;  // the item's pass: the launch mode, or gate/up or down in a fused launch
};

// Items are visited in increasing order by every role, so the group search
// resumes from the previous item's group (gh).
__device__ __forceinline__ bool gate_or_up(int mode) {
  return mode == kTcGateUp || mode == kTcPfGate || mode == kTcPfUp;
}

// Items of a fused launch: [0, s_prefix[G]) gate/up, then the down items
// listed by s_prefix2; gh holds one search hint per list.  The group offsets
// (token positions) are the shared-memory copy that follows s_prefix2.
template <class C>
__device__ __forceinline__ void decode_item(const TcParams& p, const int* s_prefix,
                                            const int* s_prefix2, int G, int i, Item& it,
                                            int (&gh)[2]) {
  int kind = p.mode;
  const int* pre = s_prefix;
  int li = i, hl = 0;
  if (p.mode == kTcFused) {
    if (i < s_prefix[G]) {
      kind = kTcGateUp;
    } else {
      kind = kTcDown;
      pre = s_prefix2;
      li = i - s_prefix[G];
      hl = 1;
    }
  }
  int g = gh[hl];
  while (g + 1 < G && pre[g + 1] <= li) ++g;
  gh[hl] = g;
  it.kind = kind;
  const int local = li - pre[g];
  int n, pos0;
  if (p.mode == kTcLinear) {
    it.rows = p.lin_rows;
    it.cols = p.lin_cols;
    n = p.T;
    pos0 = 0;
  } else {
    const int Fg = (g == p.E) ? p.S : p.F;
    it.rows = gate_or_up(kind) ? Fg : p.H;
    it.cols = gate_or_up(kind) ? p.H : Fg;
    const int* offs = s_prefix2 + (kMaxGroups + 2);
    pos0 = offs[g];
    n = offs[g + 1] - pos0;
  }
  const int rt = (it.rows + kTileRows - 1) / kTileRows;
  const int stages = (((it.cols + 31) >> 5) + kStageWords - 1) / kStageWords;
  it.g = g;
  if constexpr (C::kPrefill) {
    // token chunks vary fastest, so the CTAs working at the same time share
    // a row tile's plane pages in L2
    const int chunks = (n + C::kNT - 1) / C::kNT;
    const int row_tile = local / chunks;
    const int chunk = local - row_tile * chunks;
    it.split = 0;
    it.row0 = row_tile * kTileRows;
    it.tok0 = chunk * C::kNT;
    it.ntok = min(C::kNT, n - it.tok0);
    it.pos0 = pos0 + it.tok0;
    it.s_begin = 0;
    it.s_end = stages;
    it.npass = 1;
    return;
  }
  const int ns = (kind == kTcDown) ? p.n_split : 1;
  const int per_tt = rt * ns;
  const int tt = local / per_tt;
  const int r = local - tt * per_tt;
  const int row_tile = r / ns;
  it.split = r - row_tile * ns;
  it.row0 = row_tile * kTileRows;
  it.tok0 = tt * C::kNT;
  it.ntok = min(C::kNT, n - it.tok0);
  it.pos0 = pos0 + it.tok0;
  it.s_begin = static_cast<int>((static_cast<long long>(stages) * it.split) / ns);
  it.s_end = static_cast<int>((static_cast<long long>(stages) * (it.split + 1)) / ns);
  it.npass = (kind == kTcGateUp) ? 2 : 1;
}

// Block, bitwidth, LUT and plane tensor map of pass q of an item.
__device__ __forceinline__ Pass get_pass(const TcParams& p, const Item& it, int q) {
  if (p.mode == kTcLinear) return Pass{-1, p.lin_bits, p.lin_lut, p.lin_planes, p.lin_n_max};
  const int proj = (it.kind == kTcGateUp) ? q
                   : (it.kind == kTcPfGate) ? 0
                   : (it.kind == kTcPfUp) ? 1 : 2;
  const int blk = 3 * it.g + proj;
  return Pass{blk, p.pt.bits[blk], p.pt.blk[blk].lut, p.pt.blk[blk].planes, p.pt.stride[blk]};
}

// ---------------------------------------------------------------- dequant
extern __shared__ __align__(1024) uint8_t pw_tc_smem[];

// Read this thread's 4 words (one 16-byte chunk) of a plane slot: chunk
// `half` of row r (32-byte swizzle: chunk index xor bit 2 of the row).
__device__ __forceinline__ uint4 read_plane_chunk(uint32_t slot_off, int r, int half) {
  const uint32_t off = slot_off + r * 32 + ((half ^ ((r >> 2) & 1)) << 4);
  return *reinterpret_cast<const uint4*>(pw_tc_smem + off);
}

// The dequantiser warps counted by `bar` meet (a bounded wait, unlike a
// hardware barrier, so a warp that gave up cannot leave the others blocked).
__device__ __forceinline__ bool dq_sync(uint64_t* bar, uint32_t& phase, const Ctl& ctl) {
  mbar_arrive_warp(bar);
  const bool ok = mbar_wait_warp(bar, phase, ctl);
  phase ^= 1u;
  return ok;
}

struct DequantState {
  uint32_t stage_ctr;  // plane stages consumed
  uint32_t ring_end;   // plane-slot placement (place_stage)
  uint32_t a_ctr;      // stages processed by this K half
};

template <class C, int B>
__device__ bool dequant_stages(const Item& it, int grp, int quad,
                               uint64_t* sf, uint64_t* se, uint64_t* af, uint64_t* ae,
                               uint32_t tmem_base, DequantState& st, const Ctl& ctl) {
  const int lane = threadIdx.x & 31;
  const int r = 32 * quad + lane;
  const uint32_t ru = static_cast<uint32_t>(r);
  const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(32 * quad) << 16);
  auto lds16 = [](uint32_t x) -> uint32_t {
    return *reinterpret_cast<const uint16_t*>(pw_tc_smem + kOffLut + x);
  };
  auto lds32 = [](uint32_t x) -> uint32_t {
    return *reinterpret_cast<const uint32_t*>(pw_tc_smem + kOffLut + x);
  };
  for (int s = it.s_begin; s < it.s_end; ++s) {
    uint32_t P[4][B];
    const uint32_t e = st.stage_ctr % kNS;
    const uint32_t slot0 = place_stage<C>(st.ring_end, B);
    if (!mbar_wait_warp(&sf[e], (st.stage_ctr / kNS) & 1u, ctl)) return false;
#pragma unroll
    for (int k = 0; k < B; ++k) {
      const uint4 q4 = read_plane_chunk(C::kOffSlots + (slot0 + k) * kSlotBytes, r, grp);
      P[0][k] = q4.x;
      P[1][k] = q4.y;
      P[2][k] = q4.z;
      P[3][k] = q4.w;
    }
    mbar_arrive_warp(&se[e]);
    st.stage_ctr++;
    const uint32_t a_idx = 2u * st.a_ctr + static_cast<uint32_t>(grp);
    const uint32_t qa = a_idx % C::kNA;
    if (!mbar_wait_warp(&ae[qa], ((a_idx / C::kNA) & 1u) ^ 1u, ctl)) return false;
    const uint32_t tcol = tmem_lane + C::kAColBase + qa * kAColsPerSlot;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t out[32];
      if constexpr (B <= C::kPairMax) {
        dq::dq_word_pair<B, C::kSplitRows>(P[2 * h], ru, lds32, out);
        dq::dq_word_pair<B, C::kSplitRows>(P[2 * h + 1], ru, lds32, out + 16);
      } else {
        dq::dq_word_single<B, C::kSplitRows>(P[2 * h], ru, lds16, out);
        dq::dq_word_single<B, C::kSplitRows>(P[2 * h + 1], ru, lds16, out + 16);
      }
      tmem_st32(tcol + 32 * h, out);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive_warp(&af[qa]);
    st.a_ctr++;
  }
  return true;
}

// This thread's share of a pass's LUT.  Pair-table bitwidths (b <= 3, and
// b = 4 in the decode configuration) keep the whole row in registers (both
// threads of a row load it) and each thread writes the entries whose first
// code lies in its half; wider tables go to shared memory as single entries,
// each of the two threads of a row writing half of them.  For b <= 6 the
// global loads are issued one pass ahead (prefetch) and installed when the
// pass starts, so their latency hides behind the previous pass; b = 7, 8
// tables load when the pass starts.
struct LutPrefetch {
  uint4 v[4];
  int bits;
  bool live;  // this thread's row exists
};

template <class C>
__device__ __forceinline__ void lut_prefetch(const Item& it, const Pass& ps, int grp, int r,
                                             LutPrefetch& f) {
  const int o = it.row0 + r;
  f.bits = ps.bits;
  f.live = o < it.rows;
  if (!f.live || ps.bits > 6) return;
  const int b = ps.bits;
  const uint16_t* row = ps.lut + (static_cast<size_t>(o) << b);
  if (b <= 3) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(row);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < (1 << b) / 2) w[i] = src[i];
    f.v[0] = make_uint4(w[0], w[1], w[2], w[3]);
    return;
  }
  if (b <= C::kPairMax) {
    const uint4* src = reinterpret_cast<const uint4*>(row);
    f.v[0] = src[0];
    f.v[1] = src[1];
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(row + grp * (1 << (b - 1)));
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (i < (1 << (b - 4))) f.v[i] = src[i];
}

template <class C>
__device__ __forceinline__ void lut_install(const Item& it, const Pass& ps, int grp, int r,
                                            const LutPrefetch& f) {
  if (!f.live) return;
  const int b = ps.bits;
  const uint32_t ru = static_cast<uint32_t>(r);
  if (b <= C::kPairMax) {
    // pair table: entry (v1, v2) = (LUT[v1], LUT[v2]); this thread writes the
    // entries with v1 in its half of the codes
    // (entries stay in registers: the second code runs over a compile-time
    // range, the first is picked by selects and shifts)
    const bool wide = b > 3;
    const uint32_t w[8] = {f.v[0].x, f.v[0].y, f.v[0].z, f.v[0].w,
                           wide ? f.v[1].x : 0u, wide ? f.v[1].y : 0u,
                           wide ? f.v[1].z : 0u, wide ? f.v[1].w : 0u};
    auto pick = [&](int v) -> uint32_t {
      const uint4 q = (v & 8) ? f.v[1] : f.v[0];
      const uint64_t x = (v & 4) ? (q.z | (static_cast<uint64_t>(q.w) << 32))
                                 : (q.x | (static_cast<uint64_t>(q.y) << 32));
      return static_cast<uint32_t>(x >> (16 * (v & 3))) & 0xFFFFu;
    };
    const int n = 1 << b, half = n >> 1;
    // offsets are linear in v2: base + v2 * step
    const uint32_t step = dq::pair_offset(0, 1, b, ru, C::kSplitRows) -
                          dq::pair_offset(0, 0, b, ru, C::kSplitRows);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= half) break;
      const int v1 = grp * half + i;
      const uint32_t lo = pick(v1);
      uint8_t* base = pw_tc_smem + kOffLut + dq::pair_offset(v1, 0, b, ru, C::kSplitRows);
#pragma unroll
      for (int v2 = 0; v2 < 16; ++v2) {
        if (v2 >= n) break;
        const uint32_t hi = (w[v2 >> 1] >> (16 * (v2 & 1))) & 0xFFFFu;
        *reinterpret_cast<uint32_t*>(base + v2 * step) = lo | (hi << 16);
      }
    }
    return;
  }
  // single table: entry v of row r at dq::single_offset(v, r, .); this thread
  // writes entries grp * half .. grp * half + half - 1
  auto put = [&](int v, uint32_t e) {
    *reinterpret_cast<uint16_t*>(pw_tc_smem + kOffLut + dq::single_offset(v, ru, C::kSplitRows)) =
        static_cast<uint16_t>(e);
  };
  const int half = 1 << (b - 1);
  if (b <= 6) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i >= (1 << (b - 4))) break;
      const uint32_t e4[4] = {f.v[i].x, f.v[i].y, f.v[i].z, f.v[i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) put(grp * half + 8 * i + e, (e & 1) ? (e4[e >> 1] >> 16) : e4[e >> 1]);
    }
    return;
  }
  const uint16_t* row = ps.lut + (static_cast<size_t>(it.row0 + r) << b);
  const uint4* src = reinterpret_cast<const uint4*>(row + grp * half);
  for (int i = 0; i < half / 8; ++i) {
    const uint4 v = src[i];
    const uint32_t e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) put(grp * half + 8 * i + e, (e & 1) ? (e4[e >> 1] >> 16) : e4[e >> 1]);
  }
}

// ---------------------------------------------------------------- token tiles
// Linear mode: the activations are bf16 in natural column order; convert,
// permute into the A slots' K order and store (generic stores; the caller
// fences).  Stage s, token rows 0..ntok-1, this lane's share.
__device__ void fill_b_linear(const TcParams& p, const Item& it, int s, int j, uint32_t buf,
                              int lane) {
  // words 4j .. 4j + 3 of stage s (columns 256 s + 128 j ..)
  for (int idx = lane; idx < it.ntok * 4; idx += 32) {
    const int n = idx >> 2, w = idx & 3;
    const int col0 = s * 256 + 128 * j + 32 * w;
    float v[32];
    if (col0 < it.cols) {  // cols is a multiple of 128: whole 32-column groups
      const uint4* src = reinterpret_cast<const uint4*>(
          p.x + static_cast<size_t>(it.tok0 + n) * p.lin_cols + col0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 r4 = src[q];
        const uint32_t e4[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * q + 2 * e] = bf16f(static_cast<uint16_t>(e4[e] & 0xFFFFu));
          v[8 * q + 2 * e + 1] = bf16f(static_cast<uint16_t>(e4[e] >> 16));
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = 0.0f;
    }
    uint32_t q16[16];
#pragma unroll
    for (int pr = 0; pr < 16; ++pr)
      q16[pr] = pack_h2(v[dq::col_of_kpos(2 * pr)], v[dq::col_of_kpos(2 * pr + 1)]);
#pragma unroll
    for (int qc = 0; qc < 4; ++qc) {
      const uint32_t dst = buf + b_chunk_off(n, 4 * w + qc, tile_rows(it.ntok));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(q16[4 * qc]),
                   "r"(q16[4 * qc + 1]), "r"(q16[4 * qc + 2]), "r"(q16[4 * qc + 3])
                   : "memory");
    }
  }
}

// ---------------------------------------------------------------- kernel
template <class C>
__global__ void __launch_bounds__(kThreads, 1) tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int kNB = C::kNB, kNA = C::kNA, kNDBuf = C::kNDBuf;
  uint8_t* smem = pw_tc_smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* sf = bars;      // plane stage full (bulk copy landed)
  uint64_t* se = sf + kNS;  // plane stage empty (all dequantisers read it)
  uint64_t* bfull = se + kNS;
  uint64_t* bempty = bfull + C::kNBB;
  uint64_t* af = bempty + C::kNBB;
  uint64_t* ae = af + kNA;
  uint64_t* df = ae + kNA;
  uint64_t* de = df + kNDBuf;
  uint64_t* drain = de + kNDBuf;
  uint64_t* dqbar = drain + 1;  // table syncs: [4] (split layout: one per row quarter)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* s_prefix = reinterpret_cast<int*>(smem + C::kOffMisc + 16);
  int* s_prefix2 = s_prefix + (kMaxGroups + 2);  // fused launch: the down items
  int* s_offs = s_prefix2 + (kMaxGroups + 2);    // group offsets (token positions)
  uint32_t* slot_user = reinterpret_cast<uint32_t*>(smem + C::kOffSlotUser);  // producer only

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = (p.mode == kTcLinear) ? 1 : p.n_groups;
  // everything below reads what earlier kernels of the forward wrote (or
  // writes what they read); the successor may launch once every CTA of this
  // grid has released it here, i.e. once all of them are resident
  pdl_wait();
  pdl_trigger();
  // group offsets into shared memory with one parallel load (the item
  // counts below and every item decode read them)
  if (p.mode != kTcLinear)
    for (int g = threadIdx.x; g <= G; g += blockDim.x) s_offs[g] = p.offsets[g];
  __syncthreads();
  // token-tile ring: the prefill configuration has kNB slots; at decode the
  // ring's kNB * kBStageBytes hold 4, 8 or 16 slots by the largest token
  // tile of this launch (every CTA derives the same count from the offsets)
  uint32_t nb_lg = 2u;
  if (!C::kPrefill && p.mode != kTcLinear) {
    int maxn = 0;
    for (int g = 0; g < G; ++g) maxn = max(maxn, s_offs[g + 1] - s_offs[g]);
    nb_lg = maxn <= 8 ? 4u : (maxn <= 16 ? 3u : 2u);
  }
  const uint32_t nb = C::kPrefill ? static_cast<uint32_t>(kNB) : (1u << nb_lg);
  const uint32_t b_bytes = C::kPrefill ? static_cast<uint32_t>(C::kBStageBytes)
                                       : static_cast<uint32_t>(kNB * C::kBStageBytes) >> nb_lg;
  auto b_slot = [&](uint32_t c) -> uint32_t { return C::kPrefill ? c % kNB : (c & (nb - 1u)); };
  auto b_par = [&](uint32_t c) -> uint32_t { return C::kPrefill ? (c / kNB) & 1u : (c >> nb_lg) & 1u; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&sf[i], 1);
      mbar_init(&se[i], kDqThreads / 32);
    }
    for (int i = 0; i < C::kNBB; ++i) {
      mbar_init(&bfull[i], p.mode == kTcLinear ? 32 : 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < kNDBuf; ++i) {
      mbar_init(&df[i], 1);
      mbar_init(&de[i], 4);
    }
    for (int i = 0; i < kNA; ++i) {
      mbar_init(&af[i], 4);
      mbar_init(&ae[i], 1);
    }
    mbar_init(drain, 1);
    // split layout: the two warps of a row quarter (K halves) share its
    // tables; packed layout: all dequantisers
    for (int i = 0; i < 4; ++i) mbar_init(&dqbar[i], C::kSplitRows ? 2 : kDqThreads / 32);
    for (int k = 0; k < C::kNSlot; ++k) slot_user[k] = 0u;
    // the table offsets assume a 1024-byte aligned dynamic shared memory base
    *s_abort = (smem_addr(smem) & 1023u) ? 1 : 0;
    if (*s_abort && p.err) atomicExch(p.err, PW_ERR_UNSUPPORTED);
    // items per group: row tiles x token tiles x K splits (gate/up items of a
    // fused launch take no split; its down items are listed in s_prefix2)
    for (int list = 0; list < (p.mode == kTcFused ? 2 : 1); ++list) {
      const int kind = (p.mode == kTcFused) ? (list == 0 ? kTcGateUp : kTcDown) : p.mode;
      int* pre = list == 0 ? s_prefix : s_prefix2;
      int acc = 0;
      for (int g = 0; g < G; ++g) {
        pre[g] = acc;
        int rows, n;
        if (p.mode == kTcLinear) {
          rows = p.lin_rows;
          n = p.T;
        } else {
          const int Fg = (g == p.E) ? p.S : p.F;
          rows = gate_or_up(kind) ? Fg : p.H;
          n = s_offs[g + 1] - s_offs[g];
        }
        const int tt = (n + C::kNT - 1) / C::kNT;
        acc += ((rows + kTileRows - 1) / kTileRows) * tt * (kind == kTcDown ? p.n_split : 1);
      }
      pre[G] = acc;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total =
      *s_abort ? 0 : s_prefix[G] + (p.mode == kTcFused ? s_prefix2[G] : 0);
  const Ctl ctl{s_abort, p.err, p.wait_ns ? p.wait_ns : kWaitNs};

  if (warp < 8) {
    // ------------------------------------------------ dequantisers
    DequantState st{0u, 0u, 0u};
    int gh[2] = {0, 0};
    const int grp = warp >> 2, quad = warp & 3;
    const int r = 32 * quad + lane;
    // split layout: a row quarter's tables are touched only by its two warps,
    // so they alone meet around a table change
    uint64_t* tbar = C::kSplitRows ? &dqbar[quad] : dqbar;
    uint32_t sync_phase = 0;
    bool ok = true;
    // walk (item, pass) pairs; the next pass's LUT loads are issued before
    // the current pass's stages
    int i = blockIdx.x, q = 0;
    Item it;
    LutPrefetch pre;
    if (i < total) {
      decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
      lut_prefetch<C>(it, get_pass(p, it, 0), grp, r, pre);
    }
    while (i < total && ok) {
      const Pass ps = get_pass(p, it, q);
      // every reader of these rows' tables is done with the previous pass's
      // table before it changes
      if (!dq_sync(tbar, sync_phase, ctl)) break;
      lut_install<C>(it, ps, grp, r, pre);
      if (!dq_sync(tbar, sync_phase, ctl)) break;
      const Item cur = it;
      int ni = i, nq = q + 1;
      if (nq >= it.npass) {
        ni = i + gridDim.x;
        nq = 0;
        if (ni < total) decode_item<C>(p, s_prefix, s_prefix2, G, ni, it, gh);
      }
      if (ni < total) lut_prefetch<C>(it, get_pass(p, it, nq), grp, r, pre);
      switch (ps.bits) {
        case 1: ok = dequant_stages<C, 1>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 2: ok = dequant_stages<C, 2>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 3: ok = dequant_stages<C, 3>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 4: ok = dequant_stages<C, 4>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 5: ok = dequant_stages<C, 5>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 6: ok = dequant_stages<C, 6>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        case 7: ok = dequant_stages<C, 7>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
        default: ok = dequant_stages<C, 8>(cur, grp, quad, sf, se, af, ae, tmem_base, st, ctl); break;
      }
      i = ni;
      q = nq;
    }
  } else if (warp == kWarpProducer) {
    // ------------------------------------------------ producer (planes)
    if (lane == 0) {
      uint32_t t = 0, ring_end = 0;
      int gh[2] = {0, 0};
      bool ok = true;
      const uint64_t stream_pol = l2_evict_first_policy();
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        Item it;
        decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
        const int n_kt = pages::k_tiles(it.cols);
        const int rt = it.row0 / kTileRows;
        for (int q = 0; q < it.npass && ok; ++q) {
          const Pass ps = get_pass(p, it, q);
          for (int s = it.s_begin; s < it.s_end; ++s, ++t) {
            const uint32_t e = t % kNS;
            const uint32_t start = place_stage<C>(ring_end, ps.bits);
            // the barrier pair of stage t - kNS is free ...
            if (!mbar_wait(&se[e], ((t / kNS) & 1u) ^ 1u, ctl)) {
              ok = false;
              break;
            }
            // ... and so are the slots: wait for the latest earlier stage that
            // used any of them (slot_user holds stage index + 1).  Stages are
            // released in order, so users older than t - kNS are already free.
            uint32_t u1 = 0;
#pragma unroll
            for (int k = 0; k < PW_MAX_BITS; ++k)
              if (k < ps.bits) u1 = max(u1, slot_user[start + k]);
            if (u1 > 0 && u1 - 1 + kNS > t) {
              const uint32_t u = u1 - 1;
              if (!mbar_wait(&se[u % kNS], (u / kNS) & 1u, ctl)) {
                ok = false;
                break;
              }
            }
#pragma unroll
            for (int k = 0; k < PW_MAX_BITS; ++k)
              if (k < ps.bits) slot_user[start + k] = t + 1;
            const int64_t grp_idx = static_cast<int64_t>(rt) * n_kt + s;
            const uint32_t bytes = static_cast<uint32_t>(ps.bits) * kSlotBytes;
            mbar_arrive_tx(&sf[e], bytes);
            if constexpr (C::kPrefill)  // row tiles are shared by several CTAs' token chunks
              bulk_load(smem_addr(smem + C::kOffSlots + start * kSlotBytes),
                        ps.planes + grp_idx * ps.stride * (kSlotBytes / 4), bytes, &sf[e]);
            else
              bulk_load_hint(smem_addr(smem + C::kOffSlots + start * kSlotBytes),
                             ps.planes + grp_idx * ps.stride * (kSlotBytes / 4), bytes, &sf[e],
                             stream_pol);
          }
        }
      }
      if (!ok) {
        // let every issued copy land before the CTA's shared memory goes away
        const uint32_t lo = t > kNS ? t - kNS : 0u;
        for (uint32_t c = lo; c < t; ++c) mbar_drain(&sf[c % kNS], (c / kNS) & 1u);
      }
    }
  } else if (warp == kWarpLoader) {
    // ------------------------------------------------ token-tile loader
    uint32_t b_ctr = 0;
    int gh[2] = {0, 0};
    bool ok = true;
    for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
      Item it;
      decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
      const int rows_b = tile_rows(it.ntok);  // token rows loaded per stage (decode)
      const bool fused_down = p.mode == kTcFused && it.kind == kTcDown;
      if (fused_down && lane == 0)
        ok = wait_gate_up(p, it.g, 4 * (s_prefix[it.g + 1] - s_prefix[it.g]), ctl);
      ok = __all_sync(0xffffffffu, ok);
      const CUtensorMap* bmaps = fused_down ? p.h_maps : p.b_maps;
      for (int q = 0; q < it.npass && ok; ++q) {
        for (int s = it.s_begin; s < it.s_end && ok; ++s) {
          for (int j = 0; j < C::kBPerStage; ++j) {
            const uint32_t jb = b_slot(b_ctr);
            if (!mbar_wait_warp(&bempty[jb], b_par(b_ctr) ^ 1u, ctl)) {
              ok = false;
              break;
            }
            const uint32_t buf = smem_addr(smem + C::kOffB + jb * b_bytes);
            if constexpr (C::kPrefill) {
              if (lane == 0) {
                // {64 columns, 256 rows, 1 atom}: atom 4 s + j of the chunk's rows
                mbar_arrive_tx(&bfull[jb], static_cast<uint32_t>(C::kNT) * 128u);
                tma_load_3d(buf, &p.pf_map, 0, it.pos0, 4 * s + j, &bfull[jb]);
              }
            } else if (p.mode == kTcLinear) {
              fill_b_linear(p, it, s, j, buf, lane);
              fence_proxy_async();
              mbar_arrive(&bfull[jb]);
            } else if (lane == 0) {
              // {64 columns, rows_b rows, 2 atoms} starting at column 256 s + 128 j
              mbar_arrive_tx(&bfull[jb], static_cast<uint32_t>(rows_b) * 2u * 128u);
              tma_load_3d(buf, &bmaps[(rows_b >> 3) - 1], 0, it.pos0, 4 * s + 2 * j, &bfull[jb]);
            }
            b_ctr++;
          }
        }
      }
    }
    if (!ok && lane == 0 && p.mode != kTcLinear) {
      // let issued copies land before the CTA's shared memory goes away
      const uint32_t lo = b_ctr > nb ? b_ctr - nb : 0u;
      for (uint32_t c = lo; c < b_ctr; ++c) mbar_drain(&bfull[b_slot(c)], b_par(c));
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------ MMA issuer
    // The whole warp walks the items and waits (so every operand address is
    // warp-uniform); one elected lane issues the MMAs and their commits.
    const bool leader = elect_one();
    int gh[2] = {0, 0};
    uint32_t a_ctr = 0, b_ctr = 0, d_ctr = 0;
    bool ok = true;
    if constexpr (C::kPrefill) {
      const uint32_t idesc = mma_idesc(C::kNT);
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        Item it;
        decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
        const uint32_t jd = d_ctr % kNDBuf;
        if (!mbar_wait_warp(&de[jd], ((d_ctr / kNDBuf) & 1u) ^ 1u, ctl)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + jd * C::kDColsPerBuf;
        uint32_t accum = 0;
        for (int s = it.s_begin; s < it.s_end && ok; ++s) {
          for (int sub = 0; sub < 2 && ok; ++sub) {
            const uint32_t qa = a_ctr % kNA;
            if (!mbar_wait_warp(&af[qa], (a_ctr / kNA) & 1u, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t at = tmem_base + C::kAColBase + qa * kAColsPerSlot;
            // two 64-column B stages per 128-column A slot
            for (int j = 0; j < 2; ++j) {
              const uint32_t jb = b_slot(b_ctr);
              if (!mbar_wait_warp(&bfull[jb], b_par(b_ctr), ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t bdesc = smem_desc_sw128(smem_addr(smem + C::kOffB + jb * b_bytes));
              if (leader) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  tc_mma(dt, at + (4 * j + kk) * 8, bdesc + 2u * kk, idesc,
                         accum | static_cast<uint32_t>(j | kk));
                tc_commit(&bempty[jb]);
              }
              __syncwarp();
              accum = 1;
              b_ctr++;
            }
            if (!ok) break;
            if (leader) tc_commit(&ae[qa]);
            __syncwarp();
            a_ctr++;
          }
        }
        if (!ok) break;
        if (leader) tc_commit(&df[jd]);
        __syncwarp();
        d_ctr++;
      }
    } else {
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        Item it;
        decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
        const int n = it.ntok <= 16 ? 16 : 32;
        const uint32_t idesc = mma_idesc(n);
        // descriptor step of one 64-column atom of the token tile (16-byte units)
        const uint32_t atom_step = static_cast<uint32_t>(tile_rows(it.ntok)) * 8u;
        const uint32_t jd = d_ctr & 1u;
        if (!mbar_wait_warp(&de[jd], ((d_ctr >> 1) & 1u) ^ 1u, ctl)) break;
        tc_fence_after();
        for (int q = 0; q < it.npass && ok; ++q) {
          const uint32_t dt = tmem_base + jd * C::kDColsPerBuf + 32 * q;
          uint32_t accum = 0;
          for (int s = it.s_begin; s < it.s_end && ok; ++s) {
            // each 128-column half of the stage: one B stage, one A slot
            for (int sub = 0; sub < 2; ++sub) {
              const uint32_t jb = b_slot(b_ctr);
              if (!mbar_wait_warp(&bfull[jb], b_par(b_ctr), ctl)) {
                ok = false;
                break;
              }
              const uint32_t qa = a_ctr % kNA;
              if (!mbar_wait_warp(&af[qa], (a_ctr / kNA) & 1u, ctl)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t bdesc = smem_desc_sw128(smem_addr(smem + C::kOffB + jb * b_bytes));
              const uint32_t at = tmem_base + C::kAColBase + qa * kAColsPerSlot;
              if (leader) {
                // K step kk: atom kk / 4 of the B stage, 32 bytes per 16
                // columns inside the atom
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint64_t bd = bdesc + (kk >> 2) * atom_step + 2u * (kk & 3);
                  tc_mma(dt, at + kk * 8, bd, idesc, accum | kk);
                }
                tc_commit(&ae[qa]);
                tc_commit(&bempty[jb]);
              }
              __syncwarp();
              accum = 1;
              a_ctr++;
              b_ctr++;
            }
          }
        }
        if (!ok) break;
        if (leader) tc_commit(&df[jd]);
        __syncwarp();
        d_ctr++;
      }
    }
    // all issued MMAs complete before TMEM is released
    if (leader) {
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue
    if constexpr (C::kPrefill) {
      const int qd = warp & 3;
      const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(32 * qd) << 16);
      uint32_t d_ctr = 0;
      int gh[2] = {0, 0};
      for (int i = blockIdx.x; i < total; i += gridDim.x) {
        Item it;
        decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
        const int o = it.row0 + 32 * qd + lane;
        const bool live = o < it.rows;
        const bool up = p.mode == kTcPfUp;
        // gate values of the next 16-token chunk are loaded one chunk ahead
        // (the first chunk's before the accumulator is ready), so their
        // latency hides behind the MMAs and the previous chunk's work; they
        // stay raw fp16 bits until used, so no instruction waits on a load
        // before the chunk that needs it
        constexpr int kCh = 16;
        uint16_t gn[kCh];
        auto load_g = [&](int c) {
          const int nv = min(kCh, it.ntok - kCh * c);
          const int pos = it.pos0 + kCh * c;
#pragma unroll
          for (int n = 0; n < kCh; ++n)
            gn[n] = (live && n < nv) ? p.gbuf[static_cast<size_t>(pos + n) * p.gbuf_ld + o]
                                     : static_cast<uint16_t>(0);
        };
        // down: the routing weights of the next chunk's tokens, one chunk
        // ahead likewise (loaded when used, each chunk waited on L2)
        const bool down = p.mode == kTcPfDown;
        float wn[kCh];
        auto load_w = [&](int c) {
          const int nv = min(kCh, it.ntok - kCh * c);
          const int pos = it.pos0 + kCh * c;
#pragma unroll
          for (int n = 0; n < kCh; ++n) wn[n] = n < nv ? p.slot_w[pos + n] : 0.0f;
        };
        if (up) load_g(0);
        if (down) load_w(0);
        const uint32_t jd = d_ctr % kNDBuf;
        if (!mbar_wait_warp(&df[jd], (d_ctr / kNDBuf) & 1u, ctl)) break;
        tc_fence_after();
        // h = silu(g) * u goes to o's position in the down pass's K order
        const int col = (o & ~31) + dq::kpos_of_col(o & 31);
        uint16_t* hp = p.h_perm + static_cast<size_t>(col >> 6) * p.h_rows * 64 + (col & 63);
        for (int c = 0; c < C::kNT / kCh; ++c) {
          if (kCh * c >= it.ntok) break;
          uint32_t v[kCh];
          tmem_ld16(tmem_lane + jd * C::kDColsPerBuf + kCh * c, v);
          uint16_t g[kCh];
          float w[kCh];
          if (up) {
#pragma unroll
            for (int n = 0; n < kCh; ++n) g[n] = gn[n];
            if (kCh * (c + 1) < it.ntok) load_g(c + 1);
          }
          if (down) {
#pragma unroll
            for (int n = 0; n < kCh; ++n) w[n] = wn[n];
            if (kCh * (c + 1) < it.ntok) load_w(c + 1);
          }
          tmem_wait_ld();
          if (!live) continue;
          const int nv = min(kCh, it.ntok - kCh * c);
          const int pos = it.pos0 + kCh * c;
          if (p.mode == kTcPfGate) {
#pragma unroll
            for (int n = 0; n < kCh; ++n) {
              if (n >= nv) break;
              p.gbuf[static_cast<size_t>(pos + n) * p.gbuf_ld + o] =
                  __half_as_ushort(__float2half_rn(__uint_as_float(v[n])));
            }
          } else if (up) {
#pragma unroll
            for (int n = 0; n < kCh; ++n) {
              if (n >= nv) break;
              // the accumulator waits for this epilogue (one buffer), so the
              // activation takes one special-function instruction:
              // silu(g) = g sigmoid(g) = g (1 + tanh(g / 2)) / 2, with the
              // hardware tanh approximation (h is rounded to fp16 anyway)
              const float gf = __half2float(__ushort_as_half(g[n]));
              const float hg = 0.5f * gf;
              const float h = fmaf(hg, tanh_approx(hg), hg) * __uint_as_float(v[n]);
              hp[static_cast<size_t>(pos + n) * 64] = __half_as_ushort(__float2half_rn(h));
            }
          } else {
#pragma unroll
            for (int n = 0; n < kCh; ++n) {
              if (n >= nv) break;
              p.ysorted[static_cast<size_t>(pos + n) * p.H + o] = w[n] * __uint_as_float(v[n]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive_warp(&de[jd]);
        d_ctr++;
      }
    } else {
      const int qd = warp & 3;
      const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(32 * qd) << 16);
      uint32_t d_ctr = 0;
      int gh[2] = {0, 0};
      for (int i = blockIdx.x; i < total; i += gridDim.x) {
        Item it;
        decode_item<C>(p, s_prefix, s_prefix2, G, i, it, gh);
        const uint32_t jd = d_ctr & 1u;
        if (!mbar_wait_warp(&df[jd], (d_ctr >> 1) & 1u, ctl)) break;
        tc_fence_after();
        uint32_t v[32], u[32];
        tmem_ld32(tmem_lane + jd * C::kDColsPerBuf, v);
        if (it.npass == 2) tmem_ld32(tmem_lane + jd * C::kDColsPerBuf + 32, u);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive_warp(&de[jd]);
        d_ctr++;
        const int o = it.row0 + 32 * qd + lane;
        if (o < it.rows) {
          if (it.kind == kTcGateUp) {
            // h = silu(g) * u, fp16, at o's position in the down pass's K order
            // atom-major [ld/64][rows][64]: column col of row pos at
            // ((col / 64) * rows + pos) * 64 + col % 64
            const int col = (o & ~31) + dq::kpos_of_col(o & 31);
            uint16_t* hp = p.h_perm + static_cast<size_t>(col >> 6) * p.h_rows * 64 + (col & 63);
#pragma unroll
            for (int n = 0; n < C::kNT; ++n) {
              if (n >= it.ntok) break;
              const float g = __uint_as_float(v[n]);
              const float h = g / (1.0f + expf(-g)) * __uint_as_float(u[n]);
              hp[static_cast<size_t>(it.pos0 + n) * 64] = __half_as_ushort(__float2half_rn(h));
            }
          } else if (it.kind == kTcDown) {
#pragma unroll
            for (int n = 0; n < C::kNT; ++n) {
              if (n >= it.ntok) break;
              p.ysorted[it.split * p.split_stride + static_cast<size_t>(it.pos0 + n) * p.H + o] =
                  p.slot_w[it.pos0 + n] * __uint_as_float(v[n]);
            }
          } else {
#pragma unroll
            for (int n = 0; n < C::kNT; ++n) {
              if (n >= it.ntok) break;
              p.y[static_cast<size_t>(it.tok0 + n) * it.rows + o] = __uint_as_float(v[n]);
            }
          }
        }
        if (p.mode == kTcFused && it.kind == kTcGateUp) {
          // this warp's h rows of the item are written: count them for the
          // group's down items (the fence makes every lane's stores visible
          // at GPU scope before the count)
          __syncwarp();
          if (lane == 0) {
            __threadfence();
            atomicAdd(p.gu_done + it.g, 1);
          }
        }
      }
  
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}

}  // namespace

// The shared-memory attribute is per device context: set it once per device
// (under a lock, since handles on different devices may launch from
// different threads).
template <class C>
cudaError_t launch_cfg(const TcParams& p, int n_sm, cudaStream_t s) {
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
      e = cudaFuncSetAttribute(tc_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(C::kSmemTotal));
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  // a fused launch's down items wait on other CTAs' gate/up items: launched
  // cooperatively, so either every CTA is resident or the launch fails
  const bool coop = p.mode == kTcFused && p.cooperative;
  return launch_pdl_ex(coop, tc_kernel<C>, dim3(n_sm), dim3(kThreads), C::kSmemTotal, s, p);
}

cudaError_t launch_tc(const TcParams& p, int n_sm, cudaStream_t s) {
  if (p.mode == kTcPfGate || p.mode == kTcPfUp || p.mode == kTcPfDown)
    return launch_cfg<Pre>(p, n_sm, s);
  return launch_cfg<Dec>(p, n_sm, s);
}

}  // namespace pw
