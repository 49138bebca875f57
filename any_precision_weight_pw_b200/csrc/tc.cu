// tc.cu -- tensor-core dequant-GEMM over Any-Precision bit-plane pages
// (sm_100a: TMA + tcgen05 + TMEM).
//
// PagedWeight (legiblepapers summary, FAQ Q5; arxivlens abstract): the fused
// mixed-precision MoE kernel reads the AP bit-planes and per-row LUTs of the
// resident pages directly, at a separate bitwidth for every linear-block.
//
// One persistent CTA per SM walks a list of work items.  An item is one
// linear-block x 128 output rows x up to 32 tokens (x one K range when the
// down pass is split).  Inside the CTA:
//   warp 4      TMA producer: streams only the b active bit-planes of the
//               block, 128 rows x 256 columns (8 words) per plane per stage,
//               into a ring of 4 KB slots (32-byte swizzle, so that the
//               thread-per-row reads below are bank-conflict free).
//   warps 0-3   dequantisers, thread r <-> output row r <-> TMEM lane r: each
//               thread unpacks its row's codes from the b plane words, looks
//               them up in its row's LUT (shared memory, one bank per thread)
//               and writes fp16 weights into a TMEM ring slot (the MMA's A
//               operand); they also stage the token tile (the B operand) in
//               shared memory: bf16 activations -> fp16 (gate/up pass) or
//               silu(g)*u -> fp16 (down pass), in the K order the A slots use.
//   warp 5      MMA issuer: tcgen05.mma kind::f16, M=128, N=16/32, K=16,
//               fp32 accumulators in TMEM (two buffers, alternating items).
//   warps 6-9   epilogue: tcgen05.ld the accumulators, write fp32 outputs
//               (gate/up values, routing-weighted down partials, or the plain
//               linear result).
// Every wait is an mbarrier try_wait bounded by a global-timer deadline; a
// timeout raises the CTA's abort flag and the device error word, and every
// role drains what it has in flight before the CTA frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pw_internal.h"
#include "tc.h"

namespace pw {
namespace {

constexpr int kTileRows = 128;
constexpr int kStageWords = 8;                 // 256 columns per stage
constexpr int kSlotBytes = kTileRows * kStageWords * 4;  // 4 KB
constexpr int kNSlot = 16;
constexpr int kNT = kTcTokens;                 // token tile (MMA N <= 32)
constexpr int kBStageBytes = kNT * 256 * 2;    // 32 rows x 256 K fp16 = 16 KB
constexpr int kNA = 6;                         // TMEM A ring slots (128 K each)
constexpr int kAColsPerSlot = 64;
constexpr int kAColBase = 128;
constexpr int kDColsPerBuf = 64;
constexpr int kTmemCols = 512;
constexpr int kLutWords = kTileRows * 128;     // 128 rows x 256 fp16
constexpr int kThreads = 320;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait

constexpr size_t kSmemSlots = size_t(kNSlot) * kSlotBytes;
constexpr size_t kSmemB = 2 * size_t(kBStageBytes);
constexpr size_t kSmemLut = size_t(kLutWords) * 4;
constexpr size_t kNumBars = 2 * kNSlot + 4 + 2 * kNA + 4 + 1;
constexpr size_t kSmemBars = kNumBars * 8;
constexpr size_t kSmemMisc = 16 + 4 * (kMaxGroups + 2) + 16;
constexpr size_t kSmemTotal = 1024 + kSmemSlots + kSmemB + kSmemLut + kSmemBars + kSmemMisc;

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
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)),
               "r"(bytes)
               : "memory");
}
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
};

// Wait for the phase with the given parity; false on timeout or abort.
__device__ __noinline__ bool mbar_wait(uint64_t* b, uint32_t parity, const Ctl& c) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try(b, parity)) return true;
    if (*c.abort) return false;
    if (global_ns() - t0 > kWaitNs) {
      *c.abort = 1;
      if (c.err) atomicExch(c.err, PW_ERR_TIMEOUT);
      return false;
    }
  }
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

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
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

// ---------------------------------------------------------------- work items
struct Item {
  int g, proj, row0, tok0, ntok, pos0, split;
  int blk, rows, cols, words, bits, s_begin, s_end;
  const uint16_t* lut;
  const CUtensorMap* tmap;
};

__device__ __forceinline__ void decode_item(const TcParams& p, const int* s_prefix, int G,
                                            int i, Item& it) {
  int g = 0;
  while (g + 1 < G && s_prefix[g + 1] <= i) ++g;
  int local = i - s_prefix[g];
  int rows, cols, nproj, n, pos0;
  if (p.mode == kTcLinear) {
    rows = p.lin_rows;
    cols = p.lin_cols;
    nproj = 1;
    n = p.T;
    pos0 = 0;
  } else {
    const int Fg = (g == p.E) ? p.S : p.F;
    nproj = (p.mode == kTcGateUp) ? 2 : 1;
    rows = (p.mode == kTcGateUp) ? Fg : p.H;
    cols = (p.mode == kTcGateUp) ? p.H : Fg;
    pos0 = p.offsets[g];
    n = p.offsets[g + 1] - pos0;
  }
  const int rt = (rows + kTileRows - 1) / kTileRows;
  const int ns = p.n_split;
  const int per_tt = nproj * rt * ns;
  const int tt = local / per_tt;
  int r = local - tt * per_tt;
  const int proj = r / (rt * ns);
  r -= proj * rt * ns;
  const int row_tile = r / ns;
  const int split = r - row_tile * ns;
  it.g = g;
  it.proj = (p.mode == kTcGateUp) ? proj : 2;
  it.row0 = row_tile * kTileRows;
  it.tok0 = tt * kNT;
  it.ntok = min(kNT, n - it.tok0);
  it.pos0 = pos0 + it.tok0;
  it.split = split;
  it.rows = rows;
  it.cols = cols;
  it.words = (cols + 31) >> 5;
  const int stages = (it.words + kStageWords - 1) / kStageWords;
  it.s_begin = static_cast<int>((static_cast<long long>(stages) * split) / ns);
  it.s_end = static_cast<int>((static_cast<long long>(stages) * (split + 1)) / ns);
  if (p.mode == kTcLinear) {
    it.blk = -1;
    it.bits = p.lin_bits;
    it.lut = p.lin_lut;
    it.tmap = &p.lin_map;
  } else {
    it.blk = 3 * g + it.proj;
    it.bits = p.pt.bits[it.blk];
    it.lut = p.pt.blk[it.blk].lut;
    it.tmap = p.tmaps + it.blk;
  }
}

// Column (0..31 of a word) held at position q of the K order of a TMEM A
// slot: pair register pr = 4m + j holds columns (8j + m, 8j + m + 4).
__host__ __device__ constexpr int col_of_kpos(int q) {
  return 8 * ((q >> 1) & 3) + (q >> 3) + 4 * (q & 1);
}

// ---------------------------------------------------------------- dequant
// Thread-private LUT: row r's entries (2j, 2j+1) packed in word j*128 + r,
// so the 32 threads of a warp always hit 32 different banks.
template <int B>
__device__ __forceinline__ uint32_t lut_get(const uint32_t* lrow, uint32_t v) {
  const uint32_t w = lrow[(v >> 1) * kTileRows];
  return (v & 1u) ? (w >> 16) : (w & 0xFFFFu);
}

// 32 columns of one row: P[k] is plane k's word (k = 0 is the MSB plane).
// out[pr] = fp16 pair (col 8j+m, col 8j+m+4), pr = 4m + j.
template <int B>
__device__ __forceinline__ void dequant_word(const uint32_t (&P)[B], const uint32_t* lrow,
                                             uint32_t* out) {
  uint32_t S[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    uint32_t s = 0;
#pragma unroll
    for (int k = 0; k < B; ++k) s |= ((P[k] >> m) & 0x01010101u) << (B - 1 - k);
    S[m] = s;  // byte n = b-bit code of column 8n + m
  }
#pragma unroll
  for (int pr = 0; pr < 16; ++pr) {
    const int m = pr >> 2, j = pr & 3;
    const uint32_t v0 = (S[m] >> (8 * j)) & 0xFFu;
    const uint32_t v1 = (S[m + 4] >> (8 * j)) & 0xFFu;
    out[pr] = lut_get<B>(lrow, v0) | (lut_get<B>(lrow, v1) << 16);
  }
}

// Read this thread's 4 words (one 16-byte chunk) of plane slot `slot` for
// sub-chunk `sub` (32-byte swizzle: chunk index xor bit 2 of the row).
__device__ __forceinline__ uint4 read_plane_chunk(const uint8_t* slot, int r, int sub) {
  const int off = r * 32 + ((sub ^ ((r >> 2) & 1)) << 4);
  return *reinterpret_cast<const uint4*>(slot + off);
}

struct DequantState {
  uint32_t slot_ctr, a_ctr, b_ctr;
};

// Stage the token tile of stage s (256 K) into B buffer `buf`, K-major in
// the 128-byte swizzle layout, columns permuted into the A slot order.
__device__ void fill_b(const TcParams& p, const Item& it, int s, uint8_t* buf, int tid) {
  const int total = it.ntok * kStageWords;
  for (int idx = tid; idx < total; idx += 128) {
    const int n = idx >> 3, w = idx & 7;
    const int col0 = s * 256 + 32 * w;
    float v[32];
    if (p.mode == kTcDown) {
      const int Fg = it.cols;
      const float* gr = p.gu + static_cast<size_t>(it.pos0 + n) * p.gu_stride;
      const float* ur = gr + Fg;
      if (col0 + 32 <= it.cols) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 g4 = *reinterpret_cast<const float4*>(gr + col0 + 4 * q);
          const float4 u4 = *reinterpret_cast<const float4*>(ur + col0 + 4 * q);
          v[4 * q + 0] = g4.x / (1.0f + expf(-g4.x)) * u4.x;
          v[4 * q + 1] = g4.y / (1.0f + expf(-g4.y)) * u4.y;
          v[4 * q + 2] = g4.z / (1.0f + expf(-g4.z)) * u4.z;
          v[4 * q + 3] = g4.w / (1.0f + expf(-g4.w)) * u4.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = col0 + c;
          if (col < it.cols) {
            const float gv = gr[col];
            v[c] = gv / (1.0f + expf(-gv)) * ur[col];
          } else {
            v[c] = 0.0f;
          }
        }
      }
    } else {
      const int t = (p.mode == kTcGateUp) ? p.slot_token[it.pos0 + n] : it.tok0 + n;
      const int ld = (p.mode == kTcGateUp) ? p.H : p.lin_cols;
      const uint16_t* src = p.x + static_cast<size_t>(t) * ld;
      if (col0 + 32 <= it.cols && (ld & 7) == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + col0 + 8 * q);
          const uint32_t r4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[8 * q + 2 * e] = bf16f(static_cast<uint16_t>(r4[e] & 0xFFFFu));
            v[8 * q + 2 * e + 1] = bf16f(static_cast<uint16_t>(r4[e] >> 16));
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = col0 + c;
          v[c] = (col < it.cols) ? bf16f(src[col]) : 0.0f;
        }
      }
    }
    uint32_t q16[16];
#pragma unroll
    for (int pr = 0; pr < 16; ++pr) q16[pr] = pack_h2(v[col_of_kpos(2 * pr)], v[col_of_kpos(2 * pr + 1)]);
    const int atom = w >> 1;
    uint8_t* rowp = buf + atom * (kNT * 128) + (n >> 3) * 1024 + (n & 7) * 128;
#pragma unroll
    for (int qc = 0; qc < 4; ++qc) {
      const int c16 = (w & 1) * 4 + qc;
      *reinterpret_cast<uint4*>(rowp + ((c16 ^ (n & 7)) << 4)) =
          make_uint4(q16[4 * qc], q16[4 * qc + 1], q16[4 * qc + 2], q16[4 * qc + 3]);
    }
  }
}

template <int B>
__device__ bool dequant_stages(const TcParams& p, const Item& it, uint8_t* slots, uint8_t* bbuf,
                               const uint32_t* lrow, uint64_t* pf, uint64_t* pe, uint64_t* bfull,
                               uint64_t* bempty, uint64_t* af, uint64_t* ae, uint32_t tmem_a_lane,
                               DequantState& st, const Ctl& ctl) {
  const int r = threadIdx.x;
  for (int s = it.s_begin; s < it.s_end; ++s) {
    // token tile for this stage
    const uint32_t jb = st.b_ctr & 1u;
    if (!mbar_wait_warp(&bempty[jb], ((st.b_ctr >> 1) & 1u) ^ 1u, ctl)) return false;
    fill_b(p, it, s, bbuf + jb * kBStageBytes, r);
    fence_proxy_async();
    mbar_arrive(&bfull[jb]);
    st.b_ctr++;
    // planes of this stage
#pragma unroll
    for (int k = 0; k < B; ++k) {
      const uint32_t c = st.slot_ctr + k;
      if (!mbar_wait_warp(&pf[c % kNSlot], (c / kNSlot) & 1u, ctl)) return false;
    }
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
      uint32_t P[4][B];
#pragma unroll
      for (int k = 0; k < B; ++k) {
        const uint4 q = read_plane_chunk(slots + ((st.slot_ctr + k) % kNSlot) * kSlotBytes, r, sub);
        P[0][k] = q.x;
        P[1][k] = q.y;
        P[2][k] = q.z;
        P[3][k] = q.w;
      }
      if (sub == 1) {
#pragma unroll
        for (int k = 0; k < B; ++k) mbar_arrive(&pe[(st.slot_ctr + k) % kNSlot]);
      }
      const uint32_t qa = st.a_ctr % kNA;
      if (!mbar_wait_warp(&ae[qa], ((st.a_ctr / kNA) & 1u) ^ 1u, ctl)) return false;
      const uint32_t tcol = tmem_a_lane + kAColBase + qa * kAColsPerSlot;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t out[32];
        dequant_word<B>(P[2 * half], lrow, out);
        dequant_word<B>(P[2 * half + 1], lrow, out + 16);
        tmem_st32(tcol + 32 * half, out);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&af[qa]);
      st.a_ctr++;
    }
    st.slot_ctr += B;
  }
  return true;
}

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1) tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* slots = base;
  uint8_t* bbuf = slots + kSmemSlots;
  uint32_t* lut = reinterpret_cast<uint32_t*>(bbuf + kSmemB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(lut) + kSmemLut);
  uint64_t* pf = bars;
  uint64_t* pe = pf + kNSlot;
  uint64_t* bfull = pe + kNSlot;
  uint64_t* bempty = bfull + 2;
  uint64_t* af = bempty + 2;
  uint64_t* ae = af + kNA;
  uint64_t* df = ae + kNA;
  uint64_t* de = df + 2;
  uint64_t* drain = de + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_holder + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = (p.mode == kTcLinear) ? 1 : p.n_groups;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNSlot; ++i) {
      mbar_init(&pf[i], 1);
      mbar_init(&pe[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bfull[i], 128);
      mbar_init(&bempty[i], 1);
      mbar_init(&df[i], 1);
      mbar_init(&de[i], 128);
    }
    for (int i = 0; i < kNA; ++i) {
      mbar_init(&af[i], 128);
      mbar_init(&ae[i], 1);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    // items per group: projections x row tiles x token tiles x K splits
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      s_prefix[g] = acc;
      int rows, n, nproj;
      if (p.mode == kTcLinear) {
        rows = p.lin_rows;
        n = p.T;
        nproj = 1;
      } else {
        const int Fg = (g == p.E) ? p.S : p.F;
        rows = (p.mode == kTcGateUp) ? Fg : p.H;
        nproj = (p.mode == kTcGateUp) ? 2 : 1;
        n = p.offsets[g + 1] - p.offsets[g];
      }
      const int tt = (n + kNT - 1) / kNT;
      acc += nproj * ((rows + kTileRows - 1) / kTileRows) * tt * p.n_split;
    }
    s_prefix[G] = acc;
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
  const int total = s_prefix[G];
  const Ctl ctl{s_abort, p.err};

  if (warp < 4) {
    // ------------------------------------------------ dequantisers
    DequantState st{0u, 0u, 0u};
    const int r = threadIdx.x;
    const uint32_t* lrow = lut + r;
    const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);
    for (int i = blockIdx.x; i < total && !__any_sync(0xffffffffu, *s_abort != 0);
         i += gridDim.x) {
      Item it;
      decode_item(p, s_prefix, G, i, it);
      // this thread's LUT row
      const int o = it.row0 + r;
      if (o < it.rows) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(it.lut) +
                              (static_cast<size_t>(o) << (it.bits - 1));
        const int nw = 1 << (it.bits - 1);
        for (int j = 0; j < nw; ++j) lut[j * kTileRows + r] = src[j];
      }
      bool ok = true;
      switch (it.bits) {
        case 1: ok = dequant_stages<1>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 2: ok = dequant_stages<2>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 3: ok = dequant_stages<3>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 4: ok = dequant_stages<4>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 5: ok = dequant_stages<5>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 6: ok = dequant_stages<6>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        case 7: ok = dequant_stages<7>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
        default: ok = dequant_stages<8>(p, it, slots, bbuf, lrow, pf, pe, bfull, bempty, af, ae, tmem_lane, st, ctl); break;
      }
      if (!ok) break;
    }
  } else if (warp == 4) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t slot_ctr = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        Item it;
        decode_item(p, s_prefix, G, i, it);
        for (int s = it.s_begin; s < it.s_end && ok; ++s) {
          for (int k = 0; k < it.bits; ++k) {
            const uint32_t sl = slot_ctr % kNSlot;
            if (!mbar_wait(&pe[sl], ((slot_ctr / kNSlot) & 1u) ^ 1u, ctl)) {
              ok = false;
              break;
            }
            mbar_arrive_tx(&pf[sl], kSlotBytes);
            tma_load_3d(slots + sl * kSlotBytes, it.tmap, s * kStageWords, it.row0, k, &pf[sl]);
            slot_ctr++;
          }
        }
      }
      if (!ok) {
        // let every issued copy land before the CTA's shared memory goes away
        const uint32_t lo = slot_ctr > kNSlot ? slot_ctr - kNSlot : 0u;
        for (uint32_t c = lo; c < slot_ctr; ++c) mbar_drain(&pf[c % kNSlot], (c / kNSlot) & 1u);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t a_ctr = 0, b_ctr = 0, d_ctr = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        Item it;
        decode_item(p, s_prefix, G, i, it);
        const int n = it.ntok <= 16 ? 16 : 32;
        const uint32_t idesc = mma_idesc(n);
        const uint32_t jd = d_ctr & 1u;
        if (!mbar_wait(&de[jd], ((d_ctr >> 1) & 1u) ^ 1u, ctl)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + jd * kDColsPerBuf;
        uint32_t accum = 0;
        for (int s = it.s_begin; s < it.s_end && ok; ++s) {
          const uint32_t jb = b_ctr & 1u;
          if (!mbar_wait(&bfull[jb], (b_ctr >> 1) & 1u, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bbase = smem_addr(bbuf + jb * kBStageBytes);
          for (int sub = 0; sub < 2; ++sub) {
            const uint32_t qa = a_ctr % kNA;
            if (!mbar_wait(&af[qa], (a_ctr / kNA) & 1u, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t at = tmem_base + kAColBase + qa * kAColsPerSlot;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const int kp = sub * 128 + kk * 16;
              const uint32_t baddr = bbase + (kp >> 6) * (kNT * 128) + (kp & 63) * 2;
              tc_mma(dt, at + kk * 8, smem_desc_sw128(baddr), idesc, accum);
              accum = 1;
            }
            tc_commit(&ae[qa]);
            a_ctr++;
          }
          if (!ok) break;
          tc_commit(&bempty[jb]);
          b_ctr++;
        }
        if (!ok) break;
        tc_commit(&df[jd]);
        d_ctr++;
      }
      // all issued MMAs complete before TMEM is released
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------ epilogue
    const int qd = warp & 3;
    const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(32 * qd) << 16);
    uint32_t d_ctr = 0;
    for (int i = blockIdx.x; i < total; i += gridDim.x) {
      Item it;
      decode_item(p, s_prefix, G, i, it);
      const uint32_t jd = d_ctr & 1u;
      if (!mbar_wait_warp(&df[jd], (d_ctr >> 1) & 1u, ctl)) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem_lane + jd * kDColsPerBuf, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&de[jd]);
      d_ctr++;
      const int o = it.row0 + 32 * qd + lane;
      if (o < it.rows) {
        for (int n = 0; n < it.ntok; ++n) {
          const float acc = __uint_as_float(v[n]);
          if (p.mode == kTcGateUp) {
            p.gu[static_cast<size_t>(it.pos0 + n) * p.gu_stride + it.proj * it.rows + o] = acc;
          } else if (p.mode == kTcDown) {
            p.ysorted[it.split * p.split_stride + static_cast<size_t>(it.pos0 + n) * p.H + o] =
                p.slot_w[it.pos0 + n] * acc;
          } else {
            p.y[static_cast<size_t>(it.tok0 + n) * it.rows + o] = acc;
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

size_t tc_smem_bytes() { return kSmemTotal; }

cudaError_t launch_tc(const TcParams& p, int n_sm, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemTotal));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  tc_kernel<<<n_sm, kThreads, kSmemTotal, s>>>(p);
  return cudaGetLastError();
}

}  // namespace pw
