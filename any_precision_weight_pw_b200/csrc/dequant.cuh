// dequant.cuh -- per-thread dequantisation of one 32-column word of one row
// of an Any-Precision bit-plane block into 16 fp16 pairs.
//
// PagedWeight (legiblepapers summary, FAQ Q5): the fused kernel reads the
// bit-planes and LUTs directly; the b-bit view of a block is its top b
// planes, and W[o][i] = LUT_b[o][code_b(o, i)].
//
// Output order (the K order of the tensor-core A operand): pair register
// pr = 4m + j (m, j in 0..3) holds the weights of columns (8j + m) in its low
// half and (8j + m + 4) in its high half.  The token tile is permuted the same
// way, so the contraction is unchanged.
//
// Lookups, chosen per bitwidth:
//   b <= 3   the row's 8-entry LUT sits in four registers as separate low-
//            and high-byte tables; one byte permute (PRMT) looks up four
//            weights' low bytes, one their high bytes, two more interleave
//            them into fp16 pairs.  Selectors are 3-bit codes in nibbles.
//   b == 4   4-bit codes in nibbles address a shared-memory table.
//   b >= 5   an 8x8 bit-matrix transpose of the planes (zero planes for
//            k >= b) gives one code per byte, which addresses the table.
// The shared-memory table holds entry v of local row r in the low half of
// word v * 128 + r, so the 32 threads of a warp (32 consecutive rows) read 32
// different banks; the byte offset of an entry is (v << 9) | 4r, formed with
// one shift and one LOP3 per weight.  Right shifts are written as high
// multiplies so they issue on the FMA pipe, not the integer ALU pipe.
//
// Everything here is __host__ __device__ so the bit manipulation can be
// checked on the CPU (tests/dequant_selftest.cpp) against a plain unpack.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define PW_HD __host__ __device__ __forceinline__
#else
#define PW_HD inline
#endif

namespace pw {
namespace dq {

// ---- the K order of a 32-column word ---------------------------------------
// Column (0..31) whose weight sits at position q of the A operand's K order
// (pair register q / 2, half q % 2), and the inverse.
PW_HD constexpr int col_of_kpos(int q) { return 8 * ((q >> 1) & 3) + (q >> 3) + 4 * (q & 1); }
PW_HD constexpr int kpos_of_col(int c) { return 8 * (c & 3) + 2 * (c >> 3) + ((c >> 2) & 1); }

// ---- primitives ----------------------------------------------------------
// Byte permute with 3-bit selectors (selector nibble bit 3 must be zero).
PW_HD uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
#ifdef __CUDA_ARCH__
  return __byte_perm(a, b, sel);
#else
  const uint64_t src = (static_cast<uint64_t>(b) << 32) | a;
  uint32_t r = 0;
  for (int i = 0; i < 4; ++i) {
    const uint32_t idx = (sel >> (4 * i)) & 7u;
    r |= static_cast<uint32_t>((src >> (8 * idx)) & 0xFFu) << (8 * i);
  }
  return r;
#endif
}
// x >> S (0 <= S < 32), as a high multiply (FMA pipe) on the device.
template <int S>
PW_HD uint32_t shr(uint32_t x) {
  if (S <= 0) return x;
#ifdef __CUDA_ARCH__
  return __umulhi(x, 1u << ((32 - S) & 31));
#else
  return x >> (S & 31);
#endif
}
// x << S for S >= 0, x >> -S for S < 0.
template <int S>
PW_HD uint32_t shl(uint32_t x) {
  if (S >= 0) return x << (S >= 0 ? S : 0);
  return shr<(S < 0 ? -S : 0)>(x);
}
// (hi << 16) | lo for 16-bit lo and hi, as a multiply-add (FMA pipe).
PW_HD uint32_t pack16(uint32_t lo, uint32_t hi) { return hi * 65536u + lo; }

// ---- nibble codes ----------------------------------------------------------
// Nibble n of the result = the NB-bit number whose bits come from planes
// P[K0] (most significant) .. P[K0+NB-1] at column 4n + M.
template <int M, int K0, int NB, int B>
PW_HD uint32_t nibble_codes(const uint32_t (&P)[B]) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int j = NB - 1 - i;  // nibble bit this plane supplies
    // bit 4n + j  <-  plane bit 4n + M
    uint32_t t;
    switch (j - M) {
      case -3: t = shl<-3>(P[K0 + i]); break;
      case -2: t = shl<-2>(P[K0 + i]); break;
      case -1: t = shl<-1>(P[K0 + i]); break;
      case 0: t = P[K0 + i]; break;
      case 1: t = shl<1>(P[K0 + i]); break;
      case 2: t = shl<2>(P[K0 + i]); break;
      default: t = shl<3>(P[K0 + i]); break;
    }
    s |= t & (0x11111111u << j);
  }
  return s;
}

// ---- b <= 3: register tables -----------------------------------------------
struct RegLut {
  uint32_t lo0, lo1, hi0, hi1;  // low/high bytes of entries 0-3 and 4-7
};

// w[i] = fp16 entries 2i (low half) and 2i+1 (high half); entries >= 2^b are
// never selected.
template <int B>
PW_HD RegLut make_reg_lut(const uint32_t* w) {
  uint32_t e[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < (1 << B) / 2; ++i) e[i] = w[i];
  RegLut L;
  L.lo0 = prmt(e[0], e[1], 0x6420);
  L.hi0 = prmt(e[0], e[1], 0x7531);
  L.lo1 = prmt(e[2], e[3], 0x6420);
  L.hi1 = prmt(e[2], e[3], 0x7531);
  return L;
}

template <int M, int B>
PW_HD void reg_quarter(const uint32_t (&P)[B], const RegLut& L, uint32_t* out) {
  const uint32_t s = nibble_codes<M, 0, B, B>(P);  // codes of columns 4n + M
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sel = h ? shr<16>(s) : s;
    const uint32_t lo = prmt(L.lo0, L.lo1, sel);
    const uint32_t hi = prmt(L.hi0, L.hi1, sel);
    out[4 * M + 2 * h + 0] = prmt(lo, hi, 0x5140);  // columns (8(2h) + M, +4)
    out[4 * M + 2 * h + 1] = prmt(lo, hi, 0x7362);  // columns (8(2h+1) + M, +4)
  }
}

template <int B>
PW_HD void dq_word_reg(const uint32_t (&P)[B], const RegLut& L, uint32_t* out) {
  static_assert(B >= 1 && B <= 3, "register tables hold at most 8 entries");
  reg_quarter<0, B>(P, L, out);
  reg_quarter<1, B>(P, L, out);
  reg_quarter<2, B>(P, L, out);
  reg_quarter<3, B>(P, L, out);
}

// ---- shared-memory tables ----------------------------------------------------
// Lds(x) returns the 16-bit entry at byte offset x of the table region.
// r4 = 4 * (local row), in bits 2..8.

// b == 4: entry offset of nibble n of s = ((s >> 4n) & 15) << 9 | r4.
template <int N>
PW_HD uint32_t nib_addr(uint32_t s, uint32_t r4) {
  return (shl<9 - 4 * N>(s) & (0xFu << 9)) | r4;
}

template <int M, class Lds>
PW_HD void smem4_quarter(const uint32_t (&P)[4], uint32_t r4, Lds lds, uint32_t* out) {
  const uint32_t s = nibble_codes<M, 0, 4, 4>(P);  // 4-bit codes of columns 4n + M
  out[4 * M + 0] = pack16(lds(nib_addr<0>(s, r4)), lds(nib_addr<1>(s, r4)));
  out[4 * M + 1] = pack16(lds(nib_addr<2>(s, r4)), lds(nib_addr<3>(s, r4)));
  out[4 * M + 2] = pack16(lds(nib_addr<4>(s, r4)), lds(nib_addr<5>(s, r4)));
  out[4 * M + 3] = pack16(lds(nib_addr<6>(s, r4)), lds(nib_addr<7>(s, r4)));
}

// b >= 5: X[q] byte n = 8-bit code (zero-padded below for b < 8) of column
// 8n + q, after transposing the 8x8 bit blocks of the planes.
template <int B>
PW_HD void transpose_codes(const uint32_t (&P)[B], uint32_t (&X)[8]) {
  // X[p] = plane 7 - p (code bit p of an 8-bit code), zero for planes >= B
#pragma unroll
  for (int p = 0; p < 8; ++p) X[p] = (7 - p < B) ? P[(7 - p < B) ? 7 - p : 0] : 0u;
  // 4x4 blocks: rows i, i+4
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t t = (shr<4>(X[i]) ^ X[i + 4]) & 0x0F0F0F0Fu;
    X[i + 4] ^= t;
    X[i] ^= t << 4;
  }
  // 2x2 blocks: rows i, i+2
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i & 2) continue;
    const uint32_t t = (shr<2>(X[i]) ^ X[i + 2]) & 0x33333333u;
    X[i + 2] ^= t;
    X[i] ^= t << 2;
  }
  // single bits: rows i, i+1
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const uint32_t t = (shr<1>(X[i]) ^ X[i + 1]) & 0x55555555u;
    X[i + 1] ^= t;
    X[i] ^= t << 1;
  }
}

// Offset of the entry for byte n of x (an 8-bit code v << (8 - B)).
template <int N, int B>
PW_HD uint32_t byte_addr(uint32_t x, uint32_t r4) {
  return (shl<B + 1 - 8 * N>(x) & (((1u << B) - 1u) << 9)) | r4;
}

template <int B, class Lds>
PW_HD void dq_word_smem(const uint32_t (&P)[B], uint32_t r4, Lds lds, uint32_t* out) {
  if constexpr (B == 4) {
    smem4_quarter<0>(P, r4, lds, out);
    smem4_quarter<1>(P, r4, lds, out);
    smem4_quarter<2>(P, r4, lds, out);
    smem4_quarter<3>(P, r4, lds, out);
  } else {
    static_assert(B >= 5 && B <= 8, "transposed codes serve b = 5..8");
    uint32_t X[8];
    transpose_codes<B>(P, X);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      // columns 8j + m (X[m] byte j) and 8j + m + 4 (X[m+4] byte j)
      out[4 * m + 0] = pack16(lds(byte_addr<0, B>(X[m], r4)), lds(byte_addr<0, B>(X[m + 4], r4)));
      out[4 * m + 1] = pack16(lds(byte_addr<1, B>(X[m], r4)), lds(byte_addr<1, B>(X[m + 4], r4)));
      out[4 * m + 2] = pack16(lds(byte_addr<2, B>(X[m], r4)), lds(byte_addr<2, B>(X[m + 4], r4)));
      out[4 * m + 3] = pack16(lds(byte_addr<3, B>(X[m], r4)), lds(byte_addr<3, B>(X[m + 4], r4)));
    }
  }
}

}  // namespace dq
}  // namespace pw
