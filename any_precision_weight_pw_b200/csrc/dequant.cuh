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
// Codes come from an 8x8 bit-matrix transpose of plane words: input row p
// becomes bit p of every byte, so byte n of output row q collects column
// 8n + q.  The byte then IS an address byte: one byte permute (PRMT) puts it
// next to the thread's row bytes, and one shared-memory load fetches the
// entry.  Two kinds of table serve 128 local rows (threads):
//   pair     the 32-bit entry for codes v1 (column c) and v2 (column c + 4) is
//            the fp16 pair (LUT[v1], LUT[v2]) -- one load gives one output
//            register.
//   single   the fp16 entry for code v; two loads and one multiply-add give
//            one output register.
// and two layouts of them (h = r >= 64 is the row half):
//   split    (128 KB region) pair tables for b <= 4, single for b >= 5.  The
//            address is (h << 16) | (byte << 8) | 4 (r mod 64), with byte =
//            (v1 << b) | v2 (pair) or v (single, entry in the low half of the
//            word).  Every row owns its words in every table, so the threads
//            of one row need not wait for any other row's threads when the
//            table changes.
//   packed   (64 KB region) pair tables for b <= 3 with byte =
//            (v1 << (b + 1)) | (v2 << 1) | h at (byte << 8) | 4 (r mod 64);
//            single tables for b >= 4 at (v << 8) | 4 (r mod 64) | 2h (rows r
//            and r + 64 share a word).
// In all of them the 32 threads of a warp (32 consecutive rows) read 32
// different banks.  Shifts are written as multiplies (left) and high multiplies
// (right) so they issue on the FMA pipe; the ALU pipe keeps the LOP3 and PRMT
// work.
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
  if (S >= 0) return x * (1u << (S >= 0 ? S : 0));
  return shr<(S < 0 ? -S : 0)>(x);
}
// (hi << 16) | lo for 16-bit lo and hi, as a multiply-add (FMA pipe).
PW_HD uint32_t pack16(uint32_t lo, uint32_t hi) { return hi * 65536u + lo; }

// ---- 8x8 bit-matrix transpose --------------------------------------------------
// One delta swap: the bits of a selected by ~m trade places with the bits of b
// selected by m, S positions apart.
template <int S>
PW_HD void delta_swap(uint32_t& a, uint32_t& b, uint32_t m) {
  const uint32_t a2 = (a & m) | (shl<S>(b) & ~m);
  const uint32_t b2 = (b & ~m) | (shr<S>(a) & m);
  a = a2;
  b = b2;
}

// In place: afterwards X[q] byte n bit p = (input X[p] bit 8n + q).
PW_HD void transpose8(uint32_t (&X)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) delta_swap<4>(X[i], X[i + 4], 0x0F0F0F0Fu);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (!(i & 2)) delta_swap<2>(X[i], X[i + 2], 0x33333333u);
#pragma unroll
  for (int i = 0; i < 8; i += 2) delta_swap<1>(X[i], X[i + 1], 0x55555555u);
}

// The same for output rows 0..3 only (X[4..7] are left undefined).
PW_HD void transpose8_lo(uint32_t (&X)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) X[i] = (X[i] & 0x0F0F0F0Fu) | (shl<4>(X[i + 4]) & 0xF0F0F0F0u);
  delta_swap<2>(X[0], X[2], 0x33333333u);
  delta_swap<2>(X[1], X[3], 0x33333333u);
  delta_swap<1>(X[0], X[1], 0x55555555u);
  delta_swap<1>(X[2], X[3], 0x55555555u);
}

// Address of the entry for byte N of x: byte 0 = byte 0 of rowb (the row
// byte), byte 1 = byte N of x, byte 2 = byte 1 of rowb (the row half in the
// split layout, else zero), byte 3 = byte 2 of rowb (zero).
template <int N>
PW_HD uint32_t code_addr(uint32_t x, uint32_t rowb) {
  return prmt(x, rowb, 0x6504u | (static_cast<uint32_t>(N) << 4));
}

// Widest bitwidth served by a pair table.
PW_HD constexpr int pair_max(bool split) { return split ? 4 : 3; }
// Bytes a layout's tables span.
PW_HD constexpr uint32_t table_bytes(bool split) { return split ? (2u << 16) : (1u << 16); }

// Row words (bytes 0-1 of every address of row r).
PW_HD uint32_t pair_row_byte(uint32_t r, bool split) {
  return split ? (4u * (r & 63u) | ((r >> 6) << 8)) : 4u * (r & 63u);
}
PW_HD uint32_t single_row_byte(uint32_t r, bool split) {
  return split ? (4u * (r & 63u) | ((r >> 6) << 8)) : 4u * (r & 63u) + 2u * (r >> 6);
}

// Byte offsets of table entries (for writing the tables).
PW_HD uint32_t pair_offset(uint32_t v1, uint32_t v2, int b, uint32_t r, bool split) {
  if (split) return ((r >> 6) << 16) | (((v1 << b) | v2) << 8) | 4u * (r & 63u);
  const uint32_t byte = (v1 << (b + 1)) | (v2 << 1) | (r >> 6);
  return (byte << 8) | 4u * (r & 63u);
}
PW_HD uint32_t single_offset(uint32_t v, uint32_t r, bool split) {
  return split ? ((r >> 6) << 16) | (v << 8) | 4u * (r & 63u) : (v << 8) | single_row_byte(r, false);
}

// Pair-table bitwidths.  Lds32(x) returns the 32-bit entry at byte offset x.
template <int B, bool SPLIT, class Lds32>
PW_HD void dq_word_pair(const uint32_t (&P)[B], uint32_t r, Lds32 lds32, uint32_t* out) {
  static_assert(B >= 1 && B <= pair_max(SPLIT), "pair tables serve b = 1..3 (packed), 1..4 (split)");
  uint32_t X[8];
  // byte bits kH..kH+B-1 = code of column c + 4 (moved down 4 columns), bits
  // kH+B..kH+2B-1 = code of column c; packed layout: bit 0 = row half.
  // Plane 0 is the code's MSB.
  constexpr int kH = SPLIT ? 0 : 1;
  if (kH) X[0] = (r >> 6) ? 0xFFFFFFFFu : 0u;
#pragma unroll
  for (int j = 0; j < B; ++j) {
    X[kH + j] = shr<4>(P[B - 1 - j]);
    X[kH + B + j] = P[B - 1 - j];
  }
#pragma unroll
  for (int p = kH + 2 * B; p < 8; ++p) X[p] = 0u;
  transpose8_lo(X);
  const uint32_t rowb = pair_row_byte(r, SPLIT);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    // byte j of X[m]: columns 8j + m and 8j + m + 4
    out[4 * m + 0] = lds32(code_addr<0>(X[m], rowb));
    out[4 * m + 1] = lds32(code_addr<1>(X[m], rowb));
    out[4 * m + 2] = lds32(code_addr<2>(X[m], rowb));
    out[4 * m + 3] = lds32(code_addr<3>(X[m], rowb));
  }
}

// Single-table bitwidths.  Lds16(x) returns the 16-bit entry at byte offset x.
template <int B, bool SPLIT, class Lds16>
PW_HD void dq_word_single(const uint32_t (&P)[B], uint32_t r, Lds16 lds16, uint32_t* out) {
  static_assert(B > pair_max(SPLIT) && B <= 8, "single tables serve the wider bitwidths");
  uint32_t X[8];
  // byte bit p = code bit p (right-aligned code); plane 0 is the MSB
#pragma unroll
  for (int p = 0; p < 8; ++p) X[p] = (p < B) ? P[(p < B) ? B - 1 - p : 0] : 0u;
  transpose8(X);
  const uint32_t rowb = single_row_byte(r, SPLIT);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    // columns 8j + m (X[m] byte j) and 8j + m + 4 (X[m + 4] byte j)
    out[4 * m + 0] = pack16(lds16(code_addr<0>(X[m], rowb)), lds16(code_addr<0>(X[m + 4], rowb)));
    out[4 * m + 1] = pack16(lds16(code_addr<1>(X[m], rowb)), lds16(code_addr<1>(X[m + 4], rowb)));
    out[4 * m + 2] = pack16(lds16(code_addr<2>(X[m], rowb)), lds16(code_addr<2>(X[m + 4], rowb)));
    out[4 * m + 3] = pack16(lds16(code_addr<3>(X[m], rowb)), lds16(code_addr<3>(X[m + 4], rowb)));
  }
}

}  // namespace dq
}  // namespace pw
