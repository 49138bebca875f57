// CPU check of the kernel's per-thread dequantisation routines
// (any_precision_weight_pw_b200/csrc/dequant.cuh) against a plain unpack:
// for every bitwidth and both table layouts, random planes and LUTs, every
// output half must equal LUT[code] of the column the K order assigns to it.
// The layout checks cover bank spread and, for the split layout, that every
// row's table words are its own in every format; the 32-row tables of the
// CUDA-core passes are checked the same way.  Exit status 0 = pass.
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <random>
#include <vector>

#include "../any_precision_weight_pw_b200/csrc/dequant.cuh"

using namespace pw::dq;

static int code_of(const uint32_t* P, int B, int c) {
  int v = 0;
  for (int k = 0; k < B; ++k) v = (v << 1) | ((P[k] >> c) & 1);
  return v;
}

template <int B, bool SPLIT>
static int check(std::mt19937& rng) {
  constexpr bool kPair = B <= pair_max(SPLIT);
  int bad = 0;
  std::vector<uint8_t> region(table_bytes(SPLIT), 0);  // emulated shared-memory table region
  for (int trial = 0; trial < 2000; ++trial) {
    const uint32_t r = rng() % 128;
    uint32_t P[B];
    for (int k = 0; k < B; ++k) P[k] = rng();
    if (trial == 0) for (int k = 0; k < B; ++k) P[k] = 0xFFFFFFFFu;
    if (trial == 1) for (int k = 0; k < B; ++k) P[k] = 0u;
    uint16_t lut[256];
    for (int v = 0; v < (1 << B); ++v) lut[v] = static_cast<uint16_t>(rng());
    std::fill(region.begin(), region.end(), 0xEE);  // unwritten bytes never match
    auto put16 = [&](uint32_t off, uint16_t v) -> bool {
      if (off + 1 >= region.size()) return false;
      region[off] = v & 0xFF;
      region[off + 1] = v >> 8;
      return true;
    };
    auto get16 = [&](uint32_t x) -> uint32_t {
      if (x + 1 >= region.size()) { std::printf("read out of range\n"); std::exit(1); }
      return region[x] | (region[x + 1] << 8);
    };
    uint32_t out[16];
    if constexpr (kPair) {
      for (int v1 = 0; v1 < (1 << B); ++v1)
        for (int v2 = 0; v2 < (1 << B); ++v2) {
          const uint32_t off = pair_offset(v1, v2, B, r, SPLIT);
          if (off % 4) { std::printf("pair entry not word aligned\n"); return 1; }
          if (!put16(off, lut[v1]) || !put16(off + 2, lut[v2])) { std::printf("offset out of range\n"); return 1; }
        }
      auto lds32 = [&](uint32_t x) -> uint32_t { return get16(x) | (get16(x + 2) << 16); };
      dq_word_pair<B, SPLIT>(P, r, lds32, out);
    } else {
      for (int v = 0; v < (1 << B); ++v)
        if (!put16(single_offset(v, r, SPLIT), lut[v])) { std::printf("offset out of range\n"); return 1; }
      dq_word_single<B, SPLIT>(P, r, get16, out);
    }
    for (int pr = 0; pr < 16; ++pr) {
      const int m = pr >> 2, j = pr & 3;
      const int c0 = 8 * j + m, c1 = c0 + 4;
      const uint32_t want = lut[code_of(P, B, c0)] | (static_cast<uint32_t>(lut[code_of(P, B, c1)]) << 16);
      if (out[pr] != want) {
        if (bad < 5) std::printf("b=%d split=%d trial %d pair %d: got %08x want %08x\n", B, SPLIT, trial, pr, out[pr], want);
        ++bad;
      }
    }
  }
  return bad;
}

// Byte offsets of every entry of row r's table for bitwidth b (2 bytes each).
static std::vector<uint32_t> entries(int b, uint32_t r, bool split) {
  std::vector<uint32_t> o;
  if (b <= pair_max(split)) {
    for (uint32_t v1 = 0; v1 < (1u << b); ++v1)
      for (uint32_t v2 = 0; v2 < (1u << b); ++v2) {
        o.push_back(pair_offset(v1, v2, b, r, split));
        o.push_back(pair_offset(v1, v2, b, r, split) + 2);
      }
  } else {
    for (uint32_t v = 0; v < (1u << b); ++v) o.push_back(single_offset(v, r, split));
  }
  return o;
}

static int check_layout(bool split) {
  int bad = 0;
  for (int b = 1; b <= 8; ++b) {
    // distinct rows never share a 2-byte entry, and every entry is in range
    std::vector<int> owner(table_bytes(split) / 2, -1);
    for (uint32_t r = 0; r < 128; ++r)
      for (uint32_t off : entries(b, r, split)) {
        if (off + 2 > table_bytes(split)) { ++bad; continue; }
        if (owner[off / 2] >= 0 && owner[off / 2] != static_cast<int>(r)) ++bad;
        owner[off / 2] = static_cast<int>(r);
      }
    // the 32 rows of a warp read 32 different banks, whatever their codes
    for (uint32_t q = 0; q < 4; ++q) {
      bool bank[32] = {};
      for (uint32_t l = 0; l < 32; ++l) {
        const uint32_t r = 32 * q + l;
        const uint32_t v1 = (l * 7) % (1u << b), v2 = (l * 5 + 3) % (1u << b);
        const uint32_t off = b <= pair_max(split) ? pair_offset(v1, v2, b, r, split)
                                                  : single_offset(v1, r, split);
        const uint32_t bk = (off / 4) % 32;
        if (bank[bk]) ++bad;
        bank[bk] = true;
      }
    }
  }
  if (split) {
    // every 4-byte word of row r's tables, in every format, encodes r: row
    // half in bit 14 of the word index, r mod 64 in bits 0-5
    for (int b = 1; b <= 8; ++b)
      for (uint32_t r = 0; r < 128; ++r)
        for (uint32_t off : entries(b, r, true)) {
          const uint32_t w = off / 4;
          if ((((w >> 14) & 1u) << 6 | (w & 63u)) != r) ++bad;
        }
  }
  if (bad) std::printf("layout (split=%d): %d problems\n", split, bad);
  return bad;
}

// The CUDA-core passes' 32-row tables (gv.cu): entry (code, row l) at
// code * 128 + 4 l (pair tables up to b = 4 with code = (v1 << b) | v2,
// single tables above in the low half), looked up through the split-layout
// routines with row 2 l and the address halved.  Every entry lies inside
// the 32 KB table, the 32 rows of a warp hit 32 banks, and the outputs equal
// the plain unpack.
template <int B>
static int check_gv(std::mt19937& rng) {
  constexpr bool kPair = B <= pair_max(true);
  constexpr uint32_t kTab = 32768;
  int bad = 0;
  std::vector<uint8_t> region(kTab, 0);
  for (int trial = 0; trial < 500; ++trial) {
    const uint32_t lane = rng() % 32;
    uint32_t P[B];
    for (int k = 0; k < B; ++k) P[k] = rng();
    uint16_t lut[256];
    for (int v = 0; v < (1 << B); ++v) lut[v] = static_cast<uint16_t>(rng());
    std::fill(region.begin(), region.end(), 0xEE);
    auto put16 = [&](uint32_t off, uint16_t v) {
      if (off + 2 > kTab) { std::printf("gv entry out of range\n"); std::exit(1); }
      region[off] = v & 0xFF;
      region[off + 1] = v >> 8;
    };
    auto get16 = [&](uint32_t a) -> uint32_t {
      const uint32_t x = a >> 1;
      if (x + 2 > kTab) { std::printf("gv read out of range\n"); std::exit(1); }
      return region[x] | (region[x + 1] << 8);
    };
    uint32_t out[16];
    if constexpr (kPair) {
      for (int v1 = 0; v1 < (1 << B); ++v1)
        for (int v2 = 0; v2 < (1 << B); ++v2) {
          const uint32_t off = ((v1 << B) | v2) * 128u + 4u * lane;
          put16(off, lut[v1]);
          put16(off + 2, lut[v2]);
        }
      auto lds32 = [&](uint32_t a) -> uint32_t { return get16(a) | (get16(a + 4) << 16); };
      dq_word_pair<B, true>(P, 2 * lane, lds32, out);
    } else {
      for (int v = 0; v < (1 << B); ++v) put16(v * 128u + 4u * lane, lut[v]);
      dq_word_single<B, true>(P, 2 * lane, get16, out);
    }
    for (int pr = 0; pr < 16; ++pr) {
      const int m = pr >> 2, j = pr & 3;
      const int c0 = 8 * j + m, c1 = c0 + 4;
      const uint32_t want = lut[code_of(P, B, c0)] | (static_cast<uint32_t>(lut[code_of(P, B, c1)]) << 16);
      if (out[pr] != want) {
        if (bad < 5) std::printf("gv b=%d trial %d pair %d: got %08x want %08x\n", B, trial, pr, out[pr], want);
        ++bad;
      }
    }
  }
  // bank spread: lanes l read word (code * 32 + l), bank l
  for (uint32_t l = 0; l < 32; ++l)
    if ((((7u * l) % (1u << B)) * 128u + 4u * l) / 4 % 32 != l) ++bad;
  return bad;
}

int main() {
  std::mt19937 rng(12345);
  int bad = check<1, false>(rng) + check<2, false>(rng) + check<3, false>(rng) + check<4, false>(rng) +
            check<5, false>(rng) + check<6, false>(rng) + check<7, false>(rng) + check<8, false>(rng);
  bad += check<1, true>(rng) + check<2, true>(rng) + check<3, true>(rng) + check<4, true>(rng) +
         check<5, true>(rng) + check<6, true>(rng) + check<7, true>(rng) + check<8, true>(rng);
  bad += check_layout(false) + check_layout(true);
  bad += check_gv<1>(rng) + check_gv<2>(rng) + check_gv<3>(rng) + check_gv<4>(rng) +
         check_gv<5>(rng) + check_gv<6>(rng) + check_gv<7>(rng) + check_gv<8>(rng);
  std::printf(bad ? "FAIL %d\n" : "ok\n", bad);
  return bad ? 1 : 0;
}
