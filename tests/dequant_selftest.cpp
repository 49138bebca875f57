// CPU check of the kernel's per-thread dequantisation routines
// (any_precision_weight_pw_b200/csrc/dequant.cuh) against a plain unpack:
// for every bitwidth, random planes and LUTs, every output half must equal
// LUT[code] of the column the K order assigns to it.  Exit status 0 = pass.
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

// PAIR: take the pair table (b <= 4) rather than the single one (b >= 4).
template <int B, bool PAIR>
static int check(std::mt19937& rng) {
  int bad = 0;
  // emulated shared-memory table: 64 KB, 128 KB for the b = 4 pair table
  std::vector<uint8_t> region(PAIR ? pair_table_bytes(B) : (1u << 16), 0);
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
    if constexpr (PAIR) {
      for (int v1 = 0; v1 < (1 << B); ++v1)
        for (int v2 = 0; v2 < (1 << B); ++v2) {
          const uint32_t off = pair_offset(v1, v2, B, r);
          if (off % 4) { std::printf("pair entry not word aligned\n"); return 1; }
          if (!put16(off, lut[v1]) || !put16(off + 2, lut[v2])) { std::printf("offset out of range\n"); return 1; }
        }
      auto lds32 = [&](uint32_t x) -> uint32_t { return get16(x) | (get16(x + 2) << 16); };
      dq_word_pair<B>(P, r, lds32, out);
    } else {
      for (int v = 0; v < (1 << B); ++v)
        if (!put16(single_offset(v, r), lut[v])) { std::printf("offset out of range\n"); return 1; }
      dq_word_single<B>(P, r, get16, out);
    }
    for (int pr = 0; pr < 16; ++pr) {
      const int m = pr >> 2, j = pr & 3;
      const int c0 = 8 * j + m, c1 = c0 + 4;
      const uint32_t want = lut[code_of(P, B, c0)] | (static_cast<uint32_t>(lut[code_of(P, B, c1)]) << 16);
      if (out[pr] != want) {
        if (bad < 5) std::printf("b=%d trial %d pair %d: got %08x want %08x\n", B, trial, pr, out[pr], want);
        ++bad;
      }
    }
  }
  return bad;
}

// The tables of all rows of a warp-quarter: distinct rows never share a
// 2-byte entry, and the 32 rows of a warp address 32 different banks.
static int check_layout() {
  int bad = 0;
  for (int b = 4; b <= 8; ++b)
    for (uint32_t v = 0; v < (1u << b); ++v)
      for (uint32_t r = 0; r < 128; ++r)
        for (uint32_t r2 = r + 1; r2 < 128; ++r2)
          if (single_offset(v, r) == single_offset(v, r2)) ++bad;
  for (uint32_t q = 0; q < 4; ++q) {
    bool bank[32] = {};
    for (uint32_t l = 0; l < 32; ++l) {
      const uint32_t r = 32 * q + l;
      const uint32_t bk = (single_offset(l % 7, r) / 4) % 32;  // any codes
      if (bank[bk]) ++bad;
      bank[bk] = true;
    }
  }
  for (uint32_t q = 0; q < 4; ++q) {
    bool bank[32] = {};
    for (uint32_t l = 0; l < 32; ++l) {
      const uint32_t r = 32 * q + l;
      const uint32_t bk = (pair_offset(l % 5, l % 3, 3, r) / 4) % 32;
      if (bank[bk]) ++bad;
      bank[bk] = true;
    }
  }
  // b = 4 pair table: every (v1, v2, r) has its own word, and a warp's 32 rows
  // hit 32 banks
  {
    std::vector<uint8_t> seen(pair_table_bytes(4) / 4, 0);
    for (uint32_t v1 = 0; v1 < 16; ++v1)
      for (uint32_t v2 = 0; v2 < 16; ++v2)
        for (uint32_t r = 0; r < 128; ++r) {
          const uint32_t w = pair_offset(v1, v2, 4, r) / 4;
          if (w >= seen.size() || seen[w]) ++bad;
          else seen[w] = 1;
        }
    for (uint32_t q = 0; q < 4; ++q) {
      bool bank[32] = {};
      for (uint32_t l = 0; l < 32; ++l) {
        const uint32_t bk = (pair_offset(l % 7, l % 11, 4, 32 * q + l) / 4) % 32;
        if (bank[bk]) ++bad;
        bank[bk] = true;
      }
    }
  }
  if (bad) std::printf("layout: %d problems\n", bad);
  return bad;
}

int main() {
  std::mt19937 rng(12345);
  int bad = check<1, true>(rng) + check<2, true>(rng) + check<3, true>(rng) +
            check<4, true>(rng) + check<4, false>(rng) + check<5, false>(rng) +
            check<6, false>(rng) + check<7, false>(rng) + check<8, false>(rng) + check_layout();
  std::printf(bad ? "FAIL %d\n" : "ok\n", bad);
  return bad ? 1 : 0;
}
