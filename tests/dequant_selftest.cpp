// CPU check of the kernel's per-thread dequantisation routines
// (any_precision_weight_pw_b200/csrc/dequant.cuh) against a plain unpack:
// for every bitwidth, random planes and LUTs, every output half must equal
// LUT[code] of the column the K order assigns to it.  Exit status 0 = pass.
#include <cstdio>
#include <cstdlib>
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

template <int B>
static int check(std::mt19937& rng) {
  int bad = 0;
  std::vector<uint8_t> region(1u << 17, 0);  // emulated shared-memory table
  for (int trial = 0; trial < 2000; ++trial) {
    const int r = rng() % 128;
    uint32_t P[B];
    for (int k = 0; k < B; ++k) P[k] = rng();
    if (trial == 0) for (int k = 0; k < B; ++k) P[k] = 0xFFFFFFFFu;
    if (trial == 1) for (int k = 0; k < B; ++k) P[k] = 0u;
    uint16_t lut[256];
    for (int v = 0; v < (1 << B); ++v) lut[v] = static_cast<uint16_t>(rng());
    uint32_t out[16];
    if constexpr (B <= 3) {
      uint32_t w[4] = {0, 0, 0, 0};
      for (int v = 0; v < (1 << B); ++v) w[v / 2] |= static_cast<uint32_t>(lut[v]) << (16 * (v & 1));
      RegLut L = make_reg_lut<B>(w);
      dq_word_reg<B>(P, L, out);
    } else {
      for (int v = 0; v < (1 << B); ++v) {
        const uint32_t off = (static_cast<uint32_t>(v) << 9) | (4u * r);
        region[off] = lut[v] & 0xFF;
        region[off + 1] = lut[v] >> 8;
      }
      auto lds = [&](uint32_t x) -> uint32_t { return region[x] | (region[x + 1] << 8); };
      dq_word_smem<B>(P, 4u * r, lds, out);
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

int main() {
  std::mt19937 rng(12345);
  int bad = check<1>(rng) + check<2>(rng) + check<3>(rng) + check<4>(rng) + check<5>(rng) +
            check<6>(rng) + check<7>(rng) + check<8>(rng);
  std::printf(bad ? "FAIL %d\n" : "ok\n", bad);
  return bad ? 1 : 0;
}
