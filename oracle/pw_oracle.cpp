// pw_oracle.cpp -- plain, slow, CPU reference of the PagedWeight fused
// mixed-precision MoE layer.  TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the benchmark's CPU-baseline leg may
// load this library.  The product path (the CUDA library under
// any_precision_weight_pw_b200/) shares no code, header, table or helper with
// it, and never calls it.
//
// What it computes (sources are the public summaries of the paper
// "PagedWeight: Efficient MoE LLM Serving with Dynamic Quality-Aware Weight
// Quantization"):
//   * arxivlens summary, abstract paragraph: the fused mixed-precision MoE
//     kernel works directly on Any-Precision (AP) bit-planes and lookup
//     tables (LUTs) of GPU-resident weight pages.
//   * legiblepapers summary, "Key Takeaways" and FAQ Q5: the kernel reads
//     bit-plane and LUT buffers directly, with a separate bitwidth for every
//     linear-block, and fuses routing, expert activation and output
//     accumulation.
// The pages fix neither the bit layout nor the routing formula nor the
// activation; the reading taken for each is stated at the function that
// uses it below.
//
// Arithmetic: router logits and the top-k decision in fp32 with one fixed
// summation order (the decision is integer-valued, so both sides take it in
// the kernel's precision); everything else in double.
//
// Parity status of each function (what pins it is in tests/test_oracle_*.py):
//   pwo_pack_planes / pwo_unpack_codes  pinned (hand-derived golden words,
//                                       top-b-bits invariant, round trip)
//   pwo_linear                          pinned (identity LUT == integer matmul,
//                                       exact; golden LUT-gather example)
//   pwo_router_logits                   pinned (exact small-integer cases,
//                                       fp64 bound on random inputs)
//   pwo_topk_softmax                    pinned (brute force with ties,
//                                       closed forms for E=2 and k=E)
//   pwo_expert_ffn / pwo_moe_forward    pinned (hand-worked 2-expert example,
//                                       shared-expert linearity, SiLU limits)
//   pwo_plan_greedy / pwo_plan_exact    pinned (hand-worked instance; greedy
//                                       equals the brute-force optimum where
//                                       the exchange argument holds; greedy
//                                       never beats the optimum)
//   pwo_routing_stats                   pinned (hand-worked example, totals
//                                       T*k and T, k = E column sums equal
//                                       a softmax written out in numpy)

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

// ---- scalar conversions (exact) -------------------------------------------

// IEEE binary16 -> double, exact for every finite input, subnormals included.
double half_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int expo = (h >> 10) & 0x1f;
  const int frac = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = std::ldexp(static_cast<double>(frac), -24);          // subnormal
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = std::ldexp(static_cast<double>(frac | 0x400), expo - 25);
  }
  return sign ? -v : v;
}

// bfloat16 -> float is a 16-bit left shift of the bit pattern (exact).
float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// ---- the Any-Precision bit-plane view -------------------------------------
//
// Layout (a reading: the pages name "bit-plane buffers" without a layout):
//   planes[k][o][w], k = 0 .. n_max-1, plane 0 holds the MOST significant bit.
//   words = ceil(cols / 32); bit (i % 32) of word planes[k][o][i / 32] is bit
//   (n_max - 1 - k) of the n_max-bit code of element (o, i).
//   A b-bit view reads planes 0 .. b-1 only: its code is
//     code_b(o, i) = sum_{k < b} bit_k(o, i) * 2^(b - 1 - k).

inline int plane_bit(const uint32_t* planes, int rows, int words, int k, int o,
                     int i) {
  const uint32_t w =
      planes[(static_cast<size_t>(k) * rows + o) * words + (i >> 5)];
  return static_cast<int>((w >> (i & 31)) & 1u);
}

inline int code_of(const uint32_t* planes, int rows, int words, int b, int o,
                   int i) {
  int c = 0;
  for (int k = 0; k < b; ++k) c = (c << 1) | plane_bit(planes, rows, words, k, o, i);
  return c;
}

// Run fn(lo, hi) over [0, n) split into n_threads contiguous ranges.
template <class F>
void parallel_for(int n, int n_threads, F fn) {
  if (n_threads <= 1 || n < 2) {
    fn(0, n);
    return;
  }
  n_threads = std::min(n_threads, n);
  std::vector<std::thread> pool;
  pool.reserve(n_threads);
  for (int t = 0; t < n_threads; ++t) {
    const int lo = static_cast<int>(static_cast<long long>(n) * t / n_threads);
    const int hi = static_cast<int>(static_cast<long long>(n) * (t + 1) / n_threads);
    pool.emplace_back([=] { fn(lo, hi); });
  }
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// One linear-block of the layer as the oracle sees it: W (rows x cols),
// y = W x, stored as n_max bit-planes plus the LUT of the current bitwidth.
typedef struct {
  const uint32_t* planes;  // [n_max][rows][ceil(cols/32)]
  const uint16_t* lut;     // [rows][2^bits] fp16 bit patterns
  int32_t rows, cols, bits;
} pwo_block_t;

// The layer: E routed SwiGLU experts (gate, up: F x H; down: H x F), top-k
// routing, optional ungated shared SwiGLU expert of width S.
typedef struct {
  int32_t hidden, ffn, n_experts, top_k, shared_ffn, n_max, renorm_topk;
  const pwo_block_t* blocks;  // 3*E (+3 if shared_ffn > 0); id = expert*3 + proj,
                              // proj 0 = gate, 1 = up, 2 = down; shared = E*3 + proj
} pwo_layer_t;

// Pack n_max-bit codes [rows][cols] into bit-planes (the encoder of the
// layout above; pad bits are zero).  Returns 0 on success.
int pwo_pack_planes(const uint8_t* codes, int rows, int cols, int n_max,
                    uint32_t* planes) {
  if (!codes || !planes || rows < 0 || cols < 0 || n_max < 1 || n_max > 8) return 1;
  const int words = (cols + 31) / 32;
  std::memset(planes, 0, sizeof(uint32_t) * static_cast<size_t>(n_max) * rows * words);
  for (int k = 0; k < n_max; ++k)
    for (int o = 0; o < rows; ++o)
      for (int i = 0; i < cols; ++i) {
        const int bit = (codes[static_cast<size_t>(o) * cols + i] >> (n_max - 1 - k)) & 1;
        if (bit)
          planes[(static_cast<size_t>(k) * rows + o) * words + (i >> 5)] |= 1u << (i & 31);
      }
  return 0;
}

// Codes of the b-bit view, [rows][cols].  Returns 0 on success.
int pwo_unpack_codes(const uint32_t* planes, int rows, int cols, int n_max,
                     int b, uint8_t* codes) {
  if (!planes || !codes || b < 1 || b > n_max || n_max > 8) return 1;
  const int words = (cols + 31) / 32;
  for (int o = 0; o < rows; ++o)
    for (int i = 0; i < cols; ++i)
      codes[static_cast<size_t>(o) * cols + i] =
          static_cast<uint8_t>(code_of(planes, rows, words, b, o, i));
  return 0;
}

// y[o] = sum_i W_b[o][i] * x[i],  W_b[o][i] = LUT_b[o][code_b(o, i)]
// (the dequantised linear of one linear-block at bitwidth b).  The codes
// are unpacked bit by bit and looked up per element, in double.
int pwo_linear(const uint32_t* planes, const uint16_t* lut, int rows, int cols,
               int b, const double* x, double* y, int n_threads) {
  if (!planes || !lut || !x || !y || b < 1 || b > 8) return 1;
  const int words = (cols + 31) / 32;
  const int nlut = 1 << b;
  parallel_for(rows, n_threads, [&](int lo, int hi) {
    for (int o = lo; o < hi; ++o) {
      double acc = 0.0;
      for (int i = 0; i < cols; ++i) {
        const int c = code_of(planes, rows, words, b, o, i);
        acc += half_to_double(lut[static_cast<size_t>(o) * nlut + c]) * x[i];
      }
      y[o] = acc;
    }
  });
  return 0;
}

// Router logits in fp32, in one fixed order that the GPU path also uses:
// 32 partial sums s_j (j = 0..31) accumulate fmaf(x[i], Wr[e][i], s_j) over
// i = j, j+32, j+64, ... ascending; then s_j <- s_j + s_{j xor m} for
// m = 16, 8, 4, 2, 1 (all j at once); the logit is s_0, plus bias[e] if a
// bias is given.  (Reading: the pages only say routing is fused; bit-exact
// top-k across CPU and GPU needs a shared order.)
int pwo_router_logits(const uint16_t* x_bf16, int T, int H, const float* Wr,
                      const float* bias, int E, float* logits) {
  if ((!x_bf16 && T > 0) || !Wr || !logits || H < 1 || E < 1) return 1;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      float s[32], nxt[32];
      for (int j = 0; j < 32; ++j) {
        s[j] = 0.0f;
        for (int i = j; i < H; i += 32)
          s[j] = std::fmaf(bf16_to_float(x_bf16[static_cast<size_t>(t) * H + i]),
                           Wr[static_cast<size_t>(e) * H + i], s[j]);
      }
      for (int m = 16; m >= 1; m >>= 1) {
        for (int j = 0; j < 32; ++j) nxt[j] = s[j] + s[j ^ m];
        std::memcpy(s, nxt, sizeof(s));
      }
      float l = s[0];
      if (bias) l = l + bias[e];
      logits[static_cast<size_t>(t) * E + e] = l;
    }
  return 0;
}

// Top-k and routing weights.  Experts are ranked by logit, descending, ties
// to the lower expert index; the first k are selected in that order.  The
// probabilities are the softmax over all E logits (double); the weight of
// slot j is p[idx[j]], divided by the sum over the k selected when renorm.
int pwo_topk_softmax(const float* logits, int T, int E, int k, int renorm,
                     int32_t* idx, double* w) {
  if ((!logits && T > 0) || !idx || !w || k < 1 || k > E) return 1;
  std::vector<int> order(E);
  std::vector<double> p(E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + static_cast<size_t>(t) * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
      return l[a] > l[b];  // stable: equal logits keep ascending index
    });
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e) mx = std::max(mx, static_cast<double>(l[e]));
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = std::exp(static_cast<double>(l[e]) - mx);
      z += p[e];
    }
    double sel = 0.0;
    for (int j = 0; j < k; ++j) sel += p[order[j]] / z;
    for (int j = 0; j < k; ++j) {
      idx[static_cast<size_t>(t) * k + j] = order[j];
      const double pj = p[order[j]] / z;
      w[static_cast<size_t>(t) * k + j] = renorm ? pj / sel : pj;
    }
  }
  return 0;
}

// Routing statistics of a batch: the online "routing mass" the planner
// weighs (legiblepapers summary, "Summary & Methodology Analysis": routing
// mass is how frequently an expert is used).  Reading: per expert e, the
// number of (token, slot) assignments to e and the sum of their routing
// weights, ADDED to counts[e] and mass[e] so that calls accumulate over
// forwards.  idx / w are [T][k] as pwo_topk_softmax returns them.
int pwo_routing_stats(const int32_t* idx, const double* w, int T, int k, int E,
                      uint64_t* counts, double* mass) {
  if ((T > 0 && (!idx || !w)) || !counts || !mass || k < 1 || E < 1) return 1;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[static_cast<size_t>(t) * k + j];
      if (e < 0 || e >= E) return 1;
      counts[e] += 1;
      mass[e] += w[static_cast<size_t>(t) * k + j];
    }
  return 0;
}

// ---- the quality-aware planner (host-side decision) ------------------------
//
// legiblepapers summary, "Summary & Methodology Analysis" and FAQ Q8: the
// runtime planner takes a target number of bytes to free and greedily picks
// weight quantisation actions with the least damage per released byte; the
// damage combines offline sensitivity, online routing mass and prompt
// residuals.  The pages give no formula; the reading taken here:
//   action (i, b): lower block i from b to b - 1 bits (b > min_bits[i]); it
//     releases plane page b - 1 and shrinks the LUT from 2^b to 2^(b-1)
//     fp16 entries per row:  bytes(i, b) = plane_bytes[i] + rows[i] * 2^(b-1) * 2
//   damage(i, b) = sens[i][b] * mass[i] * (1 + resid[i])   (in double, in
//     this order), sens[i][b] the offline sensitivity of that step, mass[i]
//     the routing mass of the block's expert, resid[i] >= 0 a prompt-residual
//     weight.
//   greedy: while released < target, take the action with the smallest
//     damage / bytes (double division; ties to the lower block index) and
//     apply it.
typedef struct {
  int32_t bits, min_bits;   // current width, lowest allowed width
  int64_t plane_bytes;      // bytes of one plane page of the block
  int32_t rows;             // LUT rows
  double mass, resid;       // routing mass of the block's expert, residual weight
  double sens[9];           // sens[b]: damage of the step b -> b - 1 (b = 1..8)
} pwo_plan_block_t;

static int64_t plan_step_bytes(const pwo_plan_block_t& k, int b) {
  return k.plane_bytes + static_cast<int64_t>(k.rows) * (int64_t{1} << (b - 1)) * 2;
}
static double plan_step_damage(const pwo_plan_block_t& k, int b) {
  return k.sens[b] * k.mass * (1.0 + k.resid);
}

// Greedy: new_bits[n], *released, *damage.  Returns 0 when the target was
// reached, 2 when no action was left before reaching it (new_bits then holds
// every block at its lowest width), 1 on bad arguments.
int pwo_plan_greedy(const pwo_plan_block_t* blocks, int n, int64_t target, int32_t* new_bits,
                    int64_t* released, double* damage) {
  if (!blocks || !new_bits || !released || !damage || n < 0) return 1;
  for (int i = 0; i < n; ++i) {
    if (blocks[i].bits < 1 || blocks[i].bits > 8 || blocks[i].min_bits < 1 ||
        blocks[i].min_bits > blocks[i].bits)
      return 1;
    new_bits[i] = blocks[i].bits;
  }
  *released = 0;
  *damage = 0.0;
  while (*released < target) {
    int best = -1;
    double best_ratio = 0.0;
    for (int i = 0; i < n; ++i) {
      const int b = new_bits[i];
      if (b <= blocks[i].min_bits) continue;
      const double ratio = plan_step_damage(blocks[i], b) /
                           static_cast<double>(plan_step_bytes(blocks[i], b));
      if (best < 0 || ratio < best_ratio) {
        best = i;
        best_ratio = ratio;
      }
    }
    if (best < 0) return 2;
    const int b = new_bits[best];
    *released += plan_step_bytes(blocks[best], b);
    *damage += plan_step_damage(blocks[best], b);
    new_bits[best] = b - 1;
  }
  return 0;
}

// The exact optimum of the same problem by brute force over every width
// vector (min_bits[i] .. bits[i] per block): the smallest total damage whose
// released bytes reach the target (ties: the first vector in lexicographic
// order of (w_0, w_1, ...) descending from the current widths).  For tiny
// instances only.  Returns 0, or 2 if no vector reaches the target.
int pwo_plan_exact(const pwo_plan_block_t* blocks, int n, int64_t target, int32_t* best_bits,
                   int64_t* released, double* damage) {
  if (!blocks || !best_bits || !released || !damage || n < 0 || n > 12) return 1;
  std::vector<int> w(n);
  for (int i = 0; i < n; ++i) w[i] = blocks[i].bits;
  bool found = false;
  double best_d = 0.0;
  int64_t best_r = 0;
  while (true) {
    int64_t r = 0;
    double d = 0.0;
    for (int i = 0; i < n; ++i)
      for (int b = blocks[i].bits; b > w[i]; --b) {
        r += plan_step_bytes(blocks[i], b);
        d += plan_step_damage(blocks[i], b);
      }
    if (r >= target && (!found || d < best_d)) {
      found = true;
      best_d = d;
      best_r = r;
      for (int i = 0; i < n; ++i) best_bits[i] = w[i];
    }
    int i = n - 1;  // next vector: odometer, each digit counting down
    while (i >= 0 && w[i] == blocks[i].min_bits) {
      w[i] = blocks[i].bits;
      --i;
    }
    if (i < 0) break;
    --w[i];
  }
  if (!found) return 2;
  *released = best_r;
  *damage = best_d;
  return 0;
}

// One SwiGLU expert on one token: g = W_gate x, u = W_up x,
// h = silu(g) * u with silu(g) = g / (1 + exp(-g)), y = W_down h.
// The expert's three blocks are blocks[3*e + 0..2] of the layer
// (e == n_experts selects the shared expert).  h_out may be NULL.
int pwo_expert_ffn(const pwo_layer_t* L, int e, const double* x, double* y,
                   double* h_out, int n_threads) {
  if (!L || !x || !y || e < 0 || e > L->n_experts) return 1;
  if (e == L->n_experts && L->shared_ffn <= 0) return 1;
  const pwo_block_t& g = L->blocks[3 * e + 0];
  const pwo_block_t& u = L->blocks[3 * e + 1];
  const pwo_block_t& d = L->blocks[3 * e + 2];
  const int F = g.rows;
  std::vector<double> gv(F), uv(F), h(F);
  if (pwo_linear(g.planes, g.lut, g.rows, g.cols, g.bits, x, gv.data(), n_threads)) return 1;
  if (pwo_linear(u.planes, u.lut, u.rows, u.cols, u.bits, x, uv.data(), n_threads)) return 1;
  for (int f = 0; f < F; ++f) h[f] = gv[f] / (1.0 + std::exp(-gv[f])) * uv[f];
  if (pwo_linear(d.planes, d.lut, d.rows, d.cols, d.bits, h.data(), y, n_threads)) return 1;
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * F);
  return 0;
}

// The whole layer: out[t] = sum_{j<k} w[t][j] * expert_{idx[t][j]}(x_t)
//                           + shared(x_t)   (shared added with weight 1).
// x is bf16 [T][H]; out is double [T][H].  idx/w (optional, [T][k]) receive
// the routing.  Tokens run one after another; rows of each projection are
// split over n_threads threads.
int pwo_moe_forward(const pwo_layer_t* L, const uint16_t* x_bf16, int T,
                    const float* Wr, const float* bias, double* out,
                    int32_t* idx_out, double* w_out, int n_threads) {
  if (!L || (!x_bf16 && T > 0) || !Wr || (!out && T > 0)) return 1;
  const int H = L->hidden, E = L->n_experts, k = L->top_k;
  std::vector<float> logits(static_cast<size_t>(T) * E);
  std::vector<int32_t> idx(static_cast<size_t>(T) * k);
  std::vector<double> w(static_cast<size_t>(T) * k);
  if (T > 0) {
    if (pwo_router_logits(x_bf16, T, H, Wr, bias, E, logits.data())) return 1;
    if (pwo_topk_softmax(logits.data(), T, E, k, L->renorm_topk, idx.data(), w.data())) return 1;
  }
  std::vector<double> xt(H), ye(H);
  for (int t = 0; t < T; ++t) {
    for (int i = 0; i < H; ++i) xt[i] = bf16_to_float(x_bf16[static_cast<size_t>(t) * H + i]);
    double* o = out + static_cast<size_t>(t) * H;
    for (int i = 0; i < H; ++i) o[i] = 0.0;
    for (int j = 0; j < k; ++j) {
      if (pwo_expert_ffn(L, idx[static_cast<size_t>(t) * k + j], xt.data(), ye.data(), nullptr, n_threads)) return 1;
      const double wj = w[static_cast<size_t>(t) * k + j];
      for (int i = 0; i < H; ++i) o[i] += wj * ye[i];
    }
    if (L->shared_ffn > 0) {
      if (pwo_expert_ffn(L, E, xt.data(), ye.data(), nullptr, n_threads)) return 1;
      for (int i = 0; i < H; ++i) o[i] += ye[i];
    }
  }
  if (idx_out) std::memcpy(idx_out, idx.data(), sizeof(int32_t) * idx.size());
  if (w_out) std::memcpy(w_out, w.data(), sizeof(double) * w.size());
  return 0;
}

}  // extern "C"
