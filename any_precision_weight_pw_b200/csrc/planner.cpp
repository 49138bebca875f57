// planner.cpp -- the quality-aware release planner (host code).
//
// PagedWeight (legiblepapers summary, "Summary & Methodology Analysis" and
// FAQ Q8): given a number of bytes to free, the runtime planner greedily
// picks weight quantisation actions with the least damage per released
// byte, the damage combining offline sensitivity, online routing mass and
// prompt residuals.  The library's reading (pw.h, pw_plan_release):
//   one action lowers a block by one bit, releasing its plane page b-1 and
//   half of its LUT;  damage = sens[b] * mass * (1 + resid).
// Each block's next action sits in a min-heap keyed by (damage per byte,
// block index), so a plan of m actions over n blocks costs O((n + m) log n);
// after a block's action only that block's next action changes.
#include <cstdint>
#include <queue>
#include <vector>

#include "pw_internal.h"

namespace {

struct Cand {
  double ratio;
  int32_t block;
};
// std::priority_queue is a max-heap: "greater" puts the smallest ratio (then
// the lowest block index) on top.
struct Later {
  bool operator()(const Cand& a, const Cand& b) const {
    return a.ratio > b.ratio || (a.ratio == b.ratio && a.block > b.block);
  }
};

int64_t step_bytes(const pw_plan_block_t& k, int b) {
  return k.plane_bytes + static_cast<int64_t>(k.rows) * (static_cast<int64_t>(1) << (b - 1)) * 2;
}
double step_damage(const pw_plan_block_t& k, int b) {
  return k.sens[b] * k.mass * (1.0 + k.resid);
}

}  // namespace

extern "C" pw_status_t pw_plan_release(const pw_plan_block_t* blocks, int32_t n,
                                       int64_t target_bytes, int32_t* new_bits,
                                       int64_t* released, double* damage, int32_t* reached) {
  if (n < 0 || (n > 0 && (!blocks || !new_bits)) || !released || !damage || !reached)
    return pw::record_error(PW_ERR_INVALID_ARG, "pw_plan_release: null argument or n < 0");
  for (int32_t i = 0; i < n; ++i) {
    const pw_plan_block_t& k = blocks[i];
    if (k.bits < 1 || k.bits > PW_MAX_BITS || k.min_bits < 1 || k.min_bits > k.bits ||
        k.plane_bytes < 0 || k.rows < 0 || !(k.mass >= 0.0) || !(k.resid >= 0.0))
      return pw::record_error(PW_ERR_INVALID_ARG,
                              "pw_plan_release: a block needs 1 <= min_bits <= bits <= 8, "
                              "non-negative sizes, mass and resid");
  }
  std::priority_queue<Cand, std::vector<Cand>, Later> heap;
  auto push = [&](int32_t i, int b) {
    if (b > blocks[i].min_bits)
      heap.push(Cand{step_damage(blocks[i], b) / static_cast<double>(step_bytes(blocks[i], b)), i});
  };
  for (int32_t i = 0; i < n; ++i) {
    new_bits[i] = blocks[i].bits;
    push(i, blocks[i].bits);
  }
  int64_t rel = 0;
  double dmg = 0.0;
  while (rel < target_bytes && !heap.empty()) {
    const int32_t i = heap.top().block;
    heap.pop();
    const int b = new_bits[i];
    rel += step_bytes(blocks[i], b);
    dmg += step_damage(blocks[i], b);
    new_bits[i] = b - 1;
    push(i, b - 1);
  }
  *released = rel;
  *damage = dmg;
  *reached = rel >= target_bytes ? 1 : 0;
  return PW_OK;
}
