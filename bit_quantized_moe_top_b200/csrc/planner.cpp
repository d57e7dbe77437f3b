// Greedy bitwidth planner of the weight pages (host only): the reduction and
// restore plans declared in moe_layer.h. One action moves one block by one
// bit-plane; candidates sit in a binary heap ordered by damage per byte, ties
// to the lower block index, and a block's next action enters the heap when
// its previous one is taken.
#include <algorithm>
#include <cmath>
#include <queue>
#include <vector>

#include "../../include/moe_layer.h"

namespace {

struct Action {
  double key;  // damage per byte (reduce: ascending; restore: descending, stored negated)
  int block;
};
struct Later {
  bool operator()(const Action& a, const Action& b) const {
    return a.key > b.key || (a.key == b.key && a.block > b.block);
  }
};

// predicted damage of the transition b -> b-1 of block p
double damage(const moe_plan_block_t& p, int b, float eps) {
  const double d = (double)p.routing_mult * (double)p.sensitivity[b] * (double)p.prompt_factor;
  return std::max((double)eps, d);
}

bool valid(const moe_plan_block_t& p) {
  return p.committed_bits >= 2 && p.committed_bits <= 4 && p.floor_bits >= 2 && p.floor_bits <= p.committed_bits &&
         p.max_steps >= 0 && p.plane_bytes > 0 && p.routing_mult >= 0.f && p.prompt_factor >= 0.f &&
         std::isfinite(p.routing_mult) && std::isfinite(p.prompt_factor) && std::isfinite(p.sensitivity[3]) &&
         std::isfinite(p.sensitivity[4]) && p.sensitivity[3] >= 0.f && p.sensitivity[4] >= 0.f;
}

}  // namespace

extern "C" moe_status_t moe_plan_reduce(const moe_plan_block_t* blocks, int n, long long bytes_target, float eps,
                                        int* new_bits, long long* bytes_released) {
  if (n < 0 || (n > 0 && (!blocks || !new_bits)) || !bytes_released || bytes_target < 0 || !(eps >= 0.f))
    return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!valid(blocks[i])) return MOE_ERR_INVALID_ARG;
  std::vector<int> bits(n), lowest(n);
  std::priority_queue<Action, std::vector<Action>, Later> heap;
  auto push = [&](int i) {
    if (bits[i] > lowest[i]) heap.push({damage(blocks[i], bits[i], eps) / (double)blocks[i].plane_bytes, i});
  };
  for (int i = 0; i < n; ++i) {
    bits[i] = blocks[i].committed_bits;
    lowest[i] = std::max(blocks[i].floor_bits, blocks[i].committed_bits - blocks[i].max_steps);
    push(i);
  }
  long long released = 0;
  while (released < bytes_target && !heap.empty()) {
    const Action a = heap.top();
    heap.pop();
    --bits[a.block];
    released += blocks[a.block].plane_bytes;
    push(a.block);
  }
  for (int i = 0; i < n; ++i) new_bits[i] = bits[i];
  *bytes_released = released;
  return released >= bytes_target ? MOE_OK : MOE_ERR_TOO_LARGE;
}

extern "C" moe_status_t moe_plan_restore(const moe_plan_block_t* blocks, int n, const int* max_bits,
                                         long long bytes_budget, float eps, int* new_bits, long long* bytes_used) {
  if (n < 0 || (n > 0 && (!blocks || !new_bits || !max_bits)) || !bytes_used || bytes_budget < 0 || !(eps >= 0.f))
    return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!valid(blocks[i]) || max_bits[i] < blocks[i].committed_bits || max_bits[i] > 4) return MOE_ERR_INVALID_ARG;
  std::vector<int> bits(n), highest(n);
  std::priority_queue<Action, std::vector<Action>, Later> heap;
  auto push = [&](int i) {
    if (bits[i] < highest[i])
      heap.push({-damage(blocks[i], bits[i] + 1, eps) / (double)blocks[i].plane_bytes, i});
  };
  for (int i = 0; i < n; ++i) {
    bits[i] = blocks[i].committed_bits;
    highest[i] = std::min(max_bits[i], blocks[i].committed_bits + blocks[i].max_steps);
    push(i);
  }
  long long used = 0;
  // the most damage removed per byte first; an action that does not fit ends
  // that block's restores in this plan (its later planes depend on it)
  while (!heap.empty()) {
    const Action a = heap.top();
    heap.pop();
    if (used + blocks[a.block].plane_bytes > bytes_budget) continue;
    ++bits[a.block];
    used += blocks[a.block].plane_bytes;
    push(a.block);
  }
  for (int i = 0; i < n; ++i) new_bits[i] = bits[i];
  *bytes_used = used;
  return MOE_OK;
}
