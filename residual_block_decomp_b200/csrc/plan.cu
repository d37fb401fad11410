// Host-side planning of which residual blocks to keep loaded: the global order of
// the blocks of all weights, and the per-weight block counts a memory budget allows.
//
// BitStack keeps the residual blocks of every weight of every layer in one universal
// stack on the storage device and loads or offloads them, per weight in a presorted
// order, as the available memory changes (review page "BitStack: Fine-Grained Size
// Control...", Fig. 2 caption; OpenReview discussion, reply A1.B).  The pages compare
// three orders -- Average, Greedy, Random (review page, Fig. 6 caption) -- and name a
// scoring step (README, "Decomposition", --score_importance) without printing it.
// This file implements the three orders for scores the caller provides (for example
// the drop of the scaled residual norm per byte that each block brings) and the
// budget fill; no GPU is involved.
#include <algorithm>
#include <queue>
#include <vector>

#include "internal.h"

namespace {

struct Next {
  double score;
  int weight;
};
// max-heap on score; equal scores: the lower weight index first
struct NextLess {
  bool operator()(const Next& a, const Next& b) const {
    if (a.score != b.score) return a.score < b.score;
    return a.weight > b.weight;
  }
};

}  // namespace

extern "C" {

bs_status bs_plan_order(int n_weights, const int* n_blocks, const double* scores, int score_stride,
                        bs_order_kind kind, const double* draws, int* out_weight, int* out_block) {
  if (n_weights <= 0 || n_blocks == nullptr || out_weight == nullptr || out_block == nullptr)
    return BS_ERR_INVALID_ARG;
  long long total = 0;
  int levels = 0;
  for (int w = 0; w < n_weights; ++w) {
    if (n_blocks[w] < 0) return BS_ERR_INVALID_ARG;
    total += n_blocks[w];
    levels = std::max(levels, n_blocks[w]);
  }
  if (total > (1ll << 30)) return BS_ERR_INVALID_ARG;
  std::vector<int> next(n_weights, 0);
  long long t = 0;
  auto emit = [&](int w) {
    out_weight[t] = w;
    out_block[t] = next[w]++;
    ++t;
  };
  switch (kind) {
    case BS_ORDER_GREEDY: {
      if (scores == nullptr || score_stride < levels) return BS_ERR_INVALID_ARG;
      std::priority_queue<Next, std::vector<Next>, NextLess> heap;
      for (int w = 0; w < n_weights; ++w)
        if (n_blocks[w] > 0) heap.push({scores[static_cast<size_t>(w) * score_stride], w});
      while (!heap.empty()) {
        const int w = heap.top().weight;
        heap.pop();
        emit(w);
        if (next[w] < n_blocks[w]) heap.push({scores[static_cast<size_t>(w) * score_stride + next[w]], w});
      }
      break;
    }
    case BS_ORDER_AVERAGE:
      for (int i = 0; i < levels; ++i)
        for (int w = 0; w < n_weights; ++w)
          if (i < n_blocks[w]) emit(w);
      break;
    case BS_ORDER_RANDOM: {
      if (draws == nullptr) return BS_ERR_INVALID_ARG;
      std::vector<int> live;
      for (int w = 0; w < n_weights; ++w)
        if (n_blocks[w] > 0) live.push_back(w);
      while (!live.empty()) {
        const double u = draws[t];
        if (!(u >= 0.0 && u < 1.0)) return BS_ERR_INVALID_ARG;
        const size_t pick = std::min(static_cast<size_t>(u * static_cast<double>(live.size())), live.size() - 1);
        const int w = live[pick];
        emit(w);
        if (next[w] == n_blocks[w]) live.erase(live.begin() + static_cast<long>(pick));
      }
      break;
    }
    default:
      return BS_ERR_INVALID_ARG;
  }
  return BS_OK;
}

bs_status bs_plan_budget(long long n_steps, const int* order_weight, int n_weights, const unsigned long long* block_bytes,
                         unsigned long long budget_bytes, int* out_loaded) {
  if (n_steps < 0 || n_weights <= 0 || block_bytes == nullptr || out_loaded == nullptr ||
      (n_steps > 0 && order_weight == nullptr))
    return BS_ERR_INVALID_ARG;
  std::fill(out_loaded, out_loaded + n_weights, 0);
  unsigned long long used = 0;
  for (long long t = 0; t < n_steps; ++t) {
    const int w = order_weight[t];
    if (w < 0 || w >= n_weights) return BS_ERR_INVALID_ARG;
    if (block_bytes[w] > budget_bytes - used) break;   // the longest prefix that fits
    used += block_bytes[w];
    out_loaded[w] += 1;
  }
  return BS_OK;
}

}  // extern "C"
