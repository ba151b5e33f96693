// plan.cu -- host-side split of the path's work over several GPUs.
//
// The pages describe no distributed step. The path shards without any
// exchange: every query row of a prefill, and every sequence of a decode
// batch, is an independent problem over caches the caller holds on every GPU.
// The causal prefix makes the cost of a row grow with its position, so a
// balanced split cannot be equal row counts. These functions assign whole
// units (prefill chunks, decode sequences) to workers with the longest-first
// greedy rule: units sorted by estimated cost, largest first (ties: lower
// unit first), each given to the currently least-loaded worker (ties: lower
// worker). The makespan is at most 4/3 of the optimum (Graham's bound for
// that rule), and in practice within one small unit of the mean.
//
// Cost of one query row that sees n keys, in BF16-flop equivalents (the FP8
// indexer runs at twice the BF16 rate):
//   indexer  2 * 128 * Hi * n / 2
//   MLA      2 * (576 + 512) * H * min(n, k)
// Host code only: no CUDA call, no device memory.
#include "dsa_internal.h"
#include "dsa.h"

#include <algorithm>
#include <cstdint>
#include <numeric>
#include <vector>

namespace {

double row_cost(long long n, int Hi, int H, int k) {
  return 128.0 * Hi * static_cast<double>(n) +
         2176.0 * H * static_cast<double>(std::min<long long>(n, k));
}

// Longest-first assignment; returns the units of `part`, ascending.
std::vector<int> assign(const std::vector<double>& cost, int parts, int part) {
  std::vector<int> order(cost.size());
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<double> load(parts, 0.0);
  std::vector<int> mine;
  for (int u : order) {
    const int w = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
    load[w] += cost[u];
    if (w == part) mine.push_back(u);
  }
  std::sort(mine.begin(), mine.end());
  return mine;
}

bool plan_args_ok(int parts, int part, const int32_t* out, int max_out, int k, int Hi, int H) {
  return parts >= 1 && parts <= 4096 && part >= 0 && part < parts && out && max_out >= 0 &&
         k > 0 && Hi >= 1 && H >= 1;
}

}  // namespace

int dsa_plan_prefill_chunks(int T, int S, int q_pos0, int Hi, int H, int k, int chunk, int parts,
                            int part, int32_t* first_rows, int max_chunks) {
  if (T < 0 || S <= 0 || q_pos0 < 0 || chunk <= 0 ||
      !plan_args_ok(parts, part, first_rows, max_chunks, k, Hi, H))
    return DSA_ERR_INVALID_ARG;
  const int nchunks = (T + chunk - 1) / chunk;
  std::vector<double> cost(nchunks, 0.0);
  for (int c = 0; c < nchunks; ++c) {
    const int n = std::min(chunk, T - c * chunk);
    for (int r = 0; r < n; ++r) {
      const long long pos = std::min<long long>(static_cast<long long>(q_pos0) + c * chunk + r,
                                                S - 1);
      cost[c] += row_cost(pos + 1, Hi, H, k);
    }
  }
  const std::vector<int> mine = assign(cost, parts, part);
  if (static_cast<int>(mine.size()) > max_chunks) return DSA_ERR_INVALID_ARG;
  for (size_t i = 0; i < mine.size(); ++i) first_rows[i] = mine[i] * chunk;
  return static_cast<int>(mine.size());
}

int dsa_plan_decode_sequences(const int32_t* seq_len, int B, int nq, int Hi, int H, int k,
                              int parts, int part, int32_t* seqs, int max_seqs) {
  if (!seq_len || B < 0 || nq < 1 || !plan_args_ok(parts, part, seqs, max_seqs, k, Hi, H))
    return DSA_ERR_INVALID_ARG;
  std::vector<double> cost(B, 0.0);
  for (int b = 0; b < B; ++b) {
    if (seq_len[b] < nq) return DSA_ERR_INVALID_ARG;
    for (int j = 0; j < nq; ++j)                 // query j sees seq_len - nq + j + 1 keys
      cost[b] += row_cost(static_cast<long long>(seq_len[b]) - nq + j + 1, Hi, H, k);
  }
  const std::vector<int> mine = assign(cost, parts, part);
  if (static_cast<int>(mine.size()) > max_seqs) return DSA_ERR_INVALID_ARG;
  for (size_t i = 0; i < mine.size(); ++i) seqs[i] = mine[i];
  return static_cast<int>(mine.size());
}
