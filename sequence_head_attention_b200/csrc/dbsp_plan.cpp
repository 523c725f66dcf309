// dbsp_plan.cpp -- host-side work partition of block-sparse attention over P sequence-parallel ranks.
//
// "db-SP: ... Sparsity-Aware Sequence Parallelism ..." (abstract) balances block-sparse attention over ranks
// at two levels, heads and blocks, and measures balance by a "sparse imbalance ratio"; the page gives
// neither the ratio's formula nor the partition algorithm.  This file's reading:
//   * a work unit is (head h, query-tile pair qp): the kernel's work item, 256 query rows of one head;
//   * its cost is the number of 128 x 128 tiles the mask keeps in its two query-tile rows (keys j <= i only
//     when causal), i.e. its tensor-core work;
//   * a rank's load is the sum of its units' costs, and the imbalance ratio is max load / mean load;
//   * level 1 (heads): heads whole, in decreasing total cost (ties: lower head first), each to the least
//     loaded rank (ties: lower rank);
//   * level 2 (blocks): while some unit of the most loaded rank has a cost c with 0 < c < (max load - min
//     load), move the one with 2c closest to that gap (ties: larger c, then lower head, then lower qp) to
//     the least loaded rank (ties between ranks: lower rank).  Each move lowers the sum of squared loads,
//     so this ends; it splits only the heads it has to.
// Everything here is plain host code on host arrays.
#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <vector>

#include "sp_internal.h"

namespace {

int argmax_load(const std::vector<long long>& load) {
  int r = 0;
  for (int i = 1; i < (int)load.size(); ++i)
    if (load[i] > load[r]) r = i;
  return r;
}

int argmin_load(const std::vector<long long>& load) {
  int r = 0;
  for (int i = 1; i < (int)load.size(); ++i)
    if (load[i] < load[r]) r = i;
  return r;
}

}  // namespace

extern "C" {

sp_status sp_dbsp_unit_costs(const uint8_t* block_mask, int H, int T, int causal, long long* cost) {
  if (H < 1 || T < 1 || !cost || (causal != 0 && causal != 1)) return SP_ERR_INVALID_ARG;
  if ((long long)H * T * T > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
  const int NP = (T + 1) / 2;
  for (int h = 0; h < H; ++h)
    for (int qp = 0; qp < NP; ++qp) {
      long long c = 0;
      for (int i = 2 * qp; i < 2 * qp + 2 && i < T; ++i) {
        const int jmax = causal ? i + 1 : T;  // exclusive
        if (!block_mask) {
          c += jmax;
          continue;
        }
        const uint8_t* row = block_mask + ((size_t)h * T + i) * T;
        for (int j = 0; j < jmax; ++j) c += row[j] != 0;
      }
      cost[(size_t)h * NP + qp] = c;
    }
  return SP_OK;
}

sp_status sp_dbsp_plan(const long long* cost, int H, int NP, int P, int* unit_rank, long long* rank_load,
                       double* imbalance) {
  if (!cost || !unit_rank || H < 1 || NP < 1 || P < 1 || P > SP_MAX_RANKS) return SP_ERR_INVALID_ARG;
  const size_t n_units = (size_t)H * NP;
  for (size_t u = 0; u < n_units; ++u)
    if (cost[u] < 0) return SP_ERR_INVALID_ARG;
  std::vector<long long> load(P, 0);
  // Level 1: whole heads, longest first, each to the least loaded rank.
  std::vector<long long> head_cost(H, 0);
  for (int h = 0; h < H; ++h)
    for (int qp = 0; qp < NP; ++qp) head_cost[h] += cost[(size_t)h * NP + qp];
  std::vector<int> order(H);
  for (int h = 0; h < H; ++h) order[h] = h;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return head_cost[a] > head_cost[b]; });
  for (int h : order) {
    const int r = argmin_load(load);
    for (int qp = 0; qp < NP; ++qp) unit_rank[(size_t)h * NP + qp] = r;
    load[r] += head_cost[h];
  }
  // Level 2: single units from the most to the least loaded rank while that lowers the spread.
  const long long max_moves = (long long)n_units * 4 + 16;  // a bound far above what the argument needs
  for (long long move = 0; move < max_moves; ++move) {
    const int rmax = argmax_load(load), rmin = argmin_load(load);
    const long long gap = load[rmax] - load[rmin];
    if (gap <= 1) break;
    long long best_c = -1, best_score = 0;
    size_t best_u = 0;
    for (size_t u = 0; u < n_units; ++u) {
      if (unit_rank[u] != rmax) continue;
      const long long c = cost[u];
      if (c <= 0 || c >= gap) continue;
      const long long score = std::llabs(2 * c - gap);
      if (best_c < 0 || score < best_score || (score == best_score && c > best_c)) {
        best_c = c;
        best_score = score;
        best_u = u;
      }
    }
    if (best_c < 0) break;
    unit_rank[best_u] = rmin;
    load[rmax] -= best_c;
    load[rmin] += best_c;
  }
  if (rank_load)
    for (int r = 0; r < P; ++r) rank_load[r] = load[r];
  if (imbalance) {
    long long total = 0, mx = 0;
    for (int r = 0; r < P; ++r) {
      total += load[r];
      mx = std::max(mx, load[r]);
    }
    *imbalance = total > 0 ? (double)mx * P / (double)total : 1.0;
  }
  return SP_OK;
}

sp_status sp_dbsp_rank_items(const long long* cost, const int* unit_rank, int B, int H, int NP, int rank,
                             int* items, int capacity, int* n_items) {
  if (!cost || !unit_rank || !n_items || B < 1 || H < 1 || NP < 1 || rank < 0 || capacity < 0)
    return SP_ERR_INVALID_ARG;
  if ((long long)B * H * NP > 0x7fffffffLL) return SP_ERR_INVALID_ARG;
  std::vector<int> units;
  for (int u = 0; u < H * NP; ++u)
    if (unit_rank[u] == rank) units.push_back(u);
  // longest first, so that the kernel's in-order claiming leaves the short units for the end
  std::stable_sort(units.begin(), units.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  const long long n = (long long)units.size() * B;
  *n_items = (int)n;
  if (n > capacity) return items ? SP_ERR_INVALID_ARG : SP_OK;  // size query with items == NULL
  if (!items) return SP_OK;
  int k = 0;
  for (int u : units)
    for (int b = 0; b < B; ++b) items[k++] = (b * H + u / NP) * NP + u % NP;
  return SP_OK;
}

}  // extern "C"
