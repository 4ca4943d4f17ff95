// L1 microbatch planner: compression-oriented packing of many rollout trees under a budget of
// unique token rows per microbatch (HARTS abstract: a two-level planner first constructs
// compression-oriented microbatches; Figure 1(c): L1 forms microbatches; Table 4: L1 compression,
// balance and planning time; work is counted in unique non-replayed rows).  The pages give no
// algorithm; the one implemented (contract in include/tpc.h):
//   1. trees in increasing root id, the leaves of a tree in depth-first order (children by id);
//   2. a tree that fits the budget is one piece; a larger one is cut along its depth-first leaf
//      order, a piece closing before the leaf whose new path tokens would exceed the budget;
//   3. pieces by decreasing cost (ties: smaller first leaf id) go first-fit into microbatches.
// Linear in nodes + leaves for steps 1-2 (each node is marked once per piece) and O(pieces x
// microbatches) for the first-fit pass.
#include <algorithm>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/tpc.h"
#include "abi_internal.h"

namespace {

using tpc_abi::fail;

struct Piece {
  int64_t cost;
  std::vector<int32_t> leaves;
};

}  // namespace

extern "C" int tpc_microbatch_plan(const int32_t* parent, const int32_t* length, int32_t n, int64_t budget,
                                   int32_t* leaf_mb, int64_t* mb_unique, int64_t* mb_expanded, int32_t max_mb,
                                   tpc_microbatch_stats* stats) {
  if (!parent || !length || !leaf_mb || !stats) return fail(TPC_ERR_NULL, "parent, length, leaf_mb and stats are required");
  if (n <= 0) return fail(TPC_ERR_INVALID_TREE, "tree has no nodes");
  if (budget < 1) return fail(TPC_ERR_BAD_SHAPE, "budget must be >= 1");
  for (int32_t i = 0; i < n; ++i) {
    if (parent[i] != -1 && (parent[i] < 0 || parent[i] >= i))
      return fail(TPC_ERR_INVALID_TREE, "node " + std::to_string(i) + ": parent must be -1 or a smaller id");
    if (length[i] < 1) return fail(TPC_ERR_INVALID_TREE, "node " + std::to_string(i) + ": zero-length segment");
  }
  std::vector<int32_t> nch(n, 0), cb(n + 1, 0), ch(n);
  for (int32_t i = 0; i < n; ++i)
    if (parent[i] >= 0) nch[parent[i]]++;
  for (int32_t i = 0; i < n; ++i) cb[i + 1] = cb[i] + nch[i];
  {
    std::vector<int32_t> fill(cb.begin(), cb.end() - 1);
    for (int32_t i = 0; i < n; ++i)
      if (parent[i] >= 0) ch[fill[parent[i]]++] = i;
  }
  // path tokens (expanded length of the trajectory ending at a node) and subtree unique tokens
  std::vector<int64_t> depth_tok(n), sub(n, 0);
  for (int32_t v = 0; v < n; ++v) depth_tok[v] = (parent[v] < 0 ? 0 : depth_tok[parent[v]]) + length[v];
  for (int32_t v = n - 1; v >= 0; --v) {
    sub[v] += length[v];
    if (parent[v] >= 0) sub[parent[v]] += sub[v];
  }
  std::vector<int32_t> leaf_ord(n, -1);
  int32_t n_leaves = 0;
  for (int32_t v = 0; v < n; ++v)
    if (nch[v] == 0) leaf_ord[v] = n_leaves++;

  // pieces
  std::vector<Piece> pieces;
  std::vector<int32_t> mark(n, -1);  // piece id that already holds the node
  for (int32_t r = 0; r < n; ++r) {
    if (parent[r] >= 0) continue;
    std::vector<int32_t> leaves, stack{r};
    while (!stack.empty()) {
      int32_t v = stack.back();
      stack.pop_back();
      if (nch[v] == 0) leaves.push_back(v);
      for (int32_t j = cb[v + 1] - 1; j >= cb[v]; --j) stack.push_back(ch[j]);
    }
    if (sub[r] <= budget) {
      pieces.push_back({sub[r], leaves});
      continue;
    }
    Piece cur{0, {}};
    int32_t pid = (int32_t)pieces.size();
    for (int32_t l : leaves) {
      // new tokens: the path from the leaf up to (excluding) the deepest node the piece holds
      int64_t fresh = 0;
      for (int32_t u = l; u >= 0 && mark[u] != pid; u = parent[u]) fresh += length[u];
      if (!cur.leaves.empty() && cur.cost + fresh > budget) {
        pieces.push_back(cur);
        cur = Piece{0, {}};
        pid = (int32_t)pieces.size();
        fresh = depth_tok[l];
      }
      for (int32_t u = l; u >= 0 && mark[u] != pid; u = parent[u]) mark[u] = pid;
      cur.leaves.push_back(l);
      cur.cost += fresh;
    }
    pieces.push_back(cur);
  }
  // first fit, largest pieces first
  std::vector<int32_t> order(pieces.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = (int32_t)i;
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    if (pieces[a].cost != pieces[b].cost) return pieces[a].cost > pieces[b].cost;
    return pieces[a].leaves.front() < pieces[b].leaves.front();
  });
  std::vector<int64_t> load;
  std::vector<std::vector<int32_t>> bins;
  for (int32_t pi : order) {
    const Piece& p = pieces[pi];
    size_t b = 0;
    while (b < load.size() && load[b] + p.cost > budget) ++b;
    if (b == load.size()) { load.push_back(0); bins.emplace_back(); }
    load[b] += p.cost;
    bins[b].insert(bins[b].end(), p.leaves.begin(), p.leaves.end());
  }
  const int32_t nmb = (int32_t)bins.size();
  std::memset(stats, 0, sizeof(*stats));
  stats->n_microbatches = nmb;
  if (nmb > max_mb && (mb_unique || mb_expanded))
    return fail(TPC_ERR_BAD_SHAPE, "max_mb too small: the plan has " + std::to_string(nmb) + " microbatches");
  // per microbatch: unique tokens of the union of its paths, expanded tokens
  std::vector<int32_t> seen(n, -1);
  int64_t tu = 0, te = 0, mx = 0;
  for (int32_t m = 0; m < nmb; ++m) {
    int64_t u = 0, e = 0;
    for (int32_t l : bins[m]) {
      leaf_mb[leaf_ord[l]] = m;
      e += depth_tok[l];
      for (int32_t v = l; v >= 0 && seen[v] != m; v = parent[v]) {
        seen[v] = m;
        u += length[v];
      }
    }
    if (mb_unique) mb_unique[m] = u;
    if (mb_expanded) mb_expanded[m] = e;
    tu += u;
    te += e;
    mx = std::max(mx, u);
  }
  stats->unique_tokens = tu;
  stats->expanded_tokens = te;
  stats->max_unique = mx;
  stats->compression = (double)te / (double)tu;
  stats->balance = ((double)tu / nmb) / (double)mx;
  return TPC_OK;
}
