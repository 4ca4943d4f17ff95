// Host round planner and index tables for tree-packed chunkwise KDA.
//
// HARTS (abstract; Figure 2): a planner of linear cost reaches the minimum
// number of sequential packed linear-attention calls.  Model: chunk grids
// aligned to absolute trajectory positions; a node either continues its
// parent's sequence or starts its own at b_v = floor(s_v / C) * C from the
// boundary state after token b_v - 1 (held by its anchor a(v)), replaying
// positions b_v .. s_v - 1 without outputs, one round after the anchor's
// round (round 1 if b_v = 0).  Each internal node continues exactly one
// child, so every sequence is a chain ending at a leaf.
//
// Dynamic program (both values of e in {0, 1} per node, children via their
// top-2 "independent" costs, so O(children) per node):
//   delta_c(e) = 1 if the parent v holds token b_c - 1 (s_v < b_c), else e
//   H(v, e)    = min_{c*} max(H(c*, delta_c*(e)), max_{c != c*} delta_c(e) + H(c, 0))
// Ties: smaller H, then larger replay saved (s_c - b_c), then smaller id.
//
// Two ablation modes reuse everything else (HARTS Figure 4 "Node-wise LA", Figure 5 "No-replay"):
//   node-wise: no node continues its parent; every node is a sequence of its own that starts at
//     b_v from its anchor's boundary state (with the same bounded replay), one round after the
//     anchor's round, so the rounds equal the anchor depth;
//   no replay: a side sequence starts exactly at its fork point s_v from the state after token
//     s_v - 1 (held by the parent), so b_v = s_v and nothing is replayed; the producing sequence
//     cuts a chunk at s_v to export that state mid-grid, and the side sequence's own chunk grid
//     starts at s_v.  The same dynamic program then yields the fewest rounds under that rule.
#include <algorithm>
#include <climits>
#include <cstring>
#include <map>
#include <tuple>

#include "plan.h"

namespace tpc {

std::string build_plan(const int32_t* parent, const int32_t* length, int32_t n, int32_t C, Plan& P, int mode,
                       int32_t n_ext, const int32_t* ext_node, const int64_t* ext_pos) {
  if (n <= 0) return "tree has no nodes";
  if (C != 16 && C != 32 && C != 64) return "chunk size must be 16, 32 or 64";
  if (mode != kPlanMinRounds && mode != kPlanNodewise && mode != kPlanNoReplay) return "unknown plan mode";
  P = Plan();
  P.C = C;
  P.mode = mode;
  P.n = n;
  P.parent.assign(parent, parent + n);
  P.length.assign(length, length + n);
  int64_t total = 0;
  for (int32_t i = 0; i < n; ++i) {
    if (parent[i] != -1 && (parent[i] < 0 || parent[i] >= i))
      return "node " + std::to_string(i) + ": parent must be -1 or a smaller id";
    if (length[i] < 1) return "node " + std::to_string(i) + ": zero-length segment";
    total += length[i];
  }
  if (total >= (int64_t(1) << 31) - 1) return "too many tokens for int32 row indices";
  P.n_unique = total;

  // children lists (CSR, increasing id)
  std::vector<int32_t> nch(n, 0), ch_begin(n + 1, 0), ch(n);
  for (int32_t i = 0; i < n; ++i)
    if (parent[i] >= 0) nch[parent[i]]++;
  for (int32_t i = 0; i < n; ++i) ch_begin[i + 1] = ch_begin[i] + nch[i];
  {
    std::vector<int32_t> fill(ch_begin.begin(), ch_begin.end() - 1);
    for (int32_t i = 0; i < n; ++i)
      if (parent[i] >= 0) ch[fill[parent[i]]++] = i;
  }

  // positions, aligned starts, anchors
  P.s.assign(n, 0);
  P.b.assign(n, 0);
  P.anchor.assign(n, -1);
  for (int32_t v = 0; v < n; ++v) {
    int32_t p = parent[v];
    P.s[v] = p < 0 ? 0 : P.s[p] + length[p];
    P.b[v] = mode == kPlanNoReplay ? P.s[v] : (P.s[v] / C) * C;
    if (P.b[v] > 0) {
      int32_t u = p;
      while (P.s[u] > P.b[v] - 1) u = parent[u];
      P.anchor[v] = u;
    }
  }
  if (P.s.empty()) return "internal";
  // external exports (sharing windows): the state after token pos - 1 of node u's path, u holding it
  if (n_ext < 0 || (n_ext > 0 && (!ext_node || !ext_pos))) return "exports: count or arrays invalid";
  for (int32_t e = 0; e < n_ext; ++e) {
    const int32_t u = ext_node[e];
    const int64_t b = ext_pos[e];
    if (u < 0 || u >= n) return "export " + std::to_string(e) + ": node out of range";
    if (b % C != 0 || b <= P.s[u] || b > P.s[u] + length[u])
      return "export " + std::to_string(e) + ": position must be a multiple of the chunk inside node " +
             std::to_string(u) + " (s < pos <= s + length)";
  }
  for (int32_t v = 0; v < n; ++v)
    if (P.s[v] + length[v] >= (int64_t(1) << 31)) return "trajectory longer than 2^31 tokens";

  // bottom-up DP (node-wise plans continue nothing: choice stays -1)
  std::vector<int64_t> H(2 * n, 0);
  std::vector<int32_t> choice(2 * n, -1);
  for (int32_t v = n - 1; v >= 0; --v) {
    if (nch[v] == 0 || mode == kPlanNodewise) continue;
    for (int e = 0; e < 2; ++e) {
      // top-2 of the independent cost y_c = delta_c(e) + H(c, 0)
      int64_t m1 = -1, m2 = -1;
      int32_t a1 = -1;
      for (int32_t j = ch_begin[v]; j < ch_begin[v + 1]; ++j) {
        int32_t c = ch[j];
        int64_t d = (P.s[v] < P.b[c]) ? 1 : e;
        int64_t y = d + H[2 * c + 0];
        if (y > m1) { m2 = m1; m1 = y; a1 = c; }
        else if (y > m2) { m2 = y; }
      }
      int64_t best_h = 0, best_save = 0;
      int32_t best_c = -1;
      for (int32_t j = ch_begin[v]; j < ch_begin[v + 1]; ++j) {
        int32_t c = ch[j];
        int64_t d = (P.s[v] < P.b[c]) ? 1 : e;
        int64_t x = H[2 * c + d];
        int64_t others = (c == a1) ? m2 : m1;  // -1 when there is no other child
        int64_t h = std::max(x, others);
        int64_t save = P.s[c] - P.b[c];
        if (best_c < 0 || h < best_h || (h == best_h && (save > best_save || (save == best_save && c < best_c)))) {
          best_h = h; best_save = save; best_c = c;
        }
      }
      H[2 * v + e] = best_h;
      choice[2 * v + e] = best_c;
    }
  }

  // top-down rounds
  P.round.assign(n, 0);
  P.is_cont.assign(n, 0);
  P.cont_child.assign(n, -1);
  std::vector<int32_t> ee(n, 0);
  for (int32_t v = 0; v < n; ++v) {
    if (parent[v] < 0) { P.round[v] = 1; ee[v] = 0; P.roots.push_back(v); }
    if (mode == kPlanNodewise) {  // one sequence per node, one round after its anchor's
      if (parent[v] >= 0) P.round[v] = P.b[v] == 0 ? 1 : P.round[P.anchor[v]] + 1;
      continue;
    }
    if (nch[v] == 0) continue;
    int32_t cs = choice[2 * v + ee[v]];
    P.cont_child[v] = cs;
    for (int32_t j = ch_begin[v]; j < ch_begin[v + 1]; ++j) {
      int32_t c = ch[j];
      int32_t d = (P.s[v] < P.b[c]) ? 1 : ee[v];
      if (c == cs) { P.round[c] = P.round[v]; ee[c] = d; P.is_cont[c] = 1; }
      else { P.round[c] = P.round[v] + d; ee[c] = 0; }
    }
  }
  P.n_rounds = 0;
  for (int32_t v = 0; v < n; ++v) P.n_rounds = std::max(P.n_rounds, P.round[v]);

  // compact layout: DFS preorder, continuation child first, then others by id
  P.row_offset.assign(n, 0);
  {
    int64_t nxt = 0;
    std::vector<int32_t> stack(P.roots.rbegin(), P.roots.rend());
    while (!stack.empty()) {
      int32_t v = stack.back();
      stack.pop_back();
      P.row_offset[v] = nxt;
      nxt += length[v];
      for (int32_t j = ch_begin[v + 1] - 1; j >= ch_begin[v]; --j)
        if (ch[j] != P.cont_child[v]) stack.push_back(ch[j]);
      if (P.cont_child[v] >= 0) stack.push_back(P.cont_child[v]);
    }
  }

  // occurrences, leaves, ordinals
  P.occurrence.assign(n, 0);
  for (int32_t v = n - 1; v >= 0; --v) {
    if (nch[v] == 0) P.occurrence[v] = 1;
    if (parent[v] >= 0) P.occurrence[parent[v]] += P.occurrence[v];
  }
  P.leaf_ordinal.assign(n, -1);
  P.root_ordinal.assign(n, -1);
  for (int32_t v = 0; v < n; ++v)
    if (nch[v] == 0) { P.leaf_ordinal[v] = (int32_t)P.leaves.size(); P.leaves.push_back(v); }
  for (size_t i = 0; i < P.roots.size(); ++i) P.root_ordinal[P.roots[i]] = (int32_t)i;
  std::vector<int32_t> root_of(n);
  for (int32_t v = 0; v < n; ++v) root_of[v] = parent[v] < 0 ? v : root_of[parent[v]];

  // sequences, ordered by (round, head id)
  std::vector<int32_t> heads;
  for (int32_t v = 0; v < n; ++v)
    if (parent[v] < 0 || !P.is_cont[v]) heads.push_back(v);
  std::stable_sort(heads.begin(), heads.end(), [&](int32_t a, int32_t b) { return P.round[a] < P.round[b]; });
  P.replay_start.assign(n, -1);
  P.replay_len.assign(n, -1);
  std::vector<int32_t> seq_of(n, -1);
  std::vector<int32_t> seq_leaf;
  for (size_t si = 0; si < heads.size(); ++si) {
    int32_t h = heads[si];
    int32_t u = h;
    seq_of[u] = (int32_t)si;
    while (P.cont_child[u] >= 0) { u = P.cont_child[u]; seq_of[u] = (int32_t)si; }
    SeqRec r{};
    r.head = h;
    r.round = P.round[h];
    r.start_pos = parent[h] < 0 ? 0 : (int32_t)P.b[h];
    r.n_replay = (int32_t)(P.s[h] - r.start_pos);
    r.leaf = P.leaf_ordinal[u];
    r.import_id = -(P.root_ordinal[root_of[h]] + 1);
    P.replay_start[h] = r.start_pos;
    P.replay_len[h] = r.n_replay;
    P.seqs.push_back(r);
    seq_leaf.push_back(u);
  }

  // slots: distinct (anchor, b) over heads with b > 0, and the external exports
  std::map<std::pair<int32_t, int64_t>, std::vector<int32_t>> keyset;
  for (size_t si = 0; si < P.seqs.size(); ++si) {
    int32_t h = P.seqs[si].head;
    if (parent[h] >= 0 && P.b[h] > 0) keyset[{P.anchor[h], P.b[h]}].push_back((int32_t)si);
  }
  for (int32_t e = 0; e < n_ext; ++e) keyset[{ext_node[e], ext_pos[e]}];  // (no in-tree consumer needed)
  std::vector<std::tuple<int32_t, int32_t, int64_t, int32_t>> skeys;  // (round, producer seq, b, anchor)
  for (auto& kv : keyset)
    skeys.emplace_back(P.round[kv.first.first], seq_of[kv.first.first], kv.first.second, kv.first.first);
  std::sort(skeys.begin(), skeys.end());
  std::map<std::pair<int32_t, int64_t>, int32_t> slot_at;  // (producer seq, b) -> slot
  for (auto& t : skeys) {
    int32_t an = std::get<3>(t);
    int64_t bb = std::get<2>(t);
    auto& cons = keyset[{an, bb}];
    std::sort(cons.begin(), cons.end(), [&](int32_t a, int32_t b) { return P.seqs[a].head < P.seqs[b].head; });
    SlotRec sr{};
    sr.producer_seq = seq_of[an];
    sr.export_chunk = -1;
    sr.cons_begin = (int32_t)P.slot_cons.size();
    sr.n_cons = (int32_t)cons.size();
    int32_t sid = (int32_t)P.slots.size();
    for (int32_t c : cons) { P.slot_cons.push_back(c); P.seqs[c].import_id = sid; }
    // external consumers after the in-tree ones: pseudo-sequence ids n_seqs + e, whose start-state
    // gradients the caller provides (tpc_kda_backward_window)
    for (int32_t e = 0; e < n_ext; ++e)
      if (ext_node[e] == an && ext_pos[e] == bb) {
        P.slot_cons.push_back((int32_t)P.seqs.size() + e);
        sr.n_cons++;
      }
    slot_at[{sr.producer_seq, bb}] = sid;
    P.slots.push_back(sr);
  }
  P.ext_slot.assign(n_ext, -1);
  for (int32_t e = 0; e < n_ext; ++e) {
    const int32_t pseudo = (int32_t)P.seqs.size() + e;
    for (size_t sid = 0; sid < P.slots.size(); ++sid)
      for (int32_t m = 0; m < P.slots[sid].n_cons; ++m)
        if (P.slot_cons[P.slots[sid].cons_begin + m] == pseudo) P.ext_slot[e] = (int32_t)sid;
  }

  // root consumers (sequences reading an initial state), by head id
  P.root_cons_begin.assign(P.roots.size() + 1, 0);
  {
    std::vector<std::vector<int32_t>> rc(P.roots.size());
    for (size_t si = 0; si < P.seqs.size(); ++si)
      if (P.seqs[si].import_id < 0) rc[-(P.seqs[si].import_id + 1)].push_back((int32_t)si);
    for (size_t r = 0; r < rc.size(); ++r) {
      std::sort(rc[r].begin(), rc[r].end(), [&](int32_t a, int32_t b) { return P.seqs[a].head < P.seqs[b].head; });
      P.root_cons_begin[r + 1] = P.root_cons_begin[r] + (int32_t)rc[r].size();
      for (int32_t s : rc[r]) P.root_cons.push_back(s);
    }
  }

  // chunks and replay rows
  P.replay_total = 0;
  P.round_seq_begin.assign(P.n_rounds + 1, 0);
  P.round_chunk_begin.assign(P.n_rounds + 1, 0);
  for (size_t si = 0; si < P.seqs.size(); ++si) {
    SeqRec& r = P.seqs[si];
    int32_t h = r.head, leaf = seq_leaf[si];
    int64_t end = P.s[leaf] + length[leaf];
    int64_t s_h = P.s[h];
    r.chunk_begin = (int32_t)P.chunks.size();
    int32_t replay_base = (int32_t)P.replay_rows.size();
    // replayed rows: positions start .. s_h - 1 along h's path
    for (int64_t pos = r.start_pos; pos < s_h; ++pos) {
      int32_t u = parent[h];
      while (P.s[u] > pos) u = parent[u];
      P.replay_rows.push_back((int32_t)(P.row_offset[u] + (pos - P.s[u])));
    }
    // chunk boundaries: the sequence's grid (multiples of C from its start) and every position at
    // which it exports a boundary state (grid points, except in no-replay plans)
    std::vector<int64_t> cuts;
    for (auto it = slot_at.lower_bound({(int32_t)si, INT64_MIN}); it != slot_at.end() && it->first.first == (int32_t)si;
         ++it)
      cuts.push_back(it->first.second);
    size_t next_cut = 0;
    int32_t idx = 0;
    for (int64_t p0 = r.start_pos; p0 < end; ++idx) {
      while (next_cut < cuts.size() && cuts[next_cut] <= p0) ++next_cut;
      int64_t p1 = std::min<int64_t>(r.start_pos + ((p0 - r.start_pos) / C + 1) * C, end);
      if (next_cut < cuts.size()) p1 = std::min<int64_t>(p1, cuts[next_cut]);
      ChunkRec c{};
      c.seq = (int32_t)si;
      c.pos0 = (int32_t)p0;
      c.n_rows = (int32_t)(p1 - p0);
      c.n_replay = (int32_t)std::max<int64_t>(0, std::min<int64_t>(s_h, p1) - p0);
      int64_t first_own = std::max<int64_t>(p0, s_h);
      c.row_start = (int32_t)(P.row_offset[h] + (first_own - s_h));
      c.replay_base = replay_base;  // replayed rows (< C of them) all fall in the first chunk
      auto it = slot_at.find({(int32_t)si, p1});
      c.export_slot = -1;
      if (it != slot_at.end()) {
        c.export_slot = it->second;
        P.slots[it->second].export_chunk = (int32_t)P.chunks.size();
      }
      c.idx_in_seq = idx;
      P.chunks.push_back(c);
      p0 = p1;
    }
    r.n_chunks = idx;
    P.max_seq_chunks = std::max(P.max_seq_chunks, idx);
    P.replay_total += r.n_replay;
    P.round_seq_begin[r.round] = (int32_t)si + 1;
    P.round_chunk_begin[r.round] = (int32_t)P.chunks.size();
  }
  for (int32_t i = 1; i <= P.n_rounds; ++i) {
    P.round_seq_begin[i] = std::max(P.round_seq_begin[i], P.round_seq_begin[i - 1]);
    P.round_chunk_begin[i] = std::max(P.round_chunk_begin[i], P.round_chunk_begin[i - 1]);
  }
  for (auto& sr : P.slots)
    if (sr.export_chunk < 0) return "internal: slot without exporting chunk";

  // replay targets: rows replayed somewhere; their partials in ascending replay index
  P.row_tgt.assign((size_t)P.n_unique, -1);
  {
    std::vector<std::pair<int32_t, int32_t>> rp;
    for (size_t i = 0; i < P.replay_rows.size(); ++i) rp.emplace_back(P.replay_rows[i], (int32_t)i);
    std::sort(rp.begin(), rp.end());
    P.tgt_begin.push_back(0);
    for (size_t i = 0; i < rp.size(); ++i) {
      if (i == 0 || rp[i].first != rp[i - 1].first) {
        if (i) P.tgt_begin.push_back((int32_t)P.tgt_parts.size());
        P.row_tgt[rp[i].first] = (int32_t)P.tgt_row.size();
        P.tgt_row.push_back(rp[i].first);
      }
      P.tgt_parts.push_back(rp[i].second);
    }
    if (!rp.empty()) P.tgt_begin.push_back((int32_t)P.tgt_parts.size());
  }

  // attention tables: subtree ends, ancestor row ranges (merged when contiguous), query / key tiles
  {
    std::vector<int64_t> sub(n, 0);
    for (int32_t v = n - 1; v >= 0; --v) {
      sub[v] += length[v];
      if (parent[v] >= 0) sub[parent[v]] += sub[v];
    }
    std::vector<std::vector<std::pair<int32_t, int32_t>>> rg(n);
    for (int32_t v = 0; v < n; ++v) {
      const int32_t p = parent[v];
      if (p >= 0) {
        rg[v] = rg[p];
        const int32_t a = (int32_t)P.row_offset[p], b = a + length[p];
        if (!rg[v].empty() && rg[v].back().second == a) rg[v].back().second = b;
        else rg[v].push_back({a, b});
      }
    }
    P.attn_nodes.resize(n + 1);
    for (int32_t v = 0; v < n; ++v) {
      AttnNode an{};
      an.row_offset = (int32_t)P.row_offset[v];
      an.length = length[v];
      an.subtree_end = (int32_t)(P.row_offset[v] + sub[v]);
      an.range_begin = (int32_t)(P.attn_ranges.size() / 2);
      an.pos0 = (int32_t)P.s[v];
      for (auto& r : rg[v]) { P.attn_ranges.push_back(r.first); P.attn_ranges.push_back(r.second); }
      P.attn_nodes[v] = an;
      for (int32_t r = 0; r < length[v]; r += 128)
        P.attn_qtiles.push_back({v, (int32_t)P.row_offset[v] + r, std::min(128, length[v] - r), 0});
      for (int32_t r = 0; r < length[v]; r += 128)
        P.attn_ktiles.push_back({v, (int32_t)P.row_offset[v] + r, std::min(128, length[v] - r), 0});
    }
    P.attn_nodes[n] = AttnNode{0, 0, 0, (int32_t)(P.attn_ranges.size() / 2), 0, {0, 0, 0}};
    // query tiles by decreasing work (the keys they read: the node's ancestor rows and its own rows up
    // to the tile's end), so that the longest forward and dQ blocks start first; ties keep node order
    std::stable_sort(P.attn_qtiles.begin(), P.attn_qtiles.end(), [&](const AttnTile& a, const AttnTile& b) {
      const AttnNode &na = P.attn_nodes[a.node], &nb = P.attn_nodes[b.node];
      return na.pos0 + (a.row - na.row_offset) + a.n > nb.pos0 + (b.row - nb.row_offset) + b.n;
    });
    // key tiles by decreasing work (the query rows that read them: the subtree from the tile on), so
    // that the dK / dV blocks with the longest query ranges start first; ties keep node order
    std::stable_sort(P.attn_ktiles.begin(), P.attn_ktiles.end(), [&](const AttnTile& a, const AttnTile& b) {
      return P.attn_nodes[a.node].subtree_end - a.row > P.attn_nodes[b.node].subtree_end - b.row;
    });
  }

  // expanded maps
  P.traj_offset.push_back(0);
  for (int32_t leaf : P.leaves) {
    std::vector<int32_t> path;
    for (int32_t u = leaf; u >= 0; u = parent[u]) path.push_back(u);
    for (auto it = path.rbegin(); it != path.rend(); ++it)
      for (int32_t j = 0; j < length[*it]; ++j) {
        P.exp_rows64.push_back(P.row_offset[*it] + j);
      }
    P.traj_offset.push_back((int64_t)P.exp_rows64.size());
  }
  P.n_expanded = (int64_t)P.exp_rows64.size();
  if (P.n_expanded >= (int64_t(1) << 31)) return "expanded size exceeds int32";
  P.exp_rows.resize(P.exp_rows64.size());
  for (size_t i = 0; i < P.exp_rows64.size(); ++i) P.exp_rows[i] = (int32_t)P.exp_rows64[i];
  P.occ_begin.assign((size_t)P.n_unique + 1, 0);
  for (int32_t r : P.exp_rows) P.occ_begin[r + 1]++;
  for (int64_t r = 0; r < P.n_unique; ++r) P.occ_begin[r + 1] += P.occ_begin[r];
  P.occ_list.assign(P.exp_rows.size(), 0);
  {
    std::vector<int32_t> fill(P.occ_begin.begin(), P.occ_begin.end() - 1);
    for (size_t j = 0; j < P.exp_rows.size(); ++j) P.occ_list[fill[P.exp_rows[j]]++] = (int32_t)j;
  }
  return "";
}

namespace {
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}

size_t device_layout(const Plan& p, std::vector<size_t>& off) {
  const size_t sizes[] = {
      p.seqs.size() * sizeof(SeqRec), p.chunks.size() * sizeof(ChunkRec), p.slots.size() * sizeof(SlotRec),
      p.slot_cons.size() * 4, p.root_cons_begin.size() * 4, p.root_cons.size() * 4, p.replay_rows.size() * 4,
      p.tgt_row.size() * 4, p.tgt_begin.size() * 4, p.tgt_parts.size() * 4, p.row_tgt.size() * 4,
      p.exp_rows.size() * 4, p.occ_begin.size() * 4, p.occ_list.size() * 4, p.occurrence.size() * 0 + (size_t)p.n_unique * 4,
      p.attn_nodes.size() * sizeof(AttnNode), p.attn_ranges.size() * 4, p.attn_qtiles.size() * sizeof(AttnTile),
      p.attn_ktiles.size() * sizeof(AttnTile)};
  off.clear();
  size_t o = 0;
  for (size_t s : sizes) { off.push_back(o); o += align256(s); }
  off.push_back(o);
  return o;
}

void pack_device_blob(const Plan& p, const std::vector<size_t>& off, std::vector<uint8_t>& blob) {
  blob.assign(off.back(), 0);
  auto put = [&](int i, const void* src, size_t bytes) { if (bytes) std::memcpy(blob.data() + off[i], src, bytes); };
  put(0, p.seqs.data(), p.seqs.size() * sizeof(SeqRec));
  put(1, p.chunks.data(), p.chunks.size() * sizeof(ChunkRec));
  put(2, p.slots.data(), p.slots.size() * sizeof(SlotRec));
  put(3, p.slot_cons.data(), p.slot_cons.size() * 4);
  put(4, p.root_cons_begin.data(), p.root_cons_begin.size() * 4);
  put(5, p.root_cons.data(), p.root_cons.size() * 4);
  put(6, p.replay_rows.data(), p.replay_rows.size() * 4);
  put(7, p.tgt_row.data(), p.tgt_row.size() * 4);
  put(8, p.tgt_begin.data(), p.tgt_begin.size() * 4);
  put(9, p.tgt_parts.data(), p.tgt_parts.size() * 4);
  put(10, p.row_tgt.data(), p.row_tgt.size() * 4);
  put(11, p.exp_rows.data(), p.exp_rows.size() * 4);
  put(12, p.occ_begin.data(), p.occ_begin.size() * 4);
  put(13, p.occ_list.data(), p.occ_list.size() * 4);
  // occurrence count per compact row
  std::vector<int32_t> cnt((size_t)p.n_unique);
  for (int64_t r = 0; r < p.n_unique; ++r) cnt[r] = p.occ_begin[r + 1] - p.occ_begin[r];
  put(14, cnt.data(), cnt.size() * 4);
  put(15, p.attn_nodes.data(), p.attn_nodes.size() * sizeof(AttnNode));
  put(16, p.attn_ranges.data(), p.attn_ranges.size() * 4);
  put(17, p.attn_qtiles.data(), p.attn_qtiles.size() * sizeof(AttnTile));
  put(18, p.attn_ktiles.data(), p.attn_ktiles.size() * sizeof(AttnTile));
}

DevTables device_view(const Plan& p, void* base, const std::vector<size_t>& off) {
  (void)p;
  auto at = [&](int i) { return static_cast<const void*>(static_cast<const uint8_t*>(base) + off[i]); };
  DevTables d;
  d.seqs = (const SeqRec*)at(0);
  d.chunks = (const ChunkRec*)at(1);
  d.slots = (const SlotRec*)at(2);
  d.slot_cons = (const int32_t*)at(3);
  d.root_cons_begin = (const int32_t*)at(4);
  d.root_cons = (const int32_t*)at(5);
  d.replay_rows = (const int32_t*)at(6);
  d.tgt_row = (const int32_t*)at(7);
  d.tgt_begin = (const int32_t*)at(8);
  d.tgt_parts = (const int32_t*)at(9);
  d.row_tgt = (const int32_t*)at(10);
  d.exp_rows = (const int32_t*)at(11);
  d.occ_begin = (const int32_t*)at(12);
  d.occ_list = (const int32_t*)at(13);
  d.occ_count = (const int32_t*)at(14);
  d.attn_nodes = (const AttnNode*)at(15);
  d.attn_ranges = (const RowRange*)at(16);
  d.attn_qtiles = (const AttnTile*)at(17);
  d.attn_ktiles = (const AttnTile*)at(18);
  return d;
}

}  // namespace tpc
