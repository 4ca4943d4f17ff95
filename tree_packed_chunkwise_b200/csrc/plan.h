// Internal plan representation shared by the host planner and the kernels.
#pragma once
#include <cstdint>
#include <string>
#include <vector>

namespace tpc {

// One packed-call sequence (a continuation chain, HARTS Figure 2(a) thick edges).
struct SeqRec {
  int32_t chunk_begin;  // first chunk (chunks of a sequence are consecutive)
  int32_t n_chunks;
  int32_t import_id;    // >= 0: boundary-state slot; < 0: initial state of root ordinal -(id+1)
  int32_t leaf;         // leaf ordinal whose final state this sequence produces; -1 when the chain
                        // ends at an internal node (node-wise plans), which has no final state
  int32_t head;         // head node id
  int32_t round;        // 1-based
  int32_t start_pos;    // absolute position of the first (possibly replayed) row
  int32_t n_replay;     // replayed rows at the start (< chunk)
};

// One chunk of C consecutive positions of a sequence, aligned to multiples of C.
struct ChunkRec {
  int32_t seq;
  int32_t n_rows;       // <= C (the last chunk of a sequence may be short)
  int32_t n_replay;     // leading rows that are replays (first chunk only)
  int32_t row_start;    // compact row of the first own (non-replay) row; own rows are contiguous
  int32_t replay_base;  // index of the first replayed row in the replay tables
  int32_t export_slot;  // slot written with the state at the end of this chunk, or -1
  int32_t pos0;         // absolute position of the chunk's first row
  int32_t idx_in_seq;
};

// A boundary state at an aligned position, produced by one sequence, read by later ones.
struct SlotRec {
  int32_t producer_seq;
  int32_t export_chunk;
  int32_t cons_begin;   // into slot_cons
  int32_t n_cons;
};

// Tree-masked attention: a query in node v reads the rows of v's proper ancestors (a few
// contiguous ranges: one per chain on the path) and the earlier rows of v itself.
struct AttnNode {
  int32_t row_offset, length, subtree_end;  // subtree rows = [row_offset, subtree_end)
  int32_t range_begin;                      // ancestor ranges [range_begin, next node's range_begin)
  int32_t pos0;                             // trajectory position of the node's first token
  int32_t pad[3];
};
struct RowRange {
  int32_t start, end;
};
struct AttnTile {
  int32_t node, row, n, pad;  // n <= 128 query or key rows of one node
};

// Device view of the uploaded tables (all pointers into the caller's buffer).
struct DevTables {
  const SeqRec* seqs;
  const ChunkRec* chunks;
  const SlotRec* slots;
  const int32_t* slot_cons;        // consumer sequence ids, per slot, by head id
  const int32_t* root_cons_begin;  // [n_roots + 1]
  const int32_t* root_cons;        // sequences importing a root's initial state, by id
  const int32_t* replay_rows;      // compact row of each replayed row [R]
  const int32_t* tgt_row;          // rows that are replayed somewhere [n_tgt]
  const int32_t* tgt_begin;        // [n_tgt + 1] into tgt_parts
  const int32_t* tgt_parts;        // replay indices contributing to each target, ascending
  const int32_t* row_tgt;          // [N] target index or -1
  const int32_t* exp_rows;         // [n_expanded] compact row of each trajectory position
  const int32_t* occ_begin;        // [N + 1] occurrence CSR (trajectory order)
  const int32_t* occ_list;         // [n_expanded] expanded positions
  const int32_t* occ_count;        // [N]
  const AttnNode* attn_nodes;      // [n_nodes + 1] (last entry: range_begin sentinel)
  const RowRange* attn_ranges;     // ancestor row ranges [start, end)
  const AttnTile* attn_qtiles;
  const AttnTile* attn_ktiles;
};

// planner modes (tpc_plan_create_mode)
enum : int { kPlanMinRounds = 0, kPlanNodewise = 1, kPlanNoReplay = 2 };

struct Plan {
  int32_t C = 0, n = 0, mode = 0;
  std::vector<int32_t> parent, length;
  std::vector<int64_t> s, b;
  std::vector<int32_t> anchor, round, is_cont, cont_child, replay_start, replay_len, occurrence;
  std::vector<int64_t> row_offset;
  std::vector<int32_t> leaves, roots, root_ordinal, leaf_ordinal;
  int32_t n_rounds = 0;
  int64_t n_unique = 0, n_expanded = 0, replay_total = 0;
  int32_t max_seq_chunks = 0;

  std::vector<SeqRec> seqs;
  std::vector<ChunkRec> chunks;
  std::vector<SlotRec> slots;
  std::vector<int32_t> slot_cons, root_cons_begin, root_cons, replay_rows;
  std::vector<int32_t> tgt_row, tgt_begin, tgt_parts, row_tgt;
  std::vector<int32_t> exp_rows, occ_begin, occ_list;
  std::vector<int64_t> exp_rows64, traj_offset;
  std::vector<int32_t> round_seq_begin, round_chunk_begin;  // [n_rounds + 1], host only
  std::vector<int32_t> ext_slot;  // slot of each external export (its consumer id is n_seqs + e)
  std::vector<AttnNode> attn_nodes;
  std::vector<int32_t> attn_ranges;  // pairs
  std::vector<AttnTile> attn_qtiles, attn_ktiles;

  // device upload
  void* dev = nullptr;
  size_t dev_bytes = 0;
  DevTables dt{};
  std::vector<size_t> blob_offsets;
};

// Builds the plan; returns an empty string or an error message.
// ext_node / ext_pos: external boundary-state exports (sharing windows), n_ext of them.
std::string build_plan(const int32_t* parent, const int32_t* length, int32_t n, int32_t C, Plan& out,
                       int mode = kPlanMinRounds, int32_t n_ext = 0, const int32_t* ext_node = nullptr,
                       const int64_t* ext_pos = nullptr);
// Packs the device blob; returns the layout (offsets per table) and the total bytes.
size_t device_layout(const Plan& p, std::vector<size_t>& offsets);
void pack_device_blob(const Plan& p, const std::vector<size_t>& offsets, std::vector<uint8_t>& blob);
DevTables device_view(const Plan& p, void* base, const std::vector<size_t>& offsets);

}  // namespace tpc
