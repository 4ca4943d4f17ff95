// C ABI of the tree-packed chunkwise KDA library: device-table checks (index and bounds mode).
// Declarations and contracts in include/tpc.h.
//
// Every kernel indexes rows, chunks, slots and replay entries through the plan's uploaded tables
// (HARTS Figure 2(c): the packed rounds, their boundary-state slots and the replayed rows).  With
// checks on, each call that reads those tables first runs one kernel that bounds every index field
// of every table on the device, then waits for it on the host: a bad entry returns
// TPC_ERR_DEVICE_CHECK before any compute kernel could follow it out of bounds.  The check reads
// only inside the tables (their sizes come from the host plan), so a corrupt entry is reported, not
// followed.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/tpc.h"
#include "abi_internal.h"
#include "plan.h"

namespace {
using tpc_abi::fail;

// One bound: for records first .. first+count-1 of a table (stride int32 words each), the value
// w[f0] + s1 * w[f1] + s2 * w[f2] (fields -1 absent) must lie in [lo, hi]; with fc >= 0 only records
// whose field fc is non-zero are checked.  Field indices may reach into the next record (stride 1
// monotonicity), the host keeps every read inside the table.
struct FieldCheck {
  int64_t word0;  // first int32 word of the table in the blob
  int64_t first, count;
  int64_t lo, hi;
  int32_t stride;
  int8_t f0, f1, f2, fc, s1, s2;
  int8_t pad[2];
};
constexpr int kMaxChecks = 64;
struct CheckList {
  int n;
  FieldCheck c[kMaxChecks];
};
static_assert(sizeof(CheckList) < 4000, "kernel parameter size");

__device__ unsigned long long g_check_first;  // (check id << 40) | record of the first failure

__global__ void table_check_kernel(const int32_t* __restrict__ blob, CheckList list) {
  const FieldCheck& k = list.c[blockIdx.y];
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < k.count; r += (int64_t)gridDim.x * blockDim.x) {
    const int32_t* w = blob + k.word0 + (k.first + r) * k.stride;
    if (k.fc >= 0 && w[k.fc] == 0) continue;
    int64_t v = w[k.f0];
    if (k.f1 >= 0) v += (int64_t)k.s1 * w[k.f1];
    if (k.f2 >= 0) v += (int64_t)k.s2 * w[k.f2];
    if (v < k.lo || v > k.hi)
      atomicMin(&g_check_first, ((unsigned long long)blockIdx.y << 40) | (unsigned long long)(k.first + r));
  }
}

std::atomic<int> g_checks{-1};  // -1: not yet read from TPC_CHECKS

struct Named {
  FieldCheck c;
  int table_id;  // blob order
  const char* table;
  const char* what;
};

// The bounds the kernels rely on, table by table (blob order of the plan's device layout).
std::vector<Named> plan_checks_list(const tpc::Plan& p, const std::vector<size_t>& off) {
  const int64_t N = p.n_unique, R = (int64_t)p.replay_rows.size(), C = p.C, NE = p.n_expanded;
  const int64_t ns = (int64_t)p.seqs.size(), nc = (int64_t)p.chunks.size(), nsl = (int64_t)p.slots.size();
  const int64_t nroots = (int64_t)p.root_cons_begin.size() - 1, nrc = (int64_t)p.root_cons.size();
  const int64_t ntgt = (int64_t)p.tgt_row.size(), nnodes = (int64_t)p.attn_nodes.size() - 1;
  const int64_t nranges = (int64_t)p.attn_ranges.size() / 2, nleaves = (int64_t)p.leaves.size();
  const int64_t next = (int64_t)p.ext_slot.size();
  std::vector<Named> v;
  auto add = [&](int table, int32_t stride, int64_t first, int64_t count, int f0, int f1, int s1, int f2, int s2,
                 int fc, int64_t lo, int64_t hi, const char* tname, const char* what) {
    if (count <= 0) return;
    FieldCheck c{};
    c.word0 = (int64_t)(off[table] / 4);
    c.first = first; c.count = count; c.lo = lo; c.hi = hi; c.stride = stride;
    c.f0 = (int8_t)f0; c.f1 = (int8_t)f1; c.f2 = (int8_t)f2; c.fc = (int8_t)fc; c.s1 = (int8_t)s1; c.s2 = (int8_t)s2;
    v.push_back({c, table, tname, what});
  };
  auto one = [&](int table, int32_t stride, int64_t count, int f, int64_t lo, int64_t hi, const char* t, const char* w) {
    add(table, stride, 0, count, f, -1, 0, -1, 0, -1, lo, hi, t, w);
  };
  auto mono = [&](int table, int64_t len, const char* t) {  // w[i+1] - w[i] >= 0
    add(table, 1, 0, len - 1, 1, 0, -1, -1, 0, -1, 0, INT64_MAX, t, "non-decreasing");
  };
  // sequences: chunk_begin, n_chunks, import_id, leaf, head, round, start_pos, n_replay
  one(0, 8, ns, 0, 0, nc - 1, "seqs", "chunk_begin in [0, n_chunks)");
  add(0, 8, 0, ns, 0, 1, 1, -1, 0, -1, 1, nc, "seqs", "chunk_begin + n_chunks in [1, n_chunks]");
  one(0, 8, ns, 1, 1, nc, "seqs", "n_chunks in [1, n_chunks]");
  one(0, 8, ns, 2, -nroots, nsl - 1, "seqs", "import_id in [-n_roots, n_slots)");
  one(0, 8, ns, 3, -1, nleaves - 1, "seqs", "leaf in [-1, n_leaves)");
  one(0, 8, ns, 5, 1, p.n_rounds, "seqs", "round in [1, n_rounds]");
  one(0, 8, ns, 7, 0, C - 1, "seqs", "n_replay in [0, C)");
  // chunks: seq, n_rows, n_replay, row_start, replay_base, export_slot, pos0, idx_in_seq
  one(1, 8, nc, 0, 0, ns - 1, "chunks", "seq in [0, n_seqs)");
  one(1, 8, nc, 1, 1, C, "chunks", "n_rows in [1, C]");
  one(1, 8, nc, 2, 0, C, "chunks", "n_replay in [0, C]");
  add(1, 8, 0, nc, 1, 2, -1, -1, 0, -1, 0, C, "chunks", "n_rows - n_replay in [0, C]");
  one(1, 8, nc, 3, 0, N, "chunks", "row_start in [0, N]");
  add(1, 8, 0, nc, 3, 1, 1, 2, -1, -1, 0, N, "chunks", "row_start + n_rows - n_replay in [0, N]");
  add(1, 8, 0, nc, 4, -1, 0, -1, 0, 2, 0, R, "chunks", "replay_base in [0, R] (chunks with replays)");
  add(1, 8, 0, nc, 4, 2, 1, -1, 0, 2, 0, R, "chunks", "replay_base + n_replay in [0, R] (chunks with replays)");
  one(1, 8, nc, 5, -1, nsl - 1, "chunks", "export_slot in [-1, n_slots)");
  // slots: producer_seq, export_chunk, cons_begin, n_cons
  one(2, 4, nsl, 0, 0, ns - 1, "slots", "producer_seq in [0, n_seqs)");
  one(2, 4, nsl, 1, 0, nc - 1, "slots", "export_chunk in [0, n_chunks)");
  one(2, 4, nsl, 2, 0, (int64_t)p.slot_cons.size(), "slots", "cons_begin in [0, n_slot_cons]");
  add(2, 4, 0, nsl, 2, 3, 1, -1, 0, -1, 0, (int64_t)p.slot_cons.size(), "slots", "cons_begin + n_cons in [0, n_slot_cons]");
  one(3, 1, (int64_t)p.slot_cons.size(), 0, 0, ns + next - 1, "slot_cons", "consumer in [0, n_seqs + n_exports)");
  one(4, 1, nroots + 1, 0, 0, nrc, "root_cons_begin", "in [0, n_root_cons]");
  mono(4, nroots + 1, "root_cons_begin");
  one(5, 1, nrc, 0, 0, ns - 1, "root_cons", "consumer in [0, n_seqs)");
  one(6, 1, R, 0, 0, N - 1, "replay_rows", "row in [0, N)");
  one(7, 1, ntgt, 0, 0, N - 1, "tgt_row", "row in [0, N)");
  one(8, 1, (int64_t)p.tgt_begin.size(), 0, 0, R, "tgt_begin", "in [0, R]");
  mono(8, (int64_t)p.tgt_begin.size(), "tgt_begin");
  one(9, 1, (int64_t)p.tgt_parts.size(), 0, 0, R - 1, "tgt_parts", "replay index in [0, R)");
  one(10, 1, (int64_t)p.row_tgt.size(), 0, -1, ntgt - 1, "row_tgt", "target in [-1, n_targets)");
  one(11, 1, (int64_t)p.exp_rows.size(), 0, 0, N - 1, "exp_rows", "row in [0, N)");
  one(12, 1, (int64_t)p.occ_begin.size(), 0, 0, NE, "occ_begin", "in [0, n_expanded]");
  mono(12, (int64_t)p.occ_begin.size(), "occ_begin");
  one(13, 1, (int64_t)p.occ_list.size(), 0, 0, NE - 1, "occ_list", "position in [0, n_expanded)");
  one(14, 1, N, 0, 1, NE, "occ_count", "in [1, n_expanded]");
  // attention nodes (row_offset, length, subtree_end, range_begin, pos0, pad x3; one sentinel entry)
  one(15, 8, nnodes, 0, 0, N, "attn_nodes", "row_offset in [0, N]");
  add(15, 8, 0, nnodes, 0, 1, 1, -1, 0, -1, 0, N, "attn_nodes", "row_offset + length in [0, N]");
  one(15, 8, nnodes, 2, 0, N, "attn_nodes", "subtree_end in [0, N]");
  one(15, 8, nnodes + 1, 3, 0, nranges, "attn_nodes", "range_begin in [0, n_ranges]");
  add(15, 8, 0, nnodes, 11, 3, -1, -1, 0, -1, 0, INT64_MAX, "attn_nodes", "range_begin non-decreasing");
  one(16, 2, nranges, 0, 0, N, "attn_ranges", "start in [0, N]");
  one(16, 2, nranges, 1, 0, N, "attn_ranges", "end in [0, N]");
  add(16, 2, 0, nranges, 1, 0, -1, -1, 0, -1, 0, N, "attn_ranges", "end - start in [0, N]");
  for (int t = 17; t <= 18; ++t) {
    const int64_t nt = (int64_t)(t == 17 ? p.attn_qtiles.size() : p.attn_ktiles.size());
    const char* name = t == 17 ? "attn_qtiles" : "attn_ktiles";
    one(t, 4, nt, 0, 0, nnodes - 1, name, "node in [0, n_nodes)");
    one(t, 4, nt, 1, 0, N - 1, name, "row in [0, N)");
    one(t, 4, nt, 2, 1, 128, name, "n in [1, 128]");
    add(t, 4, 0, nt, 1, 2, 1, -1, 0, -1, 1, N, name, "row + n in [1, N]");
  }
  return v;
}

// table sizes in int32 words (blob order), for the poke hook's bounds
int64_t table_words(const tpc::Plan& p, int table) {
  switch (table) {
    case 0: return (int64_t)p.seqs.size() * 8;
    case 1: return (int64_t)p.chunks.size() * 8;
    case 2: return (int64_t)p.slots.size() * 4;
    case 3: return (int64_t)p.slot_cons.size();
    case 4: return (int64_t)p.root_cons_begin.size();
    case 5: return (int64_t)p.root_cons.size();
    case 6: return (int64_t)p.replay_rows.size();
    case 7: return (int64_t)p.tgt_row.size();
    case 8: return (int64_t)p.tgt_begin.size();
    case 9: return (int64_t)p.tgt_parts.size();
    case 10: return (int64_t)p.row_tgt.size();
    case 11: return (int64_t)p.exp_rows.size();
    case 12: return (int64_t)p.occ_begin.size();
    case 13: return (int64_t)p.occ_list.size();
    case 14: return p.n_unique;
    case 15: return (int64_t)p.attn_nodes.size() * 8;
    case 16: return (int64_t)p.attn_ranges.size();
    case 17: return (int64_t)p.attn_qtiles.size() * 4;
    case 18: return (int64_t)p.attn_ktiles.size() * 4;
    default: return -1;
  }
}

std::mutex g_check_mu;

// Reads that each check makes stay inside its table (sizes from the host plan).
int bound_reads(const tpc::Plan& p, const std::vector<Named>& all) {
  if (all.size() > (size_t)kMaxChecks) return fail(TPC_ERR_STATE, "internal: more table checks than one launch holds");
  for (const Named& n : all) {
    const FieldCheck& c = n.c;
    const int maxf = std::max<int>(c.f0, std::max<int>(c.f1, std::max<int>(c.f2, c.fc)));
    if ((c.first + c.count - 1) * c.stride + maxf >= table_words(p, n.table_id))
      return fail(TPC_ERR_STATE, std::string("internal: a check reads past ") + n.table);
  }
  return TPC_OK;
}

int report(const std::vector<Named>& all, unsigned long long first) {
  if (first == ~0ull) return TPC_OK;
  const size_t id = (size_t)(first >> 40);
  const unsigned long long rec = first & ((1ull << 40) - 1);
  if (id >= all.size()) return fail(TPC_ERR_DEVICE_CHECK, "device table check failed");
  return fail(TPC_ERR_DEVICE_CHECK, std::string("device table check failed: ") + all[id].table + "[" +
                                        std::to_string(rec) + "]: " + all[id].what);
}

int run_checks(const tpc::Plan& p, const void* dev, const std::vector<size_t>& off, cudaStream_t st) {
  if (!dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  const std::vector<Named> all = plan_checks_list(p, off);
  if (int rc = bound_reads(p, all)) return rc;
  CheckList list{};
  list.n = (int)all.size();
  int64_t most = 1;
  for (int i = 0; i < list.n; ++i) {
    list.c[i] = all[i].c;
    most = std::max(most, all[i].c.count);
  }
  std::lock_guard<std::mutex> lock(g_check_mu);
  const unsigned long long none = ~0ull;
  TPC_CUDA(cudaMemcpyToSymbolAsync(g_check_first, &none, sizeof(none), 0, cudaMemcpyHostToDevice, st));
  const unsigned gx = (unsigned)std::min<int64_t>((most + 255) / 256, 4 * (int64_t)tpc_abi::sm_count());
  TPC_LAUNCH("table_check", st, table_check_kernel<<<dim3(gx, list.n), 256, 0, st>>>(
                                    static_cast<const int32_t*>(dev), list));
  unsigned long long first = none;
  TPC_CUDA(cudaMemcpyFromSymbolAsync(&first, g_check_first, sizeof(first), 0, cudaMemcpyDeviceToHost, st));
  TPC_CUDA(cudaStreamSynchronize(st));
  return report(all, first);
}

// The same checks on the host copy of the tables (the packed blob), with one word optionally
// replaced: the checks' own test, runnable without a GPU.
int run_checks_host(const tpc::Plan& p, int table, int64_t word, int32_t value) {
  std::vector<size_t> off;
  tpc::device_layout(p, off);
  std::vector<uint8_t> blob;
  tpc::pack_device_blob(p, off, blob);
  if (table >= 0) {
    const int64_t words = table_words(p, table);
    if (words < 0 || word < 0 || word >= words) return fail(TPC_ERR_BAD_SHAPE, "poke: word outside the table");
    std::memcpy(blob.data() + off[table] + 4 * word, &value, 4);
  }
  std::vector<Named> all = plan_checks_list(p, off);
  if (int rc = bound_reads(p, all)) return rc;
  const int32_t* b = reinterpret_cast<const int32_t*>(blob.data());
  unsigned long long first = ~0ull;
  for (size_t id = 0; id < all.size() && first == ~0ull; ++id) {
    const FieldCheck& k = all[id].c;
    for (int64_t r = 0; r < k.count; ++r) {
      const int32_t* w = b + k.word0 + (k.first + r) * k.stride;
      if (k.fc >= 0 && w[k.fc] == 0) continue;
      int64_t v = w[k.f0];
      if (k.f1 >= 0) v += (int64_t)k.s1 * w[k.f1];
      if (k.f2 >= 0) v += (int64_t)k.s2 * w[k.f2];
      if (v < k.lo || v > k.hi) {
        first = ((unsigned long long)id << 40) | (unsigned long long)(k.first + r);
        break;
      }
    }
  }
  return report(all, first);
}
}  // namespace

namespace tpc_abi {
bool checks_on() {
  int v = g_checks.load();
  if (v < 0) {
    const char* e = std::getenv("TPC_CHECKS");
    v = (e && *e && std::strcmp(e, "0") != 0) ? 1 : 0;
    int expect = -1;
    g_checks.compare_exchange_strong(expect, v);
    v = g_checks.load();
  }
  return v == 1;
}

int plan_checks(const tpc_plan* plan, cudaStream_t st) {
  if (!checks_on()) return TPC_OK;
  return run_checks(plan->p, plan->p.dev, plan->p.blob_offsets, st);
}

int table_checks_at(const tpc::Plan& p, const void* dev, const std::vector<size_t>& off, cudaStream_t st) {
  return run_checks(p, dev, off, st);
}
}  // namespace tpc_abi

extern "C" {

void tpc_checks_enable(int on) { g_checks.store(on ? 1 : 0); }

int tpc_checks_enabled(void) { return tpc_abi::checks_on() ? 1 : 0; }

int tpc_plan_check_device(const tpc_plan* plan, tpc_stream_t stream) {
  if (!plan) return fail(TPC_ERR_NULL, "plan is NULL");
  return run_checks(plan->p, plan->p.dev, plan->p.blob_offsets, reinterpret_cast<cudaStream_t>(stream));
}

int tpc_plan_check_host(const tpc_plan* plan, int32_t table, int64_t word, int32_t value) {
  if (!plan) return fail(TPC_ERR_NULL, "plan is NULL");
  return run_checks_host(plan->p, table, word, value);
}

int tpc_debug_poke_table(tpc_plan* plan, int32_t table, int64_t word, int32_t value, int32_t* old_value,
                         tpc_stream_t stream) {
  if (!plan) return fail(TPC_ERR_NULL, "plan is NULL");
  const tpc::Plan& p = plan->p;
  if (!p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  const int64_t words = table_words(p, table);
  if (words < 0) return fail(TPC_ERR_BAD_SHAPE, "poke: table id outside [0, 18]");
  if (word < 0 || word >= words) return fail(TPC_ERR_BAD_SHAPE, "poke: word outside the table");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* dst = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(p.dev) + p.blob_offsets[table]) + word;
  int32_t old = 0;
  TPC_CUDA(cudaMemcpyAsync(&old, dst, 4, cudaMemcpyDeviceToHost, st));
  TPC_CUDA(cudaStreamSynchronize(st));
  TPC_CUDA(cudaMemcpyAsync(dst, &value, 4, cudaMemcpyHostToDevice, st));
  TPC_CUDA(cudaStreamSynchronize(st));
  if (old_value) *old_value = old;
  return TPC_OK;
}

}  // extern "C"
