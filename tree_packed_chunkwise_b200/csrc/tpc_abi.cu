// C ABI of the tree-packed chunkwise KDA library (declarations and contracts in include/tpc.h).
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <type_traits>
#include <vector>

#include "../../include/tpc.h"
#include "kda_kernels.cuh"
#include "kda_tc.cuh"
#include "kda_scan_tc.cuh"
#include <cudaTypedefs.h>
#include "abi_internal.h"
#include "plan.h"
#include "rowmap_kernels.cuh"

namespace tpc_abi {

thread_local std::string g_err;
Profiler g_prof;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

// ------------------------------------------------------------------------------------------------
// TMA tensor maps (driver entry point looked up through the runtime; no link against libcuda)
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

// multiprocessors of the current device (persistent grids)
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n < 1)
    return 148;
  return n;
}

// the driver's tensor-map encoder (looked up once)
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", reinterpret_cast<void**>(&g_encode), cudaEnableDefault,
                                &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      g_encode = nullptr;
  });
  return g_encode;
}

// 2-D bf16 tensor map over [rows][cols] (leading dimension ld_elems): boxes of 64 columns x box_rows
// rows, each box row one 128-byte swizzled line.
bool tensor_map(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t ld_elems,
                uint32_t box_rows) {
  const auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over a [rows][heads][features] tensor (feature dimension contiguous): boxes
// of 64 features x 1 head x box_rows rows, each box row one 128-byte swizzled line; rows past the
// end read as zeros.
bool tensor_map_rows(CUtensorMap* m, const void* ptr, uint64_t features, uint64_t heads, uint64_t rows,
                     uint32_t box_rows) {
  const auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {features, heads, rows};
  cuuint64_t strides[2] = {features * 2, heads * features * 2};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tpc_abi

namespace {

using tpc_abi::a256;
using tpc_abi::fail;
using tpc_abi::g_prof;
using tpc_abi::set_smem;

#define TPC_TRY_ABI(call)        \
  do {                           \
    const int r_ = (call);       \
    if (r_ != TPC_OK) return r_; \
  } while (0)

// workspace layout (bytes) for a plan + shape
struct WsLayout {
  size_t status, W, U, Khat, decay, S0, slot, dU, dS, dS0seq, pdk, pdG, rdk, rdv, rdg, rdb, tdk, tdv, tdg, tdb, Mt, Bc,
      At, Tm, Pm, total;
};

WsLayout ws_layout(const tpc::Plan& p, int H, int C, int D) {
  WsLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += a256(bytes); return r; };
  const size_t nc = p.chunks.size(), cd = (size_t)C * D, dd = (size_t)D * D;
  const size_t R = (size_t)p.replay_total, T = p.tgt_row.size();
  L.status = take(256);
  L.W = take(nc * H * cd * 4);
  L.U = take(nc * H * cd * 4);
  L.Khat = take(nc * H * cd * 4);
  L.decay = take(nc * H * D * 4);
  L.S0 = take(nc * H * dd * 4);
  L.slot = take(p.slots.size() * H * dd * 4);
  L.dU = take(nc * H * cd * 4);
  L.dS = take(nc * H * dd * 4);
  L.dS0seq = take((p.seqs.size() + p.ext_slot.size()) * H * dd * 4);  // + external consumers' gradients
  L.pdk = take(nc * H * cd * 4);
  L.pdG = take(nc * H * cd * 4);
  L.rdk = take(R * H * D * 4);
  L.rdv = take(R * H * D * 4);
  L.rdg = take(R * H * D * 4);
  L.rdb = take(R * H * 4);
  L.tdk = take(T * H * D * 4);
  L.tdv = take(T * H * D * 4);
  L.tdg = take(T * H * D * 4);
  L.tdb = take(T * H * 4);
  const bool tensor_cores = (C == tpc::kTcC && D == tpc::kTcD);  // (bf16 inputs; sized for either)
  L.Mt = take(tensor_cores ? nc * H * (size_t)tpc::kMtileBytes : 0);
  L.Bc = take(tensor_cores ? nc * H * dd * 4 : 0);
  L.At = take(tensor_cores ? nc * H * (size_t)C * C * 4 : 0);
  L.Tm = take(tensor_cores ? nc * H * (size_t)C * C * 4 : 0);
  L.Pm = take(tensor_cores ? nc * H * (size_t)C * C * 4 : 0);
  L.total = o;
  return L;
}

tpc::KdaWs ws_view(const WsLayout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  tpc::KdaWs w;
  w.status = reinterpret_cast<int*>(b + L.status);
  auto f = [&](size_t off) { return reinterpret_cast<float*>(b + off); };
  w.W = f(L.W); w.U = f(L.U); w.Khat = f(L.Khat); w.decay = f(L.decay); w.S0 = f(L.S0); w.slot = f(L.slot);
  w.dU = f(L.dU); w.dS = f(L.dS); w.dS0seq = f(L.dS0seq); w.pdk = f(L.pdk); w.pdG = f(L.pdG);
  w.rdk = f(L.rdk); w.rdv = f(L.rdv); w.rdg = f(L.rdg); w.rdb = f(L.rdb);
  w.tdk = f(L.tdk); w.tdv = f(L.tdv); w.tdg = f(L.tdg); w.tdb = f(L.tdb);
  w.Mt = f(L.Mt); w.Bc = f(L.Bc); w.At = f(L.At); w.Tm = f(L.Tm); w.Pm = f(L.Pm);
  w.dUt = f(L.Khat);  // the tensor-core path keeps its dU tile where the CUDA-core path keeps Khat
  return w;
}

// Heads one chunk CTA runs in turn (the largest divisor of H up to `most`): the next head's inputs
// load while the current head computes, and the CTA's set-up is paid once.
constexpr int kOutHeadsPerCta = 2, kPrepHeadsPerCta = 4, kBwdHeadsPerCta = 4;
int heads_per_cta(int H, int most) {
  for (int k = most; k > 1; --k)
    if (H % k == 0) return k;
  return 1;
}

bool shape_supported(int C, int D) { return (C == 16 && D == 32) || (C == 64 && D == 128) || (C == 32 && D == 64); }

int check_shape(const tpc_plan* plan, const tpc_kda_shape* s) {
  if (!plan || !s) return fail(TPC_ERR_NULL, "plan or shape is NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded (tpc_plan_upload)");
  if (s->H < 1 || s->dk < 1 || s->dv < 1) return fail(TPC_ERR_BAD_SHAPE, "H, dk, dv must be >= 1");
  if (s->dk != s->dv) return fail(TPC_ERR_UNSUPPORTED, "dk != dv is not built");
  if (!shape_supported(plan->p.C, s->dk))
    return fail(TPC_ERR_UNSUPPORTED, "built (chunk, d) pairs: (16,32), (32,64), (64,128)");
  if ((s->in_dtype != TPC_F32 && s->in_dtype != TPC_BF16 && s->in_dtype != TPC_F32_SPLIT) ||
      (s->out_dtype != TPC_F32 && s->out_dtype != TPC_BF16))
    return fail(TPC_ERR_UNSUPPORTED, "in_dtype TPC_F32, TPC_BF16 or TPC_F32_SPLIT; out_dtype TPC_F32 or TPC_BF16");
  if (s->in_dtype == TPC_F32_SPLIT && !(plan->p.C == tpc::kTcC && s->dk == tpc::kTcD))
    return fail(TPC_ERR_UNSUPPORTED, "TPC_F32_SPLIT is built for chunk 64, d 128 (the tensor-core path)");
  return TPC_OK;
}

// A high-priority stream per device for the sequential state scans (created once, non-blocking,
// ordered against the caller's stream by events): the scans are the critical path of a step, so
// when an SM frees up their CTAs go before the caller-stream chunk kernels that overlap them.
cudaStream_t scan_stream() {
  static std::mutex mu;
  static std::vector<cudaStream_t> streams;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)streams.size() <= dev) streams.resize(dev + 1, nullptr);
  if (!streams[dev]) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&streams[dev], cudaStreamNonBlocking, greatest) != cudaSuccess)
      streams[dev] = nullptr;
  }
  return streams[dev];
}

// work queued on `to` from now on runs after everything already queued on `from`
int stream_after(cudaStream_t to, cudaStream_t from) {
  cudaEvent_t e;
  TPC_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  TPC_CUDA(cudaEventRecord(e, from));
  TPC_CUDA(cudaStreamWaitEvent(to, e, 0));
  TPC_CUDA(cudaEventDestroy(e));
  return TPC_OK;
}

// Chunk kernels run on grids (heads, chunks): the heads of one chunk are neighbouring CTAs, so the
// CTAs in flight read whole token rows ([N, H, D] inputs) and consecutive workspace tiles; a round
// with more chunks than a grid's y extent allows is launched in pieces.
constexpr int kMaxGridY = 65535;

// Columns per state-scan CTA (one scan CTA per SM).  With several rounds the scans overlap the chunk
// kernels of neighbouring rounds, so they take 128 columns (fewest CTAs: each reads the M tile once for
// all columns, and the most SMs stay with the chunk kernels).  A plan of one round has nothing to
// overlap: its scan takes the narrowest width whose CTAs fit one wave (more CTAs, a shorter chain
// step), 128 if none does.  (Measured on the single-fork and agentic trees: 128 columns for every
// round beat 32 / 64 by 2-4 % of the step.)
int scan_width(int n_seqs, int H, int n_rounds) {
  if (n_rounds > 1) return 128;
  const long long pairs = (long long)n_seqs * H, sm = tpc_abi::sm_count();
  for (int W = 32; W < 128; W *= 2)
    if (pairs * (tpc::kTcD / W) <= sm) return W;
  return 128;
}

// launches the state scan of a round with the chosen width
template <bool REVERSE, typename Tin>
int launch_scan(cudaStream_t hs, const tpc::Plan& p, int s0, int s1, int H, const float* init, float* final_state,
                const float* d_final, const tpc::KdaWs& w, const Tin* dO) {
  using namespace tpc;
  const char* name = REVERSE ? "kda_bwd_scan_tc" : "kda_fwd_scan_tc";
  auto go = [&](auto wc) -> int {
    constexpr int W = decltype(wc)::value;
    TPC_CUDA(set_smem(kda_scan_tc<REVERSE, W, Tin>, ScanTcSmemT<REVERSE, W>::total));
    TPC_LAUNCH(name, hs,
               (kda_scan_tc<REVERSE, W, Tin><<<dim3(s1 - s0, H, kTcD / W), 128 * (W / 32), ScanTcSmemT<REVERSE, W>::total,
                                               hs>>>(p.dt, s0, H, init, final_state, d_final, w, dO)));
    return TPC_OK;
  };
  switch (scan_width(s1 - s0, H, p.n_rounds)) {
    case 128: return go(std::integral_constant<int, 128>{});
    case 64: return go(std::integral_constant<int, 64>{});
    default: return go(std::integral_constant<int, 32>{});
  }
}

template <int C, int D, typename Tin, typename Tout, bool TC>
int forward_impl(const tpc::Plan& p, const tpc_kda_shape* s, const tpc_kda_fwd_io* io, void* ws, cudaStream_t st) {
  using namespace tpc;
  constexpr int DVT = D < 32 ? D : 32;
  const int H = s->H;
  const WsLayout L = ws_layout(p, H, C, D);
  KdaWs w = ws_view(L, ws);
  const int nc = (int)p.chunks.size();
  TPC_CUDA(cudaMemsetAsync(w.status, 0, 4, st));
  TPC_CUDA(set_smem(kda_fwd_prep<C, D, Tin>, fwd_prep_smem<C, D>()));
  TPC_CUDA(set_smem(kda_fwd_scan<C, D, DVT>, scan_smem<C, D, DVT>()));
  TPC_CUDA(set_smem(kda_fwd_out<C, D, Tin, Tout>, out_smem<C, D>()));
  const Tin* q = static_cast<const Tin*>(io->q);
  const Tin* k = static_cast<const Tin*>(io->k);
  const Tin* v = static_cast<const Tin*>(io->v);
  const Tin* g = static_cast<const Tin*>(io->g);
  const Tin* b = static_cast<const Tin*>(io->beta);
  // tensor cores at chunk 64 / d 128 for bf16 inputs and for fp32 inputs given as TPC_F32_SPLIT;
  // TPC_F32 inputs take the exact CUDA-core path
  std::vector<cudaEvent_t> scans;
  if constexpr (TC) {
    // Per round r: prep(r) and then out(r) on the caller's stream, scan(r) on the high-priority scan
    // stream after prep(r) and scan(r - 1).  The caller's stream runs prep(1..R), out(1..R) in that
    // order, so the later rounds' prep overlaps scan(1) and out(r) overlaps scan(r + 1).
    TPC_CUDA(set_smem(kda_fwd_prep_tc<Tin>, PrepTcSmemT<Tin>::total));
    TPC_CUDA(set_smem(kda_fwd_out_tc<Tin, Tout>, OutTcSmem::total));
    cudaStream_t hs = scan_stream();
    if (!hs) return fail(TPC_ERR_CUDA, "could not create the library's scan stream");
    for (int r = 1; r <= p.n_rounds; ++r) {
      tpc_abi::NvtxRange nvtx_round("kda forward prep + scan", r);
      const int c0 = p.round_chunk_begin[r - 1], c1 = p.round_chunk_begin[r];
      const int s0 = p.round_seq_begin[r - 1], s1 = p.round_seq_begin[r];
      const int hpc = heads_per_cta(H, kPrepHeadsPerCta);
      for (int a = c0; a < c1; a += kMaxGridY)
        TPC_LAUNCH("kda_fwd_prep_tc", st,
                   (kda_fwd_prep_tc<Tin><<<dim3(H / hpc, std::min(c1 - a, kMaxGridY)), kTcThreads,
                                           PrepTcSmemT<Tin>::total, st>>>(p.dt, H, k, v, g, b, w, a, hpc)));
      TPC_TRY_ABI(stream_after(hs, st));  // scan(r) after prep(r)
      if (s1 > s0)
        TPC_TRY_ABI((launch_scan<false, Tin>(hs, p, s0, s1, H, io->init_state, io->final_state, nullptr, w,
                                             static_cast<const Tin*>(nullptr))));
      scans.emplace_back();
      TPC_CUDA(cudaEventCreateWithFlags(&scans.back(), cudaEventDisableTiming));
      TPC_CUDA(cudaEventRecord(scans.back(), hs));
    }
    for (int r = 1; r <= p.n_rounds; ++r) {
      tpc_abi::NvtxRange nvtx_round("kda forward out", r);
      const int c0 = p.round_chunk_begin[r - 1], c1 = p.round_chunk_begin[r];
      TPC_CUDA(cudaStreamWaitEvent(st, scans[r - 1], 0));
      TPC_CUDA(cudaEventDestroy(scans[r - 1]));
      const int hpc = heads_per_cta(H, kOutHeadsPerCta);
      for (int a = c0; a < c1; a += kMaxGridY)
        TPC_LAUNCH("kda_fwd_out_tc", st,
                   (kda_fwd_out_tc<Tin, Tout><<<dim3(H / hpc, std::min(c1 - a, kMaxGridY)), kTcThreads,
                                                OutTcSmem::total, st>>>(p.dt, H, q, k, g,
                                                                         static_cast<Tout*>(io->o), w, a, hpc)));
    }
  } else {
    TPC_LAUNCH("kda_fwd_prep", st,
               (kda_fwd_prep<C, D, Tin><<<dim3(nc, H), kThreads, fwd_prep_smem<C, D>(), st>>>(p.dt, H, k, v, g, b, w)));
    for (int r = 1; r <= p.n_rounds; ++r) {
      const int s0 = p.round_seq_begin[r - 1], s1 = p.round_seq_begin[r];
      TPC_LAUNCH("kda_fwd_scan", st,
                 (kda_fwd_scan<C, D, DVT><<<dim3(s1 - s0, H, D / DVT), kThreads, scan_smem<C, D, DVT>(), st>>>(
                     p.dt, s0, H, io->init_state, io->final_state, w)));
    }
    TPC_LAUNCH("kda_fwd_out", st,
               (kda_fwd_out<C, D, Tin, Tout><<<dim3(nc, H), kThreads, out_smem<C, D>(), st>>>(
                   p.dt, H, q, k, g, static_cast<Tout*>(io->o), w)));
  }
  return TPC_OK;
}

template <int C, int D, typename Tin, typename Tout, bool TC>
int backward_impl(const tpc::Plan& p, const tpc_kda_shape* s, const tpc_kda_bwd_io* io, void* ws, cudaStream_t st) {
  using namespace tpc;
  constexpr int DVT = D < 32 ? D : 32;
  const int H = s->H;
  const WsLayout L = ws_layout(p, H, C, D);
  KdaWs w = ws_view(L, ws);
  const int nc = (int)p.chunks.size();
  TPC_CUDA(set_smem(kda_bwd_prep<C, D, Tin>, bprep_smem<C, D>()));
  TPC_CUDA(set_smem(kda_bwd_scan<C, D, DVT>, scan_smem<C, D, DVT>() + sizeof(float) * D * (DVT + 1)));
  TPC_CUDA(set_smem(kda_bwd_dq<C, D, Tin, Tout>, bdq_smem<C, D>()));
  TPC_CUDA(set_smem(kda_bwd_dkv<C, D, Tin, Tout>, bdkv_smem<C, D>()));
  const Tin* q = static_cast<const Tin*>(io->q);
  const Tin* k = static_cast<const Tin*>(io->k);
  const Tin* v = static_cast<const Tin*>(io->v);
  const Tin* g = static_cast<const Tin*>(io->g);
  const Tin* b = static_cast<const Tin*>(io->beta);
  const Tin* dO = static_cast<const Tin*>(io->d_o);
  // tensor-core or exact CUDA-core path, as in forward_impl
  std::vector<cudaEvent_t> scans;
  if constexpr (TC) {
    // Rounds in reverse: the reverse scan(r) (which also forms the output's contribution Qeff^T dO)
    // on the high-priority scan stream after the caller's prior work and scan(r + 1); then dq(r),
    // dk/dv(r) on the caller's stream after scan(r), so dq / dk-dv(r) overlap scan(r - 1).
    TPC_CUDA(set_smem(kda_bwd_dq_tc<Tin, Tout>, BdqTcSmem::total));
    TPC_CUDA(set_smem(kda_bwd_dkv_tc<Tin, Tout>, BdkvTcSmemT<Tin>::total));
    cudaStream_t hs = scan_stream();
    if (!hs) return fail(TPC_ERR_CUDA, "could not create the library's scan stream");
    TPC_TRY_ABI(stream_after(hs, st));  // the scans after the caller's prior work (forward, d_o)
    for (int r = p.n_rounds; r >= 1; --r) {
      tpc_abi::NvtxRange nvtx_round("kda backward scan", r);
      const int s0 = p.round_seq_begin[r - 1], s1 = p.round_seq_begin[r];
      if (s1 > s0) TPC_TRY_ABI((launch_scan<true, Tin>(hs, p, s0, s1, H, nullptr, nullptr, io->d_final, w, dO)));
      scans.emplace_back();
      TPC_CUDA(cudaEventCreateWithFlags(&scans.back(), cudaEventDisableTiming));
      TPC_CUDA(cudaEventRecord(scans.back(), hs));
    }
    for (int r = p.n_rounds, i = 0; r >= 1; --r, ++i) {
      tpc_abi::NvtxRange nvtx_round("kda backward dq + dkv", r);
      const int c0 = p.round_chunk_begin[r - 1], c1 = p.round_chunk_begin[r];
      TPC_CUDA(cudaStreamWaitEvent(st, scans[i], 0));
      TPC_CUDA(cudaEventDestroy(scans[i]));
      const int hpc = heads_per_cta(H, kBwdHeadsPerCta);
      for (int a = c0; a < c1; a += kMaxGridY)
        TPC_LAUNCH("kda_bwd_dq_tc", st,
                   (kda_bwd_dq_tc<Tin, Tout><<<dim3(H / hpc, std::min(c1 - a, kMaxGridY)), kTcThreads,
                                               BdqTcSmem::total, st>>>(p.dt, H, q, k, g, dO,
                                                                       static_cast<Tout*>(io->dq), w, a, hpc)));
      for (int a = c0; a < c1; a += kMaxGridY)
        TPC_LAUNCH("kda_bwd_dkv_tc", st,
                   (kda_bwd_dkv_tc<Tin, Tout><<<dim3(H / hpc, std::min(c1 - a, kMaxGridY)), kTcThreads,
                                                BdkvTcSmemT<Tin>::total, st>>>(
                       p.dt, H, k, v, g, b, static_cast<Tout*>(io->dk), static_cast<Tout*>(io->dv), io->dg,
                       io->dbeta, w, a, hpc)));
    }
  } else {
    TPC_LAUNCH("kda_bwd_prep", st,
               (kda_bwd_prep<C, D, Tin><<<dim3(nc, H), kThreads, bprep_smem<C, D>(), st>>>(p.dt, H, q, k, g, dO, w)));
    for (int r = p.n_rounds; r >= 1; --r) {
      const int s0 = p.round_seq_begin[r - 1], s1 = p.round_seq_begin[r];
      TPC_LAUNCH("kda_bwd_scan", st,
                 (kda_bwd_scan<C, D, DVT><<<dim3(s1 - s0, H, D / DVT), kThreads,
                                            scan_smem<C, D, DVT>() + sizeof(float) * D * (DVT + 1), st>>>(
                     p.dt, s0, H, io->d_final, w)));
    }
    TPC_LAUNCH("kda_bwd_dq", st,
               (kda_bwd_dq<C, D, Tin, Tout><<<dim3(nc, H), kThreads, bdq_smem<C, D>(), st>>>(
                   p.dt, H, q, k, g, dO, static_cast<Tout*>(io->dq), w)));
    TPC_LAUNCH("kda_bwd_dkv", st,
               (kda_bwd_dkv<C, D, Tin, Tout><<<dim3(nc, H), kThreads, bdkv_smem<C, D>(), st>>>(
                   p.dt, H, k, v, g, b, static_cast<Tout*>(io->dk), static_cast<Tout*>(io->dv), io->dg, io->dbeta,
                   w)));
  }
  if (!p.tgt_row.empty()) {
    TPC_LAUNCH("kda_replay_reduce", st,
               (kda_replay_reduce<D, Tout><<<dim3((unsigned)p.tgt_row.size(), H), 128, 0, st>>>(
                   p.dt, H, static_cast<Tout*>(io->dk), static_cast<Tout*>(io->dv), io->dg, io->dbeta, w)));
  }
  if (io->d_init) {
    TPC_LAUNCH("kda_init_reduce", st,
               (kda_init_reduce<D><<<dim3((unsigned)p.roots.size(), H), 256, 0, st>>>(p.dt, H, io->d_init, w)));
  }
  return TPC_OK;
}

// Calls f(C, D, Tin{}, Tout{}, TC) with the shape's compile-time parameters.  TC (tensor cores):
// chunk 64 / d 128 with bf16 inputs or with fp32 inputs given as TPC_F32_SPLIT.
template <class F>
int dispatch(const tpc_plan* plan, const tpc_kda_shape* s, F&& f) {
  const int C = plan->p.C, D = s->dk;
  const bool ib = s->in_dtype == TPC_BF16, ob = s->out_dtype == TPC_BF16, split = s->in_dtype == TPC_F32_SPLIT;
  using Y = std::true_type;
  using N = std::false_type;
#define TPC_CASE(CC, DD, TCB, TCF)                                                                          \
  if (C == CC && D == DD) {                                                                                 \
    using IC = std::integral_constant<int, CC>;                                                             \
    using ID = std::integral_constant<int, DD>;                                                             \
    if (ib && ob) return f(IC{}, ID{}, __nv_bfloat16{}, __nv_bfloat16{}, TCB{});                            \
    if (ib) return f(IC{}, ID{}, __nv_bfloat16{}, float{}, TCB{});                                          \
    if (ob) return split ? f(IC{}, ID{}, float{}, __nv_bfloat16{}, TCF{}) : f(IC{}, ID{}, float{}, __nv_bfloat16{}, N{}); \
    return split ? f(IC{}, ID{}, float{}, float{}, TCF{}) : f(IC{}, ID{}, float{}, float{}, N{});          \
  }
  TPC_CASE(16, 32, N, N)
  TPC_CASE(32, 64, N, N)
  TPC_CASE(64, 128, Y, Y)
#undef TPC_CASE
  return fail(TPC_ERR_UNSUPPORTED, "unsupported (chunk, d)");
}

// ------------------------------------------------------------------------------------------------
// Allocation-free forward (tpc_kda_forward_static).  Its plan tables and workspace live in one
// file-scope device array, so a caller that may not allocate device memory can still run the
// forward pass.  Host code must not pass the array's name to a kernel: in host code that name is a
// host-side stand-in, not a device address.  The device address is looked up once per device with
// cudaGetSymbolAddress and cached.
static __device__ __align__(256) unsigned char g_static_scratch[TPC_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_static_ptr[kMaxDevices] = {};
cudaError_t g_static_rc[kMaxDevices] = {};
std::once_flag g_static_once[kMaxDevices];

// The array starts with the status word (a fixed place, read by tpc_kda_static_status), then the
// plan tables, then the forward-only workspace: W, U, Khat, decay, S0 and slot states.
constexpr size_t kStaticStatusBytes = 256;

size_t static_ws_layout(const tpc::Plan& p, int H, int C, int D, size_t base, tpc::KdaWs* w, char* dev) {
  size_t o = base;
  auto take = [&](size_t bytes) { size_t r = o; o += a256(bytes); return r; };
  const size_t nc = p.chunks.size(), cd = (size_t)C * D, dd = (size_t)D * D;
  const size_t W = take(nc * H * cd * 4), U = take(nc * H * cd * 4), K = take(nc * H * cd * 4);
  const size_t dec = take(nc * H * D * 4), S0 = take(nc * H * dd * 4), sl = take(p.slots.size() * H * dd * 4);
  if (w && dev) {
    *w = tpc::KdaWs{};
    w->status = reinterpret_cast<int*>(dev);
    w->W = reinterpret_cast<float*>(dev + W);
    w->U = reinterpret_cast<float*>(dev + U);
    w->Khat = reinterpret_cast<float*>(dev + K);
    w->decay = reinterpret_cast<float*>(dev + dec);
    w->S0 = reinterpret_cast<float*>(dev + S0);
    w->slot = reinterpret_cast<float*>(dev + sl);
  }
  return o;
}

// Device address of the scratch array on the current device: looked up once per device, with that
// device current (cudaGetSymbolAddress), and cached.
int static_base(char** out) {
  int dev = 0;
  TPC_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(TPC_ERR_UNSUPPORTED, "device ordinal out of range");
  std::call_once(g_static_once[dev], [dev] {
    g_static_rc[dev] = cudaGetSymbolAddress(&g_static_ptr[dev], g_static_scratch);
  });
  if (g_static_rc[dev] != cudaSuccess || !g_static_ptr[dev])
    return fail(TPC_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(g_static_rc[dev]));
  *out = static_cast<char*>(g_static_ptr[dev]);
  return TPC_OK;
}

template <int C, int D, typename Tin, typename Tout>
int forward_static_impl(const tpc::Plan& p, const tpc::DevTables& dt, tpc::KdaWs w, const tpc_kda_shape* s,
                        const tpc_kda_fwd_io* io, cudaStream_t st) {
  using namespace tpc;
  constexpr int DVT = D < 32 ? D : 32;
  const int H = s->H;
  const int nc = (int)p.chunks.size();
  TPC_CUDA(cudaMemsetAsync(w.status, 0, 4, st));  // the array keeps the previous call's contents
  TPC_CUDA(set_smem(kda_fwd_prep<C, D, Tin>, fwd_prep_smem<C, D>()));
  TPC_CUDA(set_smem(kda_fwd_scan<C, D, DVT>, scan_smem<C, D, DVT>()));
  TPC_CUDA(set_smem(kda_fwd_out<C, D, Tin, Tout>, out_smem<C, D>()));
  const Tin* q = static_cast<const Tin*>(io->q);
  const Tin* k = static_cast<const Tin*>(io->k);
  const Tin* v = static_cast<const Tin*>(io->v);
  const Tin* g = static_cast<const Tin*>(io->g);
  const Tin* b = static_cast<const Tin*>(io->beta);
  TPC_LAUNCH("kda_fwd_prep", st,
             (kda_fwd_prep<C, D, Tin><<<dim3(nc, H), kThreads, fwd_prep_smem<C, D>(), st>>>(dt, H, k, v, g, b, w)));
  for (int r = 1; r <= p.n_rounds; ++r) {
    const int s0 = p.round_seq_begin[r - 1], s1 = p.round_seq_begin[r];
    TPC_LAUNCH("kda_fwd_scan", st,
               (kda_fwd_scan<C, D, DVT><<<dim3(s1 - s0, H, D / DVT), kThreads, scan_smem<C, D, DVT>(), st>>>(
                   dt, s0, H, io->init_state, io->final_state, w)));
  }
  TPC_LAUNCH("kda_fwd_out", st,
             (kda_fwd_out<C, D, Tin, Tout><<<dim3(nc, H), kThreads, out_smem<C, D>(), st>>>(
                 dt, H, q, k, g, static_cast<Tout*>(io->o), w)));
  return TPC_OK;
}

// ------------------------------------------------------------------------------------------------
// Diagnostics: the bounded mbarrier wait every tensor-core kernel uses, on a barrier that nothing
// arrives on and with no copy or MMA in flight, so that the wait runs out and the timeout path
// (status word set, kernel returns, context intact) can be checked from the host.
__global__ void wait_timeout_probe(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tpc::tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const bool ok = tpc::tc::mbar_wait(&bar, 0, timeout_ns);
  const int failed = __syncthreads_or(ok ? 0 : 1);
  if (failed && threadIdx.x == 0) tpc::set_status(status, tpc::kStatusTimeout);
}


}  // namespace

extern "C" {

const char* tpc_last_error(void) { return tpc_abi::g_err.c_str(); }
const char* tpc_version(void) { return "tpc 0.1 (sm_100a)"; }

int tpc_plan_create_window(const int32_t* parent, const int32_t* length, int32_t n_nodes, int32_t chunk, int32_t mode,
                           int32_t n_exports, const int32_t* export_node, const int64_t* export_pos, tpc_plan** out) {
  if (!parent || !length || !out) return fail(TPC_ERR_NULL, "parent, length and out must be non-NULL");
  if (n_exports < 0 || (n_exports > 0 && (!export_node || !export_pos)))
    return fail(TPC_ERR_NULL, "export_node and export_pos are required when n_exports > 0");
  *out = nullptr;
  tpc_plan* p = new (std::nothrow) tpc_plan();
  if (!p) return fail(TPC_ERR_CUDA, "out of host memory");
  std::string err;
  try {
    err = tpc::build_plan(parent, length, n_nodes, chunk, p->p, mode, n_exports, export_node, export_pos);
  } catch (const std::exception& e) {
    err = std::string("planner: ") + e.what();
  }
  if (!err.empty()) {
    delete p;
    const bool unsup = err.find("chunk size") != std::string::npos || err.find("plan mode") != std::string::npos;
    return fail(unsup ? TPC_ERR_UNSUPPORTED : TPC_ERR_INVALID_TREE, err);
  }
  *out = p;
  return TPC_OK;
}

int tpc_plan_create_mode(const int32_t* parent, const int32_t* length, int32_t n_nodes, int32_t chunk, int32_t mode,
                         tpc_plan** out) {
  return tpc_plan_create_window(parent, length, n_nodes, chunk, mode, 0, nullptr, nullptr, out);
}

int tpc_plan_create(const int32_t* parent, const int32_t* length, int32_t n_nodes, int32_t chunk, tpc_plan** out) {
  return tpc_plan_create_mode(parent, length, n_nodes, chunk, TPC_PLAN_MIN_ROUNDS, out);
}

void tpc_plan_destroy(tpc_plan* plan) { delete plan; }

int tpc_plan_get_info(const tpc_plan* plan, tpc_plan_info* info) {
  if (!plan || !info) return fail(TPC_ERR_NULL, "plan or info is NULL");
  const tpc::Plan& p = plan->p;
  info->n_unique = p.n_unique;
  info->n_expanded = p.n_expanded;
  info->replay_total = p.replay_total;
  info->n_seq_tokens = p.n_unique + p.replay_total;
  info->n_nodes = p.n;
  info->n_rounds = p.n_rounds;
  info->n_seqs = (int32_t)p.seqs.size();
  info->n_chunks = (int32_t)p.chunks.size();
  info->n_slots = (int32_t)p.slots.size();
  info->n_leaves = (int32_t)p.leaves.size();
  info->n_roots = (int32_t)p.roots.size();
  info->chunk = p.C;
  info->max_seq_chunks = p.max_seq_chunks;
  info->n_replay_targets = (int32_t)p.tgt_row.size();
  info->n_exports = (int32_t)p.ext_slot.size();
  return TPC_OK;
}

int tpc_plan_export(const tpc_plan* plan, tpc_plan_tables* t) {
  if (!plan || !t) return fail(TPC_ERR_NULL, "plan or tables is NULL");
  const tpc::Plan& p = plan->p;
  auto cp = [](auto* dst, const auto& src) {
    if (dst) for (size_t i = 0; i < src.size(); ++i) dst[i] = src[i];
  };
  cp(t->round, p.round);
  cp(t->is_cont, p.is_cont);
  cp(t->anchor, p.anchor);
  cp(t->replay_start, p.replay_start);
  cp(t->replay_len, p.replay_len);
  cp(t->row_offset, p.row_offset);
  cp(t->occurrence, p.occurrence);
  cp(t->leaves, p.leaves);
  cp(t->expanded_rows, p.exp_rows64);
  cp(t->traj_offset, p.traj_offset);
  return TPC_OK;
}

int tpc_plan_debug_tables(const tpc_plan* plan, int32_t* seqs, int32_t* chunks, int32_t* slots, int32_t* slot_cons,
                          int32_t* replay_rows) {
  if (!plan) return fail(TPC_ERR_NULL, "plan is NULL");
  const tpc::Plan& p = plan->p;
  static_assert(sizeof(tpc::SeqRec) == 8 * 4 && sizeof(tpc::ChunkRec) == 8 * 4 && sizeof(tpc::SlotRec) == 4 * 4,
                "table records are rows of int32");
  if (seqs) std::memcpy(seqs, p.seqs.data(), p.seqs.size() * sizeof(tpc::SeqRec));
  if (chunks) std::memcpy(chunks, p.chunks.data(), p.chunks.size() * sizeof(tpc::ChunkRec));
  if (slots) std::memcpy(slots, p.slots.data(), p.slots.size() * sizeof(tpc::SlotRec));
  if (slot_cons) std::memcpy(slot_cons, p.slot_cons.data(), p.slot_cons.size() * 4);
  if (replay_rows) std::memcpy(replay_rows, p.replay_rows.data(), p.replay_rows.size() * 4);
  return TPC_OK;
}

size_t tpc_plan_device_bytes(const tpc_plan* plan) {
  if (!plan) return 0;
  std::vector<size_t> off;
  return tpc::device_layout(plan->p, off);
}

int tpc_plan_upload(tpc_plan* plan, void* dev, size_t bytes, tpc_stream_t stream) {
  if (!plan || !dev) return fail(TPC_ERR_NULL, "plan or device buffer is NULL");
  if (reinterpret_cast<uintptr_t>(dev) % 256) return fail(TPC_ERR_WORKSPACE, "device table buffer must be 256-byte aligned");
  std::vector<size_t> off;
  const size_t need = tpc::device_layout(plan->p, off);
  if (bytes < need) return fail(TPC_ERR_WORKSPACE, "device table buffer too small");
  std::vector<uint8_t> blob;
  tpc::pack_device_blob(plan->p, off, blob);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TPC_CUDA(cudaMemcpyAsync(dev, blob.data(), need, cudaMemcpyHostToDevice, st));
  // the pageable source is copied before cudaMemcpyAsync returns for host->device staging,
  // but make it explicit so that `blob` can be released
  TPC_CUDA(cudaStreamSynchronize(st));
  plan->p.dev = dev;
  plan->p.dev_bytes = bytes;
  plan->p.blob_offsets = off;
  plan->p.dt = tpc::device_view(plan->p, dev, off);
  return TPC_OK;
}

size_t tpc_kda_workspace_bytes(const tpc_plan* plan, const tpc_kda_shape* s) {
  if (!plan || !s || s->dk != s->dv || !shape_supported(plan->p.C, s->dk) || s->H < 1) return 0;
  return ws_layout(plan->p, s->H, plan->p.C, s->dk).total;
}

int tpc_kda_forward(const tpc_plan* plan, const tpc_kda_shape* s, const tpc_kda_fwd_io* io, void* ws, size_t ws_bytes,
                    tpc_stream_t stream) {
  if (int rc = check_shape(plan, s)) return rc;
  if (!io || !io->q || !io->k || !io->v || !io->g || !io->beta || !io->o || !ws)
    return fail(TPC_ERR_NULL, "forward: q, k, v, g, beta, o and ws are required");
  if (ws_bytes < tpc_kda_workspace_bytes(plan, s)) return fail(TPC_ERR_WORKSPACE, "workspace too small");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(TPC_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_kda_forward");
  return dispatch(plan, s, [&](auto CC, auto DD, auto tin, auto tout, auto tc) {
    return forward_impl<decltype(CC)::value, decltype(DD)::value, decltype(tin), decltype(tout), decltype(tc)::value>(
        plan->p, s, io, ws, st);
  });
}

int tpc_kda_backward_window(const tpc_plan* plan, const tpc_kda_shape* s, const tpc_kda_bwd_io* io,
                            const float* export_grads, void* ws, size_t ws_bytes, tpc_stream_t stream) {
  if (int rc = check_shape(plan, s)) return rc;
  if (!io || !io->q || !io->k || !io->v || !io->g || !io->beta || !io->d_o || !io->dq || !io->dk || !io->dv ||
      !io->dg || !io->dbeta || !ws)
    return fail(TPC_ERR_NULL, "backward: inputs, d_o, gradient outputs and ws are required");
  if (ws_bytes < tpc_kda_workspace_bytes(plan, s)) return fail(TPC_ERR_WORKSPACE, "workspace too small");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_kda_backward_window");
  // the external consumers' start-state gradients enter the reverse scans like in-tree consumers'
  const tpc::Plan& pl = plan->p;
  if (!pl.ext_slot.empty()) {
    const WsLayout L = ws_layout(pl, s->H, pl.C, s->dk);
    const size_t per = (size_t)s->H * s->dk * s->dv * 4;
    char* dst = static_cast<char*>(ws) + L.dS0seq + pl.seqs.size() * per;
    if (export_grads)
      TPC_CUDA(cudaMemcpyAsync(dst, export_grads, pl.ext_slot.size() * per, cudaMemcpyDeviceToDevice, st));
    else
      TPC_CUDA(cudaMemsetAsync(dst, 0, pl.ext_slot.size() * per, st));
  }
  return dispatch(plan, s, [&](auto CC, auto DD, auto tin, auto tout, auto tc) {
    return backward_impl<decltype(CC)::value, decltype(DD)::value, decltype(tin), decltype(tout), decltype(tc)::value>(
        plan->p, s, io, ws, st);
  });
}

int tpc_kda_backward(const tpc_plan* plan, const tpc_kda_shape* s, const tpc_kda_bwd_io* io, void* ws, size_t ws_bytes,
                     tpc_stream_t stream) {
  return tpc_kda_backward_window(plan, s, io, nullptr, ws, ws_bytes, stream);
}

int tpc_kda_export_states(const tpc_plan* plan, const tpc_kda_shape* s, const void* ws, float* states,
                          tpc_stream_t stream) {
  if (int rc = check_shape(plan, s)) return rc;
  if (!ws || !states) return fail(TPC_ERR_NULL, "ws and states are required");
  const tpc::Plan& pl = plan->p;
  const WsLayout L = ws_layout(pl, s->H, pl.C, s->dk);
  const size_t per = (size_t)s->H * s->dk * s->dv * 4;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  for (size_t e = 0; e < pl.ext_slot.size(); ++e)
    TPC_CUDA(cudaMemcpyAsync(reinterpret_cast<char*>(states) + e * per,
                             static_cast<const char*>(ws) + L.slot + (size_t)pl.ext_slot[e] * per, per,
                             cudaMemcpyDeviceToDevice, st));
  return TPC_OK;
}

int tpc_gather_rows(const void* src, const int32_t* rows, void* dst, int64_t n_rows, int64_t width, int32_t elem_bytes,
                    tpc_stream_t stream) {
  if (!src || !rows || !dst) return fail(TPC_ERR_NULL, "src, rows and dst are required");
  if (n_rows < 0 || width < 1 || (elem_bytes != 2 && elem_bytes != 4))
    return fail(TPC_ERR_BAD_SHAPE, "n_rows >= 0, width >= 1, elem_bytes 2 or 4");
  if (n_rows == 0) return TPC_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (elem_bytes == 2)
    TPC_LAUNCH("gather_rows", st, (tpc::gather_list_kernel<uint16_t><<<(unsigned)n_rows, 128, 0, st>>>(
                                      (const uint16_t*)src, rows, (uint16_t*)dst, width)));
  else
    TPC_LAUNCH("gather_rows", st, (tpc::gather_list_kernel<uint32_t><<<(unsigned)n_rows, 128, 0, st>>>(
                                      (const uint32_t*)src, rows, (uint32_t*)dst, width)));
  return TPC_OK;
}

int tpc_add_rows(const float* src, const int32_t* rows, float* dst, int64_t n_rows, int64_t width, tpc_stream_t stream) {
  if (!src || !rows || !dst) return fail(TPC_ERR_NULL, "src, rows and dst are required");
  if (n_rows < 0 || width < 1) return fail(TPC_ERR_BAD_SHAPE, "n_rows >= 0, width >= 1");
  if (n_rows == 0) return TPC_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TPC_LAUNCH("add_rows", st, (tpc::add_list_kernel<<<(unsigned)n_rows, 128, 0, st>>>(src, rows, dst, width)));
  return TPC_OK;
}

int tpc_status(const tpc_plan* plan, const tpc_kda_shape* s, void* ws, tpc_stream_t stream) {
  if (!plan || !s || !ws) return fail(TPC_ERR_NULL, "plan, shape or ws is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int code = 0;
  TPC_CUDA(cudaStreamSynchronize(st));
  TPC_CUDA(cudaMemcpy(&code, ws, 4, cudaMemcpyDeviceToHost));
  TPC_CUDA(cudaMemset(ws, 0, 4));
  if (code == TPC_ERR_RANGE) return fail(TPC_ERR_RANGE, "gate decay inside a 16-row sub-block exceeds 80 (log units)");
  if (code) return fail(TPC_ERR_DEVICE_CHECK, "kernel-side check failed with code " + std::to_string(code));
  return TPC_OK;
}

int tpc_reduce_expanded_to_unique(const tpc_plan* plan, const float* x_exp, float* x_unique, int64_t width,
                                  tpc_stream_t stream) {
  if (!plan || !x_exp || !x_unique) return fail(TPC_ERR_NULL, "plan or buffers NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (width < 1) return fail(TPC_ERR_BAD_SHAPE, "width must be >= 1");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  const int64_t N = plan->p.n_unique;
  TPC_LAUNCH("reduce_expanded", st,
             (tpc::reduce_expanded_kernel<<<(unsigned)N, 128, 0, st>>>(plan->p.dt, x_exp, x_unique, width)));
  return TPC_OK;
}

int tpc_gather_expanded(const tpc_plan* plan, const void* x_unique, void* x_exp, int64_t width, int32_t elem_bytes,
                        tpc_stream_t stream) {
  if (!plan || !x_unique || !x_exp) return fail(TPC_ERR_NULL, "plan or buffers NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (width < 1 || (elem_bytes != 2 && elem_bytes != 4)) return fail(TPC_ERR_BAD_SHAPE, "width >= 1, elem_bytes 2 or 4");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  const int64_t M = plan->p.n_expanded;
  if (elem_bytes == 2)
    TPC_LAUNCH("gather_expanded", st,
               (tpc::gather_rows_kernel<uint16_t><<<(unsigned)M, 128, 0, st>>>(
                   plan->p.dt, (const uint16_t*)x_unique, (uint16_t*)x_exp, width)));
  else
    TPC_LAUNCH("gather_expanded", st,
               (tpc::gather_rows_kernel<uint32_t><<<(unsigned)M, 128, 0, st>>>(
                   plan->p.dt, (const uint32_t*)x_unique, (uint32_t*)x_exp, width)));
  return TPC_OK;
}

int tpc_occurrence_counts(const tpc_plan* plan, int32_t* counts, tpc_stream_t stream) {
  if (!plan || !counts) return fail(TPC_ERR_NULL, "plan or counts NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  const int64_t N = plan->p.n_unique;
  TPC_LAUNCH("occurrence_count", st,
             (tpc::occurrence_count_kernel<<<(unsigned)((N + 255) / 256), 256, 0, st>>>(plan->p.dt, counts, N)));
  return TPC_OK;
}

int tpc_rope_positions(const tpc_plan* plan, int32_t* pos, tpc_stream_t stream) {
  if (!plan || !pos) return fail(TPC_ERR_NULL, "plan or pos is NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  TPC_LAUNCH("rope_positions", st, (tpc::rope_positions_kernel<<<plan->p.n, 128, 0, st>>>(plan->p.dt, pos)));
  return TPC_OK;
}

void tpc_profile_enable(int on) { g_prof.on = on != 0; }

long long tpc_launch_count(void) { return g_prof.launches; }

int tpc_profile_read(char* buf, size_t len) {
  if (!buf || len == 0) return fail(TPC_ERR_NULL, "buffer is NULL");
  std::vector<std::pair<std::string, std::pair<long long, double>>> acc;
  for (auto& r : g_prof.recs) {
    TPC_CUDA(cudaEventSynchronize(r.b));
    float ms = 0.f;
    TPC_CUDA(cudaEventElapsedTime(&ms, r.a, r.b));
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
    bool found = false;
    for (auto& e : acc)
      if (e.first == r.name) { e.second.first++; e.second.second += ms; found = true; }
    if (!found) acc.push_back({r.name, {1, (double)ms}});
  }
  g_prof.recs.clear();
  std::string out;
  for (auto& e : acc) out += e.first + " " + std::to_string(e.second.first) + " " + std::to_string(e.second.second) + "\n";
  std::snprintf(buf, len, "%s", out.c_str());
  return TPC_OK;
}

int tpc_kda_forward_static(const tpc_plan* plan, const tpc_kda_shape* s, const tpc_kda_fwd_io* io,
                           tpc_stream_t stream) {
  if (!plan || !s) return fail(TPC_ERR_NULL, "plan or shape is NULL");
  if (s->H < 1 || s->dk != s->dv) return fail(TPC_ERR_BAD_SHAPE, "H >= 1 and dk == dv required");
  if (!shape_supported(plan->p.C, s->dk)) return fail(TPC_ERR_UNSUPPORTED, "unsupported (chunk, d)");
  if ((s->in_dtype != TPC_F32 && s->in_dtype != TPC_BF16) || (s->out_dtype != TPC_F32 && s->out_dtype != TPC_BF16))
    return fail(TPC_ERR_UNSUPPORTED, "dtype must be TPC_F32 or TPC_BF16");
  if (!io || !io->q || !io->k || !io->v || !io->g || !io->beta || !io->o)
    return fail(TPC_ERR_NULL, "forward: q, k, v, g, beta and o are required");
  const tpc::Plan& p = plan->p;
  std::vector<size_t> off;
  const size_t table_bytes = tpc::device_layout(p, off);
  const size_t need = static_ws_layout(p, s->H, p.C, s->dk, kStaticStatusBytes + a256(table_bytes), nullptr, nullptr);
  if (need > (size_t)TPC_STATIC_SCRATCH_BYTES)
    return fail(TPC_ERR_WORKSPACE, "problem needs " + std::to_string(need) + " bytes of device scratch; the "
                "allocation-free forward holds at most " + std::to_string((size_t)TPC_STATIC_SCRATCH_BYTES));
  char* base = nullptr;
  if (int rc = static_base(&base)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tpc_abi::NvtxRange nvtx_call("tpc_kda_forward_static");
  // plan tables after the status word (pageable source: staged before cudaMemcpyAsync returns)
  std::vector<uint8_t> blob;
  tpc::pack_device_blob(p, off, blob);
  char* tables = base + kStaticStatusBytes;
  TPC_CUDA(cudaMemcpyAsync(tables, blob.data(), table_bytes, cudaMemcpyHostToDevice, st));
  if (tpc_abi::checks_on())  // the copy of the tables this call reads
    if (int rc = tpc_abi::table_checks_at(p, tables, off, st)) return rc;
  const tpc::DevTables dt = tpc::device_view(p, tables, off);
  tpc::KdaWs w;
  static_ws_layout(p, s->H, p.C, s->dk, kStaticStatusBytes + a256(table_bytes), &w, base);
  return dispatch(plan, s, [&](auto CC, auto DD, auto tin, auto tout, auto) {
    return forward_static_impl<decltype(CC)::value, decltype(DD)::value, decltype(tin), decltype(tout)>(p, dt, w, s, io,
                                                                                                        st);
  });
}

int tpc_debug_wait_timeout(int32_t* status, int64_t timeout_ns, tpc_stream_t stream) {
  if (!status) return fail(TPC_ERR_NULL, "status is NULL");
  if (timeout_ns < 1000 || timeout_ns > 100000000) return fail(TPC_ERR_BAD_SHAPE, "timeout_ns in [1e3, 1e8]");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  TPC_LAUNCH("wait_timeout_probe", st, (wait_timeout_probe<<<1, 32, 0, st>>>(status, (unsigned long long)timeout_ns)));
  return TPC_OK;
}

int tpc_kda_static_status(tpc_stream_t stream) {
  char* base = nullptr;
  if (int rc = static_base(&base)) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int code = 0;
  TPC_CUDA(cudaStreamSynchronize(st));
  TPC_CUDA(cudaMemcpy(&code, base, 4, cudaMemcpyDeviceToHost));
  TPC_CUDA(cudaMemset(base, 0, 4));
  if (code == TPC_ERR_RANGE) return fail(TPC_ERR_RANGE, "gate decay inside a 16-row sub-block exceeds 80 (log units)");
  if (code) return fail(TPC_ERR_DEVICE_CHECK, "kernel-side check failed with code " + std::to_string(code));
  return TPC_OK;
}

}  // extern "C"
