// C ABI of the tree-packed chunkwise KDA library: dense products (tree-masked attention).
// Declarations and contracts in include/tpc.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <string>
#include <type_traits>

#include "../../include/tpc.h"
#include <cudaTypedefs.h>
#include "abi_internal.h"
#include "plan.h"
#include "attn_tc.cuh"

namespace {
using tpc_abi::fail;
using tpc_abi::g_prof;
using tpc_abi::set_smem;
using tpc_abi::tensor_map_rows;
}  // namespace

extern "C" {

namespace {
int attn_check(const tpc_plan* plan, const tpc_attn_shape* s) {
  if (!plan || !s) return fail(TPC_ERR_NULL, "attention: plan or shape is NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (s->d_qk != tpc::kAttnQK || s->d_v != tpc::kAttnDV || s->H < 1)
    return fail(TPC_ERR_UNSUPPORTED, "attention: built for d_qk = 192, d_v = 128");
  if (s->io_dtype != TPC_F32 && s->io_dtype != TPC_BF16) return fail(TPC_ERR_UNSUPPORTED, "attention: io dtype");
  return TPC_OK;
}
}  // namespace

int tpc_tree_attn_forward(const tpc_plan* plan, const tpc_attn_shape* s, const void* q, const void* k, const void* v,
                          const tpc_attn_lo* lo, void* o, float* lse, int32_t* status, tpc_stream_t stream) {
  if (int rc = attn_check(plan, s)) return rc;
  if (!q || !k || !v || !o || !lse) return fail(TPC_ERR_NULL, "attention forward: NULL tensor");
  const tpc_attn_lo L = lo ? *lo : tpc_attn_lo{};
  const bool split = L.q || L.k || L.v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_tree_attn_forward");
  const tpc::Plan& p = plan->p;
  const dim3 grid((unsigned)(p.attn_qtiles.size() * (size_t)s->H));  // (query tile, head), query tiles fastest
  using bf = __nv_bfloat16;
  const uint64_t NR = (uint64_t)p.n_unique;
  CUtensorMap tk, tkl, tv, tvl;
  bool ok = tensor_map_rows(&tk, k, tpc::kAttnQK, s->H, NR, 64) && tensor_map_rows(&tv, v, tpc::kAttnDV, s->H, NR, 64);
  ok = ok && tensor_map_rows(&tkl, L.k ? L.k : k, tpc::kAttnQK, s->H, NR, 64) &&
       tensor_map_rows(&tvl, L.v ? L.v : v, tpc::kAttnDV, s->H, NR, 64);
  if (!ok) return fail(TPC_ERR_CUDA, "attention forward: cuTensorMapEncodeTiled failed");
  auto go = [&](auto tout, auto split) -> int {
    using T = decltype(tout);
    constexpr bool SP = decltype(split)::value;
    constexpr size_t smem = tpc::AttnFwdSmem<SP>::total;
    TPC_CUDA(set_smem(tpc::attn_fwd_tc<T, SP>, smem));
    TPC_LAUNCH("attn_fwd_tc", st,
               (tpc::attn_fwd_tc<T, SP><<<grid, tpc::kAttnFwdThreads, smem, st>>>(
                   p.dt, s->H, s->scale, (const bf*)q, (const bf*)L.q, tk, tkl, tv, tvl, (T*)o, lse, status)));
    return TPC_OK;
  };
  using Y = std::true_type;
  using N = std::false_type;
  if (s->io_dtype == TPC_BF16) return split ? go(bf{}, Y{}) : go(bf{}, N{});
  return split ? go(float{}, Y{}) : go(float{}, N{});
}

int tpc_tree_attn_backward(const tpc_plan* plan, const tpc_attn_shape* s, const void* q, const void* k,
                           const void* v, const tpc_attn_lo* lo, const void* o, const float* lse, const void* d_o,
                           void* dq, void* dk, void* dv, float* delta, int32_t* status, tpc_stream_t stream) {
  if (int rc = attn_check(plan, s)) return rc;
  if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv || !delta)
    return fail(TPC_ERR_NULL, "attention backward: NULL tensor");
  const tpc_attn_lo L = lo ? *lo : tpc_attn_lo{};
  const bool split = L.q || L.k || L.v || L.d_o;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_tree_attn_backward");
  const tpc::Plan& p = plan->p;
  using bf = __nv_bfloat16;
  const dim3 gq((unsigned)(p.attn_qtiles.size() * (size_t)s->H));  // (query tile, head), query tiles fastest
  const dim3 gk((unsigned)(p.attn_ktiles.size() * (size_t)s->H));  // (key tile, head), key tiles fastest
  const uint64_t NR = (uint64_t)p.n_unique;
  const unsigned Hh = (unsigned)s->H;
  CUtensorMap tk, tkl, tv, tvl, to, tol, tq32, tql32, to32, tol32;
  bool ok = tensor_map_rows(&tk, k, tpc::kAttnQK, Hh, NR, 64) && tensor_map_rows(&tv, v, tpc::kAttnDV, Hh, NR, 64) &&
            tensor_map_rows(&tkl, L.k ? L.k : k, tpc::kAttnQK, Hh, NR, 64) &&
            tensor_map_rows(&tvl, L.v ? L.v : v, tpc::kAttnDV, Hh, NR, 64) &&
            tensor_map_rows(&to, d_o, tpc::kAttnDV, Hh, NR, 128) &&
            tensor_map_rows(&tol, L.d_o ? L.d_o : d_o, tpc::kAttnDV, Hh, NR, 128);
  constexpr uint32_t QT = tpc::AttnDkvSmem<true>::QT;
  ok = ok && tensor_map_rows(&tq32, q, tpc::kAttnQK, Hh, NR, QT) &&
       tensor_map_rows(&tql32, L.q ? L.q : q, tpc::kAttnQK, Hh, NR, QT) &&
       tensor_map_rows(&to32, d_o, tpc::kAttnDV, Hh, NR, QT) &&
       tensor_map_rows(&tol32, L.d_o ? L.d_o : d_o, tpc::kAttnDV, Hh, NR, QT);
  CUtensorMap tk128, tkl128;  // key tiles of the dK / dV kernel
  constexpr uint32_t KT = tpc::AttnDkvSmem<true>::KT;
  ok = ok && tensor_map_rows(&tk128, k, tpc::kAttnQK, Hh, NR, KT) &&
       tensor_map_rows(&tkl128, L.k ? L.k : k, tpc::kAttnQK, Hh, NR, KT);
  if (!ok) return fail(TPC_ERR_CUDA, "attention backward: cuTensorMapEncodeTiled failed");
  auto go = [&](auto tio, auto split) -> int {
    using T = decltype(tio);
    constexpr bool SP = decltype(split)::value;
    constexpr size_t sq = tpc::AttnDqSmem<SP>::total, sk = tpc::AttnDkvSmem<SP>::total;
    TPC_CUDA(set_smem(tpc::attn_bwd_dq_tc<T, SP>, sq));
    TPC_CUDA(set_smem(tpc::attn_bwd_dkv_tc<T, SP>, sk));
    TPC_LAUNCH("attn_bwd_dq_tc", st,
               (tpc::attn_bwd_dq_tc<T, SP><<<gq, tpc::kAttnDqThreads, sq, st>>>(
                   p.dt, s->H, s->scale, (const bf*)q, (const bf*)L.q, tk, tkl, tv, tvl, to, tol, (const T*)o, lse,
                   (const bf*)d_o, (const bf*)L.d_o, (T*)dq, delta, status)));
    TPC_LAUNCH("attn_bwd_dkv_tc", st,
               (tpc::attn_bwd_dkv_tc<T, SP><<<gk, tpc::kAttnDkvThreads, sk, st>>>(
                   p.dt, s->H, s->scale, (const bf*)v, (const bf*)L.v, tq32, tql32, tk128, tkl128, to32, tol32, lse,
                   delta, (T*)dk, (T*)dv, status)));
    return TPC_OK;
  };
  using Y = std::true_type;
  using N = std::false_type;
  if (s->io_dtype == TPC_BF16) return split ? go(bf{}, Y{}) : go(bf{}, N{});
  return split ? go(float{}, Y{}) : go(float{}, N{});
}



}  // extern "C"
