// C ABI of the tree-packed chunkwise KDA library: compact MoE routing with occurrence counts.
// Declarations and contracts in include/tpc.h.
#include <algorithm>
#include <cuda_runtime.h>

#include <string>

#include "../../include/tpc.h"
#include "abi_internal.h"
#include "moe_kernels.cuh"
#include "plan.h"

namespace {
using tpc_abi::a256;
using tpc_abi::fail;
using tpc_abi::g_prof;
using tpc_abi::set_smem;

int moe_parts(const tpc_plan* plan) { return (int)((plan->p.n_unique + tpc::kMoeRows - 1) / tpc::kMoeRows); }
}  // namespace

extern "C" {

size_t tpc_moe_scratch_bytes(const tpc_plan* plan, int32_t E) {
  if (!plan || E < 1 || E > tpc::kMoeMaxE) return 0;
  const size_t parts = (size_t)moe_parts(plan);
  return a256(parts * E * 8) + a256(parts * E * 4) + a256(((size_t)plan->p.n_unique / 8 + 1) * 4);
}

int tpc_moe_route(const tpc_plan* plan, const void* h, const void* w_router, int64_t Dh, int32_t E, int32_t k,
                  float* logits, float* lse, int32_t* topk_idx, float* topk_gate, int64_t* expert_load,
                  float* prob_sum, void* scratch, size_t scratch_bytes, tpc_stream_t stream) {
  if (!plan || !h || !w_router || !logits || !lse || !topk_idx || !topk_gate || !expert_load || !prob_sum || !scratch)
    return fail(TPC_ERR_NULL, "moe route: NULL argument");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (E < 1 || E > tpc::kMoeMaxE || k < 1 || k > tpc::kMoeMaxK || k > E)
    return fail(TPC_ERR_UNSUPPORTED, "moe route: 1 <= k <= min(E, 8), E <= 256");
  if (Dh < tpc::kMoeCK || Dh % tpc::kMoeCK) return fail(TPC_ERR_BAD_SHAPE, "moe route: Dh a multiple of 64");
  if (scratch_bytes < tpc_moe_scratch_bytes(plan, E)) return fail(TPC_ERR_WORKSPACE, "moe route: scratch too small");
  const int N = (int)plan->p.n_unique, parts = moe_parts(plan);
  char* sc = static_cast<char*>(scratch);
  auto* part_load = reinterpret_cast<long long*>(sc);
  auto* part_prob = reinterpret_cast<float*>(sc + a256((size_t)parts * E * 8));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_moe_route");
  // rows per thread of the logits tiling: 32 rows x QP expert quads over the CTA's threads
  const int rt = std::max(1, tpc::kMoeRows * tpc::moe_quads_p2(E) / tpc::kMoeThreads);
  auto go = [&](auto rpt) -> int {
    constexpr int RT = decltype(rpt)::value;
    TPC_CUDA(set_smem(tpc::moe_route_kernel<RT>, tpc::MoeSmem::total));
    TPC_LAUNCH("moe_route", st, (tpc::moe_route_kernel<RT><<<parts, tpc::kMoeThreads, tpc::MoeSmem::total, st>>>(
                                    plan->p.dt, (const __nv_bfloat16*)h, (const __nv_bfloat16*)w_router, (int)Dh, E, k,
                                    N, logits, lse, topk_idx, topk_gate, part_load, part_prob)));
    return TPC_OK;
  };
  int rc;
  if (rt <= 1) rc = go(std::integral_constant<int, 1>{});
  else if (rt <= 2) rc = go(std::integral_constant<int, 2>{});
  else if (rt <= 4) rc = go(std::integral_constant<int, 4>{});
  else rc = go(std::integral_constant<int, 8>{});
  if (rc) return rc;
  TPC_LAUNCH("moe_reduce", st, (tpc::moe_reduce_kernel<<<E, tpc::kMoeThreads, 0, st>>>(
                                   part_load, part_prob, parts, E, (long long*)expert_load, prob_sum)));
  return TPC_OK;
}

int tpc_moe_router_loss(const tpc_plan* plan, const float* logits, const float* lse, const int64_t* expert_load,
                        const float* prob_sum, int32_t E, int32_t k, float a, float b, float* losses, float* dlogits,
                        void* scratch, size_t scratch_bytes, tpc_stream_t stream) {
  if (!plan || !logits || !lse || !expert_load || !prob_sum || !losses || !dlogits || !scratch)
    return fail(TPC_ERR_NULL, "moe loss: NULL argument");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (E < 1 || E > tpc::kMoeMaxE || k < 1 || k > tpc::kMoeMaxK || k > E)
    return fail(TPC_ERR_UNSUPPORTED, "moe loss: 1 <= k <= min(E, 8), E <= 256");
  if (scratch_bytes < tpc_moe_scratch_bytes(plan, E)) return fail(TPC_ERR_WORKSPACE, "moe loss: scratch too small");
  const int N = (int)plan->p.n_unique, parts = moe_parts(plan);
  const double n_exp = (double)plan->p.n_expanded;
  const float alpha = (float)(E / ((double)k * n_exp * n_exp));
  char* sc = static_cast<char*>(scratch);
  auto* part_z = reinterpret_cast<float*>(sc + a256((size_t)parts * E * 8) + a256((size_t)parts * E * 4));
  const int rows_per = tpc::kMoeThreads / 32, nblk = (N + rows_per - 1) / rows_per;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_moe_router_loss");
  TPC_LAUNCH("moe_loss_grad", st, (tpc::moe_loss_grad_kernel<<<nblk, tpc::kMoeThreads, 0, st>>>(
                                      plan->p.dt, logits, lse, (const long long*)expert_load, E, N, a * alpha,
                                      (float)(b / n_exp), dlogits, part_z)));
  TPC_LAUNCH("moe_losses", st, (tpc::moe_losses_kernel<<<1, tpc::kMoeThreads, 0, st>>>(
                                   (const long long*)expert_load, prob_sum, E, part_z, nblk, alpha, (float)(1.0 / n_exp),
                                   losses)));
  return TPC_OK;
}

}  // extern "C"
