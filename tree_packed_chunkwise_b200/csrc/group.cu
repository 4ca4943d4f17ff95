// Hybrid layer group on the compact rows of a rollout tree (HARTS Table 1: KDA and MLA layers in a
// 3:1 group; Figure C.1: every layer type runs once per unique row; Table 7 and Section 4: layer
// activations are recomputed in the backward pass).  The forward keeps only each layer's input;
// the backward recomputes the layer from it, then runs the layer's adjoint.  Every step is one of
// this library's kernels: RMSNorm / projection epilogues (group_kernels.cuh), the tcgen05 GEMM,
// tree-packed KDA and tree-masked attention (reached through their C entry points).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <string>

#include "abi_internal.h"
#include "group_kernels.cuh"

namespace {

using tpc_abi::a256;
using tpc_abi::fail;
using namespace tpc;

constexpr int kRowThreads = 256;

bool group_supported(const tpc_group_shape* s) {
  return s->D == kGrpD && s->H == kGrpH && s->d_head == kGrpDH && s->d_rope == kGrpRope &&
         s->d_latent == kGrpLat && s->n_kda >= 0 && s->n_kda <= TPC_GROUP_MAX_KDA;
}

// the KDA layer runs the recurrence on fp32 inputs and outputs (tensor-core path, split products)
// fp32 activations on the tensor-core KDA kernels (bf16 hi/lo operands)
tpc_kda_shape kda_shape() { return tpc_kda_shape{kGrpH, kGrpDH, kGrpDH, TPC_F32_SPLIT, TPC_F32}; }

tpc_attn_shape attn_shape() {
  return tpc_attn_shape{kGrpH, kGrpQK, kGrpDH, 1.0f / sqrtf((float)kGrpQK), TPC_F32};
}

// a bf16 hi/lo pair of an fp32 tensor
struct Pair {
  bf16 *hi, *lo;
};

// Per-row buffers of one layer.  The KDA and MLA layouts share the same bytes (layers run one at a
// time); the first block holds what both use.
struct Bufs {
  int* status;
  int32_t* pos;
  Pair xn; float* rstd; float* P; float* o; Pair ob; Pair dy; float* dob; Pair dP; float* dxn;
  // KDA layer (fp32 recurrence inputs and gradients)
  float *q, *k, *v, *g, *beta, *knorm, *dq, *dk, *dv, *dg, *dbeta;
  // MLA layer
  Pair mq, mk, mc, mv, dob2, dKV; float *kr, *KV, *lse, *mdq, *mdk, *mdv, *delta, *dkr, *dc;
  void* kda_ws; size_t kda_ws_bytes;
  size_t total;
};

// carves the buffers for N rows from base (base == nullptr: sizes only)
Bufs carve(const tpc_plan* plan, char* base) {
  const size_t N = (size_t)plan->p.n_unique, D = kGrpD, H = kGrpH;
  Bufs b{};
  size_t o = 0;
  auto take = [&](size_t bytes) { char* r = base ? base + o : nullptr; o += a256(bytes); return r; };
  auto pair = [&](size_t n) { Pair p; p.hi = (bf16*)take(n * 2); p.lo = (bf16*)take(n * 2); return p; };
  b.status = (int*)take(256);
  b.pos = (int32_t*)take(N * 4);
  b.xn = pair(N * D);
  b.rstd = (float*)take(N * 4);
  b.P = (float*)take(N * kKdaProj * 4);
  b.o = (float*)take(N * D * 4);
  b.ob = pair(N * D);
  b.dy = pair(N * D);
  b.dob = (float*)take(N * D * 4);
  b.dP = pair(N * kKdaProj);
  b.dxn = (float*)take(N * D * 4);
  const size_t common = o;
  b.q = (float*)take(N * D * 4);
  b.k = (float*)take(N * D * 4);
  b.v = (float*)take(N * D * 4);
  b.g = (float*)take(N * D * 4);
  b.beta = (float*)take(N * H * 4);
  b.knorm = (float*)take(N * H * 4);
  b.dq = (float*)take(N * D * 4);
  b.dk = (float*)take(N * D * 4);
  b.dv = (float*)take(N * D * 4);
  b.dg = (float*)take(N * D * 4);
  b.dbeta = (float*)take(N * H * 4);
  const size_t kda_end = o;
  o = common;
  b.mq = pair(N * H * kGrpQK);
  b.mc = pair(N * kGrpLat);
  b.kr = (float*)take(N * kGrpRope * 4);
  b.KV = (float*)take(N * 2 * D * 4);
  b.mk = pair(N * H * kGrpQK);
  b.mv = pair(N * D);
  b.lse = (float*)take(N * H * 4);
  b.dob2 = pair(N * D);
  b.mdq = (float*)take(N * H * kGrpQK * 4);
  b.mdk = (float*)take(N * H * kGrpQK * 4);
  b.mdv = (float*)take(N * D * 4);
  b.delta = (float*)take(N * H * 4);
  b.dKV = pair(N * 2 * D);
  b.dkr = (float*)take(N * kGrpRope * 4);
  b.dc = (float*)take(N * kGrpLat * 4);
  o = o > kda_end ? o : kda_end;
  const tpc_kda_shape ks = kda_shape();
  b.kda_ws_bytes = tpc_kda_workspace_bytes(plan, &ks);
  b.kda_ws = take(b.kda_ws_bytes);
  b.total = o;
  return b;
}

int grid_rows(const tpc_plan* plan) { return (int)plan->p.n_unique; }

#define TPC_TRY(call)             \
  do {                            \
    const int r_ = (call);        \
    if (r_ != TPC_OK) return r_;  \
  } while (0)

// C[M][N] (fp32) = A op B with fp32 activations as hi/lo pairs: a weight operand W (exact bf16)
// takes two tensor-core passes, two activation pairs take three
int gemm_aw(const Pair& A, const void* W, float* C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
            int64_t ldc, int b_mn, float beta, int* status, cudaStream_t st) {
  return tpc_gemm_split(A.hi, A.lo, W, nullptr, C, M, N, K, lda, ldb, ldc, 0, b_mn, TPC_F32, 1.f, beta, status, st);
}
int gemm_aa(const Pair& A, const Pair& B, float* C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
            int64_t ldc, int* status, cudaStream_t st) {
  return tpc_gemm_split(A.hi, A.lo, B.hi, B.lo, C, M, N, K, lda, ldb, ldc, 1, 1, TPC_F32, 1.f, 0.f, status, st);
}

int split(const float* x, const Pair& y, int64_t n, cudaStream_t st) {
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  TPC_LAUNCH("split_bf16", st, split_bf16_kernel<<<blocks, 256, 0, st>>>(x, y.hi, y.lo, n));
  return TPC_OK;
}

// ---------------------------------------------------------------- KDA layer
// y = x + KDA(q, k, v, g, beta) W_o^T with q, k, v, g, beta from RMSNorm(x) (HARTS Table 1).
// Leaves xn, P, q..beta, knorm, o and the KDA forward workspace in b for the backward.
int kda_layer_forward(const tpc_plan* plan, const tpc_group_kda_weights& w, const float* x, float* y, Bufs& b,
                      cudaStream_t st) {
  const int64_t N = plan->p.n_unique;
  const int rows = grid_rows(plan);
  TPC_LAUNCH("rmsnorm_fwd", st,
             rmsnorm_fwd_kernel<<<rows, kRowThreads, 0, st>>>(x, b.xn.hi, b.xn.lo, b.rstd, kGrpD));
  TPC_TRY(gemm_aw(b.xn, w.w_in, b.P, N, kKdaProj, kGrpD, kGrpD, kGrpD, kKdaProj, 0, 0.f, b.status, st));
  TPC_LAUNCH("kda_post", st,
             kda_post_kernel<<<rows, kRowThreads, 0, st>>>(b.P, b.q, b.k, b.v, b.g, b.beta, b.knorm));
  const tpc_kda_shape ks = kda_shape();
  tpc_kda_fwd_io io{};
  io.q = b.q; io.k = b.k; io.v = b.v; io.g = b.g; io.beta = b.beta;
  io.init_state = nullptr; io.o = b.o; io.final_state = nullptr;
  TPC_TRY(tpc_kda_forward(plan, &ks, &io, b.kda_ws, b.kda_ws_bytes, st));
  TPC_TRY(split(b.o, b.ob, N * kGrpD, st));
  if (y) {
    if (y != x) TPC_CUDA(cudaMemcpyAsync(y, x, N * kGrpD * 4, cudaMemcpyDeviceToDevice, st));
    TPC_TRY(gemm_aw(b.ob, w.w_o, y, N, kGrpD, kGrpD, kGrpD, kGrpD, kGrpD, 0, 1.f, b.status, st));
  }
  return TPC_OK;
}

// dx (in place: holds dy on entry) of the KDA layer whose input is x; weight gradients overwritten
int kda_layer_backward(const tpc_plan* plan, const tpc_group_kda_weights& w, const tpc_group_kda_grads& gr,
                       const float* x, float* dx, Bufs& b, cudaStream_t st) {
  const int64_t N = plan->p.n_unique;
  const int rows = grid_rows(plan);
  TPC_TRY(kda_layer_forward(plan, w, x, nullptr, b, st));  // recompute
  TPC_TRY(split(dx, b.dy, N * kGrpD, st));
  // d(o) = dy W_o;  dW_o = dy^T o
  TPC_TRY(gemm_aw(b.dy, w.w_o, b.dob, N, kGrpD, kGrpD, kGrpD, kGrpD, kGrpD, 1, 0.f, b.status, st));
  TPC_TRY(gemm_aa(b.dy, b.ob, gr.w_o, kGrpD, kGrpD, N, kGrpD, kGrpD, kGrpD, b.status, st));
  const tpc_kda_shape ks = kda_shape();
  tpc_kda_bwd_io io{};
  io.q = b.q; io.k = b.k; io.v = b.v; io.g = b.g; io.beta = b.beta; io.init_state = nullptr;
  io.d_o = b.dob; io.d_final = nullptr;
  io.dq = b.dq; io.dk = b.dk; io.dv = b.dv; io.dg = b.dg; io.dbeta = b.dbeta; io.d_init = nullptr;
  TPC_TRY(tpc_kda_backward(plan, &ks, &io, b.kda_ws, b.kda_ws_bytes, st));
  TPC_LAUNCH("kda_post_bwd", st,
             kda_post_bwd_kernel<<<rows, kRowThreads, 0, st>>>(b.P, b.knorm, b.dq, b.dk, b.dv, b.dg, b.dbeta,
                                                               b.dP.hi, b.dP.lo));
  // dxn = dP W_in;  dW_in = dP^T xn
  TPC_TRY(gemm_aw(b.dP, w.w_in, b.dxn, N, kGrpD, kKdaProj, kKdaProj, kGrpD, kGrpD, 1, 0.f, b.status, st));
  TPC_TRY(gemm_aa(b.dP, b.xn, gr.w_in, kKdaProj, kGrpD, N, kKdaProj, kGrpD, kGrpD, b.status, st));
  TPC_LAUNCH("rmsnorm_bwd", st,
             rmsnorm_bwd_kernel<<<rows, kRowThreads, 0, st>>>(x, b.rstd, b.dxn, dx, dx, kGrpD));
  return TPC_OK;
}

// ---------------------------------------------------------------- MLA layer
// Latent attention: q (16 x (128 + 64 rotary)), c (512), shared rotary key kr (64) from RMSNorm(x);
// k_nope and v from c; tree-masked softmax attention at tree-depth positions; y = x + o W_o^T.
int mla_layer_forward(const tpc_plan* plan, const tpc_group_mla_weights& w, const float* x, float* y, Bufs& b,
                      cudaStream_t st) {
  const int64_t N = plan->p.n_unique;
  const int rows = grid_rows(plan);
  TPC_LAUNCH("rmsnorm_fwd", st,
             rmsnorm_fwd_kernel<<<rows, kRowThreads, 0, st>>>(x, b.xn.hi, b.xn.lo, b.rstd, kGrpD));
  TPC_TRY(gemm_aw(b.xn, w.w_a, b.P, N, kMlaProj, kGrpD, kGrpD, kGrpD, kMlaProj, 0, 0.f, b.status, st));
  TPC_LAUNCH("mla_post", st,
             mla_post_kernel<<<rows, kRowThreads, 0, st>>>(b.P, b.pos, b.mq.hi, b.mq.lo, b.mc.hi, b.mc.lo, b.kr));
  TPC_TRY(gemm_aw(b.mc, w.w_b, b.KV, N, 2 * kGrpD, kGrpLat, kGrpLat, kGrpLat, 2 * kGrpD, 0, 0.f, b.status, st));
  TPC_LAUNCH("mla_kv", st,
             mla_kv_kernel<<<rows, kRowThreads, 0, st>>>(b.KV, b.kr, b.mk.hi, b.mk.lo, b.mv.hi, b.mv.lo));
  const tpc_attn_shape as = attn_shape();
  const tpc_attn_lo lo{b.mq.lo, b.mk.lo, b.mv.lo, nullptr};
  TPC_TRY(tpc_tree_attn_forward(plan, &as, b.mq.hi, b.mk.hi, b.mv.hi, &lo, b.o, b.lse, b.status, st));
  TPC_TRY(split(b.o, b.ob, N * kGrpD, st));
  if (y) {
    if (y != x) TPC_CUDA(cudaMemcpyAsync(y, x, N * kGrpD * 4, cudaMemcpyDeviceToDevice, st));
    TPC_TRY(gemm_aw(b.ob, w.w_o, y, N, kGrpD, kGrpD, kGrpD, kGrpD, kGrpD, 0, 1.f, b.status, st));
  }
  return TPC_OK;
}

// resident: the workspace still holds this layer's forward (it was the last layer of the forward)
int mla_layer_backward(const tpc_plan* plan, const tpc_group_mla_weights& w, const tpc_group_mla_grads& gr,
                       const float* x, float* dx, Bufs& b, bool resident, cudaStream_t st) {
  const int64_t N = plan->p.n_unique;
  const int rows = grid_rows(plan);
  if (!resident) TPC_TRY(mla_layer_forward(plan, w, x, nullptr, b, st));  // recompute
  TPC_TRY(split(dx, b.dy, N * kGrpD, st));
  TPC_TRY(gemm_aw(b.dy, w.w_o, b.dob, N, kGrpD, kGrpD, kGrpD, kGrpD, kGrpD, 1, 0.f, b.status, st));
  TPC_TRY(gemm_aa(b.dy, b.ob, gr.w_o, kGrpD, kGrpD, N, kGrpD, kGrpD, kGrpD, b.status, st));
  TPC_TRY(split(b.dob, b.dob2, N * kGrpD, st));
  const tpc_attn_shape as = attn_shape();
  const tpc_attn_lo lo{b.mq.lo, b.mk.lo, b.mv.lo, b.dob2.lo};
  TPC_TRY(tpc_tree_attn_backward(plan, &as, b.mq.hi, b.mk.hi, b.mv.hi, &lo, b.o, b.lse, b.dob2.hi, b.mdq, b.mdk,
                                 b.mdv, b.delta, b.status, st));
  TPC_LAUNCH("mla_kv_bwd", st,
             mla_kv_bwd_kernel<<<rows, kRowThreads, 0, st>>>(b.mdk, b.mdv, b.dKV.hi, b.dKV.lo, b.dkr));
  // dc = dKV W_b;  dW_b = dKV^T c
  TPC_TRY(gemm_aw(b.dKV, w.w_b, b.dc, N, kGrpLat, 2 * kGrpD, 2 * kGrpD, kGrpLat, kGrpLat, 1, 0.f, b.status, st));
  TPC_TRY(gemm_aa(b.dKV, b.mc, gr.w_b, 2 * kGrpD, kGrpLat, N, 2 * kGrpD, kGrpLat, kGrpLat, b.status, st));
  TPC_LAUNCH("mla_post_bwd", st,
             mla_post_bwd_kernel<<<rows, kRowThreads, 0, st>>>(b.mdq, b.dc, b.dkr, b.pos, b.dP.hi, b.dP.lo));
  TPC_TRY(gemm_aw(b.dP, w.w_a, b.dxn, N, kGrpD, kMlaProj, kMlaProj, kGrpD, kGrpD, 1, 0.f, b.status, st));
  TPC_TRY(gemm_aa(b.dP, b.xn, gr.w_a, kMlaProj, kGrpD, N, kMlaProj, kGrpD, kGrpD, b.status, st));
  TPC_LAUNCH("rmsnorm_bwd", st,
             rmsnorm_bwd_kernel<<<rows, kRowThreads, 0, st>>>(x, b.rstd, b.dxn, dx, dx, kGrpD));
  return TPC_OK;
}

int check_group(const tpc_plan* plan, const tpc_group_shape* s, const tpc_group_weights* w, void* ws, size_t bytes,
                Bufs* b) {
  if (!plan || !s || !w || !ws) return fail(TPC_ERR_NULL, "plan, shape, weights or workspace is NULL");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded (tpc_plan_upload)");
  if (!group_supported(s))
    return fail(TPC_ERR_UNSUPPORTED, "layer group is built for D 2048, 16 heads of 128, rotary 64, latent 512, "
                                     "at most " + std::to_string(TPC_GROUP_MAX_KDA) + " KDA layers");
  if (plan->p.C != 64) return fail(TPC_ERR_UNSUPPORTED, "layer group needs a chunk-64 plan");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(TPC_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  for (int l = 0; l < s->n_kda; ++l)
    if (!w->kda[l].w_in || !w->kda[l].w_o) return fail(TPC_ERR_NULL, "KDA layer weight is NULL");
  if (!w->mla.w_a || !w->mla.w_b || !w->mla.w_o) return fail(TPC_ERR_NULL, "MLA layer weight is NULL");
  *b = carve(plan, static_cast<char*>(ws));
  if (bytes < b->total)
    return fail(TPC_ERR_WORKSPACE, "group workspace needs " + std::to_string(b->total) + " bytes");
  return TPC_OK;
}

}  // namespace

extern "C" {

size_t tpc_group_workspace_bytes(const tpc_plan* plan, const tpc_group_shape* s) {
  if (!plan || !s || !group_supported(s) || plan->p.C != 64) return 0;
  return carve(plan, nullptr).total;
}

int tpc_group_forward(const tpc_plan* plan, const tpc_group_shape* s, const tpc_group_weights* w, const float* x,
                      float* h, float* y, void* ws, size_t ws_bytes, tpc_stream_t stream) {
  Bufs b;
  TPC_TRY(check_group(plan, s, w, ws, ws_bytes, &b));
  if (!x || !y || (s->n_kda > 0 && !h)) return fail(TPC_ERR_NULL, "x, y or h is NULL");
  cudaStream_t st = stream;
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_group_forward");
  const size_t ND = (size_t)plan->p.n_unique * kGrpD;
  TPC_CUDA(cudaMemsetAsync(b.status, 0, 4, st));
  TPC_TRY(tpc_rope_positions(plan, b.pos, st));
  const float* in = x;
  for (int l = 0; l < s->n_kda; ++l) {
    float* out = h + l * ND;
    TPC_TRY(kda_layer_forward(plan, w->kda[l], in, out, b, st));
    in = out;
  }
  TPC_TRY(mla_layer_forward(plan, w->mla, in, y, b, st));
  return TPC_OK;
}

int tpc_group_backward(const tpc_plan* plan, const tpc_group_shape* s, const tpc_group_weights* w, const float* x,
                       const float* h, const float* dy, float* dx, const tpc_group_grads* g, void* ws,
                       size_t ws_bytes, tpc_stream_t stream) {
  Bufs b;
  TPC_TRY(check_group(plan, s, w, ws, ws_bytes, &b));
  if (!x || !dy || !dx || !g || (s->n_kda > 0 && !h)) return fail(TPC_ERR_NULL, "x, h, dy, dx or grads is NULL");
  for (int l = 0; l < s->n_kda; ++l)
    if (!g->kda[l].w_in || !g->kda[l].w_o) return fail(TPC_ERR_NULL, "KDA weight gradient is NULL");
  if (!g->mla.w_a || !g->mla.w_b || !g->mla.w_o) return fail(TPC_ERR_NULL, "MLA weight gradient is NULL");
  cudaStream_t st = stream;
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_group_backward");
  const size_t ND = (size_t)plan->p.n_unique * kGrpD;
  TPC_CUDA(cudaMemsetAsync(b.status, 0, 4, st));
  TPC_TRY(tpc_rope_positions(plan, b.pos, st));
  if (dx != dy) TPC_CUDA(cudaMemcpyAsync(dx, dy, ND * 4, cudaMemcpyDeviceToDevice, st));
  const float* mla_in = s->n_kda > 0 ? h + (s->n_kda - 1) * ND : x;
  TPC_TRY(mla_layer_backward(plan, w->mla, g->mla, mla_in, dx, b, s->reuse_forward != 0, st));
  for (int l = s->n_kda - 1; l >= 0; --l) {
    const float* in = l > 0 ? h + (l - 1) * ND : x;
    TPC_TRY(kda_layer_backward(plan, w->kda[l], g->kda[l], in, dx, b, st));
  }
  return TPC_OK;
}

int tpc_group_status(const tpc_plan* plan, const tpc_group_shape* s, void* ws, tpc_stream_t stream) {
  if (!plan || !s || !ws) return fail(TPC_ERR_NULL, "plan, shape or workspace is NULL");
  if (!group_supported(s)) return fail(TPC_ERR_UNSUPPORTED, "unsupported group shape");
  Bufs b = carve(plan, static_cast<char*>(ws));
  int code = 0;
  TPC_CUDA(cudaMemcpyAsync(&code, b.status, 4, cudaMemcpyDeviceToHost, stream));
  TPC_CUDA(cudaStreamSynchronize(stream));
  TPC_CUDA(cudaMemsetAsync(b.status, 0, 4, stream));
  const tpc_kda_shape ks = kda_shape();
  const int kda = tpc_status(plan, &ks, b.kda_ws, stream);
  if (code != TPC_OK) return fail(code, "layer group kernel reported status " + std::to_string(code));
  return kda;
}

}  // extern "C"
