// C ABI of the tree-packed chunkwise KDA library: dense products (tensor-core GEMM, log-probability recovery).
// Declarations and contracts in include/tpc.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <string>
#include <type_traits>

#include "../../include/tpc.h"
#include <cudaTypedefs.h>
#include "abi_internal.h"
#include "plan.h"
#include "gemm_tc.cuh"
#include "logprob_kernels.cuh"

namespace {
using tpc_abi::a256;
using tpc_abi::fail;
using tpc_abi::g_prof;
using tpc_abi::set_smem;
using tpc_abi::sm_count;
using tpc_abi::tensor_map;
}  // namespace

namespace {

// The tensor-core GEMM with an epilogue (tpc::kEpi*); tpc_gemm_split is the kEpiStore form.
int gemm_launch(const void* A, const void* A_lo, const void* B, const void* B_lo, void* C, int64_t M, int64_t N,
                int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t a_mn, int32_t b_mn, int32_t c_dtype,
                float alpha, float beta, int32_t* status, tpc_stream_t stream, int epi, const float* row_a,
                const float* row_b) {
  if (!A || !B || !C) return fail(TPC_ERR_NULL, "gemm: A, B and C are required");
  if (M < 1 || N < 1 || K < 1 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30))
    return fail(TPC_ERR_BAD_SHAPE, "gemm: sizes must be in [1, 2^30]");
  auto misaligned = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) % 16) != 0; };
  if ((lda % 8) || (ldb % 8) || misaligned(A) || misaligned(B) || misaligned(A_lo) || misaligned(B_lo))
    return fail(TPC_ERR_BAD_SHAPE, "gemm: A and B need 16-byte aligned bases and leading dimensions multiple of 8");
  if (c_dtype != TPC_F32 && c_dtype != TPC_BF16) return fail(TPC_ERR_UNSUPPORTED, "gemm: C is fp32 or bf16");
  if (c_dtype == TPC_BF16 && beta != 0.f) return fail(TPC_ERR_UNSUPPORTED, "gemm: beta needs an fp32 C");
  if (a_mn ? (lda < M) : (lda < K)) return fail(TPC_ERR_BAD_SHAPE, "gemm: lda too small");
  if (b_mn ? (ldb < N) : (ldb < K)) return fail(TPC_ERR_BAD_SHAPE, "gemm: ldb too small");
  // kEpiLsePart writes one (max, sum) pair per row and column tile, the other epilogues one value per column
  const int64_t c_cols = epi == tpc::kEpiLsePart ? (N + tpc::kGemmBN - 1) / tpc::kGemmBN : N;
  if (ldc < c_cols) return fail(TPC_ERR_BAD_SHAPE, "gemm: ldc too small");
  if (B_lo && !A_lo) return fail(TPC_ERR_UNSUPPORTED, "gemm: B_lo needs A_lo (three-product form)");
  // 128-byte-swizzled boxes 64 elements wide: K-major [mn][K] boxes of 64 (K) x tile rows,
  // MN-major [K][mn] boxes of 64 (mn) x 64 (K)
  auto encode = [&](CUtensorMap* m, const void* X, bool mn_major, int64_t mn, int64_t ld, int box) {
    return mn_major ? tensor_map(m, X, mn, K, ld, tpc::kGemmBK) : tensor_map(m, X, K, mn, ld, box);
  };
  // tile height: 256 rows (two halves) once K is long enough to hide the non-overlapped epilogue
  const int HV = K >= tpc::kGemmLongK ? 2 : 1;
  const int BM = tpc::kGemmHalf * HV;
  CUtensorMap ta, tb, talo, tblo;
  bool ok = encode(&ta, A, a_mn, M, lda, BM) && encode(&tb, B, b_mn, N, ldb, tpc::kGemmBN);
  ok = ok && encode(&talo, A_lo ? A_lo : A, a_mn, M, lda, BM);
  ok = ok && encode(&tblo, B_lo ? B_lo : B, b_mn, N, ldb, tpc::kGemmBN);
  if (!ok) return fail(TPC_ERR_CUDA, "gemm: cuTensorMapEncodeTiled failed");
  const int passes = B_lo ? 3 : (A_lo ? 2 : 1);
  tpc::GemmArgs g{(int)M, (int)N, (int)K, a_mn, b_mn, c_dtype, (long long)ldc, alpha, beta, C, status, passes,
                  M < N ? 1 : 0, epi, row_a, row_b};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t tiles = ((N + tpc::kGemmBN - 1) / tpc::kGemmBN) * ((M + BM - 1) / BM);
  if (tiles > (int64_t)1 << 31) return fail(TPC_ERR_BAD_SHAPE, "gemm: too many tiles");
  const dim3 grid((unsigned)std::min<int64_t>(tiles, sm_count()));
  auto go = [&](auto cb, auto hv) -> int {
    constexpr int CB = decltype(cb)::value, H2 = decltype(hv)::value;
    constexpr size_t smem = tpc::GemmCfg<H2>::total;
    TPC_CUDA(set_smem(tpc::gemm_bf16_tc<CB, H2>, smem));
    TPC_LAUNCH("gemm_bf16_tc", st,
               (tpc::gemm_bf16_tc<CB, H2><<<grid, tpc::kGemmThreadsP, smem, st>>>(ta, tb, talo, tblo, g)));
    return TPC_OK;
  };
  using I0 = std::integral_constant<int, 0>;
  using I1 = std::integral_constant<int, 1>;
  using I2 = std::integral_constant<int, 2>;
  if (c_dtype == TPC_BF16) return HV == 2 ? go(I1{}, I2{}) : go(I1{}, I1{});
  return HV == 2 ? go(I0{}, I2{}) : go(I0{}, I1{});
}

}  // namespace

extern "C" {

int tpc_gemm_split(const void* A, const void* A_lo, const void* B, const void* B_lo, void* C, int64_t M, int64_t N,
                   int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t a_mn, int32_t b_mn, int32_t c_dtype,
                   float alpha, float beta, int32_t* status, tpc_stream_t stream) {
  return gemm_launch(A, A_lo, B, B_lo, C, M, N, K, lda, ldb, ldc, a_mn, b_mn, c_dtype, alpha, beta, status, stream,
                     tpc::kEpiStore, nullptr, nullptr);
}

int tpc_gemm_bf16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                  int64_t ldc, int32_t a_mn, int32_t b_mn, int32_t c_dtype, float alpha, float beta, int32_t* status,
                  tpc_stream_t stream) {
  return tpc_gemm_split(A, nullptr, B, nullptr, C, M, N, K, lda, ldb, ldc, a_mn, b_mn, c_dtype, alpha, beta, status,
                        stream);
}

// Scratch of the log-probability calls (all 256-byte aligned sections):
//   forward:  per-row tile partials (max, sum) [chunk_rows][V / 256] float2
//   backward: dz [chunk_rows][V] bf16, s [N] fp32, target groups: count / begin / fill [V + 1] int32,
//             positions [n_expanded] int32
size_t tpc_logprob_scratch_bytes(const tpc_plan* plan, int64_t V, int32_t chunk_rows) {
  if (!plan || V < 1 || chunk_rows < 1) return 0;
  const size_t tiles = (size_t)((V + tpc::kGemmBN - 1) / tpc::kGemmBN);
  const size_t fwd = a256((size_t)chunk_rows * tiles * 8);
  const size_t bwd = a256((size_t)chunk_rows * V * 2) + a256((size_t)plan->p.n_unique * 4) +
                     3 * a256(((size_t)V + 1) * 4) + a256((size_t)plan->p.n_expanded * 4);
  return std::max(fwd, bwd);
}

namespace {
int logprob_check(const tpc_plan* plan, const void* h, const void* W, int64_t V, int64_t Dh, const int32_t* targets,
                  void* scratch, size_t scratch_bytes, int32_t chunk_rows) {
  if (!plan || !h || !W || !targets || !scratch) return fail(TPC_ERR_NULL, "logprob: NULL argument");
  if (!plan->p.dev) return fail(TPC_ERR_STATE, "plan tables not uploaded");
  if (V < 8 || Dh < 8 || (V % 8) || (Dh % 8)) return fail(TPC_ERR_BAD_SHAPE, "logprob: V and Dh multiples of 8");
  if (V >= (int64_t(1) << 31)) return fail(TPC_ERR_BAD_SHAPE, "logprob: V below 2^31");
  if (chunk_rows < 1) return fail(TPC_ERR_BAD_SHAPE, "logprob: chunk_rows >= 1");
  if (scratch_bytes < tpc_logprob_scratch_bytes(plan, V, chunk_rows))
    return fail(TPC_ERR_WORKSPACE, "logprob: scratch too small");
  if (reinterpret_cast<uintptr_t>(scratch) % 256) return fail(TPC_ERR_WORKSPACE, "logprob: scratch must be 256-byte aligned");
  return TPC_OK;
}
}  // namespace

int tpc_logprob_forward(const tpc_plan* plan, const void* h, const void* W, int64_t V, int64_t Dh,
                        const int32_t* targets, float* logp, float* lse, void* scratch, size_t scratch_bytes,
                        int32_t chunk_rows, int32_t* status, tpc_stream_t stream) {
  if (int rc = logprob_check(plan, h, W, V, Dh, targets, scratch, scratch_bytes, chunk_rows)) return rc;
  if (!logp || !lse) return fail(TPC_ERR_NULL, "logprob: logp and lse are required");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_logprob_forward");
  const tpc::Plan& p = plan->p;
  const int tiles = (int)((V + tpc::kGemmBN - 1) / tpc::kGemmBN);
  float2* part = static_cast<float2*>(scratch);
  const __nv_bfloat16* hb = static_cast<const __nv_bfloat16*>(h);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  constexpr int wpb = tpc::kLpThreads / 32;
  for (int64_t r0 = 0; r0 < p.n_unique; r0 += chunk_rows) {
    const int R = (int)std::min<int64_t>(chunk_rows, p.n_unique - r0);
    // logits of the chunk on tensor cores, reduced in the epilogue to per-tile (max, sum) partials
    if (int rc = gemm_launch(hb + r0 * Dh, nullptr, W, nullptr, part, R, V, Dh, Dh, Dh, tiles, 0, 0, TPC_F32, 1.f, 0.f,
                             status, stream, tpc::kEpiLsePart, nullptr, nullptr))
      return rc;
    TPC_LAUNCH("lse_combine", st,
               (tpc::lse_combine_kernel<<<(R + wpb - 1) / wpb, tpc::kLpThreads, 0, st>>>(part, tiles, R, (int)r0, lse)));
    TPC_LAUNCH("target_logp", st,
               (tpc::target_logp_kernel<<<(R + wpb - 1) / wpb, tpc::kLpThreads, 0, st>>>(
                   p.dt, hb, Wb, (int)Dh, V, (int)r0, R, lse, targets, logp, status)));
  }
  return TPC_OK;
}

int tpc_logprob_backward(const tpc_plan* plan, const void* h, const void* W, int64_t V, int64_t Dh,
                         const int32_t* targets, const float* dlogp, const float* lse, float* dh, float* dW,
                         void* scratch, size_t scratch_bytes, int32_t chunk_rows, int32_t* status,
                         tpc_stream_t stream) {
  if (int rc = logprob_check(plan, h, W, V, Dh, targets, scratch, scratch_bytes, chunk_rows)) return rc;
  if (!dlogp || !lse || !dh || !dW) return fail(TPC_ERR_NULL, "logprob backward: dlogp, lse, dh and dW are required");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = tpc_abi::plan_checks(plan, st)) return rc;
  tpc_abi::NvtxRange nvtx_call("tpc_logprob_backward");
  const tpc::Plan& p = plan->p;
  const int64_t N = p.n_unique, NE = p.n_expanded;
  char* sc = static_cast<char*>(scratch);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(sc);
  size_t o = a256((size_t)chunk_rows * V * 2);
  float* srow = reinterpret_cast<float*>(sc + o);
  o += a256((size_t)N * 4);
  int32_t* cnt = reinterpret_cast<int32_t*>(sc + o);
  o += a256(((size_t)V + 1) * 4);
  int32_t* tbegin = reinterpret_cast<int32_t*>(sc + o);
  o += a256(((size_t)V + 1) * 4);
  int32_t* tfill = reinterpret_cast<int32_t*>(sc + o);
  o += a256(((size_t)V + 1) * 4);
  int32_t* tlist = reinterpret_cast<int32_t*>(sc + o);
  const __nv_bfloat16* hb = static_cast<const __nv_bfloat16*>(h);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  // s_u = sum of the occurrence weights of each row
  TPC_LAUNCH("row_weight_sum", st,
             (tpc::row_weight_sum_kernel<<<(unsigned)((N + 255) / 256), 256, 0, st>>>(p.dt, N, dlogp, srow)));
  TPC_CUDA(cudaMemsetAsync(dW, 0, (size_t)V * Dh * 4, st));
  for (int64_t r0 = 0; r0 < N; r0 += chunk_rows) {
    const int R = (int)std::min<int64_t>(chunk_rows, N - r0);
    // dense part of dz = -s softmax(z): the recomputed logit tile's epilogue writes it as bf16
    if (int rc = gemm_launch(hb + r0 * Dh, nullptr, W, nullptr, dz, R, V, Dh, Dh, Dh, V, 0, 0, TPC_BF16, 1.f, 0.f, status,
                             stream, tpc::kEpiSoftmaxGrad, lse + r0, srow + r0))
      return rc;
    // dH = dZ W  (W as an MN-major B: [V][Dh], N = Dh contiguous)
    if (int rc = tpc_gemm_bf16(dz, W, dh + r0 * Dh, R, Dh, V, V, Dh, Dh, 0, 1, TPC_F32, 1.f, 0.f, status, stream)) return rc;
    // dW += dZ^T H  (dZ as an MN-major A: [R][V]; H as an MN-major B: [R][Dh])
    if (int rc = tpc_gemm_bf16(dz, hb + r0 * Dh, dW, V, Dh, R, V, Dh, Dh, 1, 1, TPC_F32, 1.f, 1.f, status, stream)) return rc;
  }
  // sparse part, exact in fp32: dh_u += sum_j w_j W_{y_j}; dW_y += sum_j w_j h_{u(j)}, by target
  constexpr int wpb = tpc::kLpThreads / 32;
  TPC_LAUNCH("sparse_dh", st,
             (tpc::sparse_dh_kernel<<<(unsigned)((N + wpb - 1) / wpb), tpc::kLpThreads, 0, st>>>(p.dt, N, Wb, (int)Dh, V,
                                                                                               targets, dlogp, dh)));
  TPC_CUDA(cudaMemsetAsync(cnt, 0, ((size_t)V + 1) * 4, st));
  TPC_LAUNCH("target_count", st,
             (tpc::target_count_kernel<<<(unsigned)((NE + 255) / 256), 256, 0, st>>>(targets, NE, V, cnt)));
  TPC_LAUNCH("target_scan", st, (tpc::target_scan_kernel<<<1, 1024, 0, st>>>(cnt, V, tbegin, tfill)));
  TPC_LAUNCH("target_place", st,
             (tpc::target_place_kernel<<<(unsigned)((NE + 255) / 256), 256, 0, st>>>(targets, NE, V, tfill, tlist)));
  TPC_LAUNCH("target_sort", st, (tpc::target_sort_kernel<<<(unsigned)((V + 255) / 256), 256, 0, st>>>(tbegin, V, tlist)));
  TPC_LAUNCH("sparse_dw", st,
             (tpc::sparse_dw_kernel<<<(unsigned)((V + wpb - 1) / wpb), tpc::kLpThreads, 0, st>>>(
                 p.dt, hb, (int)Dh, V, tbegin, tlist, dlogp, dW)));
  return TPC_OK;
}

}  // extern "C"
