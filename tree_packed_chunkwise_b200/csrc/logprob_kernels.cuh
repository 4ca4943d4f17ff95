// Per-position log-probability recovery on compact rows (HARTS abstract: log-probabilities are
// recovered for each original trajectory position; Figure 1: one logit row z_B serves every
// trajectory through B; Figure C.1(d): no expanded vocabulary-sized logits).
//
// Logits exist only per unique row, chunk by chunk: Z = H_chunk W^T (tensor-core GEMM), then
//   lse_u = log sum_v exp(Z_uv)                           (one CTA per row, fixed reduction order)
//   logp_j = Z_u[y_j] - lse_u  for every occurrence j of u (the plan's occurrence lists)
// Backward of L = sum_j w_j logp_j:
//   dZ_u = sum_{j of u} w_j onehot(y_j) - (sum_{j of u} w_j) softmax(Z_u)   (bf16 hi/lo pair)
//   dH = dZ W,  dW = dZ^T H  (tensor-core GEMMs, hi and lo parts accumulated)
#pragma once
#include "common.cuh"

namespace tpc {

constexpr int kLseThreads = 256;

// deterministic block reduction (max or sum) over kLseThreads values
template <bool MAX>
__device__ __forceinline__ float block_reduce(float x, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, o);
    x = MAX ? fmaxf(x, y) : x + y;
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kLseThreads / 32; ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

// lse[r0 + i] for rows i of the chunk Z [R][V]
__global__ void __launch_bounds__(kLseThreads) lse_rows_kernel(const float* __restrict__ Z, int64_t V,
                                                              float* __restrict__ lse, int r0) {
  __shared__ float red[kLseThreads / 32];
  const int i = blockIdx.x;
  const float* z = Z + (int64_t)i * V;
  float m = -INFINITY;
  for (int64_t v = threadIdx.x; v < V; v += kLseThreads) m = fmaxf(m, z[v]);
  m = block_reduce<true>(m, red);
  float s = 0.f;
  for (int64_t v = threadIdx.x; v < V; v += kLseThreads) s += expf(z[v] - m);
  s = block_reduce<false>(s, red);
  if (threadIdx.x == 0) lse[r0 + i] = m + logf(s);
}

// logp of every occurrence of the chunk's rows: one thread per row, occurrences in list order
__global__ void logprob_gather_kernel(DevTables t, const float* __restrict__ Z, int64_t V, int r0, int R,
                                      const float* __restrict__ lse, const int32_t* __restrict__ targets,
                                      float* __restrict__ logp, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R) return;
  const int u = r0 + i;
  for (int m = t.occ_begin[u]; m < t.occ_begin[u + 1]; ++m) {
    const int j = t.occ_list[m];
    const int y = targets[j];
    if (y < 0 || y >= V) {
      set_status(status, kStatusCheck);
      continue;
    }
    logp[j] = Z[(int64_t)i * V + y] - lse[u];
  }
}

// dZ of row r0 + i as a bf16 hi/lo pair; the sparse one-hot terms are added afterwards by one thread
// in occurrence order (deterministic)
__global__ void __launch_bounds__(kLseThreads) dz_rows_kernel(DevTables t, const float* __restrict__ Z, int64_t V,
                                                             int r0, const float* __restrict__ lse,
                                                             const int32_t* __restrict__ targets,
                                                             const float* __restrict__ dlogp,
                                                             __nv_bfloat16* __restrict__ dz_hi,
                                                             __nv_bfloat16* __restrict__ dz_lo, int* status) {
  __shared__ float wsum_s;
  const int i = blockIdx.x, u = r0 + i;
  const int b0 = t.occ_begin[u], b1 = t.occ_begin[u + 1];
  if (threadIdx.x == 0) {
    float ws = 0.f;
    for (int m = b0; m < b1; ++m) ws += dlogp[t.occ_list[m]];
    wsum_s = ws;
  }
  __syncthreads();
  const float ws = wsum_s, l = lse[u];
  const float* z = Z + (int64_t)i * V;
  __nv_bfloat16* hi = dz_hi + (int64_t)i * V;
  __nv_bfloat16* lo = dz_lo + (int64_t)i * V;
  for (int64_t v = threadIdx.x; v < V; v += kLseThreads) {
    const float x = -ws * expf(z[v] - l);
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[v] = h;
    lo[v] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int m = b0; m < b1; ++m) {
      const int j = t.occ_list[m];
      const int y = targets[j];
      if (y < 0 || y >= V) {
        set_status(status, kStatusCheck);
        continue;
      }
      const float x = __bfloat162float(hi[y]) + __bfloat162float(lo[y]) + dlogp[j];
      const __nv_bfloat16 h = __float2bfloat16_rn(x);
      hi[y] = h;
      lo[y] = __float2bfloat16_rn(x - __bfloat162float(h));
    }
  }
}

}  // namespace tpc
