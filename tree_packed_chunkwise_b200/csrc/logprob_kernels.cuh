// Per-position log-probability recovery on compact rows (HARTS abstract: log-probabilities are
// recovered for each original trajectory position; Figure 1: one logit row z_B serves every
// trajectory through B; Figure C.1(d): no expanded vocabulary-sized logits).
//
// No logit matrix is stored, not even per unique row.  Forward: the tensor-core GEMM
// z_u = W h_u runs chunk by chunk with an epilogue that keeps, per row and 256-column tile, the tile's
// maximum and sum of exponentials (kEpiLsePart); lse_u combines those partials in a fixed order; the
// target logit of every occurrence j of u is its own dot product W_{y_j} . h_u (fp32, fixed order),
// and logp_j = z_u[y_j] - lse_u.
// Backward of L = sum_j w_j logp_j, with s_u = sum over u's occurrences of w_j:
//   dz_u = sum_j w_j onehot(y_j) - s_u softmax(z_u).
// The dense part -s_u softmax(z_u) comes out of the recomputed GEMM tile's epilogue as bf16
// (kEpiSoftmaxGrad) and enters dH = dz W and dW = dz^T H as one tensor-core pass each; the sparse
// one-hot part is added exactly in fp32: dh_u += sum_j w_j W_{y_j} (per row, occurrence order) and
// dW_y += sum over the occurrences with target y of w_j h_{u(j)} (occurrences grouped by target and
// ordered by position, so every sum has a fixed order).
#pragma once
#include "common.cuh"

namespace tpc {

constexpr int kLpThreads = 256;

// lse of rows r0 .. r0 + R - 1 from their tiles' (max, sum) partials, tiles in order (one warp per row)
__global__ void __launch_bounds__(kLpThreads) lse_combine_kernel(const float2* __restrict__ part, int n_tiles, int R,
                                                                int r0, float* __restrict__ lse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kLpThreads / 32) + warp;
  if (i >= R) return;
  const float2* p = part + (size_t)i * n_tiles;
  float m = -INFINITY;
  for (int t = lane; t < n_tiles; t += 32) m = fmaxf(m, p[t].x);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
  for (int t = lane; t < n_tiles; t += 32) s += p[t].y * expf(p[t].x - m);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) lse[r0 + i] = m + logf(s);
}

// fp32 dot product of two bf16 rows of length Dh (a multiple of 256), lane-strided 16-byte pieces
// and a fixed butterfly; the result is on every lane
__device__ __forceinline__ float warp_dot_bf16(const __nv_bfloat16* a, const __nv_bfloat16* b, int Dh) {
  float acc = 0.f;
  for (int c = 8 * (threadIdx.x & 31); c < Dh; c += 256) {
    const uint4 ua = *reinterpret_cast<const uint4*>(a + c), ub = *reinterpret_cast<const uint4*>(b + c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ua);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&ub);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = __bfloat1622float2(a2[k]), y = __bfloat1622float2(b2[k]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// logp of every occurrence of rows r0 .. r0 + R - 1 (one warp per row, occurrences in list order)
__global__ void __launch_bounds__(kLpThreads) target_logp_kernel(DevTables t, const __nv_bfloat16* __restrict__ h,
                                                                const __nv_bfloat16* __restrict__ W, int Dh,
                                                                int64_t V, int r0, int R,
                                                                const float* __restrict__ lse,
                                                                const int32_t* __restrict__ targets,
                                                                float* __restrict__ logp, int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kLpThreads / 32) + warp;
  if (i >= R) return;
  const int u = r0 + i;
  const __nv_bfloat16* hu = h + (size_t)u * Dh;
  const float l = lse[u];
  for (int m = t.occ_begin[u]; m < t.occ_begin[u + 1]; ++m) {
    const int j = t.occ_list[m];
    const int y = targets[j];
    if (y < 0 || y >= V) {
      if (lane == 0) set_status(status, kStatusCheck);
      continue;
    }
    const float z = warp_dot_bf16(hu, W + (size_t)y * Dh, Dh);
    if (lane == 0) logp[j] = z - l;
  }
}

// s_u = sum over u's occurrences (list order) of w_j
__global__ void row_weight_sum_kernel(DevTables t, int64_t N, const float* __restrict__ w, float* __restrict__ s) {
  const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= N) return;
  float acc = 0.f;
  for (int m = t.occ_begin[u]; m < t.occ_begin[u + 1]; ++m) acc += w[t.occ_list[m]];
  s[u] = acc;
}

// dh_u += sum over u's occurrences (list order) of w_j W_{y_j} (one warp per row; Dh <= 4096)
__global__ void __launch_bounds__(kLpThreads) sparse_dh_kernel(DevTables t, int64_t N, const __nv_bfloat16* __restrict__ W,
                                                              int Dh, int64_t V, const int32_t* __restrict__ targets,
                                                              const float* __restrict__ w, float* __restrict__ dh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t u = (int64_t)blockIdx.x * (kLpThreads / 32) + warp;
  if (u >= N) return;
  float* d = dh + u * Dh;
  for (int c0 = 8 * lane; c0 < Dh; c0 += 256) {
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = d[c0 + k];
    for (int m = t.occ_begin[u]; m < t.occ_begin[u + 1]; ++m) {
      const int j = t.occ_list[m];
      const int y = targets[j];
      if (y < 0 || y >= V) continue;
      const float wj = w[j];
      const uint4 ub = *reinterpret_cast<const uint4*>(W + (size_t)y * Dh + c0);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&ub);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x = __bfloat1622float2(b2[k]);
        acc[2 * k] = fmaf(wj, x.x, acc[2 * k]);
        acc[2 * k + 1] = fmaf(wj, x.y, acc[2 * k + 1]);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) d[c0 + k] = acc[k];
  }
}

// Occurrences grouped by target: counts (integer atomics: exact), then the scanned offsets, then
// placement, then each group sorted by position (so that the order is fixed).
__global__ void target_count_kernel(const int32_t* __restrict__ targets, int64_t n, int64_t V,
                                    int32_t* __restrict__ count) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int y = targets[j];
  if (y >= 0 && y < V) atomicAdd(&count[y], 1);
}

// exclusive scan of count[0 .. V) into begin[0 .. V] (one CTA, chunks of the block size)
__global__ void __launch_bounds__(1024) target_scan_kernel(const int32_t* __restrict__ count, int64_t V,
                                                           int32_t* __restrict__ begin, int32_t* __restrict__ fill) {
  __shared__ int32_t sh[1024];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t b = 0; b < V; b += 1024) {
    const int64_t i = b + threadIdx.x;
    const int32_t x = i < V ? count[i] : 0;
    sh[threadIdx.x] = x;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int32_t y = threadIdx.x >= o ? sh[threadIdx.x - o] : 0;
      __syncthreads();
      sh[threadIdx.x] += y;
      __syncthreads();
    }
    if (i < V) {
      begin[i] = carry + sh[threadIdx.x] - x;
      fill[i] = begin[i];
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry += sh[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) begin[V] = carry;
}

__global__ void target_place_kernel(const int32_t* __restrict__ targets, int64_t n, int64_t V,
                                    int32_t* __restrict__ fill, int32_t* __restrict__ list) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int y = targets[j];
  if (y >= 0 && y < V) list[atomicAdd(&fill[y], 1)] = (int32_t)j;
}

// insertion sort of each target's positions (one thread per target)
__global__ void target_sort_kernel(const int32_t* __restrict__ begin, int64_t V, int32_t* __restrict__ list) {
  const int64_t y = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (y >= V) return;
  const int b0 = begin[y], b1 = begin[y + 1];
  for (int a = b0 + 1; a < b1; ++a) {
    const int x = list[a];
    int b = a - 1;
    while (b >= b0 && list[b] > x) {
      list[b + 1] = list[b];
      --b;
    }
    list[b + 1] = x;
  }
}

// dW_y += sum over the occurrences with target y (position order) of w_j h_{u(j)} (one warp per target)
__global__ void __launch_bounds__(kLpThreads) sparse_dw_kernel(DevTables t, const __nv_bfloat16* __restrict__ h, int Dh,
                                                              int64_t V, const int32_t* __restrict__ begin,
                                                              const int32_t* __restrict__ list,
                                                              const float* __restrict__ w, float* __restrict__ dW) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t y = (int64_t)blockIdx.x * (kLpThreads / 32) + warp;
  if (y >= V) return;
  const int b0 = begin[y], b1 = begin[y + 1];
  if (b0 == b1) return;
  float* d = dW + y * Dh;
  for (int c0 = 8 * lane; c0 < Dh; c0 += 256) {
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = d[c0 + k];
    for (int a = b0; a < b1; ++a) {
      const int j = list[a];
      const float wj = w[j];
      const uint4 uh = *reinterpret_cast<const uint4*>(h + (size_t)t.exp_rows[j] * Dh + c0);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&uh);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x = __bfloat1622float2(h2[k]);
        acc[2 * k] = fmaf(wj, x.x, acc[2 * k]);
        acc[2 * k + 1] = fmaf(wj, x.y, acc[2 * k + 1]);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) d[c0 + k] = acc[k];
  }
}

}  // namespace tpc
