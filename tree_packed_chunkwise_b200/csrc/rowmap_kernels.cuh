// Row maps between the compact (unique-row) layout and the trajectory-expanded layout.
// HARTS Figure 1: one row serves every trajectory through it, with occurrence count q.
#pragma once
#include "common.cuh"

namespace tpc {

// x_unique[r] = sum over the occurrences of r (trajectory order) of x_exp[j]; one CTA per row
__global__ void reduce_expanded_kernel(DevTables t, const float* __restrict__ x_exp, float* __restrict__ x_unique,
                                       int64_t width) {
  const int r = blockIdx.x;
  const int b0 = t.occ_begin[r], b1 = t.occ_begin[r + 1];
  for (int64_t c = threadIdx.x; c < width; c += blockDim.x) {
    float acc = 0.f;
    for (int m = b0; m < b1; ++m) acc += x_exp[(int64_t)t.occ_list[m] * width + c];
    x_unique[(int64_t)r * width + c] = acc;
  }
}

// x_exp[j] = x_unique[exp_rows[j]]; one CTA per expanded row
template <typename T>
__global__ void gather_rows_kernel(DevTables t, const T* __restrict__ src, T* __restrict__ dst, int64_t width) {
  const int j = blockIdx.x;
  const int64_t r = t.exp_rows[j];
  for (int64_t c = threadIdx.x; c < width; c += blockDim.x) dst[(int64_t)j * width + c] = src[r * width + c];
}

__global__ void occurrence_count_kernel(DevTables t, int32_t* __restrict__ counts, int64_t n) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r < n) counts[r] = t.occ_count[r];
}

// absolute trajectory position (depth) of every compact row: one CTA per node
// dst[i] = src[rows[i]] (rows of `width` elements)
template <typename T>
__global__ void gather_list_kernel(const T* __restrict__ src, const int32_t* __restrict__ rows, T* __restrict__ dst,
                                   int64_t width) {
  const int64_t i = blockIdx.x;
  const T* s = src + (int64_t)rows[i] * width;
  for (int64_t c = threadIdx.x; c < width; c += blockDim.x) dst[i * width + c] = s[c];
}

// dst[rows[i]] += src[i]; the rows of one call are distinct (one writer per row, no atomics)
__global__ void add_list_kernel(const float* __restrict__ src, const int32_t* __restrict__ rows, float* __restrict__ dst,
                                int64_t width) {
  const int64_t i = blockIdx.x;
  float* d = dst + (int64_t)rows[i] * width;
  for (int64_t c = threadIdx.x; c < width; c += blockDim.x) d[c] += src[i * width + c];
}

__global__ void rope_positions_kernel(DevTables t, int32_t* __restrict__ pos) {
  const AttnNode nd = t.attn_nodes[blockIdx.x];
  for (int i = threadIdx.x; i < nd.length; i += blockDim.x) pos[nd.row_offset + i] = nd.pos0 + i;
}

}  // namespace tpc
