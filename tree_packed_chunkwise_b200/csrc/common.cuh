// Shared device helpers for the tree-packed chunkwise KDA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "plan.h"

namespace tpc {

constexpr int kThreads = 256;   // CTA size of the per-chunk kernels
constexpr int kSub = 16;        // rows per gate sub-block (reference row = first row of the block)
constexpr float kMaxGateRange = 80.f;  // max of G[first] - G[last] inside a sub-block (exp(80) < FLT_MAX / 1e3)

// status word codes written by kernels (first error wins)
enum : int { kStatusOk = 0, kStatusRange = 9, kStatusCheck = 7 };

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// compact row of row i of chunk c
__device__ __forceinline__ int chunk_row(const ChunkRec& c, const int32_t* replay_rows, int i) {
  return i < c.n_replay ? replay_rows[c.replay_base + i] : c.row_start + (i - c.n_replay);
}

// thread tiling of an M x N CTA product over kThreads threads: each thread owns TM x TN
// outputs, interleaved (row mi + i*MM, column ni + j*NN) so that neighbouring threads touch
// neighbouring columns.
template <int M, int N>
struct TileShape {
  static constexpr int TN = (N >= 128) ? 4 : (N >= 64 ? 2 : 1);
  static constexpr int NN = N / TN;
  static constexpr int pow2_at_least(int x) { return x <= 1 ? 1 : 2 * pow2_at_least((x + 1) / 2); }
  // smallest power-of-two rows per thread so that the tiles fit in one pass of kThreads
  static constexpr int TMr = pow2_at_least((M * NN + kThreads - 1) / kThreads);
  static constexpr int TM = TMr < M ? TMr : M;
  static constexpr int MM = M / TM;
};

// Out(m, n) = sum_k a(m, k) * b(k, n), delivered to epi(m, n, value).
template <int M, int N, int K, class FA, class FB, class FE>
__device__ __forceinline__ void cta_gemm(FA a, FB b, FE epi) {
  using TS = TileShape<M, N>;
  constexpr int TM = TS::TM, TN = TS::TN, MM = TS::MM, NN = TS::NN;
  static_assert(M % TM == 0 && N % TN == 0, "tile");
  for (int t = threadIdx.x; t < MM * NN; t += blockDim.x) {
    const int mi = t / NN, ni = t % NN;
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
      float av[TM], bv[TN];
#pragma unroll
      for (int i = 0; i < TM; ++i) av[i] = a(mi + i * MM, kk);
#pragma unroll
      for (int j = 0; j < TN; ++j) bv[j] = b(kk, ni + j * NN);
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) epi(mi + i * MM, ni + j * NN, acc[i][j]);
  }
}

}  // namespace tpc
