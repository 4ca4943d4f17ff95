// Compact top-k MoE routing with occurrence counts (HARTS abstract: for deterministic top-k routing
// without token dropping, occurrence counts restore MoE objective weights and expert-load
// statistics; Figure 1: q_B = 2 restores them without repeating routing; Figure C.1(d):
// multiplicity-weighted router losses and expert-load counts).
//
// Each unique row is routed once.  Router logits z_u = W_r h_u are fp32 sums over the hidden
// dimension in a fixed order of separately rounded products (c = 0, 1, ...; no fused multiply-add),
// so the top-k decision is reproducible bit for bit.  Every statistic over trajectory positions is
// the occurrence-weighted sum over unique rows (q_u = number of positions holding row u):
//   load_e = sum_u q_u [e in topk(u)],  P_e = sum_u q_u p_ue,  sum_j lse_j^2 = sum_u q_u lse_u^2,
// and the gradient of a L_aux + b L_z (L_aux = E/(k N^2) sum_e load_e P_e, L_z = (1/N) sum lse^2,
// N = positions) with respect to z_u is q_u times the per-position gradient.  All reductions run in
// a fixed order (deterministic).
#pragma once
#include <cuda_bf16.h>

#include "common.cuh"

namespace tpc {

constexpr int kMoeRows = 32;      // rows per routing CTA
constexpr int kMoeThreads = 256;
constexpr int kMoeCK = 64;        // hidden-dimension chunk staged in shared memory
constexpr int kMoeMaxE = 256, kMoeMaxK = 8;

// Expert columns padded to a multiple of 4 (float4 reads) plus 4 (fewer bank conflicts on the stores)
constexpr int kMoeMaxEp = kMoeMaxE + 4;

struct MoeSmem {
  static constexpr size_t hs = 0;                                           // [rows][CK] fp32
  static constexpr size_t ws = hs + sizeof(float) * kMoeRows * kMoeCK;       // [CK][Ep] fp32
  static constexpr size_t zs = ws + sizeof(float) * kMoeCK * kMoeMaxEp;      // [rows][E] fp32 logits
  static constexpr size_t sel = zs + sizeof(float) * kMoeRows * kMoeMaxE;    // [rows][K] int
  static constexpr size_t lse = sel + sizeof(int) * kMoeRows * kMoeMaxK;     // [rows] fp32
  static constexpr size_t total = lse + sizeof(float) * kMoeRows;
};

// one warp's fixed-order reductions (lane-strided partial, then a butterfly)
__device__ __forceinline__ float warp_max(float x) {
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// number of expert quads rounded up to a power of two (the thread tiling of the logits)
__host__ __device__ __forceinline__ int moe_quads_p2(int E) {
  int q = 1;
  while (q < (E + 3) / 4) q <<= 1;
  return q;
}

// Routing of kMoeRows rows per CTA: logits, lse, top-k experts and gates per row, and this CTA's
// partial occurrence-weighted expert loads and probability sums.  Logits: thread (quad q, row group tr)
// owns experts 4q .. 4q+3 of rows tr, tr + TR, ... (RT rows); per hidden index c it reads one float4
// of router weights and RT hidden values and updates 4 RT sums, each in the order c = 0, 1, ...
template <int RT>  // rows per thread: max(1, 32 * QP / 256), QP = moe_quads_p2(E)
__global__ void __launch_bounds__(kMoeThreads) moe_route_kernel(DevTables t, const __nv_bfloat16* __restrict__ h,
                                                                const __nv_bfloat16* __restrict__ w, int Dh, int E,
                                                                int k, int N, float* __restrict__ logits,
                                                                float* __restrict__ lse_out, int* __restrict__ topk_idx,
                                                                float* __restrict__ topk_gate,
                                                                long long* __restrict__ part_load,
                                                                float* __restrict__ part_prob) {
  extern __shared__ __align__(16) uint8_t msm[];
  float* hs = reinterpret_cast<float*>(msm + MoeSmem::hs);
  float* wsm = reinterpret_cast<float*>(msm + MoeSmem::ws);
  float* zs = reinterpret_cast<float*>(msm + MoeSmem::zs);
  int* sel = reinterpret_cast<int*>(msm + MoeSmem::sel);
  float* slse = reinterpret_cast<float*>(msm + MoeSmem::lse);
  const int tid = threadIdx.x, r0 = blockIdx.x * kMoeRows, nr = min(kMoeRows, N - r0);
  const int QP = moe_quads_p2(E), Ep = 4 * QP + 4, TR = kMoeThreads / QP;
  const int q = tid % QP, tr = tid / QP;
  float acc[RT][4];
#pragma unroll
  for (int m = 0; m < RT; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[m][j] = 0.f;
  for (int c0 = 0; c0 < Dh; c0 += kMoeCK) {
    for (int e = tid; e < kMoeRows * kMoeCK; e += kMoeThreads) {
      const int r = e / kMoeCK, c = e % kMoeCK;
      hs[e] = (r < nr) ? __bfloat162float(h[(size_t)(r0 + r) * Dh + c0 + c]) : 0.f;
    }
    for (int e = tid; e < 4 * QP * kMoeCK; e += kMoeThreads) {
      const int x = e / kMoeCK, c = e % kMoeCK;
      wsm[c * Ep + x] = x < E ? __bfloat162float(w[(size_t)x * Dh + c0 + c]) : 0.f;
    }
    __syncthreads();
    if (tr < kMoeRows) {
#pragma unroll 4
      for (int c = 0; c < kMoeCK; ++c) {
        const float4 wv = *reinterpret_cast<const float4*>(wsm + c * Ep + 4 * q);
#pragma unroll
        for (int m = 0; m < RT; ++m) {
          const float hv = hs[(tr + TR * m) * kMoeCK + c];
          acc[m][0] = __fadd_rn(acc[m][0], __fmul_rn(hv, wv.x));
          acc[m][1] = __fadd_rn(acc[m][1], __fmul_rn(hv, wv.y));
          acc[m][2] = __fadd_rn(acc[m][2], __fmul_rn(hv, wv.z));
          acc[m][3] = __fadd_rn(acc[m][3], __fmul_rn(hv, wv.w));
        }
      }
    }
    __syncthreads();
  }
  if (tr < kMoeRows) {
#pragma unroll
    for (int m = 0; m < RT; ++m) {
      const int r = tr + TR * m;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int x = 4 * q + j;
        if (x < E) {
          zs[r * E + x] = acc[m][j];
          if (r < nr) logits[(size_t)(r0 + r) * E + x] = acc[m][j];
        }
      }
    }
  }
  __syncthreads();
  // per row (one warp): lse, top-k (larger first, ties to the lower index), gates
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < nr; r += kMoeThreads / 32) {
    const float* z = zs + r * E;
    float m = -INFINITY;
    for (int x = lane; x < E; x += 32) m = fmaxf(m, z[x]);
    m = warp_max(m);
    float s = 0.f;
    for (int x = lane; x < E; x += 32) s += expf(z[x] - m);
    s = warp_sum(s);
    const float l = m + logf(s);
    int chosen[kMoeMaxK];
    float gsum = 0.f;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = E;
      for (int x = lane; x < E; x += 32) {
        bool taken = false;
        for (int q = 0; q < j; ++q) taken |= (chosen[q] == x);
        if (!taken && (z[x] > bv || (z[x] == bv && x < bi))) { bv = z[x]; bi = x; }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      chosen[j] = bi;
      gsum += expf(bv - l);
    }
    if (lane == 0) {
      slse[r] = l;
      lse_out[r0 + r] = l;
      for (int j = 0; j < k; ++j) {
        sel[r * kMoeMaxK + j] = chosen[j];
        topk_idx[(size_t)(r0 + r) * k + j] = chosen[j];
        topk_gate[(size_t)(r0 + r) * k + j] = expf(z[chosen[j]] - l) / gsum;
      }
    }
  }
  __syncthreads();
  // this CTA's partial statistics, rows in order
  for (int x = tid; x < E; x += kMoeThreads) {
    long long ld = 0;
    float pr = 0.f;
    for (int r = 0; r < nr; ++r) {
      const int q = t.occ_count[r0 + r];
      for (int j = 0; j < k; ++j) ld += (sel[r * kMoeMaxK + j] == x) ? q : 0;
      pr += (float)q * expf(zs[r * E + x] - slse[r]);
    }
    part_load[(size_t)blockIdx.x * E + x] = ld;
    part_prob[(size_t)blockIdx.x * E + x] = pr;
  }
}

// expert statistics: the CTAs' partials summed in CTA order (one CTA per expert; threads take CTAs
// t, t + 256, ... and a fixed tree finishes)
__global__ void __launch_bounds__(kMoeThreads) moe_reduce_kernel(const long long* __restrict__ part_load,
                                                                 const float* __restrict__ part_prob, int n_part,
                                                                 int E, long long* __restrict__ load,
                                                                 float* __restrict__ prob) {
  __shared__ long long sl[kMoeThreads];
  __shared__ float sp[kMoeThreads];
  const int x = blockIdx.x, tid = threadIdx.x;
  long long a = 0;
  float b = 0.f;
  for (int i = tid; i < n_part; i += kMoeThreads) {
    a += part_load[(size_t)i * E + x];
    b += part_prob[(size_t)i * E + x];
  }
  sl[tid] = a;
  sp[tid] = b;
  __syncthreads();
  for (int s = kMoeThreads / 2; s > 0; s >>= 1) {
    if (tid < s) {
      sl[tid] += sl[tid + s];
      sp[tid] += sp[tid + s];
    }
    __syncthreads();
  }
  if (tid == 0) {
    load[x] = sl[0];
    prob[x] = sp[0];
  }
}

// Gradient of a L_aux + b L_z with respect to the logits of every unique row (one warp per row),
// and per-CTA partial sums of q_u lse_u^2 for L_z.
__global__ void __launch_bounds__(kMoeThreads) moe_loss_grad_kernel(DevTables t, const float* __restrict__ logits,
                                                                    const float* __restrict__ lse,
                                                                    const long long* __restrict__ load, int E, int N,
                                                                    float alpha_a, float beta_n, float* __restrict__ dz,
                                                                    float* __restrict__ part_z) {
  __shared__ float red[kMoeThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * (kMoeThreads / 32) + warp;
  float zpart = 0.f;
  if (u < N) {
    const float q = (float)t.occ_count[u], l = lse[u];
    const float* z = logits + (size_t)u * E;
    float dot = 0.f;  // <load, p_u>
    for (int x = lane; x < E; x += 32) dot += (float)load[x] * expf(z[x] - l);
    dot = warp_sum(dot);
    for (int x = lane; x < E; x += 32) {
      const float p = expf(z[x] - l);
      dz[(size_t)u * E + x] = q * (alpha_a * p * ((float)load[x] - dot) + beta_n * 2.f * l * p);
    }
    zpart = q * l * l;
  }
  if (lane == 0) red[warp] = zpart;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < kMoeThreads / 32; ++i) s += red[i];
    part_z[blockIdx.x] = s;
  }
}

// L_aux = alpha sum_e load_e P_e and L_z = (1/N) sum of the partials, each in a fixed order
__global__ void moe_losses_kernel(const long long* __restrict__ load, const float* __restrict__ prob, int E,
                                  const float* __restrict__ part_z, int n_part, float alpha, float inv_n,
                                  float* __restrict__ losses) {
  __shared__ float sz[kMoeThreads];
  const int tid = threadIdx.x;
  float a = 0.f;
  for (int i = tid; i < n_part; i += kMoeThreads) a += part_z[i];
  sz[tid] = a;
  __syncthreads();
  for (int s = kMoeThreads / 2; s > 0; s >>= 1) {
    if (tid < s) sz[tid] += sz[tid + s];
    __syncthreads();
  }
  if (tid == 0) {
    double aux = 0.0;
    for (int x = 0; x < E; ++x) aux += (double)load[x] * (double)prob[x];
    losses[0] = (float)(alpha * aux);
    losses[1] = sz[0] * inv_n;
  }
}

}  // namespace tpc
