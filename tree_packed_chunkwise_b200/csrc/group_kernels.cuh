// Elementwise parts of the hybrid attention group (HARTS Table 1: KDA and MLA layers in a 3:1
// group; Figure C.1: every layer type runs once per unique row).  Plain reading of the layers (the
// pages give none): pre-norm residual layers with RMSNorm (unit weight, eps 1e-6); KDA layer
// q = xn W_q, k = L2-normalised per head (eps 1e-6 under the root), v = xn W_v,
// g = -0.1 softplus(xn W_g), beta = sigmoid(xn W_beta); latent attention with a 512-wide latent,
// 16 query heads of 128 + 64 rotary dims, a 64-dim rotary key shared by all heads, rotary position
// = depth of the token on its trajectories (half-split rotation, base 10000).
//
// Precision: activations and gradients are fp32.  Where one is a tensor-core operand it is stored
// as a bf16 pair hi = bf16(x), lo = bf16(x - hi) (x = hi + lo to 2^-17 relative), which the GEMM
// and the attention kernels combine into fp32-accurate products.
#pragma once
#include "common.cuh"

namespace tpc {

constexpr int kGrpD = 2048, kGrpH = 16, kGrpDH = 128, kGrpRope = 64, kGrpLat = 512;
constexpr int kGrpQK = kGrpDH + kGrpRope;                                  // 192
constexpr int kKdaProj = 4 * kGrpD + kGrpH;                                // q | k | v | g | beta = 8208
constexpr int kMlaProj = kGrpH * kGrpQK + kGrpLat + kGrpRope;              // 3072 + 512 + 64 = 3648
constexpr float kNormEps = 1e-6f;

using bf16 = __nv_bfloat16;

__device__ __forceinline__ void split_store(float x, bf16* hi, bf16* lo, size_t i) {
  const bf16 h = __float2bfloat16_rn(x);
  hi[i] = h;
  lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
}

__device__ __forceinline__ float warp_sum(float x) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// fixed-order block sum over 256 threads
__device__ __forceinline__ float block_sum256(float x, float* red) {
  x = warp_sum(x);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < 8; ++i) s += red[i];
  return s;
}

// xn = x * rstd as a hi/lo pair, rstd = 1 / sqrt(mean(x^2) + eps); one CTA (256 threads) per row
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ x, bf16* __restrict__ xh, bf16* __restrict__ xl,
                                   float* __restrict__ rstd, int D) {
  __shared__ float red[8];
  const size_t o = (size_t)blockIdx.x * D;
  float s = 0.f;
  for (int i = threadIdx.x; i < D; i += 256) s += x[o + i] * x[o + i];
  s = block_sum256(s, red);
  const float r = rsqrtf(s / D + kNormEps);
  for (int i = threadIdx.x; i < D; i += 256) split_store(x[o + i] * r, xh, xl, o + i);
  if (threadIdx.x == 0) rstd[blockIdx.x] = r;
}

// dx = dres + r (dxn - xn mean(dxn xn)),  xn = x r  (RMSNorm backward with unit weight)
__global__ void rmsnorm_bwd_kernel(const float* __restrict__ x, const float* __restrict__ rstd,
                                   const float* __restrict__ dxn, const float* __restrict__ dres,
                                   float* __restrict__ dx, int D) {
  __shared__ float red[8];
  const size_t o = (size_t)blockIdx.x * D;
  const float r = rstd[blockIdx.x];
  float s = 0.f;
  for (int i = threadIdx.x; i < D; i += 256) s += dxn[o + i] * x[o + i] * r;
  s = block_sum256(s, red) / D;
  for (int i = threadIdx.x; i < D; i += 256) {
    const float xn = x[o + i] * r;
    dx[o + i] = dres[o + i] + r * (dxn[o + i] - xn * s);
  }
}

__device__ __forceinline__ float softplus_f(float z) { return z > 20.f ? z : log1pf(expf(z)); }
__device__ __forceinline__ float sigmoid_f(float z) { return 1.f / (1.f + expf(-z)); }

// KDA projections P [N][8208] -> q, k, v, g [N][16][128] and beta [N][16] (fp32), knorm [N][16];
// one CTA per row, one warp per two heads for the key norms
__global__ void kda_post_kernel(const float* __restrict__ P, float* __restrict__ q, float* __restrict__ k,
                                float* __restrict__ v, float* __restrict__ g, float* __restrict__ beta,
                                float* __restrict__ knorm) {
  const int row = blockIdx.x;
  const float* p = P + (size_t)row * kKdaProj;
  const size_t o = (size_t)row * kGrpD;
  for (int i = threadIdx.x; i < kGrpD; i += blockDim.x) {
    q[o + i] = p[i];
    v[o + i] = p[2 * kGrpD + i];
    g[o + i] = -0.1f * softplus_f(p[3 * kGrpD + i]);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int hh = w; hh < kGrpH; hh += blockDim.x >> 5) {
    const float* kp = p + kGrpD + hh * kGrpDH;
    float s = 0.f;
    for (int i = lane; i < kGrpDH; i += 32) s += kp[i] * kp[i];
    s = warp_sum(s);
    const float r = rsqrtf(s + kNormEps);
    for (int i = lane; i < kGrpDH; i += 32) k[o + hh * kGrpDH + i] = kp[i] * r;
    if (lane == 0) {
      knorm[(size_t)row * kGrpH + hh] = r;
      beta[(size_t)row * kGrpH + hh] = sigmoid_f(p[4 * kGrpD + hh]);
    }
  }
}

// gradient of the KDA projections (hi/lo pair) from dq, dk, dv, dg, dbeta
__global__ void kda_post_bwd_kernel(const float* __restrict__ P, const float* __restrict__ knorm,
                                    const float* __restrict__ dq, const float* __restrict__ dk,
                                    const float* __restrict__ dv, const float* __restrict__ dg,
                                    const float* __restrict__ dbeta, bf16* __restrict__ dPh, bf16* __restrict__ dPl) {
  const int row = blockIdx.x;
  const float* p = P + (size_t)row * kKdaProj;
  const size_t d = (size_t)row * kKdaProj;
  const size_t o = (size_t)row * kGrpD;
  for (int i = threadIdx.x; i < kGrpD; i += blockDim.x) {
    split_store(dq[o + i], dPh, dPl, d + i);
    split_store(dv[o + i], dPh, dPl, d + 2 * kGrpD + i);
    split_store(dg[o + i] * -0.1f * sigmoid_f(p[3 * kGrpD + i]), dPh, dPl, d + 3 * kGrpD + i);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int hh = w; hh < kGrpH; hh += blockDim.x >> 5) {
    // k = kt r, r = (|kt|^2 + eps)^(-1/2):  dkt = r (dk - k (k . dk))
    const float* kp = p + kGrpD + hh * kGrpDH;
    const float r = knorm[(size_t)row * kGrpH + hh];
    float s = 0.f;
    for (int i = lane; i < kGrpDH; i += 32) s += kp[i] * r * dk[o + hh * kGrpDH + i];
    s = warp_sum(s);
    for (int i = lane; i < kGrpDH; i += 32) {
      const float kn = kp[i] * r;
      split_store(r * (dk[o + hh * kGrpDH + i] - kn * s), dPh, dPl, d + kGrpD + hh * kGrpDH + i);
    }
    if (lane == 0) {
      const float b = sigmoid_f(p[4 * kGrpD + hh]);
      split_store(dbeta[(size_t)row * kGrpH + hh] * b * (1.f - b), dPh, dPl, d + 4 * kGrpD + hh);
    }
  }
}

// cos / sin of the rotary angles of position pos (threads 0..31 of the block): angle_i =
// pos * 10000^(-2i/64) taken in double precision, so that deep positions keep full fp32 accuracy
__device__ __forceinline__ void rope_table(int pos, float* cs, float* sn) {
  if (threadIdx.x < kGrpRope / 2) {
    const double inv = pow(10000.0, -2.0 * threadIdx.x / kGrpRope);
    double s, c;
    sincos((double)pos * inv, &s, &c);
    cs[threadIdx.x] = (float)c;
    sn[threadIdx.x] = (float)s;
  }
}

// MLA projections P [N][3648] -> q [N][16][192] (hi/lo pair, rotary half-split rotation of dims
// 128..191), latent c [N][512] (hi/lo pair), kr [N][64] (fp32, rotated).  One CTA per row.
__global__ void mla_post_kernel(const float* __restrict__ P, const int32_t* __restrict__ pos, bf16* __restrict__ qh,
                                bf16* __restrict__ ql, bf16* __restrict__ ch, bf16* __restrict__ cl,
                                float* __restrict__ kr) {
  __shared__ float cs[kGrpRope / 2], sn[kGrpRope / 2];
  const int row = blockIdx.x;
  const float* p = P + (size_t)row * kMlaProj;
  rope_table(pos[row], cs, sn);
  for (int i = threadIdx.x; i < kGrpH * kGrpDH; i += blockDim.x) {
    const int hh = i / kGrpDH, j = i % kGrpDH;
    split_store(p[hh * kGrpQK + j], qh, ql, ((size_t)row * kGrpH + hh) * kGrpQK + j);
  }
  for (int i = threadIdx.x; i < kGrpLat; i += blockDim.x)
    split_store(p[kGrpH * kGrpQK + i], ch, cl, (size_t)row * kGrpLat + i);
  __syncthreads();
  // head 16 = the rotary key shared by all heads
  for (int it = threadIdx.x; it < (kGrpH + 1) * (kGrpRope / 2); it += blockDim.x) {
    const int hh = it / (kGrpRope / 2), i = it % (kGrpRope / 2);
    const float* src = hh < kGrpH ? p + hh * kGrpQK + kGrpDH : p + kGrpH * kGrpQK + kGrpLat;
    const float a = src[i], b = src[i + kGrpRope / 2];
    const float ra = a * cs[i] - b * sn[i], rb = a * sn[i] + b * cs[i];
    if (hh < kGrpH) {
      const size_t d = ((size_t)row * kGrpH + hh) * kGrpQK + kGrpDH;
      split_store(ra, qh, ql, d + i);
      split_store(rb, qh, ql, d + i + kGrpRope / 2);
    } else {
      kr[(size_t)row * kGrpRope + i] = ra;
      kr[(size_t)row * kGrpRope + i + kGrpRope / 2] = rb;
    }
  }
}

// keys and values of the latent attention from KV [N][4096] = c W_b^T: k [N][16][192] =
// [k_nope | kr] and v [N][16][128], both hi/lo pairs
__global__ void mla_kv_kernel(const float* __restrict__ KV, const float* __restrict__ kr, bf16* __restrict__ kh,
                              bf16* __restrict__ kl, bf16* __restrict__ vh, bf16* __restrict__ vl) {
  const int row = blockIdx.x;
  const float* p = KV + (size_t)row * 2 * kGrpD;
  for (int i = threadIdx.x; i < kGrpH * kGrpQK; i += blockDim.x) {
    const int hh = i / kGrpQK, j = i % kGrpQK;
    const float x = j < kGrpDH ? p[hh * kGrpDH + j] : kr[(size_t)row * kGrpRope + j - kGrpDH];
    split_store(x, kh, kl, (size_t)row * kGrpH * kGrpQK + i);
  }
  for (int i = threadIdx.x; i < kGrpD; i += blockDim.x) split_store(p[kGrpD + i], vh, vl, (size_t)row * kGrpD + i);
}

// dKV (hi/lo pair) and dkr (fp32, summed over heads in head order) from dk, dv
__global__ void mla_kv_bwd_kernel(const float* __restrict__ dk, const float* __restrict__ dv, bf16* __restrict__ dKVh,
                                  bf16* __restrict__ dKVl, float* __restrict__ dkr) {
  const int row = blockIdx.x;
  const size_t o = (size_t)row * 2 * kGrpD;
  for (int i = threadIdx.x; i < kGrpD; i += blockDim.x) {
    const int hh = i / kGrpDH, j = i % kGrpDH;
    split_store(dk[((size_t)row * kGrpH + hh) * kGrpQK + j], dKVh, dKVl, o + i);
    split_store(dv[(size_t)row * kGrpD + i], dKVh, dKVl, o + kGrpD + i);
  }
  if (threadIdx.x < kGrpRope) {
    float s = 0.f;
    for (int hh = 0; hh < kGrpH; ++hh) s += dk[((size_t)row * kGrpH + hh) * kGrpQK + kGrpDH + threadIdx.x];
    dkr[(size_t)row * kGrpRope + threadIdx.x] = s;
  }
}

// gradient of the MLA projections (hi/lo pair): queries (the rotary part rotated back), latent dc,
// shared rotary key dkr (rotated back)
__global__ void mla_post_bwd_kernel(const float* __restrict__ dq, const float* __restrict__ dc,
                                    const float* __restrict__ dkr, const int32_t* __restrict__ pos,
                                    bf16* __restrict__ dPh, bf16* __restrict__ dPl) {
  __shared__ float cs[kGrpRope / 2], sn[kGrpRope / 2];
  const int row = blockIdx.x;
  const size_t d = (size_t)row * kMlaProj;
  rope_table(pos[row], cs, sn);
  for (int i = threadIdx.x; i < kGrpH * kGrpDH; i += blockDim.x) {
    const int hh = i / kGrpDH, j = i % kGrpDH;
    split_store(dq[((size_t)row * kGrpH + hh) * kGrpQK + j], dPh, dPl, d + hh * kGrpQK + j);
  }
  for (int i = threadIdx.x; i < kGrpLat; i += blockDim.x)
    split_store(dc[(size_t)row * kGrpLat + i], dPh, dPl, d + kGrpH * kGrpQK + i);
  __syncthreads();
  for (int it = threadIdx.x; it < (kGrpH + 1) * (kGrpRope / 2); it += blockDim.x) {
    const int hh = it / (kGrpRope / 2), i = it % (kGrpRope / 2);
    const float* src = hh < kGrpH ? dq + ((size_t)row * kGrpH + hh) * kGrpQK + kGrpDH : dkr + (size_t)row * kGrpRope;
    const float ga = src[i], gb = src[i + kGrpRope / 2];
    // transpose of the rotation
    const float da = ga * cs[i] + gb * sn[i], db = -ga * sn[i] + gb * cs[i];
    const size_t dst = d + (hh < kGrpH ? hh * kGrpQK + kGrpDH : kGrpH * kGrpQK + kGrpLat);
    split_store(da, dPh, dPl, dst + i);
    split_store(db, dPh, dPl, dst + i + kGrpRope / 2);
  }
}

// hi/lo pair of an fp32 tensor
__global__ void split_bf16_kernel(const float* __restrict__ x, bf16* __restrict__ hi, bf16* __restrict__ lo, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    split_store(x[i], hi, lo, i);
}

}  // namespace tpc
