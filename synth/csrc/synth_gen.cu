// Device twin of synth/__init__.py: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) and the
// same Box-Muller / rounding steps, so that the device writes the bits the host generator
// produces.  Holds no arithmetic of the KDA method: it only draws inputs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

__device__ __forceinline__ double normal_at(uint64_t seed, uint32_t stream, uint64_t idx) {
  uint32_t c[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), stream, 0u};
  philox(c, (uint32_t)seed, (uint32_t)(seed >> 32) ^ 0x5EEDu);
  const double a = __dadd_rn(__dmul_rn((double)(c[0] >> 5), 67108864.0), (double)(c[1] >> 6));
  const double b = __dadd_rn(__dmul_rn((double)(c[2] >> 5), 67108864.0), (double)(c[3] >> 6));
  const double u1 = __dmul_rn(__dadd_rn(a, 1.0), 1.0 / 9007199254740992.0);
  const double u2 = __dmul_rn(b, 1.0 / 9007199254740992.0);
  return __dmul_rn(sqrt(__dmul_rn(-2.0, log(u1))), cos(__dmul_rn(6.283185307179586, u2)));
}

__device__ __forceinline__ void store(void* out, int dtype, size_t i, double x) {
  const float f = __double2float_rn(x);
  if (dtype == 1) static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(f);
  else static_cast<float*>(out)[i] = f;
}

// out[r, :] = scale * normal(seed, stream, rows[r] * width + col)
__global__ void normal_rows_kernel(uint64_t seed, uint32_t stream, const int32_t* rows, int64_t n, int64_t width,
                                   double scale, int dtype, void* out) {
  const int64_t tot = n * width;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < tot; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / width, c = e % width;
    const int64_t src = rows ? (int64_t)rows[r] : r;
    double z = normal_at(seed, stream, (uint64_t)(src * width + c));
    if (scale != 1.0) z = __dmul_rn(z, scale);
    store(out, dtype, (size_t)e, z);
  }
}

// KDA inputs for rows[r] (node-order row ids) written at row r: q, k (L2-normalised), v, g, beta
__global__ void kda_inputs_kernel(uint64_t seed, const int32_t* rows, int64_t n, int H, int dk, int dv, int dtype,
                                  void* q, void* k, void* v, void* g, void* beta) {
  const int64_t tot = n * H;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < tot; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / H, h = e % H;
    const int64_t src = rows ? (int64_t)rows[r] : r;
    const uint64_t bk = (uint64_t)(src * H + h) * dk, bv = (uint64_t)(src * H + h) * dv;
    double ss = 0.0;
    for (int c = 0; c < dk; ++c) {
      const double z = normal_at(seed, 2, bk + c);
      ss = __dadd_rn(ss, __dmul_rn(z, z));
    }
    const double nrm = sqrt(ss);
    for (int c = 0; c < dk; ++c) {
      const size_t o = (size_t)(r * H + h) * dk + c;
      store(q, dtype, o, normal_at(seed, 1, bk + c));
      store(k, dtype, o, __ddiv_rn(normal_at(seed, 2, bk + c), nrm));
      const double zg = normal_at(seed, 4, bk + c);
      store(g, dtype, o, __dmul_rn(-0.1, log1p(exp(zg))));
    }
    for (int c = 0; c < dv; ++c) store(v, dtype, (size_t)(r * H + h) * dv + c, normal_at(seed, 3, bv + c));
    const double zb = normal_at(seed, 5, (uint64_t)(src * H + h));
    store(beta, dtype, (size_t)(r * H + h), __ddiv_rn(1.0, __dadd_rn(1.0, exp(-zb))));
  }
}

}  // namespace

extern "C" {

int synth_normal_rows(uint64_t seed, uint32_t stream, const int32_t* rows, int64_t n, int64_t width, double scale,
                      int dtype, void* out, cudaStream_t st) {
  const int64_t tot = n * width;
  const int blocks = (int)((tot + 255) / 256 < 148 * 32 ? (tot + 255) / 256 : 148 * 32);
  if (tot == 0) return 0;
  normal_rows_kernel<<<blocks, 256, 0, st>>>(seed, stream, rows, n, width, scale, dtype, out);
  return (int)cudaGetLastError();
}

int synth_kda_inputs(uint64_t seed, const int32_t* rows, int64_t n, int H, int dk, int dv, int dtype, void* q, void* k,
                     void* v, void* g, void* beta, cudaStream_t st) {
  const int64_t tot = n * H;
  if (tot == 0) return 0;
  const int blocks = (int)((tot + 127) / 128 < 148 * 16 ? (tot + 127) / 128 : 148 * 16);
  kda_inputs_kernel<<<blocks, 128, 0, st>>>(seed, rows, n, H, dk, dv, dtype, q, k, v, g, beta);
  return (int)cudaGetLastError();
}

}  // extern "C"
