// Tensor-core (tcgen05) per-chunk kernels of the tree-packed chunkwise KDA path, chunk C = 64,
// head dim D = 128.
//
// Every contraction of the chunkwise form runs on the 5th-generation tensor cores with fp32
// accumulators in TMEM.  Operands that are not raw bf16 inputs (gated keys, the WY factors, the
// state, U, P ...) carry ~16 significant bits as a bf16 pair x = hi + lo, and a product of two such
// operands is hi*hi + lo*hi + hi*lo (three MMA chains into one accumulator); against a raw bf16
// input two chains suffice.  Single-pass bf16 or fp16 operands miss the 2e-3 max-error bound.
//
// The intra-chunk gated products gated(a, b)_ri = sum_c a_rc b_ic e^{G_rc - G_ic} use the chunk's
// first row as the reference of every channel: a_rc e^{G_rc - G_0c} (<= 1) and b_ic e^{G_0c - G_ic}
// (>= 1) are single dense operands.  The reference is causal: nothing computed for row r depends on
// a later row of the chunk, so a row shared by several trajectories gets the same bits whether its
// chunk continues into one branch or another (each trajectory keeps its chunkwise numerical path).
// Factors stay within e^{+-80} while a channel decays by at most kMaxChunkDecay over one chunk
// (checked; TPC_ERR_RANGE otherwise).  In shared memory the cumulative gates are kept in base-2
// units (G log2 e), so every factor e^{G_a - G_b} is one hardware exp2 of a difference.
#pragma once
#include <type_traits>

#include "kda_kernels.cuh"
#include "tc.cuh"

namespace tpc {

constexpr int kTcC = 64, kTcD = 128;
// CTA size of the per-chunk tensor-core kernels: 16 warps, i.e. four warps per TMEM sub-partition
// (kTcGroups warp groups of 128 threads split the columns of every accumulator read)
constexpr int kTcThreads = 512, kTcGroups = kTcThreads / 128;
constexpr uint32_t kMtileBytes = 2u * kTcD * kTcD * 2u;  // state transition tile: hi + lo bf16, 128 x 128
// chunk-start state S0 and chunk-end state gradient dS as hi/lo bf16 operand tiles (element (c, j) at
// cm_off(c, j, 128) in the hi half, the same in the lo half): one 128 x 128 tile per chunk and head
constexpr uint32_t kStateTileBytes = 2u * kTcD * kTcD * 2u;
constexpr float kMaxChunkDecay = 80.f;  // G_first - G_last per channel over one chunk
constexpr float kLog2e = 1.4426950408889634f;
enum : int { kStatusTimeout = 8 };
// state scans: CTA size and width of the d_v slice one CTA owns
constexpr int kScanThreads = 128, kScanDVT = 32;

// offset (floats) of element (c, j) of a chunk-head's d x d additive term B in the slice-major layout
// [slice][row][32] that the forward scan reads by bulk copies; within a row the eight 16-byte groups
// are permuted by (row mod 8) so that the scan's threads (one row each) read them without bank conflicts
__host__ __device__ __forceinline__ size_t slice_major(int c, int j) {
  const int jj = j % kScanDVT;
  return ((size_t)(j / kScanDVT) * kTcD + c) * kScanDVT + ((((jj >> 2) ^ (c & 7)) << 2) | (jj & 3));
}

namespace tck {

using namespace tc;

// A x B tile (b contiguous) of bf16 hi (and lo) values val(a, b); 16-byte stores, one 8-wide
// chunk of b per thread and step; neighbouring threads take neighbouring a (conflict-free).
template <int A, int B, bool SPLIT, class F>
__device__ __forceinline__ void build_tile(uint8_t* hi, uint8_t* lo, F val) {
  for (int e = threadIdx.x; e < A * (B / 8); e += blockDim.x) {
    const int a = e % A, b0 = (e / A) * 8;
    __align__(16) __nv_bfloat16 h[8];
    __align__(16) __nv_bfloat16 l[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = val(a, b0 + j);
      if (SPLIT) split_bf16(x, h[j], l[j]);
      else h[j] = __float2bfloat16_rn(x);
    }
    *reinterpret_cast<uint4*>(hi + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(h);
    if (SPLIT) *reinterpret_cast<uint4*>(lo + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(l);
  }
}

// Same tile from a row-major global matrix: row a starts at rowp(a) (nullptr -> zeros), columns b
// contiguous.  Every thread first issues all of its 16-byte loads (8 bf16 or 2 x 4 fp32 per step),
// then converts; f(a, b, x) transforms each loaded value.
template <typename T>
__device__ __forceinline__ void ld8(const T* p, float (&x)[8]) {
  if constexpr (sizeof(T) == 4) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
    const float4 w = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
  } else {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b2[j]);
      x[2 * j] = f.x;
      x[2 * j + 1] = f.y;
    }
  }
}

template <int A, int B, bool SPLIT, typename T, int NT = kTcThreads, class RP, class F>
__device__ __forceinline__ void build_tile_ld(uint8_t* hi, uint8_t* lo, RP rowp, F f) {
  constexpr int NCH = A * (B / 8);
  static_assert(NCH % NT == 0, "tile chunks must be a multiple of the CTA size");
  constexpr int IT = NCH / NT;
  float x[IT][8];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int e = threadIdx.x + it * NT, a = e % A, b0 = (e / A) * 8;
    const T* p = rowp(a);
    if (p) ld8(p + b0, x[it]);
    else {
#pragma unroll
      for (int j = 0; j < 8; ++j) x[it][j] = 0.f;
    }
  }
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int e = threadIdx.x + it * NT, a = e % A, b0 = (e / A) * 8;
    __align__(16) __nv_bfloat16 hh[8];
    __align__(16) __nv_bfloat16 ll[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float y = f(a, b0 + j, x[it][j]);
      if (SPLIT) split_bf16(y, hh[j], ll[j]);
      else hh[j] = __float2bfloat16_rn(y);
    }
    *reinterpret_cast<uint4*>(hi + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(hh);
    if (SPLIT) *reinterpret_cast<uint4*>(lo + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(ll);
  }
}

// The 16-byte pieces of a tile's rows (the element -> thread map of build_tile_ld), loaded early into
// registers (raw_ld) and converted into tiles later (build_tile_raw, build_tile2_raw), so that the
// loads overlap other work
template <typename T, int A, int B>
struct RawTile {
  static constexpr int IT = A * (B / 8) / kTcThreads, Q = sizeof(T) / 2;  // uint4 per 8 values
  uint4 u[IT][Q];
};
template <typename T, int A, int B, class RP>
__device__ __forceinline__ void raw_ld(RawTile<T, A, B>& rt, RP rowp) {
  using RT = RawTile<T, A, B>;
#pragma unroll
  for (int it = 0; it < RT::IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e % A, b0 = (e / A) * 8;
    const T* p = rowp(a);
#pragma unroll
    for (int q = 0; q < RT::Q; ++q)
      rt.u[it][q] = p ? __ldg(reinterpret_cast<const uint4*>(p + b0) + q) : make_uint4(0u, 0u, 0u, 0u);
  }
}
template <typename T>
__device__ __forceinline__ void raw_get(const uint4* u, float (&x)[8]) {
  if constexpr (sizeof(T) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(&u[0]), b = *reinterpret_cast<const float4*>(&u[1]);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u[0]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b2[j]);
      x[2 * j] = f.x;
      x[2 * j + 1] = f.y;
    }
  }
}
template <int A, int B, typename T, class F>
__device__ __forceinline__ void build_tile_raw(uint8_t* hi, uint8_t* lo, const RawTile<T, A, B>& rt, F f) {
  using RT = RawTile<T, A, B>;
#pragma unroll
  for (int it = 0; it < RT::IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e % A, b0 = (e / A) * 8;
    float x[8];
    raw_get<T>(rt.u[it], x);
    __align__(16) __nv_bfloat16 hh[8], ll[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) split_bf16(f(a, b0 + j, x[j]), hh[j], ll[j]);
    *reinterpret_cast<uint4*>(hi + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(hh);
    *reinterpret_cast<uint4*>(lo + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(ll);
  }
}
template <int A, int B, typename T, class F1, class F2>
__device__ __forceinline__ void build_tile2_raw(uint8_t* hi1, uint8_t* lo1, uint8_t* hi2, uint8_t* lo2,
                                                const RawTile<T, A, B>& rt, F1 f1, F2 f2) {
  using RT = RawTile<T, A, B>;
#pragma unroll
  for (int it = 0; it < RT::IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e % A, b0 = (e / A) * 8;
    float x[8];
    raw_get<T>(rt.u[it], x);
    __align__(16) __nv_bfloat16 h1[8], l1[8], h2[8], l2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      split_bf16(f1(a, b0 + j, x[j]), h1[j], l1[j]);
      split_bf16(f2(a, b0 + j, x[j]), h2[j], l2[j]);
    }
    const uint32_t off = cm_off(a, b0, A);
    *reinterpret_cast<uint4*>(hi1 + off) = *reinterpret_cast<const uint4*>(h1);
    *reinterpret_cast<uint4*>(lo1 + off) = *reinterpret_cast<const uint4*>(l1);
    *reinterpret_cast<uint4*>(hi2 + off) = *reinterpret_cast<const uint4*>(h2);
    *reinterpret_cast<uint4*>(lo2 + off) = *reinterpret_cast<const uint4*>(l2);
  }
}

// Gate rows of the chunk into G (fp32, pitch LD) in two steps, so that a kernel issues these loads
// before its larger copies and stores them once they arrive: gate_ld (16-byte loads into registers)
// and gate_st (neighbouring threads take neighbouring rows: conflict-free stores).  Rows >= n are zero.
// (the loaded 16-byte pieces stay raw until gate_st, so that nothing waits for them before then)
template <typename T>
struct GateRegs {
  static constexpr int IT = kTcC * (kTcD / 8) / kTcThreads, Q = sizeof(T) / 2;  // uint4 per 8 values
  uint4 u[IT][Q];
};
template <typename T>
__device__ __forceinline__ void gate_ld(GateRegs<T>& gr, const T* g_, const int* rows, int H, int h, int n) {
#pragma unroll
  for (int it = 0; it < GateRegs<T>::IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e % kTcC, b0 = (e / kTcC) * 8;
    const T* p = g_ + ((size_t)(a < n ? rows[a] : 0) * H + h) * kTcD + b0;
#pragma unroll
    for (int q = 0; q < GateRegs<T>::Q; ++q)
      gr.u[it][q] = a < n ? __ldg(reinterpret_cast<const uint4*>(p) + q) : make_uint4(0u, 0u, 0u, 0u);
  }
}
template <typename T>
__device__ __forceinline__ void gate_st(float* G, int LD, const GateRegs<T>& gr) {
#pragma unroll
  for (int it = 0; it < GateRegs<T>::IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e % kTcC, b0 = (e / kTcC) * 8;
    float x[8];
    raw_get<T>(gr.u[it], x);
#pragma unroll
    for (int j = 0; j < 8; ++j) G[a * LD + b0 + j] = x[j];
  }
}

// Copy of the chunk's rows of an input (row pitch kTcD + 8 elements) in shared memory.
constexpr int kStagePitch = kTcD + 8;
template <typename T>
__device__ __forceinline__ void stage_rows(T* dst, const T* src, const int* rows, int H, int h, int n) {
  constexpr int VEC = 16 / sizeof(T), NCH = kTcC * (kTcD / VEC), IT = NCH / kTcThreads;
  uint4 x[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e / (kTcD / VEC), b0 = (e % (kTcD / VEC)) * VEC;
    x[it] = a < n ? __ldg(reinterpret_cast<const uint4*>(src + ((size_t)rows[a] * H + h) * kTcD + b0))
                  : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int e = threadIdx.x + it * kTcThreads, a = e / (kTcD / VEC), b0 = (e % (kTcD / VEC)) * VEC;
    *reinterpret_cast<uint4*>(dst + a * kStagePitch + b0) = x[it];
  }
}

// Asynchronous copy of the chunk's rows of a bf16 input into shared memory (row pitch kStagePitch);
// rows >= n are zero.  Completed by cp_async_wait + a barrier.
__device__ __forceinline__ void stage_rows_async(__nv_bfloat16* dst, const __nv_bfloat16* src, const int* rows, int H,
                                                 int h, int n) {
  constexpr int VEC = 8, NCH = kTcC * (kTcD / VEC);
  for (int e = threadIdx.x; e < NCH; e += blockDim.x) {
    const int a = e / (kTcD / VEC), b0 = (e % (kTcD / VEC)) * VEC;
    const bool in = a < n;
    tc::cp_async16(dst + a * kStagePitch + b0, src + ((size_t)(in ? rows[a] : 0) * H + h) * kTcD + b0, in ? 16u : 0u);
  }
  tc::cp_async_commit();
}

// A x B tile from staged bf16 rows (row a at st + a * kStagePitch), value f(a, b, x)
template <int A, int B, bool SPLIT, class F>
__device__ __forceinline__ void build_tile_st(uint8_t* hi, uint8_t* lo, const __nv_bfloat16* st, F f) {
  for (int e = threadIdx.x; e < A * (B / 8); e += blockDim.x) {
    const int a = e % A, b0 = (e / A) * 8;
    const uint4 u = *reinterpret_cast<const uint4*>(st + a * kStagePitch + b0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    __align__(16) __nv_bfloat16 hh[8];
    __align__(16) __nv_bfloat16 ll[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(b2[j]);
      const float y0 = f(a, b0 + 2 * j, x.x), y1 = f(a, b0 + 2 * j + 1, x.y);
      if (SPLIT) {
        split_bf16(y0, hh[2 * j], ll[2 * j]);
        split_bf16(y1, hh[2 * j + 1], ll[2 * j + 1]);
      } else {
        hh[2 * j] = __float2bfloat16_rn(y0);
        hh[2 * j + 1] = __float2bfloat16_rn(y1);
      }
    }
    *reinterpret_cast<uint4*>(hi + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(hh);
    if (SPLIT) *reinterpret_cast<uint4*>(lo + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(ll);
  }
}

// C x D K-major tile (element (a, b) at cm_off(a, b, A)) of raw bf16 rows gathered by 16-byte
// asynchronous copies (one per row and 8 columns); rows that rowp maps to nullptr are zero.
// Completed by cp_async_wait + a barrier.
template <int A, int B, class RP>
__device__ __forceinline__ void tile_async_bf16(uint8_t* hi, RP rowp, const void* any_valid) {
  for (int e = threadIdx.x; e < A * (B / 8); e += blockDim.x) {
    const int a = e % A, b0 = (e / A) * 8;
    const __nv_bfloat16* p = rowp(a);
    tc::cp_async16(hi + cm_off(a, b0, A), p ? static_cast<const void*>(p + b0) : any_valid, p ? 16u : 0u);
  }
  tc::cp_async_commit();
}

// 8 values (a, b0 .. b0 + 7) of a K-major hi/lo tile in shared memory, as fp32 (hi + lo)
template <int A>
__device__ __forceinline__ void tile8(const uint8_t* hi, const uint8_t* lo, int a, int b0, float (&v)[8]) {
  const uint32_t off = cm_off(a, b0, A);
  const uint4 hq = *reinterpret_cast<const uint4*>(hi + off), lq = *reinterpret_cast<const uint4*>(lo + off);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hq);
  const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lq);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 x = __bfloat1622float2(h2[k]), y = __bfloat1622float2(l2[k]);
    v[2 * k] = x.x + y.x;
    v[2 * k + 1] = x.y + y.y;
  }
}


// Two A x B tiles (hi/lo) from the same staged bf16 rows: f(a, b, x) returns both values (float2)
template <int A, int B, class F>
__device__ __forceinline__ void build_tile2_st(uint8_t* hi1, uint8_t* lo1, uint8_t* hi2, uint8_t* lo2,
                                               const __nv_bfloat16* st, F f) {
  for (int e = threadIdx.x; e < A * (B / 8); e += blockDim.x) {
    const int a = e % A, b0 = (e / A) * 8;
    const uint4 u = *reinterpret_cast<const uint4*>(st + a * kStagePitch + b0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    __align__(16) __nv_bfloat16 h1[8], l1[8], h2[8], l2[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(b2[j]);
      const float2 y0 = f(a, b0 + 2 * j, x.x), y1 = f(a, b0 + 2 * j + 1, x.y);
      split_bf16(y0.x, h1[2 * j], l1[2 * j]);
      split_bf16(y1.x, h1[2 * j + 1], l1[2 * j + 1]);
      split_bf16(y0.y, h2[2 * j], l2[2 * j]);
      split_bf16(y1.y, h2[2 * j + 1], l2[2 * j + 1]);
    }
    const uint32_t off = cm_off(a, b0, A);
    *reinterpret_cast<uint4*>(hi1 + off) = *reinterpret_cast<const uint4*>(h1);
    *reinterpret_cast<uint4*>(lo1 + off) = *reinterpret_cast<const uint4*>(l1);
    *reinterpret_cast<uint4*>(hi2 + off) = *reinterpret_cast<const uint4*>(h2);
    *reinterpret_cast<uint4*>(lo2 + off) = *reinterpret_cast<const uint4*>(l2);
  }
}

// 8 consecutive values of a staged row as fp32
template <typename T>
__device__ __forceinline__ void staged8(const T* st, int r, int c0, float (&v)[8]) {
  if constexpr (sizeof(T) == 4) {
    const float4 u = *reinterpret_cast<const float4*>(st + r * kStagePitch + c0);
    const float4 u2 = *reinterpret_cast<const float4*>(st + r * kStagePitch + c0 + 4);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; v[4] = u2.x; v[5] = u2.y; v[6] = u2.z; v[7] = u2.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(st + r * kStagePitch + c0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b2[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  }
}


__device__ __forceinline__ void ld8g(const float* p, float (&v)[8]) {
  const float4 u = *reinterpret_cast<const float4*>(p), u2 = *reinterpret_cast<const float4*>(p + 4);
  v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; v[4] = u2.x; v[5] = u2.y; v[6] = u2.z; v[7] = u2.w;
}
__device__ __forceinline__ void st8g(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <typename T>
__device__ __forceinline__ void st8_out(T* p, const float* v) {
  if constexpr (sizeof(T) == 4) {
    st8g(reinterpret_cast<float*>(p), v);
  } else {
    __align__(16) __nv_bfloat16 b[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) b[j] = __float2bfloat16_rn(v[j]);
    *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(b);
  }
}

// The dq kernel's per-chunk partials of dk and dG (C x D fp32 each) go to the dk/dv kernel in the
// order of the two kernels' epilogue lanes (the same element -> lane map in both): the 8 values of
// (warp w, iteration it, lane l) are the float4 pair pd_frag(w, it, l) and pd_frag(w, it, l) + 32, so
// that each store or load instruction of a warp covers 512 contiguous bytes.  Epilogue lane map
// (512 threads, an M = 64 accumulator read 16 columns at a time with share8): row 16 (w % 4) + l % 16,
// columns 16 (w / 4) + 64 it + 8 (l / 16) + 0 .. 7.
__device__ __forceinline__ int pd_frag(int w, int it, int lane) { return (w * 2 + it) * 64 + lane; }
// float offset of element (r, c) of a chunk's partials in that order
__device__ __forceinline__ int pd_index(int r, int c) {
  const int w = ((c >> 4) & 3) * 4 + (r >> 4), it = c >> 6, lane = (r & 15) + 16 * ((c >> 3) & 1), v = c & 7;
  return ((pd_frag(w, it, lane) + 32 * (v >> 2)) << 2) + (v & 3);
}

// The rows of an M = 64 accumulator sit in TMEM lanes 0-15 of each sub-partition.  After a 16-column
// read, lanes 16-31 take columns 8-15 of the row of lane - 16 (one shuffle per value), so that every
// lane of the warp handles 8 values: row 16 * sp + lane % 16, columns 8 * (lane / 16) + 0 .. 7.
__device__ __forceinline__ void share8u(const uint32_t (&v)[16], float (&w)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t x = __shfl_sync(0xffffffffu, v[8 + j], lane & 15);
    w[j] = __uint_as_float(lane < 16 ? v[j] : x);
  }
}
__device__ __forceinline__ void share8(const float (&v)[16], float (&w)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float x = __shfl_sync(0xffffffffu, v[8 + j], lane & 15);
    w[j] = lane < 16 ? v[j] : x;
  }
}

// Reads an M x N fp32 accumulator (N a multiple of 16) starting at TMEM column col0.  Warp w reads
// the lanes of sub-partition w % 4; the kTcGroups groups of four warps take interleaved 16-column
// chunks.  M = 128: f(m, n0, v) gets 16 consecutive columns n0 .. n0+15 of row m.  M = 64: every lane
// takes 8 of them (share8): f(m, n0, v) gets columns n0 .. n0+7.
template <int M, int N, class F>
__device__ __forceinline__ void acc_read(uint32_t tbase, int col0, F f) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, sp = w & 3, grp = w >> 2;
  for (int c = grp * 16; c < N; c += 16 * kTcGroups) {
    float v[16];
    tmem_ld16(tbase + ((uint32_t)(32 * sp) << 16) + (uint32_t)(col0 + c), v);
    if constexpr (M == 128) {
      f(32 * sp + lane, c, v);
    } else {
      float h8[8];
      share8(v, h8);
      f(16 * sp + (lane & 15), c + 8 * (lane >> 4), h8);
    }
  }
}

// Writes 8 values into a K-major/MN-major tile as bf16 hi/lo at (a, b0..b0+7) (b0 a multiple of 8).
template <int A, bool SPLIT>
__device__ __forceinline__ void put8(uint8_t* hi, uint8_t* lo, int a, int b0, const float* v) {
  __align__(16) __nv_bfloat16 h[8];
  __align__(16) __nv_bfloat16 l[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (SPLIT) split_bf16(v[j], h[j], l[j]);
    else h[j] = __float2bfloat16_rn(v[j]);
  }
  *reinterpret_cast<uint4*>(hi + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(h);
  if (SPLIT) *reinterpret_cast<uint4*>(lo + cm_off(a, b0, A)) = *reinterpret_cast<const uint4*>(l);
}

// Writes 16 values (one row chunk) into a K-major/MN-major tile as bf16 hi/lo at (a, b0..b0+15).
template <int A, bool SPLIT>
__device__ __forceinline__ void put16(uint8_t* hi, uint8_t* lo, int a, int b0, const float* v) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    __align__(16) __nv_bfloat16 h[8];
    __align__(16) __nv_bfloat16 l[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (SPLIT) split_bf16(v[8 * half + j], h[j], l[j]);
      else h[j] = __float2bfloat16_rn(v[8 * half + j]);
    }
    *reinterpret_cast<uint4*>(hi + cm_off(a, b0 + 8 * half, A)) = *reinterpret_cast<const uint4*>(h);
    if (SPLIT) *reinterpret_cast<uint4*>(lo + cm_off(a, b0 + 8 * half, A)) = *reinterpret_cast<const uint4*>(l);
  }
}

struct Sync {
  uint64_t* bar;
  uint32_t phase;
  int* status;
};

// Makes the threads' shared-memory writes visible to the tensor core, lets thread 0 issue the
// MMAs and commit, and waits (bounded) for their completion.  Returns false on every thread if
// any thread's wait ran out (CTA-wide vote), after recording TPC_ERR_TIMEOUT.
template <class F>
__device__ __forceinline__ bool run(Sync& s, F issue) {
  fence_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (threadIdx.x == 0) {
    issue();
    commit(s.bar);
  }
  const bool ok = mbar_wait(s.bar, s.phase);
  const int failed = __syncthreads_or(ok ? 0 : 1);
  if (failed) {
    if (threadIdx.x == 0) set_status(s.status, kStatusTimeout);
    mbar_wait(s.bar, s.phase, 200000000ull);  // give MMAs still in flight a last bounded chance
    return false;
  }
  s.phase ^= 1u;
  fence_after_sync();
  return true;
}

// Bulk asynchronous loads into shared memory, completion on their own mbarrier (issued by one
// thread; every thread waits with ld_wait).
struct Ld {
  uint64_t* bar;
  uint32_t phase;
  int* status;
};

// One phase of loads: the issuing thread first calls ld_expect with the phase's total bytes (the
// barrier's single arrival), then issues the copies (ld_state_tile, ld_cd_tile, ld_cc_tile).
__device__ __forceinline__ void ld_expect(Ld& l, uint32_t bytes) { tc::mbar_arrive_expect_tx(l.bar, bytes); }

// one chunk-head's state tile (S0 or dS: hi half then lo half, kStateTileBytes) into hi and lo
__device__ __forceinline__ void ld_state_tile(Ld& l, uint8_t* hi, uint8_t* lo, const float* tiles, size_t base) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(tiles) + base * kStateTileBytes;
  if (lo == hi + kStateTileBytes / 2) {  // halves adjacent in shared memory: one copy
    tc::bulk_g2s(hi, src, kStateTileBytes, l.bar);
    return;
  }
  tc::bulk_g2s(hi, src, kStateTileBytes / 2, l.bar);
  tc::bulk_g2s(lo, src + kStateTileBytes / 2, kStateTileBytes / 2, l.bar);
}

// one chunk-head's C x D hi/lo tile (hi half, then lo half: kCDTileBytes in all), and C x C tile
constexpr uint32_t kCDTileBytes = 2u * kTcC * kTcD * 2u, kCCTileBytes = 2u * kTcC * kTcC * 2u;
__device__ __forceinline__ void ld_cd_tile(Ld& l, uint8_t* hi, uint8_t* lo, const float* tiles, size_t base) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(tiles) + base * kCDTileBytes;
  if (lo == hi + kCDTileBytes / 2) {  // halves adjacent in shared memory: one copy
    tc::bulk_g2s(hi, src, kCDTileBytes, l.bar);
    return;
  }
  tc::bulk_g2s(hi, src, kCDTileBytes / 2, l.bar);
  tc::bulk_g2s(lo, src + kCDTileBytes / 2, kCDTileBytes / 2, l.bar);
}
__device__ __forceinline__ void ld_cc_tile(Ld& l, uint8_t* hi, uint8_t* lo, const float* tiles, size_t base) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(tiles) + base * kCCTileBytes;
  if (lo == hi + kCCTileBytes / 2) {  // halves adjacent in shared memory: one copy
    tc::bulk_g2s(hi, src, kCCTileBytes, l.bar);
    return;
  }
  tc::bulk_g2s(hi, src, kCCTileBytes / 2, l.bar);
  tc::bulk_g2s(lo, src + kCCTileBytes / 2, kCCTileBytes / 2, l.bar);
}
// bulk stores (issuing thread, after the tile writes were fenced and synchronised; the caller waits
// with bulk_wait_read before the shared buffers are reused or the CTA exits; the global writes
// complete with the grid)
__device__ __forceinline__ void store_cd_tile(float* tiles, size_t base, const uint8_t* hi, const uint8_t* lo) {
  uint8_t* dst = reinterpret_cast<uint8_t*>(tiles) + base * kCDTileBytes;
  if (lo == hi + kCDTileBytes / 2) {  // halves adjacent in shared memory: one copy
    tc::bulk_s2g(dst, hi, kCDTileBytes);
  } else {
    tc::bulk_s2g(dst, hi, kCDTileBytes / 2);
    tc::bulk_s2g(dst + kCDTileBytes / 2, lo, kCDTileBytes / 2);
  }
  tc::bulk_commit();
}
__device__ __forceinline__ void store_cc_tile(float* tiles, size_t base, const uint8_t* hi, const uint8_t* lo) {
  uint8_t* dst = reinterpret_cast<uint8_t*>(tiles) + base * kCCTileBytes;
  if (lo == hi + kCCTileBytes / 2) {  // halves adjacent in shared memory: one copy
    tc::bulk_s2g(dst, hi, kCCTileBytes);
  } else {
    tc::bulk_s2g(dst, hi, kCCTileBytes / 2);
    tc::bulk_s2g(dst + kCCTileBytes / 2, lo, kCCTileBytes / 2);
  }
  tc::bulk_commit();
}

// bounded wait for the loads issued on l (CTA-wide vote); false on every thread after recording
// TPC_ERR_TIMEOUT
__device__ __forceinline__ bool ld_wait(Ld& l) {
  const bool ok = tc::mbar_wait(l.bar, l.phase);
  const int failed = __syncthreads_or(ok ? 0 : 1);
  if (failed) {
    if (threadIdx.x == 0) set_status(l.status, kStatusTimeout);
    tc::mbar_wait(l.bar, l.phase, 200000000ull);  // copies still in flight get a last bounded chance
    return false;
  }
  l.phase ^= 1u;
  return true;
}

// sum over j in [j_begin, j_end) of a(c, j) b(c, j) for two state tiles in global memory (hi + lo of
// each), row c
__device__ __forceinline__ float state_row_dot(const float* ta, const float* tb, size_t base, int c, int j_begin,
                                               int j_end) {
  const uint8_t* a = reinterpret_cast<const uint8_t*>(ta) + base * kStateTileBytes;
  const uint8_t* b = reinterpret_cast<const uint8_t*>(tb) + base * kStateTileBytes;
  float acc = 0.f;
#pragma unroll 4
  for (int j0 = j_begin; j0 < j_end; j0 += 8) {
    const uint32_t off = cm_off(c, j0, kTcD);
    const uint4 ah = __ldg(reinterpret_cast<const uint4*>(a + off));
    const uint4 al = __ldg(reinterpret_cast<const uint4*>(a + kStateTileBytes / 2 + off));
    const uint4 bh = __ldg(reinterpret_cast<const uint4*>(b + off));
    const uint4 bl = __ldg(reinterpret_cast<const uint4*>(b + kStateTileBytes / 2 + off));
    const __nv_bfloat162* ah2 = reinterpret_cast<const __nv_bfloat162*>(&ah);
    const __nv_bfloat162* al2 = reinterpret_cast<const __nv_bfloat162*>(&al);
    const __nv_bfloat162* bh2 = reinterpret_cast<const __nv_bfloat162*>(&bh);
    const __nv_bfloat162* bl2 = reinterpret_cast<const __nv_bfloat162*>(&bl);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x1 = __bfloat1622float2(ah2[k]), x2 = __bfloat1622float2(al2[k]);
      const float2 y1 = __bfloat1622float2(bh2[k]), y2 = __bfloat1622float2(bl2[k]);
      acc = fmaf(x1.x + x2.x, y1.x + y2.x, acc);
      acc = fmaf(x1.y + x2.y, y1.y + y2.y, acc);
    }
  }
  return acc;
}

// three chains: hi*hi + lo*hi + hi*lo (both operands split) or two (b exact: lo of b absent)
__device__ __forceinline__ void mma3(uint32_t d, const Op& ah, const Op& al, const Op& bh, const Op& bl, int K,
                                     uint32_t id, bool acc, bool b_exact) {
  mma_chain(d, ah, bh, K, id, acc);
  mma_chain(d, al, bh, K, id, true);
  if (!b_exact) mma_chain(d, ah, bl, K, id, true);
}

// hi/lo product with either operand possibly exact (its lo part is zero and skipped)
__device__ __forceinline__ void mma4(uint32_t d, const Op& ah, const Op& al, const Op& bh, const Op& bl, int K,
                                     uint32_t id, bool acc, bool a_exact, bool b_exact) {
  mma_chain(d, ah, bh, K, id, acc);
  if (!a_exact) mma_chain(d, al, bh, K, id, true);
  if (!b_exact) mma_chain(d, ah, bl, K, id, true);
}

// T = (I + L)^{-1} for strictly lower-triangular L (64 x 64, pitch LC), fp32, in smem.
// Diagonal 16 x 16 blocks by forward substitution, one thread per block column (64 threads) with the
// column in registers: T_pp[r][c] = [r == c] - sum_{k < r} L_pp[r][k] T_pp[k][c];
// off-diagonal blocks: T_pq = -T_pp sum_{q <= s < p} L_ps T_sq, by increasing p - q.
// Row r of T depends on rows <= r of L only.  W1: 4 scratch 16 x 16 blocks (pitch 17).
template <int LC>
__device__ __forceinline__ void block_inverse(float* T, const float* L, float* W1) {
  constexpr int P = 17, BB = 16 * P;
  const int tid = threadIdx.x;
  if (tid < 64) {
    const int p = tid >> 4, c = tid & 15;
    const float* Lp = L + (16 * p) * LC + 16 * p;
    float col[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = (r == c) ? 1.f : 0.f;
#pragma unroll
      for (int k = 0; k < r; ++k) acc = fmaf(-Lp[r * LC + k], col[k], acc);
      col[r] = acc;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) T[(16 * p + r) * LC + 16 * p + c] = col[r];
  }
  __syncthreads();
  // off-diagonal blocks by distance d = p - q: T_pq = -T_pp * (sum_s L_ps T_sq); the distance loop is
  // unrolled so that every inner sum has a constant length (T_pp is zero above its diagonal, so the
  // second product runs over all 16 columns)
#pragma unroll
  for (int d = 1; d < 4; ++d) {
    const int nb = 4 - d;  // blocks (p, p - d), p = d .. 3
    // W1[j] = sum_{s=q}^{p-1} L_ps T_sq
    for (int e = tid; e < nb * 256; e += blockDim.x) {
      const int j = e >> 8, r = (e >> 4) & 15, c = e & 15;
      const int p = d + j, q = j;
      const float* Lr = L + (16 * p + r) * LC + 16 * q;
      const float* Tc = T + (16 * q) * LC + 16 * q + c;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 16 * d; ++k) acc = fmaf(Lr[k], Tc[k * LC], acc);
      W1[j * BB + r * P + c] = acc;
    }
    __syncthreads();
    for (int e = tid; e < nb * 256; e += blockDim.x) {
      const int j = e >> 8, r = (e >> 4) & 15, c = e & 15;
      const int p = d + j, q = j;
      const float* Tr = T + (16 * p + r) * LC + 16 * p;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) acc = fmaf(Tr[k], W1[j * BB + k * P + c], acc);
      T[(16 * p + r) * LC + 16 * q + c] = -acc;
    }
    __syncthreads();
  }
  // upper blocks (p < q) are zero
  for (int e = tid; e < 6 * 256; e += blockDim.x) {
    const int b = e >> 8, r = (e >> 4) & 15, c = e & 15;
    const int p = b < 3 ? 0 : (b < 5 ? 1 : 2), q = b < 3 ? b + 1 : (b < 5 ? b - 1 : 3);
    T[(16 * p + r) * LC + 16 * q + c] = 0.f;
  }
  __syncthreads();
}

// G <- inclusive cumulative gate over the chunk's rows (rows >= n repeat row n - 1), in base-2 units;
// the reference (row 0) goes to ref[c].  Flags TPC_ERR_RANGE when a channel decays by more than
// kMaxChunkDecay.  Four threads per channel, each a quarter of the rows: the quarters' totals, then
// each quarter's running sum from the earlier quarters' totals.  Row i's value depends on rows <= i
// only (the same bits whichever rows follow it in the chunk).  scratch: 4 x kTcD floats.
__device__ __forceinline__ void cumsum_ref(float* G, int LD, int n, float* ref, int* status, float* scratch) {
  static_assert(kTcThreads == 4 * kTcD && kTcC == 64, "four threads per channel, 16 rows each");
  const int c = threadIdx.x % kTcD, q = threadIdx.x / kTcD, i0 = 16 * q;
  float a = 0.f;
#pragma unroll
  for (int i = i0; i < i0 + 16; ++i)
    if (i < n) a += G[i * LD + c];
  scratch[q * kTcD + c] = a;
  __syncthreads();
  float acc = 0.f;
  for (int p = 0; p < q; ++p) acc += scratch[p * kTcD + c];
#pragma unroll
  for (int i = i0; i < i0 + 16; ++i) {
    if (i < n) acc += G[i * LD + c];
    G[i * LD + c] = acc * kLog2e;
  }
  if (q == 0) ref[c] = G[c];
  __syncthreads();  // G and ref complete
  if (q == 0 && status && !(G[c] - G[(kTcC - 1) * LD + c] <= kMaxChunkDecay * kLog2e)) set_status(status, kStatusRange);
}


}  // namespace tck

// --------------------------------------------------------------------------------- forward prep
// per (chunk, head): Atilde = gated(k, k) (strict lower), T = (I + diag(beta) Atilde)^{-1},
// W = T diag(beta) Kbar, U' = T diag(beta) V, Khat = k e^{G_C - G}, decay = e^{G_C}.
template <typename Tin>
struct PrepTcSmemT {
  static constexpr int C = kTcC, D = kTcD, LD = D + 1, LC = C + 1;
  static constexpr size_t G = 0;
  static constexpr size_t A = G + sizeof(float) * C * LD;
  static constexpr size_t T = A + sizeof(float) * C * LC;
  static constexpr size_t W1 = T + sizeof(float) * C * LC;
  static constexpr size_t vec = W1 + sizeof(float) * 4 * 16 * 17;       // beta[C], ref[D], gC[D]
  static constexpr size_t tiles = (vec + sizeof(float) * (C + 2 * D) + 1023) & ~size_t(1023);
  // phase 1: af hi/lo, bf hi/lo (C x D each); phase 2: T' hi/lo (C x C), Kbar hi/lo, V hi/lo (C x D)
  static constexpr size_t CDb = size_t(C) * D * 2, CCb = size_t(C) * C * 2;
  // bf16 inputs: the chunk's k and v rows staged once (pitch kStagePitch)
  static constexpr size_t Stage = tiles + 6 * CDb;  // phase 3: W, U' (MN) and Khat (MN) hi/lo
  static constexpr size_t StB = sizeof(Tin) == 2 ? size_t(C) * tck::kStagePitch * 2 : 0;
  static constexpr size_t total = Stage + 2 * StB;
  static_assert(total <= 227 * 1024, "shared memory");
};

template <typename Tin>
__global__ void __launch_bounds__(kTcThreads, 1)
    kda_fwd_prep_tc(DevTables t, int H, const Tin* __restrict__ k_, const Tin* __restrict__ v_,
                    const Tin* __restrict__ g_, const Tin* __restrict__ beta_, KdaWs ws, int chunk0 = 0,
                    int hpc = 1) {
  using namespace tck;
  using S = PrepTcSmemT<Tin>;
  constexpr int C = S::C, D = S::D, LD = S::LD, LC = S::LC;
  constexpr bool EX = std::is_same<Tin, __nv_bfloat16>::value;
  // grid (heads / hpc, chunks): a CTA runs hpc heads of one chunk in turn, the next head's gates and
  // beta loaded into registers while the current head computes
  const int ci = chunk0 + (int)blockIdx.y, h0 = (int)blockIdx.x * hpc;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ __align__(1024) uint8_t tsm[];
  float* sG = reinterpret_cast<float*>(tsm + S::G);
  float* sA = reinterpret_cast<float*>(tsm + S::A);
  float* sT = reinterpret_cast<float*>(tsm + S::T);
  float* sW1 = reinterpret_cast<float*>(tsm + S::W1);
  float* sb = reinterpret_cast<float*>(tsm + S::vec);
  float* sref = sb + C;
  uint8_t* tl = tsm + S::tiles;
  __shared__ int srow[C];
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x;
  for (int i = tid; i < C; i += blockDim.x) {
    srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  }
  if ((tid >> 5) == 0) tc::tmem_alloc(&tslot, 512);
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // bf16: the chunk's k and v rows into shared memory while the gates load and accumulate
  [[maybe_unused]] __nv_bfloat16* sk = reinterpret_cast<__nv_bfloat16*>(tsm + S::Stage);
  [[maybe_unused]] __nv_bfloat16* sv = reinterpret_cast<__nv_bfloat16*>(tsm + S::Stage + S::StB);
  GateRegs<Tin> gr;
  gate_ld(gr, g_, srow, H, h0, n);  // gates and beta first
  Tin bv = tid < n ? beta_[(size_t)srow[tid] * H + h0] : Tin(0.f);  // (converted when stored)
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  Sync sy{&bar, 0u, ws.status};
  bool ok = true;
  for (int hk = 0; hk < hpc && ok; ++hk) {
    const int h = h0 + hk;
    if constexpr (EX) {
      stage_rows_async(sk, k_, srow, H, h, n);
      stage_rows_async(sv, v_, srow, H, h, n);
    }
    gate_st(sG, LD, gr);
    if (tid < C) sb[tid] = to_f(bv);
    if (hk + 1 < hpc) {  // the next head's gates and beta, into the registers just consumed
      gate_ld(gr, g_, srow, H, h + 1, n);
      bv = tid < n ? beta_[(size_t)srow[tid] * H + h + 1] : Tin(0.f);
    }
    __syncthreads();
    cumsum_ref(sG, LD, n, sref, ws.status, reinterpret_cast<float*>(tl));  // (tiles not yet in use)
    if constexpr (EX) tc::cp_async_wait<0>();
    __syncthreads();
    tc::fence_after_sync();
    auto row_k = [&](int a) -> const Tin* { return a < n ? k_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    auto row_v = [&](int a) -> const Tin* { return a < n ? v_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    // a C x D tile of k (or v) transformed by f, from the staged rows (bf16) or from global memory
    auto k_tile = [&](uint8_t* hi, uint8_t* lo, auto f) {
      if constexpr (EX) build_tile_st<C, D, true>(hi, lo, sk, f);
      else build_tile_ld<C, D, true, Tin>(hi, lo, row_k, f);
    };
    // phase 1: Atilde = af bf^T with af = k e^{G - ref}, bf = k e^{ref - G}
    {
      uint8_t *afh = tl, *afl = tl + S::CDb, *bfh = tl + 2 * S::CDb, *bfl = tl + 3 * S::CDb;
      if constexpr (EX) {  // e = 2^{G - ref} (bounded by the decay check), 2^{ref - G} = 1 / e
        build_tile2_st<C, D>(afh, afl, bfh, bfl, sk, [&](int r, int c, float x) {
          const float e = tc::ex2(sG[r * LD + c] - sref[c]);
          return make_float2(x * e, x * tc::rcp_approx(e));
        });
      } else {
        k_tile(afh, afl, [&](int r, int c, float x) { return x * tc::ex2(sG[r * LD + c] - sref[c]); });
        k_tile(bfh, bfl, [&](int i, int c, float x) { return x * tc::ex2(sref[c] - sG[i * LD + c]); });
      }
      const tc::Op ah{tc::smem_u32(afh), C, false}, al{tc::smem_u32(afl), C, false};
      const tc::Op bh{tc::smem_u32(bfh), C, false}, bl{tc::smem_u32(bfl), C, false};
      ok = run(sy, [&] { mma3(tb, ah, al, bh, bl, D, tc::idesc_bf16(C, C, false, false), false, false); });
      if (ok) {
        float* Ag = ws.At + ((size_t)ci * H + h) * C * C;  // kept for the backward
        acc_read<C, C>(tb, 0, [&](int r, int i0, const float* v) {
          float a[8];
          for (int j = 0; j < 8; ++j) {
            const int i = i0 + j;
            a[j] = (i < r) ? v[j] : 0.f;
            sA[r * LC + i] = sb[r] * a[j];  // L = diag(beta) Atilde, strict lower
          }
          st8g(Ag + r * C + i0, a);
        });
      }
    }
    if (ok) {
      __syncthreads();
      block_inverse<LC>(sT, sA, sW1);
      // T as a hi/lo tile (element (r, i) at cm_off(r, i, C)) for the backward, built where L was
      uint8_t *ttH = reinterpret_cast<uint8_t*>(sA), *ttL = ttH + S::CCb;
      build_tile<C, C, true>(ttH, ttL, [&](int r, int i) { return sT[r * LC + i]; });
      // phase 2: W = T' Kbar and U' = T' V with T' = T diag(beta)
      uint8_t *th = tl, *tlo = tl + S::CCb, *kh = tl + 2 * S::CCb, *kl = kh + S::CDb, *vh = kl + S::CDb,
              *vl = vh + S::CDb;
      build_tile<C, C, true>(th, tlo, [&](int r, int i) { return sT[r * LC + i] * sb[i]; });
      k_tile(kh, kl, [&](int i, int c, float x) { return x * tc::ex2(sG[i * LD + c]); });
      if constexpr (EX) build_tile_st<C, D, false>(vh, vl, sv, [&](int, int, float x) { return x; });
      else build_tile_ld<C, D, true, Tin>(vh, vl, row_v, [&](int, int, float x) { return x; });
      const tc::Op tH{tc::smem_u32(th), C, false}, tL{tc::smem_u32(tlo), C, false};
      const tc::Op kH{tc::smem_u32(kh), C, true}, kL{tc::smem_u32(kl), C, true};
      const tc::Op vH{tc::smem_u32(vh), C, true}, vL{tc::smem_u32(vl), C, true};
      const uint32_t id = tc::idesc_bf16(C, D, false, true);
      ok = run(sy, [&] {
        store_cc_tile(ws.Tm, ((size_t)ci * H + h), ttH, ttL);
        mma3(tb + 64, tH, tL, kH, kL, C, id, false, false);
        mma3(tb + 192, tH, tL, vH, vL, C, id, false, EX);
      });
      if (ok) {
        // phase 3: the chunk's state transition S_end = M S_0 + B with M = Diag(e^{G_C}) - Khat^T W and
        // B = Khat^T U' (Khat = k e^{G_C - G})
        const size_t base = (size_t)ci * H + h;
        uint8_t *wth = tl, *wtl = tl + S::CDb, *uth = tl + 2 * S::CDb, *utl = tl + 3 * S::CDb, *khh = tl + 4 * S::CDb,
                *khl = tl + 5 * S::CDb;
        // W and U' as hi/lo tiles, element (i, c) at cm_off(i, c, C): the operands of this phase and,
        // stored as they are, of the output and backward kernels
        acc_read<C, D>(tb, 64, [&](int r, int c0, const float* v) { put8<C, true>(wth, wtl, r, c0, v); });
        acc_read<C, D>(tb, 192, [&](int r, int c0, const float* v) { put8<C, true>(uth, utl, r, c0, v); });
        const float* gC = sG + (n - 1) * LD;
        k_tile(khh, khl, [&](int i, int c, float x) { return x * tc::ex2(gC[c] - sG[i * LD + c]); });
        ok = run(sy, [&] {
          store_cd_tile(ws.W, base, wth, wtl);
          store_cd_tile(ws.U, base, uth, utl);
          const uint32_t id = tc::idesc_bf16(D, D, true, true);
          const tc::Op kH{tc::smem_u32(khh), C, true}, kL{tc::smem_u32(khl), C, true};
          const tc::Op wH{tc::smem_u32(wth), C, true}, wL{tc::smem_u32(wtl), C, true};
          const tc::Op uH{tc::smem_u32(uth), C, true}, uL{tc::smem_u32(utl), C, true};
          mma4(tb, kH, kL, wH, wL, C, id, false, false, false);        // Khat^T W
          mma4(tb + 128, kH, kL, uH, uL, C, id, false, false, false);  // Khat^T U'
        });
        if (ok) {
          // M (tile) and B (slice-major) are assembled in the consumed tile space (and the staging rows,
          // when they exist) and bulk-stored, once the W and U' stores have read their tiles
          uint8_t* Mt = reinterpret_cast<uint8_t*>(ws.Mt) + base * kMtileBytes;
          float* Bg = ws.Bc + base * D * D;
          constexpr bool kBsm = 6 * S::CDb + 2 * S::StB >= kMtileBytes + sizeof(float) * D * D;
          uint8_t* mts = tl;
          float* bs = reinterpret_cast<float*>(tl + kMtileBytes);
          if (tid == 0) tc::bulk_wait_read();
          __syncthreads();
          acc_read<D, D>(tb, 0, [&](int c, int c0, const float* v) {
            float m[16];
            const float gam = tc::ex2(gC[c]);
            for (int j = 0; j < 16; ++j) m[j] = (c0 + j == c ? gam : 0.f) - v[j];
            put16<D, true>(mts, mts + kMtileBytes / 2, c, c0, m);  // element (c, c'): K-major A (M = c)
          });
          tc::fence_async_smem();
          __syncthreads();
          if (tid == 0) {  // M leaves while B is assembled
            tc::bulk_s2g(Mt, mts, kMtileBytes);
            tc::bulk_commit();
          }
          acc_read<D, D>(tb, 128, [&](int c, int j0, const float* v) {  // slice-major for the scan's bulk loads
            float* dst = kBsm ? bs : Bg;
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(dst + slice_major(c, j0 + j)) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          });
          if constexpr (kBsm) {
            tc::fence_async_smem();
            __syncthreads();
            if (tid == 0) {
              tc::bulk_s2g(Bg, bs, sizeof(float) * D * D);
              tc::bulk_commit();
            }
          }
        }
      }
    }
    // the bulk stores have read the tiles and staging rows before the next head overwrites them
    if (tid == 0) tc::bulk_wait_read();  // (the stores complete with the grid)
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  if ((tid >> 5) == 0) tc::tmem_dealloc(tb, 512);
}

// --------------------------------------------------------------------------------- forward output
// per (chunk, head), with the chunk-start state S0 from the scan:
//   U = U' - W S0 (written back for the backward),  P = lower_incl(gated(q, k)),  O = Qbar S0 + P U,
//   and for the reverse scan Qeff = Qbar - P W (so that O = Qeff S0 + P U' and the state-independent
//   part of the reverse step is Qeff^T dO); Qeff is stored where W was (the backward recomputes W)
struct OutTcSmem {
  static constexpr int C = kTcC, D = kTcD, LD = D + 1;
  static constexpr size_t G = 0;
  static constexpr size_t vec = G + sizeof(float) * C * LD;  // ref[D]
  static constexpr size_t tiles = (vec + sizeof(float) * D + 1023) & ~size_t(1023);
  static constexpr size_t CDb = size_t(C) * D * 2, CCb = size_t(C) * C * 2, DDb = size_t(D) * D * 2;
  // R (4 CDb): run 1 qf + bf; run 2 P (2 CCb) + U (2 CDb).  Wq (2 CDb): W.  Qb (2 CDb): Qbar.
  static constexpr size_t R = tiles;
  static constexpr size_t Wq = R + 4 * CDb;
  static constexpr size_t Qb = Wq + 2 * CDb;
  static constexpr size_t S0 = Qb + 2 * CDb;    // S0 hi/lo (D x D, MN-major); then the Qeff tile
  static constexpr size_t total = S0 + 2 * DDb;
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kTcThreads, 1)
    kda_fwd_out_tc(DevTables t, int H, const Tin* __restrict__ q_, const Tin* __restrict__ k_,
                   const Tin* __restrict__ g_, Tout* __restrict__ o_, KdaWs ws, int chunk0 = 0, int hpc = 1) {
  using namespace tck;
  using S = OutTcSmem;
  constexpr int C = S::C, D = S::D, LD = S::LD;
  // grid (heads / hpc, chunks): a CTA runs hpc heads of one chunk in turn, the next head's gates, q
  // and k loaded into registers while the current head's products and epilogues run
  const int ci = chunk0 + (int)blockIdx.y, h0 = (int)blockIdx.x * hpc;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ __align__(1024) uint8_t tsm[];
  float* sG = reinterpret_cast<float*>(tsm + S::G);
  float* sref = reinterpret_cast<float*>(tsm + S::vec);
  __shared__ int srow[C];
  __shared__ __align__(8) uint64_t bar, bar_ld;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x;
  uint8_t *s0h = tsm + S::S0, *s0l = s0h + S::DDb;
  for (int i = tid; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  if ((tid >> 5) == 0) tc::tmem_alloc(&tslot, 512);
  Ld ld{&bar_ld, 0u, ws.status};
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_init(&bar_ld, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int hl = h0;  // the head whose inputs are being loaded
  auto row_q = [&](int a) -> const Tin* { return a < n ? q_ + ((size_t)srow[a] * H + hl) * D : nullptr; };
  auto row_k = [&](int a) -> const Tin* { return a < n ? k_ + ((size_t)srow[a] * H + hl) * D : nullptr; };
  GateRegs<Tin> gr;
  gate_ld(gr, g_, srow, H, hl, n);  // gates, q and k first, then the workspace tiles
  RawTile<Tin, C, D> rq, rk;
  raw_ld(rq, row_q);
  raw_ld(rk, row_k);
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  Sync sy{&bar, 0u, ws.status};
  bool ok = true;
  for (int hk = 0; hk < hpc && ok; ++hk) {
    const int h = h0 + hk;
    const size_t base = (size_t)ci * H + h;
    if (tid == 0) {
      ld_expect(ld, kStateTileBytes + kCDTileBytes);
      ld_state_tile(ld, s0h, s0l, ws.S0, base);  // the chunk-start state, as the scan left it
      ld_cd_tile(ld, tsm + S::Wq, tsm + S::Wq + S::CDb, ws.W, base);  // W, as the prep kernel left it
    }
    gate_st(sG, LD, gr);
    __syncthreads();
    uint8_t *qbh = tsm + S::Qb, *qbl = qbh + S::CDb;
    cumsum_ref(sG, LD, n, sref, nullptr, reinterpret_cast<float*>(qbh));  // (the Qbar tile comes later)
    // TMEM: P [0,64), W S0 [64,192), O [192,320), P W [320,448)
    uint8_t *qfh = tsm + S::R, *qfl = qfh + S::CDb, *bfh = qfl + S::CDb, *bfl = bfh + S::CDb;
    uint8_t *wh = tsm + S::Wq, *wl = wh + S::CDb;
    // qf = q e^{G - ref} and Qbar = q e^G from one load of q; bf = k e^{ref - G}
    build_tile2_raw<C, D, Tin>(
        qfh, qfl, qbh, qbl, rq, [&](int r, int c, float x) { return x * tc::ex2(sG[r * LD + c] - sref[c]); },
        [&](int r, int c, float x) { return x * tc::ex2(sG[r * LD + c]); });
    build_tile_raw<C, D, Tin>(bfh, bfl, rk, [&](int i, int c, float x) { return x * tc::ex2(sref[c] - sG[i * LD + c]); });
    if (hk + 1 < hpc) {  // the next head's inputs, into the registers just consumed
      hl = h + 1;
      gate_ld(gr, g_, srow, H, hl, n);
      raw_ld(rq, row_q);
      raw_ld(rk, row_k);
    }
    const tc::Op sH{tc::smem_u32(s0h), D, true}, sL{tc::smem_u32(s0l), D, true};
    ok = ld_wait(ld);
    ok = ok && run(sy, [&] {
      const tc::Op ah{tc::smem_u32(qfh), C, false}, al{tc::smem_u32(qfl), C, false};
      const tc::Op bh{tc::smem_u32(bfh), C, false}, bl{tc::smem_u32(bfl), C, false};
      const tc::Op wH{tc::smem_u32(wh), C, false}, wL{tc::smem_u32(wl), C, false};
      mma4(tb, ah, al, bh, bl, D, tc::idesc_bf16(C, C, false, false), false, false, false);
      mma4(tb + 64, wH, wL, sH, sL, D, tc::idesc_bf16(C, D, false, true), false, false, false);
    });
    uint8_t *ph = tsm + S::R, *pl = ph + S::CCb, *uh = pl + S::CCb, *ul = uh + S::CDb;
    if (ok) {
      if (tid == 0) {  // U' (as the prep kernel left it) into the consumed qf / bf space
        ld_expect(ld, kCDTileBytes);
        ld_cd_tile(ld, uh, ul, ws.U, base);
      }
      acc_read<C, C>(tb, 0, [&](int r, int i0, const float* v) {
        float m[8];
        for (int j = 0; j < 8; ++j) m[j] = (i0 + j <= r) ? v[j] : 0.f;
        put8<C, true>(ph, pl, r, i0, m);  // kept (as this tile) for the backward
      });
      ok = ld_wait(ld);
    }
    if (ok) {
      acc_read<C, D>(tb, 64, [&](int i, int j0, const float* v) {
        float u[8];
        tile8<C>(uh, ul, i, j0, u);  // U'
        for (int j = 0; j < 8; ++j) u[j] -= v[j];
        put8<C, true>(uh, ul, i, j0, u);  // U, element (i, j): MN-major (k = i); kept for the backward
      });
      ok = run(sy, [&] {
        store_cc_tile(ws.Pm, base, ph, pl);
        store_cd_tile(ws.U, base, uh, ul);  // U replaces U'

        const uint32_t id = tc::idesc_bf16(C, D, false, true);
        const tc::Op qH{tc::smem_u32(qbh), C, false}, qL{tc::smem_u32(qbl), C, false};
        const tc::Op pH{tc::smem_u32(ph), C, false}, pL{tc::smem_u32(pl), C, false};
        const tc::Op uH{tc::smem_u32(uh), C, true}, uL{tc::smem_u32(ul), C, true};
        const tc::Op wH{tc::smem_u32(wh), C, true}, wL{tc::smem_u32(wl), C, true};  // W as B (k = i, n = c)
        mma4(tb + 192, qH, qL, sH, sL, D, id, false, false, false);
        mma4(tb + 192, pH, pL, uH, uL, C, id, true, false, false);
        mma4(tb + 320, pH, pL, wH, wL, C, id, false, false, false);
      });
      if (ok) {
        acc_read<C, D>(tb, 192, [&](int r, int j0, const float* v) {
          if (r >= ch.n_replay && r < n) st8_out(o_ + ((size_t)srow[r] * H + h) * D + j0, v);
        });
        // Qeff = Qbar - P W (element (r, c)) into the S0 buffer, which the products above consumed
        uint8_t *eh = s0h, *el = s0h + S::CDb;
        acc_read<C, D>(tb, 320, [&](int r, int c0, const float* v) {
          float e[8];
          tile8<C>(qbh, qbl, r, c0, e);  // Qbar
          for (int j = 0; j < 8; ++j) e[j] -= v[j];
          put8<C, true>(eh, el, r, c0, e);
        });
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) store_cd_tile(ws.W, base, eh, el);
      }
    }
    // the bulk stores have read the tiles before the next head overwrites them
    if (tid == 0) tc::bulk_wait_read();  // (the stores complete with the grid)
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  if ((tid >> 5) == 0) tc::tmem_dealloc(tb, 512);
}

// --------------------------------------------------------------------------------- backward dq
// per (chunk, head), with S0 (chunk start state), dS (gradient of the chunk end state), U and P:
//   dU = P^T dO + Khat dS                                   (for the dk / dv kernel)
//   dP = lower_incl(dO U^T), Tq = dO S0^T, T1 = U dS^T,
//   RS = dP bf (bf = k e^{G_0 - G}),  CS = dP^T qf (qf = q e^{G - G_0})
//   dq  = e^G Tq + e^{G - G_0} RS                         (final)
//   pdk = e^{G_C - G} T1 + e^{G_0 - G} CS                 (partial dk)
//   pdG = q dq - k pdk,  pdG[n-1] += sum_i k_i e^{G_C - G_i} T1_i + e^{G_C} rowsum(dS * S0)
struct BdqTcSmem {
  static constexpr int C = kTcC, D = kTcD, LD = D + 1;
  static constexpr size_t G = 0;
  static constexpr size_t vec = G + sizeof(float) * C * LD;  // ref[D], e0[D] = 2^{G_0}, eC0[D] = 2^{G_C - G_0}
  static constexpr size_t tiles = (vec + sizeof(float) * 3 * D + 1023) & ~size_t(1023);
  static constexpr size_t CDb = size_t(C) * D * 2, CCb = size_t(C) * C * 2, DDb = size_t(D) * D * 2;
  // phase 1: dO (K-major) | U (K-major) | S0 (K-major D x D); phase 2: dS in the S0 slot;
  // phase 3: dP | bf (MN) | qf (MN) over the dO/U/S0 space; epilogue row buffer (C x LD fp32) after.
  // Pt: the forward's P tile (element (r, i)), read as P^T for dU = P^T dO + Khat dS.
  static constexpr size_t R = tiles;
  static constexpr size_t Pt = R + 4 * CDb + 2 * DDb;
  static constexpr size_t Stage = Pt + 2 * CCb;  // bf16 inputs: the chunk's q and k rows (pitch kStagePitch)
  static constexpr size_t StB = size_t(C) * tck::kStagePitch * 2;
  static constexpr size_t Scr = Stage + 2 * StB;  // 4 x D fp32 scratch of the gate accumulation
  static constexpr size_t total = Scr + sizeof(float) * 4 * D;
  // epilogue, inside R: row buffer (C x LD fp32), fp32 staging of q and k (fp32 inputs), column partials
  static constexpr size_t Part = sizeof(float) * C * LD + 2 * sizeof(float) * C * tck::kStagePitch;
  static_assert(Part + sizeof(float) * 8 * D <= 4 * CDb + 2 * DDb, "epilogue scratch exceeds R");
  static_assert(total <= 227 * 1024, "shared memory");
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kTcThreads, 1)
    kda_bwd_dq_tc(DevTables t, int H, const Tin* __restrict__ q_, const Tin* __restrict__ k_,
                  const Tin* __restrict__ g_, const Tin* __restrict__ do_, Tout* __restrict__ dq_, KdaWs ws,
                  int chunk0 = 0, int hpc = 1) {
  using namespace tck;
  using S = BdqTcSmem;
  constexpr int C = S::C, D = S::D, LD = S::LD;
  constexpr bool EX = std::is_same<Tin, __nv_bfloat16>::value;
  // grid (heads / hpc, chunks): a CTA runs hpc heads of one chunk in turn, the next head's gates
  // loaded into registers while the current head computes
  const int ci = chunk0 + (int)blockIdx.y, h0 = (int)blockIdx.x * hpc;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ __align__(1024) uint8_t tsm[];
  float* sG = reinterpret_cast<float*>(tsm + S::G);
  float* sref = reinterpret_cast<float*>(tsm + S::vec);
  __shared__ int srow[C];
  __shared__ __align__(8) uint64_t bar, bar_ld;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x;
  uint8_t *doh = tsm + S::R, *dol = doh + S::CDb, *uh = dol + S::CDb, *ul = uh + S::CDb;
  uint8_t *sh = ul + S::CDb, *sl = sh + S::DDb;
  for (int i = tid; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  if ((tid >> 5) == 0) tc::tmem_alloc(&tslot, 512);
  Ld ld{&bar_ld, 0u, ws.status};
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_init(&bar_ld, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  GateRegs<Tin> gr;
  gate_ld(gr, g_, srow, H, h0, n);  // gates first, then the workspace tiles and the row gathers
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  Sync sy{&bar, 0u, ws.status};
  bool ok = true;
  for (int hk = 0; hk < hpc && ok; ++hk) {
    const int h = h0 + hk;
    const size_t base = (size_t)ci * H + h;
    if (tid == 0) {
      ld_expect(ld, kStateTileBytes + kCDTileBytes + kCCTileBytes);
      ld_state_tile(ld, sh, sl, ws.S0, base);  // chunk-start state
      ld_cd_tile(ld, uh, ul, ws.U, base);        // U, as the output kernel left it
      ld_cc_tile(ld, tsm + S::Pt, tsm + S::Pt + S::CCb, ws.Pm, base);  // P, as the output kernel left it
    }
    // bf16: the chunk's q and k rows into shared memory while the gates load and accumulate
    [[maybe_unused]] __nv_bfloat16* stq = reinterpret_cast<__nv_bfloat16*>(tsm + S::Stage);
    [[maybe_unused]] __nv_bfloat16* stk = reinterpret_cast<__nv_bfloat16*>(tsm + S::Stage + S::StB);
    auto row_q = [&](int a) -> const Tin* { return a < n ? q_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    auto row_k = [&](int a) -> const Tin* { return a < n ? k_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    auto row_do = [&](int a) -> const Tin* {
      return (a >= ch.n_replay && a < n) ? do_ + ((size_t)srow[a] * H + h) * D : nullptr;
    };
    if constexpr (EX) {  // dO straight into its operand tile (raw bf16: no lo part)
      stage_rows_async(stq, q_, srow, H, h, n);
      stage_rows_async(stk, k_, srow, H, h, n);
      tile_async_bf16<C, D>(doh, row_do, do_);
    }
    gate_st(sG, LD, gr);
    if (hk + 1 < hpc) gate_ld(gr, g_, srow, H, h + 1, n);  // the next head's gates
    __syncthreads();
    cumsum_ref(sG, LD, n, sref, nullptr, reinterpret_cast<float*>(tsm + S::Scr));
    float* se0 = sref + D;  // per channel 2^{G_0} and 2^{G_C - G_0} (ready long before the epilogue)
    float* seC0 = se0 + D;
    for (int c = tid; c < D; c += blockDim.x) {
      se0[c] = tc::ex2(sref[c]);
      seC0[c] = tc::ex2(sG[(n - 1) * LD + c] - sref[c]);
    }
    if constexpr (EX) tc::cp_async_wait<0>();
    __syncthreads();
    tc::fence_after_sync();
    // TMEM columns: Tq [0,128), T1 [128,256), RS [256,384), dP [384,448) then CS [384,512)
    constexpr int cTq = 0, cT1 = 128, cRS = 256, cCS = 384;
    if constexpr (!EX) build_tile_ld<C, D, true, Tin>(doh, dol, row_do, [&](int, int, float x) { return x; });
    const tc::Op oH{tc::smem_u32(doh), C, false}, oL{tc::smem_u32(dol), C, false};
    const tc::Op uH{tc::smem_u32(uh), C, false}, uL{tc::smem_u32(ul), C, false};
    const tc::Op sH{tc::smem_u32(sh), D, false}, sL{tc::smem_u32(sl), D, false};
    ok = ld_wait(ld);
    ok = ok && run(sy, [&] {
      mma4(tb + cCS, oH, oL, uH, uL, D, tc::idesc_bf16(C, C, false, false), false, EX, false);   // dP (raw)
      {  // dU = P^T dO, accumulated further in phase 2 (P^T: the P tile read MN-major; dO read MN-major)
        const tc::Op pH{tc::smem_u32(tsm + S::Pt), C, true}, pL{tc::smem_u32(tsm + S::Pt + S::CCb), C, true};
        const tc::Op dH{tc::smem_u32(doh), C, true}, dL{tc::smem_u32(dol), C, true};
        mma4(tb + cRS, pH, pL, dH, dL, C, tc::idesc_bf16(C, D, true, true), false, false, EX);
      }
      mma4(tb + cTq, oH, oL, sH, sL, D, tc::idesc_bf16(C, D, false, false), false, EX, false);  // Tq
    });
    if (ok) {
      // phase 2: T1 = U dS^T and dU = dU0 + Khat dS (Khat = k e^{G_C - G}, K-major in the dO slot);
      // the gradient of the chunk-end state replaces S0 in its buffer
      if (tid == 0) {
        ld_expect(ld, kStateTileBytes);
        ld_state_tile(ld, sh, sl, ws.dS, base);
      }
      const float* gC = sG + (n - 1) * LD;
      auto khf = [&](int i, int c, float x) { return x * tc::ex2(gC[c] - sG[i * LD + c]); };
      if constexpr (EX) build_tile_st<C, D, true>(doh, dol, stk, khf);
      else build_tile_ld<C, D, true, Tin>(doh, dol, row_k, khf);
      ok = ld_wait(ld);
      ok = ok && run(sy, [&] {
        mma4(tb + cT1, uH, uL, sH, sL, D, tc::idesc_bf16(C, D, false, false), false, false, false);
        const tc::Op kH{tc::smem_u32(doh), C, false}, kL{tc::smem_u32(dol), C, false};
        const tc::Op dH{tc::smem_u32(sh), D, true}, dL{tc::smem_u32(sl), D, true};
        mma4(tb + cRS, kH, kL, dH, dL, D, tc::idesc_bf16(C, D, false, true), true, false, false);
      });
      if (ok) {
        // dU = dU0 + Khat dS as a hi/lo tile (element (i, j) at cm_off(i, j, C), in the consumed Khat
        // slot) for the dk / dv kernel
        acc_read<C, D>(tb, cRS, [&](int i, int j0, const float* v) { put8<C, true>(doh, dol, i, j0, v); });
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
          store_cd_tile(ws.dUt, base, doh, dol);
          tc::bulk_wait_read();
        }
        __syncthreads();
      }
    }
    uint8_t *pH8 = tsm + S::R, *pL8 = pH8 + S::CCb, *bh = pL8 + S::CCb, *bl = bh + S::CDb, *qh = bl + S::CDb,
            *ql = qh + S::CDb;
    if (ok) {
      acc_read<C, C>(tb, cCS, [&](int r, int i0, const float* v) {
        float m[8];
        for (int j = 0; j < 8; ++j) m[j] = (i0 + j <= r) ? v[j] : 0.f;
        put8<C, true>(pH8, pL8, r, i0, m);  // element (r, i)
      });
      auto bff = [&](int i, int c, float x) { return x * tc::ex2(sref[c] - sG[i * LD + c]); };
      auto qff = [&](int r, int c, float x) { return x * tc::ex2(sG[r * LD + c] - sref[c]); };
      if constexpr (EX) {
        build_tile_st<C, D, true>(bh, bl, stk, bff);
        build_tile_st<C, D, true>(qh, ql, stq, qff);
      } else {
        build_tile_ld<C, D, true, Tin>(bh, bl, row_k, bff);
        build_tile_ld<C, D, true, Tin>(qh, ql, row_q, qff);
      }
      ok = run(sy, [&] {
        const uint32_t id = tc::idesc_bf16(C, D, false, true), idT = tc::idesc_bf16(C, D, true, true);
        const tc::Op pK{tc::smem_u32(pH8), C, false}, pKl{tc::smem_u32(pL8), C, false};  // dP (r, i), K-major
        const tc::Op pM{tc::smem_u32(pH8), C, true}, pMl{tc::smem_u32(pL8), C, true};    // dP^T (i, r), MN-major
        const tc::Op bH{tc::smem_u32(bh), C, true}, bL{tc::smem_u32(bl), C, true};
        const tc::Op qH{tc::smem_u32(qh), C, true}, qL{tc::smem_u32(ql), C, true};
        mma4(tb + cRS, pK, pKl, bH, bL, C, id, false, false, false);
        mma4(tb + cCS, pM, pMl, qH, qL, C, idT, false, false, false);
      });
    }
    if (ok) {
      float* pdk = ws.pdk + base * C * D;
      float* pdG = ws.pdG + base * C * D;
      float* sbuf = reinterpret_cast<float*>(tsm + S::R);  // [C][LD]: k e^{G_C - G} T1 per row
      Tin* sq = reinterpret_cast<Tin*>(tsm + S::R + sizeof(float) * C * LD);
      Tin* sk = sq + C * kStagePitch;
      if constexpr (EX) {  // staged at the start
        sq = reinterpret_cast<Tin*>(stq);
        sk = reinterpret_cast<Tin*>(stk);
      } else {
        stage_rows(sq, q_, srow, H, h, n);
        stage_rows(sk, k_, srow, H, h, n);
      }
      __syncthreads();
      const int w = tid >> 5, lane = tid & 31, sp = w & 3, grp = w >> 2;
      const int r = 16 * sp + (lane & 15);  // accumulator row; this lane's 8 columns: share8
      const uint32_t la = tb + ((uint32_t)(32 * sp) << 16);
      static_assert(D == 2 * 16 * kTcGroups && C == 64 && kTcGroups == 4, "the pd_frag lane map");
      for (int it = 0; it < 2; ++it) {
        const int cc = grp * 16 + 16 * kTcGroups * it;
        float tq[8], t1[8], rs[8], cs[8];
        {
          uint32_t a0[16], a1[16], a2[16], a3[16];  // four loads in flight, one wait
          tc::tmem_ld16_nowait(la + cTq + cc, a0);
          tc::tmem_ld16_nowait(la + cT1 + cc, a1);
          tc::tmem_ld16_nowait(la + cRS + cc, a2);
          tc::tmem_ld16_nowait(la + cCS + cc, a3);
          tc::tmem_wait_ld();
          tc::tmem_regs16(a0);
          tc::tmem_regs16(a1);
          tc::tmem_regs16(a2);
          tc::tmem_regs16(a3);
          share8u(a0, tq);
          share8u(a1, t1);
          share8u(a2, rs);
          share8u(a3, cs);
        }
        const int c0 = cc + 8 * (lane >> 4);
        float qv[8], kv[8], dq[8], dk[8], dG[8];
        staged8(sq, r, c0, qv);
        staged8(sk, r, c0, kv);
  #pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = c0 + j;
          // a = 2^{G_r - G_0} (bounded by the chunk's decay check), 1/a = 2^{G_0 - G_r};
          // 2^{G_r} = 2^{G_0} a and 2^{G_C - G_r} = 2^{G_C - G_0} / a
          const float a = tc::ex2(sG[r * LD + c] - sref[c]), ia = tc::rcp_approx(a);
          dq[j] = a * fmaf(se0[c], tq[j], rs[j]);
          const float dks = seC0[c] * ia * t1[j];
          dk[j] = fmaf(ia, cs[j], dks);
          dG[j] = qv[j] * dq[j] - kv[j] * dk[j];
          sbuf[r * LD + c] = r < n ? kv[j] * dks : 0.f;
        }
        {
          float4* pk = reinterpret_cast<float4*>(pdk) + pd_frag(w, it, lane);
          float4* pg = reinterpret_cast<float4*>(pdG) + pd_frag(w, it, lane);
          pk[0] = make_float4(dk[0], dk[1], dk[2], dk[3]);
          pk[32] = make_float4(dk[4], dk[5], dk[6], dk[7]);
          pg[0] = make_float4(dG[0], dG[1], dG[2], dG[3]);
          pg[32] = make_float4(dG[4], dG[5], dG[6], dG[7]);
        }
        if (r >= ch.n_replay && r < n) st8_out(dq_ + ((size_t)srow[r] * H + h) * D + c0, dq);
      }
      __syncthreads();
      // per column c: sum over rows of the row buffer and sum_j dS_cj S0_cj, each split over four
      // threads (rows and j in quarters) and combined in a fixed order
      static_assert(kTcThreads == 4 * D, "four threads per column");
      float* part = reinterpret_cast<float*>(tsm + S::R + S::Part);  // [2][4][D]
      {
        const int c = tid % D, q4 = tid / D;
        float a = 0.f;
        for (int i = 16 * q4; i < 16 * q4 + 16; ++i) a += sbuf[i * LD + c];  // rows >= n hold zeros
        part[q4 * D + c] = a;
        part[(4 + q4) * D + c] = state_row_dot(ws.dS, ws.S0, base, c, 32 * q4, 32 * q4 + 32);
      }
      __syncthreads();
      if (tid < D) {
        const int c = tid;
        const float acc = (part[c] + part[D + c]) + (part[2 * D + c] + part[3 * D + c]);
        const float acc2 = (part[4 * D + c] + part[5 * D + c]) + (part[6 * D + c] + part[7 * D + c]);
        pdG[pd_index(n - 1, c)] += acc + tc::ex2(sG[(n - 1) * LD + c]) * acc2;
      }
    }
    // the bulk stores have read their tiles before the next head overwrites them
    if (tid == 0) tc::bulk_wait_read();  // (the stores complete with the grid)
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  if ((tid >> 5) == 0) tc::tmem_dealloc(tb, 512);
}

// --------------------------------------------------------------------------------- backward dk/dv
// per (chunk, head), the WY part of the backward:
//   Atilde = gated(k, k) (strict lower), T = (I + diag(beta) Atilde)^{-1}, X = [W | U'] = T diag(beta) [Kbar | V]
//   dX = [-dU S0^T | dU],  dB = T^T dX,  dA = -strict_lower(dB X^T),  dAt = diag(beta) dA
//   dk  = pdk + e^G beta dB_k + e^{G-G_0} (dAt bf) + e^{G_0-G} (dAt^T af)
//   dG  = pdG + Kbar beta dB_k + k (e^{G-G_0} (dAt bf) - e^{G_0-G} (dAt^T af)),  dg = reverse cumsum of dG
//   dv  = beta dB_v,  dbeta = rowsum(dB_k Kbar + dB_v v + dA Atilde)
// Replayed rows go to the replay partials, rows replayed elsewhere to the target staging.
// bf16 inputs stage the chunk's k rows in shared memory; fp32 inputs (twice the bytes, which do not
// fit beside the other tiles) read them from global memory instead.
template <typename Tin>
struct BdkvTcSmemT {
  static constexpr bool kStageK = sizeof(Tin) == 2;
  static constexpr int C = kTcC, D = kTcD, LD = D + 1, LC = C + 1;
  static constexpr size_t G = 0;
  static constexpr size_t At = G + sizeof(float) * C * LD;        // Atilde fp32 [C][LC]
  // beta[C], ref[D], dbeta parts[3][groups][C], e0[D] = 2^{G_0}
  static constexpr size_t vec = At + sizeof(float) * C * LC;
  static constexpr size_t Ks = (vec + sizeof(float) * (C + 2 * D + 3 * kTcGroups * C) + 15) & ~size_t(15);  // staged k
  static constexpr size_t Tt = (Ks + (kStageK ? sizeof(Tin) * C * tck::kStagePitch : 0) + 1023) & ~size_t(1023);  // T tile
  static constexpr size_t CCb = size_t(C) * C * 2, CDb = size_t(C) * D * 2, DDb = size_t(D) * D * 2;
  static constexpr size_t R = Tt + 2 * CCb;
  static constexpr size_t Rbytes = 128 * 1024;
  static constexpr size_t total = R + Rbytes;
  // offsets inside R by phase
  static constexpr size_t p2_Tp = 44 * 1024, p2_Kb = p2_Tp + 2 * CCb, p2_V = p2_Kb + 2 * CDb;  // T', Kbar, V
  static constexpr size_t p2_S0 = 0;                                                   // S0 (K); dU in dX
  static constexpr size_t p3_X = 0, p3_dX = 4 * CDb;                                   // X (K, C x 2D), dX (MN)
  static constexpr size_t p4_dB = 4 * CDb;                                             // dB (K, C x 2D)
  static constexpr size_t p5_dA = 0, p5_bf = 2 * CCb, p5_af = p5_bf + 2 * CDb;         // dAt, bf (MN), af (MN)
  static_assert(p2_V + 2 * CDb <= Rbytes && p2_S0 + 2 * DDb <= p3_dX && p3_dX + 4 * CDb <= Rbytes, "R");
  static_assert(total <= 227 * 1024, "shared memory");
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kTcThreads, 1)
    kda_bwd_dkv_tc(DevTables t, int H, const Tin* __restrict__ k_, const Tin* __restrict__ v_,
                   const Tin* __restrict__ g_, const Tin* __restrict__ beta_, Tout* __restrict__ dk_,
                   Tout* __restrict__ dv_, float* __restrict__ dg_, float* __restrict__ dbeta_, KdaWs ws,
                   int chunk0 = 0, int hpc = 1) {
  using namespace tck;
  using S = BdkvTcSmemT<Tin>;
  constexpr int C = S::C, D = S::D, LD = S::LD, LC = S::LC;
  constexpr bool EX = std::is_same<Tin, __nv_bfloat16>::value;
  // grid (heads / hpc, chunks): a CTA runs hpc heads of one chunk in turn, the next head's gates
  // loaded into registers while the current head computes
  const int ci = chunk0 + (int)blockIdx.y, h0 = (int)blockIdx.x * hpc;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ __align__(1024) uint8_t tsm[];
  float* sG = reinterpret_cast<float*>(tsm + S::G);
  float* sAt = reinterpret_cast<float*>(tsm + S::At);
  float* sb = reinterpret_cast<float*>(tsm + S::vec);
  float* sref = sb + C;
  float* sdb = sref + D;  // [3][kTcGroups][C] partial dbeta (dB_k, dB_v, dA parts per warp group), fixed-order sum
  uint8_t* tTh = tsm + S::Tt;
  uint8_t* tTl = tTh + S::CCb;
  uint8_t* R = tsm + S::R;
  __shared__ int srow[C];
  // where row r's gradients go: kind 0 the replay partials (row idx), 1 the target staging (row idx),
  // 2 the outputs (row idx = srow)
  __shared__ int skind[C], sidx[C];
  __shared__ __align__(8) uint64_t bar, bar_ld;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x;
  for (int i = tid; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  if ((tid >> 5) == 0) tc::tmem_alloc(&tslot, 512);
  Ld ld{&bar_ld, 0u, ws.status};
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_init(&bar_ld, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  GateRegs<Tin> gr;
  gate_ld(gr, g_, srow, H, h0, n);  // gates and beta first, then the copies
  Tin bv = tid < n ? beta_[(size_t)srow[tid] * H + h0] : Tin(0.f);  // (converted when stored)
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  Sync sy{&bar, 0u, ws.status};
  bool ok = true;
  for (int hk = 0; hk < hpc && ok; ++hk) {
    const int h = h0 + hk;
    const size_t base = (size_t)ci * H + h;
    for (int e = tid; e < 3 * kTcGroups * C; e += blockDim.x) sdb[e] = 0.f;
    Tin* sk = reinterpret_cast<Tin*>(tsm + S::Ks);
    auto row_v = [&](int a) -> const Tin* { return a < n ? v_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    if constexpr (S::kStageK) {
      stage_rows_async(reinterpret_cast<__nv_bfloat16*>(sk), reinterpret_cast<const __nv_bfloat16*>(k_), srow, H, h, n);
      tile_async_bf16<C, D>(R + S::p2_V, row_v, v_);  // V straight into its phase-2a operand tile
    }
    {  // Atilde (fp32, padded rows) by 4-byte asynchronous copies; T (hi/lo tile) by a bulk copy
      const size_t cb = (size_t)ci * H + h;
      const float* Ag = ws.At + cb * C * C;
      for (int e = tid; e < C * C; e += blockDim.x) tc::cp_async4(sAt + (e / C) * LC + (e % C), Ag + e, 4u);
      tc::cp_async_commit();
      if (tid == 0) {
        ld_expect(ld, kCCTileBytes);
        ld_cc_tile(ld, tTh, tTl, ws.Tm, cb);
      }
    }
    if (tid < C) {  // where row tid's gradients go (read while the gates are in flight)
      const int i = tid, row = srow[i];
      int kind = 2, idx = row;
      if (i < ch.n_replay) {
        kind = 0;
        idx = ch.replay_base + i;
      } else if (i < n) {
        const int tg = t.row_tgt[row];
        if (tg >= 0) {
          kind = 1;
          idx = tg;
        }
      }
      skind[i] = kind;
      sidx[i] = idx;
    }
    gate_st(sG, LD, gr);
    if (tid < C) sb[tid] = to_f(bv);
    if (hk + 1 < hpc) {  // the next head's gates and beta, into the registers just consumed
      gate_ld(gr, g_, srow, H, h + 1, n);
      bv = tid < n ? beta_[(size_t)srow[tid] * H + h + 1] : Tin(0.f);
    }
    __syncthreads();
    cumsum_ref(sG, LD, n, sref, nullptr, reinterpret_cast<float*>(R));  // (R's first phase comes later)
    float* se0 = sdb + 3 * kTcGroups * C;  // per channel 2^{G_0}
    for (int c = tid; c < D; c += blockDim.x) se0[c] = tc::ex2(sref[c]);
    tc::cp_async_wait<0>();  // staged k, V and Atilde
    __syncthreads();
    tc::fence_after_sync();
    auto row_k = [&](int a) -> const Tin* { return a < n ? k_ + ((size_t)srow[a] * H + h) * D : nullptr; };
    // 8 values of k row r from column c0 on (zero for r >= n)
    auto k8 = [&](int r, int c0, float(&kv)[8]) {
      if constexpr (S::kStageK) {
        staged8(sk, r, c0, kv);
      } else if (r < n) {
        ld8(k_ + ((size_t)srow[r] * H + h) * D + c0, kv);
      } else {
  #pragma unroll
        for (int j = 0; j < 8; ++j) kv[j] = 0.f;
      }
    };
    float* pdk = ws.pdk + base * C * D;
    float* pdG = ws.pdG + base * C * D;
    const int w = tid >> 5, lane = tid & 31, sp = w & 3, grp = w >> 2;
    const int myrow = 16 * sp + (lane & 15);  // M = 64 accumulator row; this lane's 8 columns: share8
    const int half8 = 8 * (lane >> 4);
    float pre_dk[2][8], pre_dG[2][8];  // the final phase's dq-kernel partials (loaded ahead)
    uint4 vraw[2][sizeof(Tin) / 2];     // phase 4's v values (loaded ahead, raw)
    // 8 gradient values of row r from column c0 on, to where the row's gradients go
    auto out8 = [&](float* replay_buf, float* tgt_buf, Tout* out, int r, int c0, const float* v) {
      const size_t o = ((size_t)sidx[r] * H + h) * D + c0;
      if (skind[r] == 0) st8g(replay_buf + o, v);
      else if (skind[r] == 1) st8g(tgt_buf + o, v);
      else st8_out(out + o, v);
    };
    const uint32_t la = tb + ((uint32_t)(32 * sp) << 16);
    // TMEM columns
    // dB_k [0, 128) stays in TMEM until the last phase; CS reuses the dB_v columns [128, 256)
    constexpr int cW = 64, cU = 192, cdW = 320, cdB = 0, cdA = 256, cRS = 320, cCS = 128;

    // ---- phase 1: Atilde and T as the forward left them (loaded above)
    ok = ld_wait(ld);
    // element (r, i) of T from its hi/lo tile
    auto tval = [&](int r, int i) {
      const uint32_t o = cm_off(r, i, C);
      return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tTh + o)) +
             __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tTl + o));
    };
    if (ok) {
      // ---- phase 2a: W = T' Kbar, U' = T' V (T' = T diag(beta)); the T tile for T^T dX
      uint8_t *tph = R + S::p2_Tp, *tpl = tph + S::CCb, *kbh = R + S::p2_Kb, *kbl = kbh + S::CDb, *vh = R + S::p2_V,
              *vl = vh + S::CDb;
      build_tile<C, C, true>(tph, tpl, [&](int r, int i) { return tval(r, i) * sb[i]; });
      auto kbf = [&](int i, int c, float x) { return x * tc::ex2(sG[i * LD + c]); };
      if constexpr (S::kStageK) build_tile_st<C, D, true>(kbh, kbl, reinterpret_cast<const __nv_bfloat16*>(sk), kbf);
      else build_tile_ld<C, D, true, Tin>(kbh, kbl, row_k, kbf);
      if constexpr (!EX) build_tile_ld<C, D, true, Tin>(vh, vl, row_v, [&](int i, int c, float x) { return x; });
      ok = run(sy, [&] {
        const uint32_t id = tc::idesc_bf16(C, D, false, true);
        const tc::Op tH{tc::smem_u32(tph), C, false}, tL{tc::smem_u32(tpl), C, false};
        const tc::Op kH{tc::smem_u32(kbh), C, true}, kL{tc::smem_u32(kbl), C, true};
        const tc::Op vH{tc::smem_u32(vh), C, true}, vL{tc::smem_u32(vl), C, true};
        mma4(tb + cW, tH, tL, kH, kL, C, id, false, false, false);
        mma4(tb + cU, tH, tL, vH, vL, C, id, false, false, EX);
      });
    }
    if (ok) {
      // ---- phase 2b: dW' = dU S0^T.  dU is loaded where phase 3's dX keeps its columns [D, 2D) (a
      // C x D sub-tile of the K-major C x 2D layout is itself a C x D K-major tile), S0 where X goes.
      uint8_t *dxh0 = R + S::p3_dX, *dxl0 = dxh0 + 2 * S::CDb;
      uint8_t *duh = dxh0 + tc::cm_off(0, D, C), *dul = dxl0 + tc::cm_off(0, D, C);
      uint8_t *s0h = R + S::p2_S0, *s0l = s0h + S::DDb;
      if (tid == 0) {  // the phase 2a operands are consumed
        ld_expect(ld, kStateTileBytes + kCDTileBytes);
        ld_state_tile(ld, s0h, s0l, ws.S0, base);
        ld_cd_tile(ld, duh, dul, ws.dUt, base);
      }
      ok = ld_wait(ld);
      ok = ok && run(sy, [&] {
        const tc::Op aH{tc::smem_u32(duh), C, false}, aL{tc::smem_u32(dul), C, false};
        const tc::Op bH{tc::smem_u32(s0h), D, false}, bL{tc::smem_u32(s0l), D, false};
        mma4(tb + cdW, aH, aL, bH, bL, D, tc::idesc_bf16(C, D, false, false), false, false, false);
      });
    }
    if (ok) {
      // ---- phase 3: X (K-major, rows i, columns n in [0, 2D)) and dX (MN-major, k = r, n)
      uint8_t *xh = R + S::p3_X, *xl = xh + 2 * S::CDb, *dxh = R + S::p3_dX, *dxl = dxh + 2 * S::CDb;
      // this lane's v values for phase 4 (its rows' columns of dB_v), loaded now and converted there
      static_assert(2 * D == 4 * 16 * kTcGroups, "four 16-column chunks of dB per warp group");
      for (int t2 = 0; t2 < 2; ++t2) {
        const int c1 = grp * 16 + 16 * kTcGroups * t2 + half8;
        const Tin* p = v_ + ((size_t)srow[myrow] * H + h) * D + c1;
  #pragma unroll
        for (int q = 0; q < (int)(sizeof(Tin) / 2); ++q)
          vraw[t2][q] = myrow < n ? __ldg(reinterpret_cast<const uint4*>(p) + q) : make_uint4(0u, 0u, 0u, 0u);
      }
      acc_read<C, D>(tb, cW, [&](int i, int c0, const float* v) { put8<C, true>(xh, xl, i, c0, v); });
      acc_read<C, D>(tb, cU, [&](int i, int c0, const float* v) { put8<C, true>(xh, xl, i, D + c0, v); });
      acc_read<C, D>(tb, cdW, [&](int r, int c0, const float* v) {
        float m[8];
        for (int j = 0; j < 8; ++j) m[j] = -v[j];
        put8<C, true>(dxh, dxl, r, c0, m);
      });
      // (dX columns [D, 2D) = dU, loaded in phase 2b)
      ok = run(sy, [&] {
        const tc::Op aH{tc::smem_u32(tTh), C, true}, aL{tc::smem_u32(tTl), C, true};
        const tc::Op bH{tc::smem_u32(dxh), C, true}, bL{tc::smem_u32(dxl), C, true};
        mma4(tb + cdB, aH, aL, bH, bL, C, tc::idesc_bf16(C, 2 * D, true, true), false, false, false);
      });
    }
    if (ok) {
      // ---- read dB: dB tile for dA; dv; dk / dG / dbeta contributions
      uint8_t *dbh = R + S::p4_dB, *dbl = dbh + 2 * S::CDb;
  #pragma unroll
      for (int t4 = 0; t4 < 4; ++t4) {
        const int cc = grp * 16 + 16 * kTcGroups * t4;
        float v[8];
        {
          float v16[16];
          tc::tmem_ld16(la + cdB + cc, v16);
          share8(v16, v);
        }
        const int i = myrow, c0 = cc + half8;
        put8<C, true>(dbh, dbl, i, c0, v);
        float part = 0.f;
        if (t4 < 2) {  // columns < D: dB_k (its dk / dG terms are added in the last phase, from TMEM)
          float kv[8];
          k8(i, c0, kv);
  #pragma unroll
          for (int j = 0; j < 8; ++j) part = fmaf(v[j], kv[j] * tc::ex2(sG[i * LD + c0 + j]), part);
        } else if (i < n) {
          const int c1 = c0 - D;
          float vv[8], val[8];
          raw_get<Tin>(vraw[t4 - 2], vv);
  #pragma unroll
          for (int j = 0; j < 8; ++j) {
            part = fmaf(v[j], vv[j], part);
            val[j] = sb[i] * v[j];
          }
          out8(ws.rdv, ws.tdv, dv_, i, c1, val);
        }
        part += __shfl_sync(0xffffffffu, part, (lane + 16) & 31);  // columns 0-7 + 8-15 of the chunk
        if (lane < 16) sdb[((t4 < 2 ? 0 : 1) * kTcGroups + grp) * C + i] += part;  // one slot per (half, group)
      }
      uint8_t *xh = R + S::p3_X, *xl = xh + 2 * S::CDb;
      ok = run(sy, [&] {
        const tc::Op aH{tc::smem_u32(dbh), C, false}, aL{tc::smem_u32(dbl), C, false};
        const tc::Op bH{tc::smem_u32(xh), C, false}, bL{tc::smem_u32(xl), C, false};
        mma4(tb + cdA, aH, aL, bH, bL, 2 * D, tc::idesc_bf16(C, C, false, false), false, false, false);
      });
    }
    if (ok) {
      // ---- dA = -(dB X^T) strict lower; dAt = beta dA (tile); dbeta += rowsum(dA Atilde)
      uint8_t *dah = R + S::p5_dA, *dal = dah + S::CCb;
      for (int cc = grp * 16; cc < C; cc += 16 * kTcGroups) {
        float v[8];
        {
          float v16[16];
          tc::tmem_ld16(la + cdA + cc, v16);
          share8(v16, v);
        }
        const int r = myrow, c0 = cc + half8;
        float m[8], part = 0.f;
        for (int j = 0; j < 8; ++j) {
          const int i = c0 + j;
          const float dA = (i < r) ? -v[j] : 0.f;
          part = fmaf(dA, sAt[r * LC + i], part);
          m[j] = sb[r] * dA;
        }
        put8<C, true>(dah, dal, r, c0, m);  // element (r, i)
        part += __shfl_sync(0xffffffffu, part, (lane + 16) & 31);
        if (lane < 16) sdb[(2 * kTcGroups + grp) * C + r] += part;
      }
      // the dq kernel's partials of this lane's final-phase rows and columns, loaded ahead of phase 5
      static_assert(D == 2 * 16 * kTcGroups, "two 16-column chunks per warp group in the final phase");
      for (int it = 0; it < 2; ++it) {  // (the pd_frag order of the dq kernel's epilogue)
        const float4* pk = reinterpret_cast<const float4*>(pdk) + pd_frag(w, it, lane);
        const float4* pg = reinterpret_cast<const float4*>(pdG) + pd_frag(w, it, lane);
        const float4 a0 = pk[0], a1 = pk[32], b0 = pg[0], b1 = pg[32];
        pre_dk[it][0] = a0.x; pre_dk[it][1] = a0.y; pre_dk[it][2] = a0.z; pre_dk[it][3] = a0.w;
        pre_dk[it][4] = a1.x; pre_dk[it][5] = a1.y; pre_dk[it][6] = a1.z; pre_dk[it][7] = a1.w;
        pre_dG[it][0] = b0.x; pre_dG[it][1] = b0.y; pre_dG[it][2] = b0.z; pre_dG[it][3] = b0.w;
        pre_dG[it][4] = b1.x; pre_dG[it][5] = b1.y; pre_dG[it][6] = b1.z; pre_dG[it][7] = b1.w;
      }
      // ---- phase 5: RS = dAt bf, CS = dAt^T af (bf, af as MN-major B operands)
      uint8_t *bfh = R + S::p5_bf, *bfl = bfh + S::CDb, *afh = R + S::p5_af, *afl = afh + S::CDb;
      auto bff = [&](int i, int c, float x) { return x * tc::ex2(sref[c] - sG[i * LD + c]); };
      auto aff = [&](int r, int c, float x) { return x * tc::ex2(sG[r * LD + c] - sref[c]); };
      if constexpr (S::kStageK) {  // e = 2^{G - ref} (bounded by the decay check), 2^{ref - G} = 1 / e
        build_tile2_st<C, D>(afh, afl, bfh, bfl, reinterpret_cast<const __nv_bfloat16*>(sk), [&](int r, int c, float x) {
          const float e = tc::ex2(sG[r * LD + c] - sref[c]);
          return make_float2(x * e, x * tc::rcp_approx(e));
        });
      } else {
        build_tile_ld<C, D, true, Tin>(bfh, bfl, row_k, bff);
        build_tile_ld<C, D, true, Tin>(afh, afl, row_k, aff);
      }
      ok = run(sy, [&] {
        const tc::Op pK{tc::smem_u32(dah), C, false}, pKl{tc::smem_u32(dal), C, false};
        const tc::Op pM{tc::smem_u32(dah), C, true}, pMl{tc::smem_u32(dal), C, true};
        const tc::Op bH{tc::smem_u32(bfh), C, true}, bL{tc::smem_u32(bfl), C, true};
        const tc::Op aH{tc::smem_u32(afh), C, true}, aL{tc::smem_u32(afl), C, true};
        mma4(tb + cRS, pK, pKl, bH, bL, C, tc::idesc_bf16(C, D, false, true), false, false, false);
        mma4(tb + cCS, pM, pMl, aH, aL, C, tc::idesc_bf16(C, D, true, true), false, false, false);
      });
    }
    if (ok) {
      // ---- final: dk, dG = partials + dB_k terms + gated terms; dG staged for the reverse cumulative sum
      float* sdG = reinterpret_cast<float*>(R);  // [C][LD]
  #pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int cc = grp * 16 + 16 * kTcGroups * it;
        float rs[8], cs[8], dbk[8];
        {
          uint32_t a0[16], a1[16], a2[16];  // three loads in flight, one wait
          tc::tmem_ld16_nowait(la + cRS + cc, a0);
          tc::tmem_ld16_nowait(la + cCS + cc, a1);
          tc::tmem_ld16_nowait(la + cdB + cc, a2);
          tc::tmem_wait_ld();
          tc::tmem_regs16(a0);
          tc::tmem_regs16(a1);
          tc::tmem_regs16(a2);
          share8u(a0, rs);
          share8u(a1, cs);
          share8u(a2, dbk);
        }
        const int r = myrow, c0 = cc + half8;
        float kv[8], dkv[8], pg[8];
        k8(r, c0, kv);
  #pragma unroll
        for (int j = 0; j < 8; ++j) {
          dkv[j] = pre_dk[it][j];
          pg[j] = pre_dG[it][j];
        }
  #pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = c0 + j;
          // e = 2^{G_r - G_0} (bounded by the chunk's decay check), 1/e = 2^{G_0 - G_r}, 2^{G_r} = 2^{G_0} e
          const float e = tc::ex2(sG[r * LD + c] - sref[c]), ie = tc::rcp_approx(e);
          const float a = e * rs[j], b = ie * cs[j];
          const float wb = se0[c] * e * sb[r] * dbk[j];
          dkv[j] += wb + (a + b);
          sdG[r * LD + c] = r < n ? pg[j] + kv[j] * (wb + (a - b)) : 0.f;
        }
        if (r < n) out8(ws.rdk, ws.tdk, dk_, r, c0, dkv);
      }
      __syncthreads();
      // dg = reverse cumulative sum of dG over the chunk's rows: four threads per column, each a
      // quarter of the rows; the quarters' totals first, then each quarter's running sum from below
      static_assert(kTcThreads == 4 * D, "four threads per column");
      float* qsum = sdG + C * LD;  // [4][D]
      const int c = tid % D, q4 = tid / D, r_lo = 16 * q4;
      {
        float a = 0.f;
  #pragma unroll
        for (int r = r_lo; r < r_lo + 16; ++r) a += sdG[r * LD + c];  // rows >= n hold zeros
        qsum[q4 * D + c] = a;
      }
      __syncthreads();
      {
        float acc = 0.f;
        for (int q = 3; q > q4; --q) acc += qsum[q * D + c];
        for (int r = r_lo + 15; r >= r_lo; --r) {
          acc += sdG[r * LD + c];
          if (r < n) {
            float* dst = skind[r] == 0 ? ws.rdg : (skind[r] == 1 ? ws.tdg : dg_);
            dst[((size_t)sidx[r] * H + h) * D + c] = acc;
          }
        }
      }
      for (int r = tid; r < n; r += blockDim.x) {
        float db = 0.f;
        for (int q = 0; q < 3 * kTcGroups; ++q) db += sdb[q * C + r];
        float* dst = skind[r] == 0 ? ws.rdb : (skind[r] == 1 ? ws.tdb : dbeta_);
        dst[(size_t)sidx[r] * H + h] = db;
      }
    }
    // the bulk stores have read their tiles before the next head overwrites them
    if (tid == 0) tc::bulk_wait_read();  // (the stores complete with the grid)
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  if ((tid >> 5) == 0) tc::tmem_dealloc(tb, 512);
}

}  // namespace tpc
