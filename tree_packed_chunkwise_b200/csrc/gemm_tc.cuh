// bf16 GEMM on 5th-generation tensor cores: C = alpha * op(A) op(B) (+ beta * C), fp32 accumulation
// in TMEM.  A is M x K and B is K x N; each is given either K-major (K contiguous: A as [M][K], B
// as [N][K]) or MN-major (M resp. N contiguous: A as [K][M], B as [K][N]).
//
// Split precision: an fp32 operand X is passed as two bf16 matrices, X_hi = bf16(X) and
// X_lo = bf16(X - X_hi), so that X = X_hi + X_lo to 2^-17 relative.  The kernel accumulates up to
// three products in one TMEM accumulator: A_hi B_hi (+ A_lo B_hi) (+ A_hi B_lo); the dropped
// A_lo B_lo term is below 2^-16 of the product.  The K loop simply runs once per product.
//
// Output tiles of 128 x 256 (K < 4096) or 256 x 256 (two 128-row halves, each an M = 128 MMA into
// its own TMEM accumulator), K in steps of 64 through a 4- resp. 3-stage shared-memory pipeline:
// a producer thread issues TMA loads into the 128-byte-swizzled canonical layout (K-major operand:
// one box of 64 K x tile rows, each row one 128-byte line; MN-major operand: boxes of 64 M/N x 64 K,
// each K row one 128-byte line), an MMA thread issues tcgen05.mma and frees stages by
// tcgen05.commit, all 128 threads run the epilogue (thread = row).  All waits are bounded.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace tpc {

constexpr int kGemmBN = 256, kGemmBK = 64, kGemmThreads = 128;
constexpr int kGemmHalf = 128;      // rows per MMA and per TMEM accumulator
constexpr int kGemmLongK = 4096;    // K from which the 256-row tile is used
// one MN-major 128-byte-swizzle block: 64 K rows of one 128-byte line
constexpr uint32_t kSw128Atom = kGemmBK * 128;

// Shared-memory descriptor of the 16-wide K step ks of a 128-byte-swizzled operand tile (descriptor
// version 1, layout type 2 = 128-byte swizzle).  Groups of 8 rows of 128-byte lines are 1024 bytes
// apart (SBO).  K-major: a line holds 64 K of one M/N row, the K step moves 32 bytes along it.
// MN-major: a line holds 64 M/N of one K row, the K step moves 16 lines (2048 bytes), and the
// 64-wide M/N blocks are kSw128Atom apart (LBO).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t base, bool mn, int ks) {
  const uint32_t addr = mn ? base + (uint32_t)ks * 2048u : base + (uint32_t)ks * 32u;
  const uint32_t lbo = mn ? kSw128Atom : 16u;
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((1024u >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// HV = 128-row halves per tile: 1 (two TMEM accumulators, the epilogue of a tile overlaps the next
// tile's main loop) or 2 (both accumulators hold one tile; more K in flight per stage)
template <int HV>
struct GemmCfg {
  static constexpr int BM = kGemmHalf * HV, stages = HV == 2 ? 3 : 4, nacc = HV == 2 ? 1 : 2;
  static constexpr size_t Ab = size_t(BM) * kGemmBK * 2, Bb = size_t(kGemmBN) * kGemmBK * 2;
  static constexpr size_t stage = Ab + Bb;
  static constexpr size_t total = stages * stage + 1024;  // + slack to align the stages to 1024 bytes
};

// Epilogues: kEpiStore writes alpha * acc (+ beta * C); kEpiLsePart writes, per row and 256-column
// tile, (max, sum of exp(acc - max)) over the tile's columns into C = float2 [M][ldc] at column
// tile_n (the rows' log-sum-exp is combined from these later, the accumulator is never stored);
// kEpiSoftmaxGrad writes bf16 -row_b[m] * exp(acc - row_a[m]) (row_a = log-sum-exp, row_b = the row's
// gradient weight) into C = bf16 [M][ldc].
enum : int { kEpiStore = 0, kEpiLsePart = 1, kEpiSoftmaxGrad = 2 };

struct GemmArgs {
  int M, N, K;
  int a_mn, b_mn;     // 1: MN-major
  int c_dtype;        // 0 fp32, 1 bf16
  long long ldc;      // elements
  float alpha, beta;  // beta != 0 reads C (fp32 only)
  void* C;
  int* status;
  int passes;         // 1: A B;  2: + A_lo B;  3: + A B_lo
  int m_fast;         // tile order: 1 = M blocks fastest (concurrent CTAs share B), 0 = N blocks fastest
  int epi;            // kEpi*
  const float* row_a; // per-row inputs of kEpiSoftmaxGrad (indexed by the GEMM row)
  const float* row_b;
};

// Persistent, warp-specialised: grid = min(tiles, SMs); each CTA walks tiles blockIdx.x,
// blockIdx.x + gridDim.x, ...  The tile order runs along the smaller of M and N fastest, so the
// CTAs in flight share the tiles of the larger operand and the smaller one stays in L2.  Warp 0
// lane 0 issues TMA loads into the stage ring; warp 1 lane 0 issues per 16-wide K step one MMA per
// 128-row half.  HV = 1: two TMEM accumulators of 256 columns alternate between tiles, so warps
// 2-5 drain one tile (thread = row) while the next one's main loop runs.  HV = 2: the two
// accumulators hold the two halves of one tile and are drained (thread = one row of each half)
// before the next tile starts; per MMA cycle this moves a third less operand data and keeps 1.5x
// the MMA time in flight per stage, which pays once K is long.  Every wait is bounded; a timeout
// records TPC_ERR_TIMEOUT and every role stops.
constexpr int kGemmThreadsP = 192;

template <int C_BF16, int HV>
__global__ void __launch_bounds__(kGemmThreadsP, 1)
    gemm_bf16_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                 const __grid_constant__ CUtensorMap tma_alo, const __grid_constant__ CUtensorMap tma_blo, GemmArgs g) {
  using namespace tc;
  using Cfg = GemmCfg<HV>;
  constexpr int kGemmBM = Cfg::BM, kGemmStages = Cfg::stages, NACC = Cfg::nacc;
  using GemmSmem = Cfg;
  extern __shared__ __align__(1024) uint8_t gsm_raw[];
  // the swizzle pattern is a function of the shared address: stages start on 1024-byte boundaries
  uint8_t* gsm = gsm_raw + ((1024u - (smem_u32(gsm_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages], acc_full[NACC], acc_empty[NACC], done_bar;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int KT = (g.K + kGemmBK - 1) / kGemmBK;
  const int IT = KT * g.passes;  // pass p = it / KT uses (A, B), (A_lo, B), (A, B_lo)
  const int n_tiles = (g.N + kGemmBN - 1) / kGemmBN, m_tiles = (g.M + kGemmBM - 1) / kGemmBM;
  const int tiles = n_tiles * m_tiles;
  auto tile_m = [&](int t) { return g.m_fast ? t % m_tiles : t / n_tiles; };
  auto tile_n = [&](int t) { return g.m_fast ? t / m_tiles : t % n_tiles; };
  if (w == 1) tmem_alloc(&tslot, 512);
  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tslot;
  auto give_up = [&] {
    set_status(g.status, 8);
    atomicExch(&abort_flag, 1);
  };
  auto aborted = [&] { return *((volatile int*)&abort_flag) != 0; };
  if (w == 0) {
    if (lane == 0) {  // producer
      int it_all = 0;
      for (int t = blockIdx.x; t < tiles && !aborted(); t += gridDim.x) {
        const int m0 = tile_m(t) * kGemmBM, n0 = tile_n(t) * kGemmBN;
        for (int it = 0; it < IT; ++it, ++it_all) {
          const int s = it_all % kGemmStages, pass = it / KT, kt = it - pass * KT;
          if (it_all >= kGemmStages && !mbar_wait(&empty[s], ((it_all / kGemmStages) - 1) & 1)) {
            give_up();
            break;
          }
          const CUtensorMap* ma = pass == 1 ? &tma_alo : &tma_a;
          const CUtensorMap* mb = pass == 2 ? &tma_blo : &tma_b;
          uint8_t* sa = gsm + s * GemmSmem::stage;
          uint8_t* sb = sa + GemmSmem::Ab;
          mbar_arrive_expect_tx(&full[s], (uint32_t)GemmSmem::stage);
          const int k0 = kt * kGemmBK;
          if (!g.a_mn) {
            tma_load_2d(sa, ma, k0, m0, &full[s]);
          } else {
            for (int j = 0; j < kGemmBM / 64; ++j) tma_load_2d(sa + j * kSw128Atom, ma, m0 + 64 * j, k0, &full[s]);
          }
          if (!g.b_mn) {
            tma_load_2d(sb, mb, k0, n0, &full[s]);
          } else {
            for (int j = 0; j < kGemmBN / 64; ++j) tma_load_2d(sb + j * kSw128Atom, mb, n0 + 64 * j, k0, &full[s]);
          }
        }
      }
    }
  } else if (w == 1) {
    if (lane == 0) {  // MMA issuer
      const uint32_t id = idesc_bf16(kGemmHalf, kGemmBN, g.a_mn != 0, g.b_mn != 0);
      // second 128-row half of the A stage: 128 lines on (K-major) or two 64-row blocks on (MN-major)
      const uint32_t a_half = g.a_mn ? 2u * kSw128Atom : (uint32_t)kGemmHalf * 128u;
      int it_all = 0, local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok && !aborted(); t += gridDim.x, ++local) {
        // the epilogue has drained this tile's accumulator(s) (their previous use: tile local - NACC)
        const int b = local % NACC;
        if (local >= NACC && !mbar_wait(&acc_empty[b], ((local / NACC) - 1) & 1, 4000000000ull)) {
          give_up();
          ok = false;
          break;
        }
        fence_after_sync();
        const uint32_t acc = tb + (uint32_t)(b * kGemmBN);
        for (int it = 0; it < IT; ++it, ++it_all) {
          const int s = it_all % kGemmStages;
          if (!mbar_wait(&full[s], (it_all / kGemmStages) & 1)) {
            give_up();
            ok = false;
            break;
          }
          fence_after_sync();
          const uint32_t sa = smem_u32(gsm + s * GemmSmem::stage), sb = sa + (uint32_t)GemmSmem::Ab;
#pragma unroll
          for (int ks = 0; ks < kGemmBK / 16; ++ks) {
            const uint64_t db = sw128_desc(sb, g.b_mn != 0, ks);
            const uint32_t accum = (it > 0 || ks) ? 1u : 0u;
            mma_bf16(acc, sw128_desc(sa, g.a_mn != 0, ks), db, id, accum);
            if constexpr (HV == 2)
              mma_bf16(acc + (uint32_t)kGemmBN, sw128_desc(sa + a_half, g.a_mn != 0, ks), db, id, accum);
          }
          commit(&empty[s]);
        }
        if (ok) commit(&acc_full[b]);
      }
      commit(&done_bar);  // arrives once every MMA issued above has completed
      if (!mbar_wait(&done_bar, 0, 2000000000ull)) give_up();
    }
  } else {  // epilogue warps 2..5: TMEM lanes of sub-partition w % 4, one row of each half
    const int sp = w & 3, row = 32 * sp + lane;
    int local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      // decisions are warp-uniform: the TMEM loads below are warp-collective
      const int b = local % NACC;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], (local / NACC) & 1, 4000000000ull));
      if (!got) {
        if (lane == 0) give_up();
        break;
      }
      if (__any_sync(0xffffffffu, aborted())) break;
      fence_after_sync();
      const int n0 = tile_n(t) * kGemmBN;
      for (int half = 0; half < HV; ++half) {
        const int m = tile_m(t) * kGemmBM + kGemmHalf * half + row;
        const uint32_t la = tb + ((uint32_t)(32 * sp) << 16) + (uint32_t)((b + half) * kGemmBN);
        if (g.epi == kEpiLsePart) {  // running max and sum of exponentials over the tile's columns
          float mx = -INFINITY, sm = 0.f;
          for (int c0 = 0; c0 < kGemmBN; c0 += 16) {
            float v[16];
            tmem_ld16(la + c0, v);
            const int nn = min(16, g.N - (n0 + c0));
            float lm = mx;
            for (int j = 0; j < nn; ++j) lm = fmaxf(lm, v[j]);
            if (nn > 0 && lm > -INFINITY) {
              sm *= expf(mx - lm);
              for (int j = 0; j < nn; ++j) sm += expf(v[j] - lm);
              mx = lm;
            }
          }
          if (m < g.M) reinterpret_cast<float2*>(g.C)[(size_t)m * g.ldc + tile_n(t)] = make_float2(mx, sm);
          continue;
        }
        if (g.epi == kEpiSoftmaxGrad) {  // dense part of the log-softmax gradient, as bf16
          const float ra = m < g.M ? g.row_a[m] : 0.f, rb = m < g.M ? g.row_b[m] : 0.f;
          for (int c0 = 0; c0 < kGemmBN; c0 += 16) {
            float v[16];
            tmem_ld16(la + c0, v);
            if (m >= g.M || n0 + c0 >= g.N) continue;
            const int nn = min(16, g.N - (n0 + c0));
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.C) + (size_t)m * g.ldc + n0 + c0;
            if (nn == 16 && (g.ldc & 7) == 0) {
              __align__(16) __nv_bfloat16 o[16];
              for (int j = 0; j < 16; ++j) o[j] = __float2bfloat16_rn(-rb * expf(v[j] - ra));
              reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(o)[0];
              reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(o)[1];
            } else {
              for (int j = 0; j < nn; ++j) dst[j] = __float2bfloat16_rn(-rb * expf(v[j] - ra));
            }
          }
          continue;
        }
        for (int c0 = 0; c0 < kGemmBN; c0 += 16) {
          float v[16];
          tmem_ld16(la + c0, v);
          if (m >= g.M || n0 + c0 >= g.N) continue;
          const int nn = min(16, g.N - (n0 + c0));
          if (C_BF16) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.C) + (size_t)m * g.ldc + n0 + c0;
            for (int j = 0; j < nn; ++j) dst[j] = __float2bfloat16_rn(g.alpha * v[j]);
          } else {
            float* dst = static_cast<float*>(g.C) + (size_t)m * g.ldc + n0 + c0;
            if (nn == 16 && (g.ldc & 3) == 0) {
              float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                float4 x = make_float4(g.alpha * v[4 * j], g.alpha * v[4 * j + 1], g.alpha * v[4 * j + 2],
                                       g.alpha * v[4 * j + 3]);
                if (g.beta != 0.f) {
                  const float4 c = d4[j];
                  x.x += g.beta * c.x; x.y += g.beta * c.y; x.z += g.beta * c.z; x.w += g.beta * c.w;
                }
                d4[j] = x;
              }
            } else if (g.beta != 0.f) {
              for (int j = 0; j < nn; ++j) dst[j] = g.alpha * v[j] + g.beta * dst[j];
            } else {
              for (int j = 0; j < nn; ++j) dst[j] = g.alpha * v[j];
            }
          }
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (w == 1) tmem_dealloc(tb, 512);
}

}  // namespace tpc
