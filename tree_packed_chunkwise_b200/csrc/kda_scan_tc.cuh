// Sequential state scans of the tensor-core KDA path (chunk 64, head dim 128).
//
// Per chunk the state update is affine: S_end = M S_0 + B with M = Diag(e^{G_C}) - Khat^T W and
// B = Khat^T U' (both formed in parallel by the prep kernel; M is stored as a bf16 hi/lo tile in the
// tensor-core operand layout).  The forward scan computes S <- M S + B per chunk, the backward scan
// dS <- M^T dS + X (X = Qbar^T dO - W^T dU0), each as one M = 128 tcgen05 product per chunk (three
// hi/lo chains) with the next chunk's M tile arriving by a bulk asynchronous copy meanwhile.
// One CTA of 128 threads per (sequence of the round, head, 32-column slice of d_v); thread c owns
// row c of the state slice.
#pragma once
#include "kda_tc.cuh"

namespace tpc {

constexpr int kScanThreads = 128, kScanDVT = 32;

struct ScanTcSmem {
  static constexpr size_t M0 = 0, M1 = kMtileBytes;              // double-buffered M tiles
  static constexpr size_t St = 2 * size_t(kMtileBytes);          // state slice hi/lo (MN-major, K = 128)
  static constexpr size_t StB = size_t(kTcD) * kScanDVT * 2;
  static constexpr size_t total = St + 2 * StB;
};

namespace tck {

// one bounded wait + CTA vote; false on every thread after recording the timeout
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* status) {
  const bool ok = tc::mbar_wait(bar, parity);
  const int failed = __syncthreads_or(ok ? 0 : 1);
  if (failed && threadIdx.x == 0) set_status(status, kStatusTimeout);
  return !failed;
}

__device__ __forceinline__ void load_mtile(uint8_t* dst, const uint8_t* src, uint64_t* bar) {
  tc::mbar_arrive_expect_tx(bar, kMtileBytes);
#pragma unroll
  for (int p = 0; p < 4; ++p) tc::bulk_g2s(dst + p * (kMtileBytes / 4), src + p * (kMtileBytes / 4), kMtileBytes / 4, bar);
}

// state slice (row c = this thread, 32 columns) -> MN-major hi/lo operand tile (k = c, n = j)
__device__ __forceinline__ void put_state(uint8_t* hi, uint8_t* lo, int c, const float (&s)[32]) {
  put16<kTcD, true>(hi, lo, c, 0, s);
  put16<kTcD, true>(hi, lo, c, 16, s + 16);
}

__device__ __forceinline__ void ld32g(const float* p, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p) + i);
    v[4 * i] = u.x; v[4 * i + 1] = u.y; v[4 * i + 2] = u.z; v[4 * i + 3] = u.w;
  }
}
__device__ __forceinline__ void st32g(float* p, const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

}  // namespace tck

template <bool REVERSE>
__global__ void __launch_bounds__(kScanThreads, 1)
    kda_scan_tc(DevTables t, int seq0, int H, const float* __restrict__ init, float* __restrict__ final_state,
                const float* __restrict__ d_final, KdaWs ws) {
  using namespace tck;
  using S = ScanTcSmem;
  constexpr int D = kTcD, DVT = kScanDVT;
  const int si = seq0 + blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVT;
  const SeqRec sq = t.seqs[si];
  extern __shared__ __align__(1024) uint8_t tsm[];
  uint8_t* mbuf[2] = {tsm + S::M0, tsm + S::M1};
  uint8_t *sth = tsm + S::St, *stl = sth + S::StB;
  __shared__ __align__(8) uint64_t bar_m[2];
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ uint32_t tslot;
  const int c = threadIdx.x;  // state row / TMEM lane
  if ((c >> 5) == 0) tc::tmem_alloc(&tslot, 32);
  if (c == 0) {
    tc::mbar_init(&bar_m[0], 1);
    tc::mbar_init(&bar_m[1], 1);
    tc::mbar_init(&bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  const uint32_t la = tb + ((uint32_t)(32 * (c >> 5)) << 16);
  float s[32];
  const int nch = sq.n_chunks;
  auto chunk_at = [&](int q) { return REVERSE ? sq.chunk_begin + nch - 1 - q : sq.chunk_begin + q; };
  auto mtile = [&](int ci) {
    return reinterpret_cast<const uint8_t*>(ws.Mt) + ((size_t)ci * H + h) * kMtileBytes;
  };
  // initial value: forward -> initial / imported state; reverse -> gradient of the final state
  {
    const float* src = nullptr;
    if (!REVERSE) {
      if (sq.import_id >= 0) src = ws.slot + ((size_t)sq.import_id * H + h) * D * D;
      else if (init) src = init + ((size_t)(-(sq.import_id + 1)) * H + h) * D * D;
    } else if (d_final) {
      src = d_final + ((size_t)sq.leaf * H + h) * D * D;
    }
    if (src) ld32g(src + c * D + j0, s);
    else
      for (int j = 0; j < 32; ++j) s[j] = 0.f;
  }
  if (c == 0) load_mtile(mbuf[0], mtile(chunk_at(0)), &bar_m[0]);
  uint32_t mma_phase = 0;
  bool ok = true;
  for (int q = 0; q < nch && ok; ++q) {
    const int ci = chunk_at(q);
    const size_t base = (size_t)ci * H + h;
    float add[32];
    if (!REVERSE) {
      st32g(ws.S0 + base * D * D + c * D + j0, s);               // chunk-start state
      ld32g(ws.Bc + base * D * D + c * D + j0, add);             // B of this chunk
    } else {
      const int slot = t.chunks[ci].export_slot;
      if (slot >= 0) {  // gradients of the exported boundary state, consumers in a fixed order
        const SlotRec sr = t.slots[slot];
        for (int m = 0; m < sr.n_cons; ++m) {
          float g2[32];
          ld32g(ws.dS0seq + ((size_t)t.slot_cons[sr.cons_begin + m] * H + h) * D * D + c * D + j0, g2);
          for (int j = 0; j < 32; ++j) s[j] += g2[j];
        }
      }
      float* dSg = ws.dS + base * D * D + c * D + j0;
      ld32g(dSg, add);   // X of this chunk
      st32g(dSg, s);     // gradient of the chunk-end state, for the chunk kernels
    }
    put_state(sth, stl, c, s);
    if (c == 0 && q + 1 < nch) load_mtile(mbuf[(q + 1) & 1], mtile(chunk_at(q + 1)), &bar_m[(q + 1) & 1]);
    ok = wait_all(&bar_m[q & 1], (q >> 1) & 1, ws.status);
    if (!ok) break;
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (c == 0) {
      const tc::Op mH{tc::smem_u32(mbuf[q & 1]), D, REVERSE}, mL{tc::smem_u32(mbuf[q & 1] + kMtileBytes / 2), D, REVERSE};
      const tc::Op sH{tc::smem_u32(sth), D, true}, sL{tc::smem_u32(stl), D, true};
      mma4(tb, mH, mL, sH, sL, D, tc::idesc_bf16(D, DVT, REVERSE, true), false, false, false);
      tc::commit(&bar_mma);
    }
    ok = wait_all(&bar_mma, mma_phase, ws.status);
    mma_phase ^= 1u;
    if (!ok) break;
    tc::fence_after_sync();
    float acc[32];
    tc::tmem_ld32(la, acc);
    for (int j = 0; j < 32; ++j) s[j] = acc[j] + add[j];
    if (!REVERSE) {
      const int slot = t.chunks[ci].export_slot;
      if (slot >= 0) st32g(ws.slot + ((size_t)slot * H + h) * D * D + c * D + j0, s);
    }
    tc::fence_before_sync();
    __syncthreads();  // the state tile and this M buffer are free again
  }
  if (ok) {
    if (!REVERSE) {
      if (final_state) st32g(final_state + ((size_t)sq.leaf * H + h) * D * D + c * D + j0, s);
    } else {
      st32g(ws.dS0seq + ((size_t)si * H + h) * D * D + c * D + j0, s);
    }
  } else {
    // give copies still in flight a last bounded chance before the shared memory is released
    tc::mbar_wait(&bar_m[0], 0, 200000000ull);
  }
  tc::fence_before_sync();
  __syncthreads();
  if ((c >> 5) == 0) tc::tmem_dealloc(tb, 32);
}

}  // namespace tpc
