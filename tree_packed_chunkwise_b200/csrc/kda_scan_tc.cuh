// Sequential state scans of the tensor-core KDA path (chunk 64, head dim 128).
//
// Per chunk the state update is affine: S_end = M S_0 + B with M = Diag(e^{G_C}) - Khat^T W and
// B = Khat^T U' (both formed in parallel by the prep kernel; M is stored as a bf16 hi/lo tile in the
// tensor-core operand layout).  The forward scan computes S <- M S + B per chunk; the backward scan
// dS <- M^T dS + Qeff^T dO with Qeff = Qbar - P W (formed by the output kernel; O = Qeff S0 + P U',
// so Qeff^T dO is the output's contribution to the chunk-start state gradient).  Each step is one
// accumulator of M = 128 tcgen05 products (three hi/lo chains), with the next chunk's operands
// arriving by asynchronous copies meanwhile: forward the M tile and this CTA's slice of B (stored
// slice by slice, [chunk][head][slice][row][32] fp32); backward the M tile, the Qeff tile and the
// chunk's rows of this CTA's 32 columns of dO.
// One CTA of 128 threads per (sequence of the round, head, 32-column slice of d_v); thread c owns
// row c of the state slice.
#pragma once
#include "kda_tc.cuh"

namespace tpc {

// Slice width W of d_v per CTA: 32 (128 threads) or 64 (256 threads; half the CTAs, the same M
// tile traffic per CTA, used when the round has more (sequence, head) pairs than fit in one wave of
// 32-column CTAs).  Thread c owns row c % 128 of the state and columns 32 (c / 128) .. + 31 of the
// slice.
template <bool REVERSE, int W>
struct ScanTcSmemT {
  static constexpr int NT = 128 * (W / 32);
  // M tiles double-buffered, except at W = 128 (one buffer, reloaded after each step's products)
  static constexpr int NM = W == 128 ? 1 : 2;
  static constexpr size_t M0 = 0, M1 = NM == 2 ? kMtileBytes : 0;
  static constexpr size_t St = NM * size_t(kMtileBytes);         // state slice hi/lo (MN-major, K = 128)
  static constexpr size_t StB = size_t(kTcD) * W * 2;            // one half (hi or lo) of it
  // forward: B columns [j0, j0 + W) (W / 32 consecutive 32-column slices); reverse: the Qeff tile
  static constexpr size_t XB = REVERSE ? size_t(2) * kTcC * kTcD * 2 : size_t(kTcD) * W * 4;
  static constexpr int NX = ((REVERSE && W == 64) || W == 128) ? 1 : 2;  // X buffers (one where two do not fit)
  static constexpr size_t X = St + 2 * StB;
  // reverse: double-buffered dO slices, hi/lo operand tiles of C rows x W columns (k = row, n = column)
  static constexpr size_t dOB = REVERSE ? size_t(kTcC) * W * 2 : 0;
  static constexpr size_t dO = X + NX * XB;
  static constexpr size_t total = dO + 2 * 2 * dOB;
  static_assert(total <= 224 * 1024, "shared memory");
  static_assert(W == 32 || W == 64 || W == 128, "slice width");
};

namespace tck {

// one bounded wait + CTA vote; false on every thread after recording the timeout
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* status) {
  const bool ok = tc::mbar_wait(bar, parity);
  const int failed = __syncthreads_or(ok ? 0 : 1);
  if (failed && threadIdx.x == 0) set_status(status, kStatusTimeout);
  return !failed;
}

// the chunk's M tile and a second operand (forward: this CTA's B slice; reverse: the Qeff tile), on one
// mbarrier with one expected-bytes arrival
__device__ __forceinline__ void load_mtile(uint8_t* dst, const uint8_t* src, uint8_t* x_dst, const uint8_t* x_src,
                                           uint32_t x_bytes, uint64_t* bar) {
  tc::mbar_arrive_expect_tx(bar, kMtileBytes + (x_dst ? x_bytes : 0u));
  tc::bulk_g2s(dst, src, kMtileBytes, bar);
  if (x_dst) tc::bulk_g2s(x_dst, x_src, x_bytes, bar);
}

// This CTA's W columns (j0 ..) of the chunk's dO rows as an MN-major operand tile (k = chunk row,
// n = column; element (r, j) at cm_off(r, j, C)), hi (and lo for fp32 data); rows that are replays
// or past the chunk's end are zero.  bf16: asynchronous 16-byte copies (completed by the caller with
// cp_async_wait); fp32: loaded, split and stored now.
template <typename Tin, int W>
__device__ __forceinline__ void load_do_slice(uint8_t* hi, uint8_t* lo, const Tin* d_o, const ChunkRec& ch, int H,
                                              int h, int j0) {
  constexpr int C = kTcC, G = W / 8;
  for (int p = threadIdx.x; p < C * G; p += blockDim.x) {
    const int r = p / G, g = p % G;
    const bool own = r >= ch.n_replay && r < ch.n_rows;
    const size_t row = own ? (size_t)(ch.row_start + (r - ch.n_replay)) : 0;
    const Tin* src = d_o + (row * H + h) * kTcD + j0 + 8 * g;
    const uint32_t off = cm_off(r, 8 * g, C);
    if constexpr (sizeof(Tin) == 2) {
      tc::cp_async16(hi + off, src, own ? 16u : 0u);
    } else {
      float x[8];
      if (own) ld8(src, x);
      else
        for (int j = 0; j < 8; ++j) x[j] = 0.f;
      __align__(16) __nv_bfloat16 a[8];
      __align__(16) __nv_bfloat16 b[8];
      for (int j = 0; j < 8; ++j) split_bf16(x[j], a[j], b[j]);
      *reinterpret_cast<uint4*>(hi + off) = *reinterpret_cast<const uint4*>(a);
      *reinterpret_cast<uint4*>(lo + off) = *reinterpret_cast<const uint4*>(b);
    }
  }
  if constexpr (sizeof(Tin) == 2) tc::cp_async_commit();
}

// this thread's part of the state slice (row c, 32 columns from n0) -> MN-major hi/lo operand tile
// (k = c, n = j)
__device__ __forceinline__ void put_state(uint8_t* hi, uint8_t* lo, int c, int n0, const float (&s)[32]) {
  put16<kTcD, true>(hi, lo, c, n0, s);
  put16<kTcD, true>(hi, lo, c, n0 + 16, s + 16);
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

// REVERSE: d_o [N, H, D] (Tin) is the output gradient; forward: unused
template <bool REVERSE, int W, typename Tin>
__global__ void __launch_bounds__(128 * (W / 32), 1)
    kda_scan_tc(DevTables t, int seq0, int H, const float* __restrict__ init, float* __restrict__ final_state,
                const float* __restrict__ d_final, KdaWs ws, const Tin* __restrict__ d_o) {
  using namespace tck;
  using S = ScanTcSmemT<REVERSE, W>;
  constexpr int D = kTcD, C = kTcC;
  constexpr bool EX = sizeof(Tin) == 2;  // bf16 dO: exact operand, no lo part
  const int si = seq0 + blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * W;
  const SeqRec sq = t.seqs[si];
  extern __shared__ __align__(1024) uint8_t tsm[];
  uint8_t* mbuf[2] = {tsm + S::M0, tsm + S::M1};
  uint8_t* xbuf[2] = {tsm + S::X, tsm + S::X + (S::NX == 2 ? S::XB : 0)};
  uint8_t* dobuf[2] = {tsm + S::dO, tsm + S::dO + 2 * S::dOB};  // hi, then lo at + dOB
  uint8_t *sth = tsm + S::St, *stl = sth + S::StB;
  __shared__ __align__(8) uint64_t bar_m[2];
  __shared__ __align__(8) uint64_t bar_x;  // the single-buffered operands (S::NX == 1, S::NM == 1)
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ uint32_t tslot;
  __shared__ int s_ok;  // thread 0's bounded waits, read by every thread after the following barrier
  const int c = threadIdx.x & 127, half = threadIdx.x >> 7;  // state row / TMEM lane; 32-column half
  const int jc = j0 + 32 * half;                              // this thread's first column
  const bool lead = threadIdx.x == 0;
  if ((threadIdx.x >> 5) == 0) tc::tmem_alloc(&tslot, W);
  if (lead) {
    tc::mbar_init(&bar_m[0], 1);
    tc::mbar_init(&bar_m[1], 1);
    tc::mbar_init(&bar_x, 1);
    tc::mbar_init(&bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  const uint32_t la = tb + ((uint32_t)(32 * ((threadIdx.x >> 5) & 3)) << 16) + (uint32_t)(32 * half);
  float s[32];
  const int nch = sq.n_chunks;
  auto chunk_at = [&](int q) { return REVERSE ? sq.chunk_begin + nch - 1 - q : sq.chunk_begin + q; };
  auto mtile = [&](int ci) {
    return reinterpret_cast<const uint8_t*>(ws.Mt) + ((size_t)ci * H + h) * kMtileBytes;
  };
  // forward: this CTA's columns of B (consecutive 32-column slices); reverse: the chunk's Qeff tile
  // (kept where the forward kept W)
  auto xsrc = [&](int ci) -> const uint8_t* {
    if (REVERSE) return reinterpret_cast<const uint8_t*>(ws.W) + ((size_t)ci * H + h) * S::XB;
    return reinterpret_cast<const uint8_t*>(ws.Bc + ((size_t)ci * H + h) * D * D + (size_t)j0 * D);
  };
  auto prefetch = [&](int q) {  // thread 0: bulk copies (the M tile, and X when it is double-buffered)
    const int ci = chunk_at(q);
    load_mtile(mbuf[q & 1], mtile(ci), S::NX == 2 ? xbuf[q & 1] : nullptr, xsrc(ci), (uint32_t)S::XB, &bar_m[q & 1]);
  };
  // thread 0: the single-buffered operands (X; and M at W = 128), once the previous chunk's products
  // are done with them
  auto load_x_single = [&](int q) {
    const int ci = chunk_at(q);
    tc::mbar_arrive_expect_tx(&bar_x, (uint32_t)S::XB + (S::NM == 1 ? kMtileBytes : 0u));
    if constexpr (S::NM == 1) tc::bulk_g2s(mbuf[0], mtile(ci), kMtileBytes, &bar_x);
    tc::bulk_g2s(xbuf[0], xsrc(ci), (uint32_t)S::XB, &bar_x);
  };
  // thread 0: the operands of a later chunk into L2 (the M tile once per (sequence, head), by the
  // first slice's CTA), so that the shared-memory copy a step ahead finds them there
  auto prefetch_l2 = [&](int q) {
    if (q >= nch) return;
    const int ci = chunk_at(q);
    if (blockIdx.z == 0) tc::bulk_prefetch_l2(mtile(ci), kMtileBytes);
    tc::bulk_prefetch_l2(xsrc(ci), (uint32_t)S::XB);
  };
  auto prefetch_do = [&](int q) {  // every thread
    if constexpr (REVERSE) {
      const ChunkRec ch = t.chunks[chunk_at(q)];
      load_do_slice<Tin, W>(dobuf[q & 1], dobuf[q & 1] + S::dOB, d_o, ch, H, h, j0);
    }
  };
  // initial value: forward -> initial / imported state; reverse -> gradient of the final state
  {
    const float* src = nullptr;
    if (!REVERSE) {
      if (sq.import_id >= 0) src = ws.slot + ((size_t)sq.import_id * H + h) * D * D;
      else if (init) src = init + ((size_t)(-(sq.import_id + 1)) * H + h) * D * D;
    } else if (d_final && sq.leaf >= 0) {  // a sequence ending at an internal node has no final state
      src = d_final + ((size_t)sq.leaf * H + h) * D * D;
    }
    if (src) ld32g(src + c * D + jc, s);
    else
      for (int j = 0; j < 32; ++j) s[j] = 0.f;
  }
  // The next chunk's operands are prefetched into L2 one step ahead (further ahead measured slower: the
  // prefetches then compete with the chunk kernels running beside the scan).
  constexpr int kL2Ahead = 1;
  if (lead) {
    if constexpr (S::NM == 2) prefetch(0);
    if constexpr (S::NX == 1) load_x_single(0);
    for (int q = 1; q < kL2Ahead; ++q) prefetch_l2(q);
  }
  prefetch_do(0);
  uint32_t mma_phase = 0;
  bool ok = true;
  // Per step: thread 0 alone waits (bounded) on the mbarriers and publishes the outcome in s_ok; two
  // barriers per step (operands ready; products done, and the state tile's bulk store has read it).
  for (int q = 0; q < nch && ok; ++q) {
    const int ci = chunk_at(q);
    const size_t base = (size_t)ci * H + h;
    uint8_t* xq = xbuf[S::NX == 2 ? (q & 1) : 0];
    uint8_t* mq = mbuf[S::NM == 2 ? (q & 1) : 0];
    if (REVERSE) {
      const int slot = t.chunks[ci].export_slot;
      if (slot >= 0) {  // gradients of the exported boundary state, consumers in a fixed order
        const SlotRec sr = t.slots[slot];
        for (int m = 0; m < sr.n_cons; ++m) {
          float g2[32];
          ld32g(ws.dS0seq + ((size_t)t.slot_cons[sr.cons_begin + m] * H + h) * D * D + c * D + jc, g2);
          for (int j = 0; j < 32; ++j) s[j] += g2[j];
        }
      }
    }
    put_state(sth, stl, c, 32 * half, s);
    if constexpr (REVERSE && EX) tc::cp_async_wait<0>();  // this chunk's dO slice (issued a step ago)
    if (lead) {
      if (S::NM == 2 && q + 1 < nch) prefetch(q + 1);
      prefetch_l2(q + kL2Ahead);
      bool w = S::NM == 1 || tc::mbar_wait(&bar_m[q & 1], (q >> 1) & 1);
      if constexpr (S::NX == 1) w = w && tc::mbar_wait(&bar_x, q & 1);
      if (!w) set_status(ws.status, kStatusTimeout);
      s_ok = w ? 1 : 0;
    }
    if (q + 1 < nch) prefetch_do(q + 1);
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();  // state tile written, this chunk's operands arrived
    tc::fence_after_sync();
    ok = s_ok != 0;
    if (!ok) break;
    float add[32];  // forward: B of this chunk, row c of this thread's 32-column slice (16-byte groups
                    // permuted by c mod 8)
    if constexpr (!REVERSE) {
      const float* ab = reinterpret_cast<const float*>(xq) + ((size_t)half * D + c) * 32;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 u = reinterpret_cast<const float4*>(ab)[i ^ (c & 7)];
        add[4 * i] = u.x; add[4 * i + 1] = u.y; add[4 * i + 2] = u.z; add[4 * i + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) add[j] = 0.f;
    }
    if (lead) {
      const tc::Op mH{tc::smem_u32(mq), D, REVERSE}, mL{tc::smem_u32(mq + kMtileBytes / 2), D, REVERSE};
      const tc::Op sH{tc::smem_u32(sth), D, true}, sL{tc::smem_u32(stl), D, true};
      mma4(tb, mH, mL, sH, sL, D, tc::idesc_bf16(D, W, REVERSE, true), false, false, false);
      if constexpr (REVERSE) {  // + Qeff^T dO (A: the Qeff tile read MN-major, k = chunk row)
        const tc::Op eH{tc::smem_u32(xq), C, true}, eL{tc::smem_u32(xq + S::XB / 2), C, true};
        const tc::Op oH{tc::smem_u32(dobuf[q & 1]), C, true}, oL{tc::smem_u32(dobuf[q & 1] + S::dOB), C, true};
        mma4(tb, eH, eL, oH, oL, C, tc::idesc_bf16(D, W, true, true), true, false, EX);
      }
      tc::commit(&bar_mma);
      // the state slice tile goes to the chunk kernels as it is: forward the chunk-start state S0,
      // reverse the gradient of the chunk-end state (hi/lo operand tiles; this slice's columns are
      // contiguous in each half)
      uint8_t* dst = reinterpret_cast<uint8_t*>(REVERSE ? ws.dS : ws.S0) + base * kStateTileBytes +
                     (size_t)blockIdx.z * S::StB;
      tc::bulk_s2g(dst, sth, (uint32_t)S::StB);
      tc::bulk_s2g(dst + kStateTileBytes / 2, stl, (uint32_t)S::StB);
      tc::bulk_commit();
      const bool w = tc::mbar_wait(&bar_mma, mma_phase);
      if (!w) set_status(ws.status, kStatusTimeout);
      tc::bulk_wait_read();  // (read while the products ran)
      s_ok = w ? 1 : 0;
    }
    mma_phase ^= 1u;
    tc::fence_before_sync();
    __syncthreads();  // products in TMEM; this chunk's M buffer (and the single X buffer) free again
    tc::fence_after_sync();
    ok = s_ok != 0;
    if (!ok) break;
    if constexpr (S::NX == 1)
      if (lead && q + 1 < nch) load_x_single(q + 1);
    float acc[32];
    tc::tmem_ld32(la, acc);
    for (int j = 0; j < 32; ++j) s[j] = acc[j] + add[j];
    if (!REVERSE) {
      const int slot = t.chunks[ci].export_slot;
      if (slot >= 0) st32g(ws.slot + ((size_t)slot * H + h) * D * D + c * D + jc, s);
    }
  }
  if (ok) {
    if (!REVERSE) {
      if (final_state && sq.leaf >= 0) st32g(final_state + ((size_t)sq.leaf * H + h) * D * D + c * D + jc, s);
    } else {
      st32g(ws.dS0seq + ((size_t)si * H + h) * D * D + c * D + jc, s);
    }
  } else if (lead) {
    // give copies still in flight a last bounded chance before the shared memory is released
    if constexpr (S::NM == 2) tc::mbar_wait(&bar_m[0], 0, 200000000ull);
  }
  if constexpr (REVERSE && EX) tc::cp_async_wait<0>();
  if (lead) tc::bulk_wait_read();  // (the stores complete with the grid)
  tc::fence_before_sync();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) tc::tmem_dealloc(tb, W);
}

}  // namespace tpc
