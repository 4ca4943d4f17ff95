// Tree-masked softmax attention on tcgen05 (HARTS Figure 1(b): full attention reads ancestor keys
// and values; Figure C.1(c): within a segment the diagonal blocks are causal, a later segment reads
// its ancestors and never the reverse; outputs return to compact rows).
//
// A query tile (<= 128 rows of one node) visits the node's ancestor row ranges (a few contiguous
// ranges in the compact layout, one per chain on its path) and then its own node's rows up to the
// tile's end with the causal mask, in key tiles of 64.  Forward: S = Q K^T, online softmax in fp32,
// O += P V with P a bf16 hi/lo pair.  Backward, deterministic (no atomics): dQ per query tile (S and
// dP = dO V^T recomputed, dQ += dS K accumulated in TMEM); dK, dV per key tile (<= 128 rows of one
// node), looping over the query rows that can see it: the node's subtree rows from the tile on, one
// contiguous range in the compact layout.
//
// All three kernels are warp-specialised (one MMA-issuing thread, TMA loader threads, softmax
// warps) with mbarrier-ordered pipelines and bounded waits.  Row tiles arrive by TMA from 3-D tensor
// maps (rows x heads x features) as 128-byte-swizzled boxes of 64 features; the operand that stays
// put for a whole block (Q in the forward and dQ, V in dK/dV) and the softmax outputs that feed a
// product as its M side (P, dS) live in TMEM as A operands.
//
// SPLIT kernels take q, k, v and dO as bf16 hi/lo pairs (fp32 values x = hi + lo to 2^-17
// relative) and form every product from three partial products (hi hi + lo hi + hi lo), so that
// fp32 inputs and upstream gradients enter without a bf16 rounding of their own.
#pragma once
#include "kda_tc.cuh"

namespace tpc {

constexpr int kAttnQK = 192, kAttnDV = 128;

namespace tck {

template <typename T>
__device__ __forceinline__ void st_out16(T* p, const float* v) {
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int j = 0; j < 16; j += 4)
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
    __align__(16) __nv_bfloat16 b[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) b[j] = __float2bfloat16_rn(v[j]);
    reinterpret_cast<uint4*>(p)[0] = reinterpret_cast<const uint4*>(b)[0];
    reinterpret_cast<uint4*>(p)[1] = reinterpret_cast<const uint4*>(b)[1];
  }
}

// x0, x1 as packed bf16 hi / lo pairs (element 0 in the low half): x = hi + lo to ~2^-17
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// 16 packed values (8 pairs along the contiguous index) of row a at (a, b0..b0+15) of K-major
// core-matrix tiles with A rows, hi and lo parts
template <int A>
__device__ __forceinline__ void put16_packed(uint8_t* hi, uint8_t* lo, int a, int b0, const uint32_t* ph,
                                             const uint32_t* pl) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    *reinterpret_cast<uint4*>(hi + tc::cm_off(a, b0 + 8 * half, A)) =
        make_uint4(ph[4 * half], ph[4 * half + 1], ph[4 * half + 2], ph[4 * half + 3]);
    *reinterpret_cast<uint4*>(lo + tc::cm_off(a, b0 + 8 * half, A)) =
        make_uint4(pl[4 * half], pl[4 * half + 1], pl[4 * half + 2], pl[4 * half + 3]);
  }
}

}  // namespace tck

// ------------------------------------------------------------------------------------------ forward
// Key tiles of a query tile, one at a time: the node's ancestor ranges in order, then its own rows up
// to the tile's end.
template <int KT>
struct KeyTileIter {
  const RowRange* ranges;
  int r, r1, k, own_start, own_end;
  __device__ void init(const DevTables& t, const AttnTile& qt) {
    const AttnNode nd = t.attn_nodes[qt.node];
    ranges = t.attn_ranges;
    r = nd.range_begin;
    r1 = t.attn_nodes[qt.node + 1].range_begin;
    own_start = nd.row_offset;
    own_end = qt.row + qt.n;
    k = r < r1 ? ranges[r].start : own_start;
  }
  __device__ bool next(int& k0, int& nk, bool& own) {
    while (r < r1) {
      const RowRange rr = ranges[r];
      if (k < rr.end) {
        k0 = k; nk = min(KT, rr.end - k); own = false; k += KT;
        return true;
      }
      ++r;
      k = r < r1 ? ranges[r].start : own_start;
    }
    if (k < own_end) {
      k0 = k; nk = min(KT, own_end - k); own = true; k += KT;
      return true;
    }
    return false;
  }
};



// Forward, per query tile (<= 128 rows of one node) and head, warp-specialised:
//   warp 0      issues the MMAs: S_j = Q K_j^T into one of two TMEM buffers, then O += P_j V_j;
//   warp 1      streams the key tiles K_j (and their lo parts) through a three-stage ring and
//   warp 2      V_j through a two-stage ring, by TMA (128-byte-swizzled boxes of 64 features);
//   warps 3-10  two threads per query row (key columns split in halves): Q is loaded once into TMEM
//               (the A operand of S), then per key tile the online softmax (base-2 exponentials of
//               log2-scaled scores) reads S_j (releasing its buffer), writes P_j as a bf16 hi/lo
//               pair into a TMEM buffer of its own (the A operand of P V) once P_{j-1} V_{j-1} has
//               completed, and keeps a reference maximum that is raised (O and l rescaled) only when
//               a tile's maximum exceeds it by more than a factor e^8.
// S_{j+1} and P_{j-1} V_{j-1} run on the tensor core while the softmax of tile j runs.
template <bool SPLIT>
struct AttnFwdSmem {
  static constexpr int NK = 3, NV = 2;
  static constexpr size_t X = SPLIT ? 2 : 1;  // hi (and lo) parts
  static constexpr size_t Kb = size_t(64) * kAttnQK * 2, Vb = size_t(64) * kAttnDV * 2;
  static constexpr size_t Kst = X * Kb, Vst = X * Vb;  // one ring stage
  static constexpr size_t K = 0, V = K + NK * Kst;
  static constexpr size_t total = V + NV * Vst + 1024;  // + slack to align the boxes to 1024 bytes
  static_assert(total <= 227 * 1024, "shared memory");
};

constexpr int kAttnFwdThreads = 352;

template <typename Tout, bool SPLIT>
__global__ void __launch_bounds__(kAttnFwdThreads, 1)
    attn_fwd_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ q,
                const __nv_bfloat16* __restrict__ q_lo, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_vl, Tout* __restrict__ o, float* __restrict__ lse,
                int* status) {
  using namespace tck;
  using namespace tc;
  using S = AttnFwdSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, NK = S::NK, NV = S::NV;
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  constexpr float kRaise2 = 8.f * kLog2e;  // raise threshold (e^8) in log2 units
  // TMEM columns: Q hi (96), Q lo (96), O (128), two S buffers (64 each), P hi (32) and lo (32)
  constexpr uint32_t cQh = 0, cQl = 96, cO = 192, cS = 320, cBuf = 64, cP = 448;
  // grid: one block per (query tile, head), query tiles fastest, so that the blocks resident at one
  // time read the same head's keys and values (shared in L2); the planner lists the query tiles of
  // a head by decreasing work, so the longest blocks start first
  const int n_qt = gridDim.x / H;
  const AttnTile qt = t.attn_qtiles[blockIdx.x % n_qt];
  const int h = blockIdx.x / n_qt;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t asmem_raw[];
  // the swizzle pattern is a function of the shared address: boxes start on 1024-byte boundaries
  uint8_t* asmem = asmem_raw + ((1024u - (smem_u32(asmem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t kfull[NK], kempty[NK], vfull[NV], vempty[NV], s_full[2], s_read[2], p_full,
      pv_done, q_ready, done_bar;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  __shared__ float red_sum[2][128];
  auto kst = [&](int s) { return asmem + S::K + (size_t)s * S::Kst; };
  auto vst = [&](int s) { return asmem + S::V + (size_t)s * S::Vst; };
  if (w == 0) tmem_alloc(&tslot, 512);
  if (tid == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&kfull[s], 1);  // the loader's arrival with the expected bytes
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_read[b], 8);  // one arrival per softmax warp
    }
    mbar_init(&p_full, 8);
    mbar_init(&pv_done, 1);
    mbar_init(&q_ready, 8);
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tslot;
  auto give_up = [&] {
    set_status(status, kStatusTimeout);
    atomicExch(&abort_flag, 1);
  };
  auto aborted = [&] { return *((volatile int*)&abort_flag) != 0; };
  // number of key tiles of this query tile
  int n_tiles = 0;
  {
    KeyTileIter<64> it;
    it.init(t, qt);
    int a, b;
    bool c;
    while (it.next(a, b, c)) ++n_tiles;
  }

  if (w == 0) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16(128, 64, false, false), id_o = idesc_bf16(128, DV, false, true);
      bool ok = mbar_wait(&q_ready, 0);
      if (!ok) give_up();
      for (int j = 0; ok && j <= n_tiles && !aborted(); ++j) {
        if (j < n_tiles) {  // S_j = Q K_j^T
          const int ks = j % NK, b = j & 1;
          if (!mbar_wait(&kfull[ks], (j / NK) & 1) || (j >= 2 && !mbar_wait(&s_read[b], ((j >> 1) - 1) & 1))) {
            give_up();
            break;
          }
          fence_after_sync();
          const uint32_t d = tb + cS + cBuf * b;
          const uint32_t kh = smem_u32(kst(ks)), kl = kh + (uint32_t)S::Kb;
          for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(d, tb + cQh + 8 * s, sw_desc_k(kh, 64, s), id_s, s ? 1u : 0u);
          if constexpr (SPLIT) {
            for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(d, tb + cQl + 8 * s, sw_desc_k(kh, 64, s), id_s, 1u);
            for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(d, tb + cQh + 8 * s, sw_desc_k(kl, 64, s), id_s, 1u);
          }
          commit(&kempty[ks]);
          commit(&s_full[b]);
        }
        if (j >= 1) {  // O += P_{j-1} V_{j-1}
          const int jp = j - 1, vs = jp % NV;
          if (!mbar_wait(&p_full, jp & 1) || !mbar_wait(&vfull[vs], (jp / NV) & 1)) {
            give_up();
            break;
          }
          fence_after_sync();
          const uint32_t ph = tb + cP, pl = ph + 32;
          const uint32_t vh = smem_u32(vst(vs)), vl = vh + (uint32_t)S::Vb;
          for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cO, ph + 8 * s, sw_desc_mn(vh, 64, s), id_o, (jp > 0 || s) ? 1u : 0u);
          for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cO, pl + 8 * s, sw_desc_mn(vh, 64, s), id_o, 1u);
          if constexpr (SPLIT)
            for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cO, ph + 8 * s, sw_desc_mn(vl, 64, s), id_o, 1u);
          commit(&vempty[vs]);
          commit(&pv_done);
        }
      }
      commit(&done_bar);  // arrives once every MMA issued above has completed
      if (!mbar_wait(&done_bar, 0, 2000000000ull)) give_up();
    }
  } else if (w <= 2) {  // ------------------------------------------------ loaders (one thread each)
    if (lane == 0) {
      const bool is_k = w == 1;
      const int NS = is_k ? NK : NV, F = is_k ? DQ : DV;
      const uint32_t part = (uint32_t)(is_k ? S::Kb : S::Vb), bytes = (uint32_t)(SPLIT ? 2 : 1) * part;
      KeyTileIter<64> it;
      it.init(t, qt);
      int k0 = 0, nk = 0, j = 0;
      bool own = false;
      for (; it.next(k0, nk, own); ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(is_k ? &kempty[s] : &vempty[s], ((j / NS) - 1) & 1)) {
          give_up();
          break;
        }
        if (aborted()) break;
        uint64_t* bar = is_k ? &kfull[s] : &vfull[s];
        uint8_t* dst = is_k ? kst(s) : vst(s);
        // rows k0 .. k0 + 63 of head h (rows past the tile's end are masked by the softmax; rows past
        // the tensor's end are filled with zeros)
        mbar_arrive_expect_tx(bar, bytes);
        for (int c = 0; c < F / 64; ++c) {
          tma_load_3d(dst + c * 64 * 128, is_k ? (const void*)&tm_k : (const void*)&tm_v, 64 * c, h, k0, bar);
          if constexpr (SPLIT)
            tma_load_3d(dst + part + c * 64 * 128, is_k ? (const void*)&tm_kl : (const void*)&tm_vl, 64 * c, h, k0, bar);
        }
      }
    }
  } else if (w >= 3) {  // ------------------------------------------------ softmax (warps 3-10)
    // warp w holds the TMEM lanes (query rows) of sub-partition w % 4 and the key columns of half
    // (w - 3) / 4 for the exponentials; each thread reads the whole row of S for the row maximum, so
    // the two threads of a row take the same decisions without exchanging data per key tile
    const int sp = w & 3, half = (w - 3) >> 2, row = 32 * sp + lane, qrow = qt.row + row;
    const uint32_t la = tb + ((uint32_t)(32 * sp) << 16);
    const float sl2 = scale * kLog2e;  // scores in log2 units: t = s scale log2(e)
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar, parity));
      if (!got && lane == 0) give_up();
      return got && !__any_sync(0xffffffffu, aborted());
    };
    // the two warps of a row pair meet once, after the last key tile (named barrier, 64 threads)
    auto pair_sync = [&] { asm volatile("bar.sync %0, 64;" ::"r"(1 + sp) : "memory"); };
    {  // this half of Q (and its lo part) into TMEM: a bf16 pair per 32-bit column, as in memory
      const bool in = row < qt.n;
      constexpr int HC = DQ / 4;  // 48 columns per half
      for (int part = 0; part < (SPLIT ? 2 : 1); ++part) {
        const bf* src = part ? q_lo : q;
        const uint4* g4 = (in && src) ? reinterpret_cast<const uint4*>(src + ((size_t)qrow * H + h) * DQ) + HC / 4 * half
                                      : nullptr;
        for (int c0 = 0; c0 < HC; c0 += 16) {
          float r[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 x = g4 ? g4[c0 / 4 + i] : make_uint4(0u, 0u, 0u, 0u);
            r[4 * i] = __uint_as_float(x.x); r[4 * i + 1] = __uint_as_float(x.y);
            r[4 * i + 2] = __uint_as_float(x.z); r[4 * i + 3] = __uint_as_float(x.w);
          }
          tmem_st16(la + (part ? cQl : cQh) + HC * half + c0, r);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }
    KeyTileIter<64> it;
    it.init(t, qt);
    int k0 = 0, nk = 0;
    bool own = false, ok = true;
    float m_ref = -INFINITY, l = 0.f;  // m_ref in log2 units; l: this half's share of the row sum
    for (int j = 0; j < n_tiles; ++j) {
      it.next(k0, nk, own);
      const int b = j & 1;
      if (!(ok = wait_all(&s_full[b], (j >> 1) & 1))) break;
      fence_after_sync();
      const uint32_t sb = la + cS + cBuf * b;
      float tv[32], mx = -INFINITY;  // tv: this half's scores
      {
        uint32_t r0[32], r1[32];
        tmem_ld32_nowait(sb, r0);
        tmem_ld32_nowait(sb + 32, r1);
        tmem_wait_ld();
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_read[b]);  // the buffer may take S_{j+2}
        const bool masked = own || nk < 64;  // ragged key tile or the node's own (causal) rows
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0 = __uint_as_float(r0[c]) * sl2, x1 = __uint_as_float(r1[c]) * sl2;
          if (masked) {
            if (c >= nk || (own && k0 + c > qrow)) x0 = -INFINITY;
            if (32 + c >= nk || (own && k0 + 32 + c > qrow)) x1 = -INFINITY;
          }
          mx = fmaxf(mx, fmaxf(x0, x1));
          tv[c] = half ? x1 : x0;
        }
      }
      // raise the reference where the tile's maximum exceeds it by more than kRaise; O (all tiles so
      // far, so the previous P V must have completed) and l follow.  Both threads of a row take the
      // same decision; TMEM loads and stores are warp-collective, so a warp rescales its 32 rows
      // together when any of them raised.
      const bool raise = mx > m_ref + kRaise2;
      const float corr = !raise ? 1.f : (m_ref == -INFINITY ? 0.f : exp2f(m_ref - mx));
      if (raise) {
        l *= corr;
        m_ref = mx;
      }
      // P_{j-1} V_{j-1} has completed: O is final up to tile j - 1 and the P buffer is free
      if (j > 0) {
        if (!(ok = wait_all(&pv_done, (j - 1) & 1))) break;
        fence_after_sync();
      }
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        for (int c0 = 0; c0 < DV / 2; c0 += 32) {
          uint32_t r[32];
          tmem_ld32_nowait(la + cO + DV / 2 * half + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * corr);
          tmem_st32_nowait(la + cO + DV / 2 * half + c0, r);
        }
        tmem_wait_st();
      }
      const float mb = m_ref == -INFINITY ? 0.f : m_ref;
      float psum = 0.f;
      float ph[16], pl[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = exp2f(tv[c] - mb), p1 = exp2f(tv[c + 1] - mb);
        psum += p0 + p1;
        const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
        const float2 hf = __bfloat1622float2(hi);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
        ph[c / 2] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&hi));
        pl[c / 2] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&lo));
      }
      l += psum;
      // P hi in columns 0..31 of its buffer, lo in 32..63; this half's keys are 16 columns of each
      tmem_st16(la + cP + 16 * half, ph);
      tmem_st16(la + cP + 32 + 16 * half, pl);
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && n_tiles > 0) ok = wait_all(&pv_done, (n_tiles - 1) & 1);
    red_sum[half][row] = l;
    pair_sync();
    if (ok) {
      fence_after_sync();
      const float lt = l + red_sum[half ^ 1][row];
      const float inv = n_tiles > 0 ? 1.f / lt : 0.f;
      Tout* dst = o + ((size_t)qrow * H + h) * DV + DV / 2 * half;
      for (int c0 = 0; c0 < DV / 2; c0 += 32) {
        uint32_t r[32];
        tmem_ld32_nowait(la + cO + DV / 2 * half + c0, r);  // warp-collective: every row takes part
        tmem_wait_ld();
        if (row < qt.n) {
          float ov[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __uint_as_float(r[c]) * inv;
          st_out16(dst + c0, ov);
          st_out16(dst + c0 + 16, ov + 16);
        }
      }
      if (row < qt.n && half == 0) lse[(size_t)qrow * H + h] = (m_ref + log2f(lt)) * kLn2;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (w == 0) tmem_dealloc(tb, 512);
}


// ------------------------------------------------------------------------------------------ backward dQ
// per query tile (<= 128 rows of one node) and head: delta = rowsum(dO * O) (also written for the
// dK/dV kernel), then over the key tiles P = exp(scale S - lse), dP = dO V^T, dS = P (dP - delta),
// dQ += dS K; dq = scale dQ.  Warp-specialised like the forward:
//   warp 0      issues S_j = Q K_j^T, then dQ += dS_{j-1} K_{j-1}, then dP_j = dO V_j^T;
//   warp 1      streams K_j through a two-stage ring; warp 2 loads dO once, then streams V_j (TMA,
//               128-byte-swizzled boxes of 64 features);
//   warps 3-18  four threads per query row (key columns in quarters of 16): Q into TMEM once, delta;
//               per key tile they read S_j (releasing it for S_{j+1}) and dP_j, and write dS_j as
//               bf16 hi/lo pairs over their own 16 dP_j columns (hi in the first 8, lo in the last 8:
//               the A operand of the dQ product, one K step per quarter).
template <bool SPLIT>
struct AttnDqSmem {
  static constexpr int NK = 2, NV = 2;
  static constexpr size_t X = SPLIT ? 2 : 1;
  static constexpr size_t Ob = size_t(128) * kAttnDV * 2, Kb = size_t(64) * kAttnQK * 2, Vb = size_t(64) * kAttnDV * 2;
  static constexpr size_t dO = 0, K = dO + X * Ob, V = K + NK * X * Kb;
  static constexpr size_t total = V + NV * X * Vb + 1024;  // + slack to align the boxes to 1024 bytes
  static_assert(total <= 227 * 1024, "shared memory");
};

constexpr int kAttnDqThreads = 608;

template <typename Tio, bool SPLIT>
__global__ void __launch_bounds__(kAttnDqThreads, 1)
    attn_bwd_dq_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ q_lo, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_vl, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_ol, const Tio* __restrict__ o, const float* __restrict__ lse,
                   const __nv_bfloat16* __restrict__ d_o, const __nv_bfloat16* __restrict__ d_o_lo,
                   Tio* __restrict__ dq, float* __restrict__ delta, int* status) {
  using namespace tck;
  using namespace tc;
  using S = AttnDqSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, NK = S::NK, NV = S::NV;
  constexpr float kLog2e = 1.4426950408889634f;
  // TMEM columns: Q hi (96), Q lo (96), dQ (192), S (64), dP / dS (64)
  constexpr uint32_t cQh = 0, cQl = 96, cG = 192, cS = 384, cP = 448;
  // grid: one block per (query tile, head), query tiles fastest (see the forward)
  const int n_qt = gridDim.x / H;
  const AttnTile qt = t.attn_qtiles[blockIdx.x % n_qt];
  const int h = blockIdx.x / n_qt;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t asmem_raw[];
  uint8_t* asmem = asmem_raw + ((1024u - (smem_u32(asmem_raw) & 1023u)) & 1023u);  // 1024-byte aligned boxes
  __shared__ __align__(8) uint64_t kfull[NK], kempty[NK], vfull[NV], vempty[NV], do_full, q_ready, s_full, s_read,
      dp_full, ds_full, dq_done, done_bar;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  uint8_t* sO = asmem + S::dO;
  auto kst = [&](int s) { return asmem + S::K + (size_t)s * S::X * S::Kb; };
  auto vst = [&](int s) { return asmem + S::V + (size_t)s * S::X * S::Vb; };
  if (w == 0) tmem_alloc(&tslot, 512);
  if (tid == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&kfull[s], 1);  // the loader's arrival with the expected bytes
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    mbar_init(&do_full, 1);
    mbar_init(&q_ready, 8);  // one arrival per warp of the first two column quarters
    mbar_init(&s_full, 1);
    mbar_init(&s_read, 16);  // one arrival per P / dS warp
    mbar_init(&dp_full, 1);
    mbar_init(&ds_full, 16);
    mbar_init(&dq_done, 1);
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tslot;
  auto give_up = [&] {
    set_status(status, kStatusTimeout);
    atomicExch(&abort_flag, 1);
  };
  auto aborted = [&] { return *((volatile int*)&abort_flag) != 0; };
  int n_tiles = 0;
  {
    KeyTileIter<64> it;
    it.init(t, qt);
    int a, b;
    bool c;
    while (it.next(a, b, c)) ++n_tiles;
  }

  if (w == 0) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16(128, 64, false, false), id_g = idesc_bf16(128, DQ, false, true);
      bool ok = mbar_wait(&q_ready, 0) && mbar_wait(&do_full, 0);
      if (!ok) give_up();
      const uint32_t oh = smem_u32(sO), ol = oh + (uint32_t)S::Ob;
      for (int j = 0; ok && j <= n_tiles && !aborted(); ++j) {
        if (j < n_tiles) {  // S_j = Q K_j^T, once the softmax warps have read S_{j-1}
          const int ks = j % NK;
          if (!mbar_wait(&kfull[ks], (j / NK) & 1) || (j >= 1 && !mbar_wait(&s_read, (j - 1) & 1))) {
            give_up();
            break;
          }
          fence_after_sync();
          const uint32_t kh = smem_u32(kst(ks)), kl = kh + (uint32_t)S::Kb;
          for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(tb + cS, tb + cQh + 8 * s, sw_desc_k(kh, 64, s), id_s, s ? 1u : 0u);
          if constexpr (SPLIT) {
            for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(tb + cS, tb + cQl + 8 * s, sw_desc_k(kh, 64, s), id_s, 1u);
            for (int s = 0; s < DQ / 16; ++s) mma_bf16_ts(tb + cS, tb + cQh + 8 * s, sw_desc_k(kl, 64, s), id_s, 1u);
          }
          commit(&s_full);
        }
        if (j >= 1) {  // dQ += dS_{j-1} K_{j-1}: dS in the dP columns, hi / lo in each half's 32 columns
          const int jp = j - 1, ks = jp % NK;
          if (!mbar_wait(&ds_full, jp & 1)) {
            give_up();
            break;
          }
          fence_after_sync();
          const uint32_t kh = smem_u32(kst(ks)), kl = kh + (uint32_t)S::Kb;
          auto a_hi = [&](int s) { return tb + cP + 16 * s; };  // K step s: keys 16 s .. 16 s + 15
          for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cG, a_hi(s), sw_desc_mn(kh, 64, s), id_g, (jp > 0 || s) ? 1u : 0u);
          for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cG, a_hi(s) + 8, sw_desc_mn(kh, 64, s), id_g, 1u);
          if constexpr (SPLIT)
            for (int s = 0; s < 4; ++s) mma_bf16_ts(tb + cG, a_hi(s), sw_desc_mn(kl, 64, s), id_g, 1u);
          commit(&kempty[ks]);
          commit(&dq_done);
        }
        if (j < n_tiles) {  // dP_j = dO V_j^T, once dQ has read dS_{j-1} from the same columns
          const int vs = j % NV;
          if (!mbar_wait(&vfull[vs], (j / NV) & 1) || (j >= 1 && !mbar_wait(&dq_done, (j - 1) & 1))) {
            give_up();
            break;
          }
          fence_after_sync();
          const uint32_t vh = smem_u32(vst(vs)), vl = vh + (uint32_t)S::Vb;
          for (int s = 0; s < DV / 16; ++s) mma_bf16(tb + cP, sw_desc_k(oh, 128, s), sw_desc_k(vh, 64, s), id_s, s ? 1u : 0u);
          if constexpr (SPLIT) {
            for (int s = 0; s < DV / 16; ++s) mma_bf16(tb + cP, sw_desc_k(ol, 128, s), sw_desc_k(vh, 64, s), id_s, 1u);
            for (int s = 0; s < DV / 16; ++s) mma_bf16(tb + cP, sw_desc_k(oh, 128, s), sw_desc_k(vl, 64, s), id_s, 1u);
          }
          commit(&vempty[vs]);
          commit(&dp_full);
        }
      }
      commit(&done_bar);  // arrives once every MMA issued above has completed
      if (!mbar_wait(&done_bar, 0, 2000000000ull)) give_up();
    }
  } else if (w <= 2) {  // ------------------------------------------------ loaders (one thread each)
    if (lane == 0) {
      const bool is_k = w == 1;
      if (!is_k) {  // dO rows of the query tile (rows past the tile are masked, past the tensor zero)
        mbar_arrive_expect_tx(&do_full, (uint32_t)(SPLIT ? 2 : 1) * (uint32_t)S::Ob);
        for (int c = 0; c < DV / 64; ++c) {
          tma_load_3d(sO + c * 128 * 128, &tm_o, 64 * c, h, qt.row, &do_full);
          if constexpr (SPLIT) tma_load_3d(sO + S::Ob + c * 128 * 128, &tm_ol, 64 * c, h, qt.row, &do_full);
        }
      }
      const int NS = is_k ? NK : NV, F = is_k ? DQ : DV;
      const uint32_t part = (uint32_t)(is_k ? S::Kb : S::Vb), bytes = (uint32_t)(SPLIT ? 2 : 1) * part;
      KeyTileIter<64> it;
      it.init(t, qt);
      int k0 = 0, nk = 0, j = 0;
      bool own = false;
      for (; it.next(k0, nk, own); ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(is_k ? &kempty[s] : &vempty[s], ((j / NS) - 1) & 1)) {
          give_up();
          break;
        }
        if (aborted()) break;
        uint64_t* bar = is_k ? &kfull[s] : &vfull[s];
        uint8_t* dst = is_k ? kst(s) : vst(s);
        mbar_arrive_expect_tx(bar, bytes);
        for (int c = 0; c < F / 64; ++c) {
          tma_load_3d(dst + c * 64 * 128, is_k ? (const void*)&tm_k : (const void*)&tm_v, 64 * c, h, k0, bar);
          if constexpr (SPLIT)
            tma_load_3d(dst + part + c * 64 * 128, is_k ? (const void*)&tm_kl : (const void*)&tm_vl, 64 * c, h, k0, bar);
        }
      }
    }
  } else if (w >= 3) {  // ------------------------------------------------ P, dS (warps 3-18)
    const int sp = w & 3, quarter = (w - 3) >> 2, row = 32 * sp + lane, qrow = qt.row + row;
    const bool in = row < qt.n;
    const uint32_t la = tb + ((uint32_t)(32 * sp) << 16);
    const float sl2 = scale * kLog2e;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar, parity));
      if (!got && lane == 0) give_up();
      return got && !__any_sync(0xffffffffu, aborted());
    };
    if (quarter < 2) {  // half `quarter` of Q (and its lo part) into TMEM
      const int half = quarter;
      constexpr int HC = DQ / 4;
      for (int part = 0; part < (SPLIT ? 2 : 1); ++part) {
        const bf* src = part ? q_lo : q;
        const uint4* g4 = (in && src) ? reinterpret_cast<const uint4*>(src + ((size_t)qrow * H + h) * DQ) + HC / 4 * half
                                      : nullptr;
        for (int c0 = 0; c0 < HC; c0 += 16) {
          float r[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 x = g4 ? g4[c0 / 4 + i] : make_uint4(0u, 0u, 0u, 0u);
            r[4 * i] = __uint_as_float(x.x); r[4 * i + 1] = __uint_as_float(x.y);
            r[4 * i + 2] = __uint_as_float(x.z); r[4 * i + 3] = __uint_as_float(x.w);
          }
          tmem_st16(la + (part ? cQl : cQh) + HC * half + c0, r);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_ready);
    }
    // delta = rowsum(dO O) over the whole row (both threads of a row), lse of the row
    float dl = 0.f, ls2 = 0.f;
    if (in) {
      const Tio* orow = o + ((size_t)qrow * H + h) * DV;
      const bf* grow = d_o + ((size_t)qrow * H + h) * DV;
      const bf* glow = SPLIT && d_o_lo ? d_o_lo + ((size_t)qrow * H + h) * DV : nullptr;
      for (int c = 0; c < DV; ++c)
        dl = fmaf(to_f(orow[c]), __bfloat162float(grow[c]) + (glow ? __bfloat162float(glow[c]) : 0.f), dl);
      if (quarter == 0) delta[(size_t)qrow * H + h] = dl;
      ls2 = lse[(size_t)qrow * H + h] * kLog2e;
    }
    KeyTileIter<64> it;
    it.init(t, qt);
    int k0 = 0, nk = 0;
    bool own = false, ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      it.next(k0, nk, own);
      if (!(ok = wait_all(&s_full, j & 1)) || !(ok = wait_all(&dp_full, j & 1))) break;
      fence_after_sync();
      float rs[16], rp[16];
      tmem_ld16(la + cS + 16 * quarter, rs);
      tmem_ld16(la + cP + 16 * quarter, rp);
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_read);  // S may take S_{j+1}
      const bool masked = !in || own || nk < 64;
      float g[16];  // dS of the quarter's 16 keys: 8 hi pairs, then 8 lo pairs
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kc = 16 * quarter + c + e;
          const bool valid = !masked || (in && kc < nk && !(own && k0 + kc > qrow));
          const float pv = valid ? exp2f(rs[c + e] * sl2 - ls2) : 0.f;
          ds[e] = pv * (rp[c + e] - dl);
        }
        uint32_t hi, lo;
        split2(ds[0], ds[1], hi, lo);
        g[c / 2] = __uint_as_float(hi);
        g[8 + c / 2] = __uint_as_float(lo);
      }
      tmem_st16(la + cP + 16 * quarter, g);  // over this quarter's own dP columns
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full);
    }
    if (ok && n_tiles > 0) ok = wait_all(&dq_done, (n_tiles - 1) & 1);
    if (ok) {
      fence_after_sync();
      for (int c0 = 0; c0 < DQ / 4; c0 += 16) {
        float g[16];
        tmem_ld16(la + cG + DQ / 4 * quarter + c0, g);  // warp-collective: every row takes part
        if (in) {
#pragma unroll
          for (int c = 0; c < 16; ++c) g[c] = n_tiles > 0 ? g[c] * scale : 0.f;
          st_out16(dq + ((size_t)qrow * H + h) * DQ + DQ / 4 * quarter + c0, g);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (w == 0) tmem_dealloc(tb, 512);
}

// ------------------------------------------------------------------------------------------ backward dK, dV
// per key tile of node u (<= 128 rows): query rows [row of the tile, subtree end of u) in tiles of 32
// (queries of u itself only from the key row on), S^T = K Q^T, dP^T = V dO^T, P^T = exp(scale S^T -
// lse), dS^T = P^T (dP^T - delta); dV += P^T dO, dK += dS^T Q; dk = scale dK.  M = 128 accumulators.
//
// Warp-specialised: warp 0 issues the MMAs, warp 1 loads K and then streams the query tiles (Q, dO
// and their lo parts) through a two-stage ring by TMA (128-byte-swizzled boxes of 64 features),
// warp 2 adds lse and delta of each query tile by cp.async, warps 3-10 load V into TMEM (the A
// operand of dP^T) and turn S^T, dP^T into P^T, dS^T.  The products of query tile j + 1 run on the
// tensor core while the P / dS math of tile j runs.  Every wait is bounded; a timeout records
// TPC_ERR_TIMEOUT and every role stops.
template <bool SPLIT>
struct AttnDkvSmem {
  static constexpr int KT = 128, QT = 32, NS = 2;  // key rows, query rows per tile, ring stages
  static constexpr size_t X = SPLIT ? 2 : 1;
  static constexpr size_t Kb = size_t(KT) * kAttnQK * 2;
  static constexpr size_t Qb = size_t(QT) * kAttnQK * 2, Ob = size_t(QT) * kAttnDV * 2, Pb = size_t(KT) * QT * 2;
  // one ring stage: Q, Q_lo, dO, dO_lo (swizzled boxes), lse[QT], delta[QT]; stages 1024-byte aligned
  static constexpr size_t sQ = 0, sQl = sQ + Qb, sO = sQ + X * Qb, sOl = sO + Ob, sL = sO + X * Ob, sD = sL + QT * 4;
  static constexpr size_t stage = (sD + QT * 4 + 1023) & ~size_t(1023);
  static constexpr size_t K = 0, ring = K + X * Kb;
  static constexpr size_t P = ring + NS * stage, Pl = P + Pb, dS = Pl + Pb, dSl = dS + Pb;
  static constexpr size_t total = dSl + Pb + 1024;  // + slack to align the boxes to 1024 bytes
  static_assert(total <= 227 * 1024, "shared memory");
  static_assert(stage % 1024 == 0, "stage alignment");
};

constexpr int kAttnDkvThreads = 352;

template <typename Tio, bool SPLIT>
__global__ void __launch_bounds__(kAttnDkvThreads, 1)
    attn_bwd_dkv_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ v,
                    const __nv_bfloat16* __restrict__ v_lo, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_ql, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_ol, const float* __restrict__ lse,
                    const float* __restrict__ delta, Tio* __restrict__ dk, Tio* __restrict__ dv, int* status) {
  using namespace tck;
  using namespace tc;
  using S = AttnDkvSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, KT = S::KT, QT = S::QT, NS = S::NS;
  constexpr float kLog2e = 1.4426950408889634f;
  const float sl2 = scale * kLog2e;
  // TMEM columns: dV (128), dK (192), V hi (64) and lo (64) as bf16 pairs, S^T (32), dP^T (32)
  constexpr uint32_t cDV = 0, cDK = 128, cVh = 320, cVl = 384, cS = 448, cP = 480;
  // grid: one block per (key tile, head), key tiles fastest, so that the blocks resident at one
  // time read the same head's query rows (shared in L2); the planner lists the key tiles of a head
  // by decreasing work, so the longest blocks start first
  const int n_kt = gridDim.x / H;
  const AttnTile kt = t.attn_ktiles[blockIdx.x % n_kt];
  const int h = blockIdx.x / n_kt;
  const AttnNode nd = t.attn_nodes[kt.node];
  const int k0 = kt.row, nk = kt.n, own_end = nd.row_offset + nd.length, q_end = nd.subtree_end;
  const int n_tiles = (q_end - k0 + QT - 1) / QT;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t asmem_raw[];
  uint8_t* asmem = asmem_raw + ((1024u - (smem_u32(asmem_raw) & 1023u)) & 1023u);  // 1024-byte aligned boxes
  __shared__ __align__(8) uint64_t full[NS], empty[NS], v_ready, s_full, s_read, p_full, p_empty, done_bar;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  uint8_t *sK = asmem + S::K, *sKl = sK + S::Kb;
  uint8_t *sPh = asmem + S::P, *sPl = asmem + S::Pl, *sDh = asmem + S::dS, *sDl = asmem + S::dSl;
  auto stage = [&](int s) { return asmem + S::ring + (size_t)s * S::stage; };
  if (w == 0) tmem_alloc(&tslot, 512);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 33);  // the TMA thread's arrival with the expected bytes, the lse / delta warp
      mbar_init(&empty[s], 1);
    }
    mbar_init(&v_ready, 8);  // one arrival per P / dS warp
    mbar_init(&s_full, 1);
    mbar_init(&s_read, 8);
    mbar_init(&p_full, 8);
    mbar_init(&p_empty, 1);
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  fence_after_sync();
  const uint32_t tb = tslot;
  auto give_up = [&] {
    set_status(status, kStatusTimeout);
    atomicExch(&abort_flag, 1);
  };
  auto aborted = [&] { return *((volatile int*)&abort_flag) != 0; };

  if (w == 0) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      const uint32_t id_s = idesc_bf16(128, QT, false, false);
      const uint32_t id_dv = idesc_bf16(128, DV, false, true), id_dk = idesc_bf16(128, DQ, false, true);
      bool ok = mbar_wait(&v_ready, 0);
      if (!ok) give_up();
      // S^T, dP^T of tile jS (needs its stage loaded and the previous S^T read) and dV, dK of tile jD
      // (needs P^T, dS^T of tile jD in shared memory) are independent: issue whichever is ready,
      // dV / dK first, since they release the stage that the load of tile jD + 2 waits for.
      auto issue_s = [&](int j) {
        const uint32_t st = smem_u32(stage(j % NS));
        const uint32_t kh = smem_u32(sK), kl = smem_u32(sKl);
        const uint32_t qh = st + (uint32_t)S::sQ, ql = st + (uint32_t)S::sQl, oh = st + (uint32_t)S::sO,
                       ol = st + (uint32_t)S::sOl;
        for (int s2 = 0; s2 < DQ / 16; ++s2) mma_bf16(tb + cS, sw_desc_k(kh, KT, s2), sw_desc_k(qh, QT, s2), id_s, s2 ? 1u : 0u);
        for (int s2 = 0; s2 < DV / 16; ++s2) mma_bf16_ts(tb + cP, tb + cVh + 8 * s2, sw_desc_k(oh, QT, s2), id_s, s2 ? 1u : 0u);
        if constexpr (SPLIT) {
          for (int s2 = 0; s2 < DQ / 16; ++s2) {
            mma_bf16(tb + cS, sw_desc_k(kl, KT, s2), sw_desc_k(qh, QT, s2), id_s, 1u);
            mma_bf16(tb + cS, sw_desc_k(kh, KT, s2), sw_desc_k(ql, QT, s2), id_s, 1u);
          }
          for (int s2 = 0; s2 < DV / 16; ++s2) {
            mma_bf16_ts(tb + cP, tb + cVl + 8 * s2, sw_desc_k(oh, QT, s2), id_s, 1u);
            mma_bf16_ts(tb + cP, tb + cVh + 8 * s2, sw_desc_k(ol, QT, s2), id_s, 1u);
          }
        }
        commit(&s_full);
      };
      auto issue_d = [&](int jp) {
        const int s = jp % NS;
        const uint32_t st = smem_u32(stage(s));
        const uint32_t qh = st + (uint32_t)S::sQ, ql = st + (uint32_t)S::sQl, oh = st + (uint32_t)S::sO,
                       ol = st + (uint32_t)S::sOl;
        const Op ph{smem_u32(sPh), KT, false}, pl{smem_u32(sPl), KT, false};
        const Op gh{smem_u32(sDh), KT, false}, gl{smem_u32(sDl), KT, false};
        for (int s2 = 0; s2 < QT / 16; ++s2) {
          const uint32_t acc = (jp > 0 || s2) ? 1u : 0u;
          mma_bf16(tb + cDV, op_desc(ph, s2), sw_desc_mn(oh, QT, s2), id_dv, acc);
          mma_bf16(tb + cDV, op_desc(pl, s2), sw_desc_mn(oh, QT, s2), id_dv, 1u);
          if constexpr (SPLIT) mma_bf16(tb + cDV, op_desc(ph, s2), sw_desc_mn(ol, QT, s2), id_dv, 1u);
          mma_bf16(tb + cDK, op_desc(gh, s2), sw_desc_mn(qh, QT, s2), id_dk, acc);
          mma_bf16(tb + cDK, op_desc(gl, s2), sw_desc_mn(qh, QT, s2), id_dk, 1u);
          if constexpr (SPLIT) mma_bf16(tb + cDK, op_desc(gh, s2), sw_desc_mn(ql, QT, s2), id_dk, 1u);
        }
        commit(&p_empty);   // P^T, dS^T may be overwritten
        commit(&empty[s]);  // the stage may be refilled
      };
      int jS = 0, jD = 0;
      uint64_t t_last = globaltimer();
      while (ok && jD < n_tiles) {
        if (aborted()) break;
        bool issued = false;
        if (jD < jS && mbar_try_wait(&p_full, jD & 1)) {
          fence_after_sync();
          issue_d(jD++);
          issued = true;
        } else if (jS < n_tiles && mbar_try_wait(&full[jS % NS], (jS / NS) & 1) &&
                   (jS == 0 || mbar_try_wait(&s_read, (jS - 1) & 1))) {
          fence_after_sync();
          issue_s(jS++);
          issued = true;
        }
        if (issued) {
          t_last = globaltimer();
        } else if (globaltimer() - t_last > 1000000000ull) {  // nothing became ready for a second
          give_up();
          ok = false;
        }
      }
      commit(&done_bar);  // arrives once every MMA issued above has completed
      if (!mbar_wait(&done_bar, 0, 2000000000ull)) give_up();
    }
  } else if (w <= 2) {  // ------------------------------------------------ loads
    // warp 1 (one thread): TMA of K (with the first query tile) and of each query tile's Q, dO;
    // warp 2: lse and delta of the tile (rows past the subtree are masked, past the tensor zero)
    const bool tma = w == 1;
    if (!tma || lane == 0) {
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(&empty[s], ((j / NS) - 1) & 1)) {
          give_up();
          break;
        }
        if (aborted()) break;
        const int q0 = k0 + j * QT, nq = min(QT, q_end - q0);
        uint8_t* st = stage(s);
        if (tma) {
          const uint32_t kb = j == 0 ? (uint32_t)(SPLIT ? 2 : 1) * (uint32_t)S::Kb : 0u;
          mbar_arrive_expect_tx(&full[s], kb + (uint32_t)(SPLIT ? 2 : 1) * (uint32_t)(S::Qb + S::Ob));
          if (j == 0) {
            for (int c = 0; c < DQ / 64; ++c) {
              tma_load_3d(sK + c * KT * 128, &tm_k, 64 * c, h, k0, &full[s]);
              if constexpr (SPLIT) tma_load_3d(sKl + c * KT * 128, &tm_kl, 64 * c, h, k0, &full[s]);
            }
          }
          for (int c = 0; c < DQ / 64; ++c) {
            tma_load_3d(st + S::sQ + c * QT * 128, &tm_q, 64 * c, h, q0, &full[s]);
            if constexpr (SPLIT) tma_load_3d(st + S::sQl + c * QT * 128, &tm_ql, 64 * c, h, q0, &full[s]);
          }
          for (int c = 0; c < DV / 64; ++c) {
            tma_load_3d(st + S::sO + c * QT * 128, &tm_o, 64 * c, h, q0, &full[s]);
            if constexpr (SPLIT) tma_load_3d(st + S::sOl + c * QT * 128, &tm_ol, 64 * c, h, q0, &full[s]);
          }
        } else {
          const size_t src = (size_t)(q0 + min(lane, nq - 1)) * H + h;
          cp_async4(st + S::sL + 4 * lane, lse + src, lane < nq ? 4u : 0u);
          cp_async4(st + S::sD + 4 * lane, delta + src, lane < nq ? 4u : 0u);
          cp_async_commit();
          cp_async_wait<0>();
          mbar_arrive(&full[s]);
        }
      }
      if (!tma) cp_async_wait<0>();
    }
  } else if (w >= 3) {  // ------------------------------------------------ P^T, dS^T (warps 3-10)
    // warp w holds the TMEM lanes (key rows) of sub-partition w % 4 and the query columns of half
    // (w - 3) / 4 of each tile (and of dV / dK at the end)
    const int sp = w & 3, half = (w - 3) >> 2, r = 32 * sp + lane;
    const bool in = r < nk;
    const uint32_t la = tb + ((uint32_t)(32 * sp) << 16);
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar, parity));
      if (!got && lane == 0) give_up();
      return got && !__any_sync(0xffffffffu, aborted());
    };
    {  // this half of the key row's V (and its lo part) into TMEM: a bf16 pair per 32-bit column
      for (int part = 0; part < (SPLIT ? 2 : 1); ++part) {
        const bf* src = part ? v_lo : v;
        const uint4* g4 =
            (in && src) ? reinterpret_cast<const uint4*>(src + ((size_t)(k0 + r) * H + h) * DV) + 8 * half : nullptr;
        uint32_t rr[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 x = g4 ? g4[i] : make_uint4(0u, 0u, 0u, 0u);
          rr[4 * i] = x.x; rr[4 * i + 1] = x.y; rr[4 * i + 2] = x.z; rr[4 * i + 3] = x.w;
        }
        tmem_st32_nowait(la + (part ? cVl : cVh) + 32 * half, rr);
      }
      tmem_wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_ready);
    }
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % NS;
      if (!(ok = wait_all(&s_full, j & 1))) break;
      fence_after_sync();
      uint32_t rs[16], rp[16];
      {
        float a[16], b[16];
        tmem_ld16(la + cS + 16 * half, a);
        tmem_ld16(la + cP + 16 * half, b);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          rs[c] = __float_as_uint(a[c]);
          rp[c] = __float_as_uint(b[c]);
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_read);  // S^T, dP^T may take the next tile
      if (!(ok = wait_all(&full[s], (j / NS) & 1))) break;  // lse and delta of the tile
      const uint8_t* st = stage(s);
      const float* sl = reinterpret_cast<const float*>(st + S::sL);
      const float* sd = reinterpret_cast<const float*>(st + S::sD);
      const int q0 = k0 + j * QT, nq = min(QT, q_end - q0);
      // P^T and dS^T of this thread's 16 entries as packed bf16 hi / lo pairs (base-2 exponentials)
      uint32_t ph[8], pl[8], gh[8], gl[8];
#pragma unroll
      for (int jj = 0; jj < 16; jj += 2) {
        float pv[2], dsv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 16 * half + jj + e, qrow = q0 + c;
          const bool valid = in && c < nq && !(qrow < own_end && qrow < k0 + r);
          pv[e] = valid ? exp2f(fmaf(__uint_as_float(rs[jj + e]), sl2, -sl[c] * kLog2e)) : 0.f;
          dsv[e] = pv[e] * (__uint_as_float(rp[jj + e]) - sd[c]);
        }
        split2(pv[0], pv[1], ph[jj / 2], pl[jj / 2]);
        split2(dsv[0], dsv[1], gh[jj / 2], gl[jj / 2]);
      }
      if (j >= 1 && !(ok = wait_all(&p_empty, (j - 1) & 1))) break;  // dV, dK of tile j - 1 are done
      put16_packed<KT>(sPh, sPl, r, 16 * half, ph, pl);
      put16_packed<KT>(sDh, sDl, r, 16 * half, gh, gl);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && n_tiles > 0) ok = wait_all(&p_empty, (n_tiles - 1) & 1);
    if (ok) {
      fence_after_sync();
      const bool none = n_tiles == 0;
      for (int c = DV / 2 * half; c < DV / 2 * (half + 1); c += 32) {
        float g[32];
        tmem_ld32(la + cDV + c, g);
        if (in) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) g[jj] = none ? 0.f : g[jj];
          Tio* dst = dv + ((size_t)(k0 + r) * H + h) * DV + c;
          st_out16(dst, g);
          st_out16(dst + 16, g + 16);
        }
      }
      for (int c = DQ / 2 * half; c < DQ / 2 * (half + 1); c += 32) {
        float g[32];
        tmem_ld32(la + cDK + c, g);
        if (in) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) g[jj] = none ? 0.f : g[jj] * scale;
          Tio* dst = dk + ((size_t)(k0 + r) * H + h) * DQ + c;
          st_out16(dst, g);
          st_out16(dst + 16, g + 16);
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (w == 0) tmem_dealloc(tb, 512);
}

}  // namespace tpc
