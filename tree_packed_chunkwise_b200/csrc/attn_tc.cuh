// Tree-masked softmax attention on tcgen05 (HARTS Figure 1(b): full attention reads ancestor keys
// and values; Figure C.1(c): within a segment the diagonal blocks are causal, a later segment reads
// its ancestors and never the reverse; outputs return to compact rows).
//
// A query tile (<= 128 rows of one node) visits the node's ancestor row ranges (a few contiguous
// ranges in the compact layout, one per chain on its path) and then its own node's rows up to the
// tile's end with the causal mask.  Forward: S = Q K^T (bf16 inputs, exact products), online
// softmax in fp32 (one query row per thread), O += P V with P a bf16 hi/lo pair.  Backward,
// deterministic: dQ per query tile (S and dP = dO V^T recomputed, dQ += dS K accumulated in TMEM);
// dK, dV per key tile (<= 64 rows of one node), looping over the query rows that can see it: the
// node's subtree rows from the tile on, one contiguous range in the compact layout.
//
// SPLIT kernels take q, k, v and dO as bf16 hi/lo pairs (fp32 values x = hi + lo to 2^-17
// relative) and form every product from three partial products (hi hi + lo hi + hi lo), so that
// fp32 inputs and upstream gradients enter without a bf16 rounding of their own.  The dQ kernel
// then walks the keys in tiles of 32 (the split tiles take twice the shared memory).
#pragma once
#include "kda_tc.cuh"

namespace tpc {

constexpr int kAttnQK = 192, kAttnDV = 128, kAttnThreads = 128;

namespace tck {

// key tiles of a query tile: f(row start, rows, own-node flag) in a fixed order; stops on false
template <int KT = 64, class F>
__device__ __forceinline__ bool for_key_tiles(const DevTables& t, const AttnTile& qt, F f) {
  const AttnNode nd = t.attn_nodes[qt.node];
  const int r1 = t.attn_nodes[qt.node + 1].range_begin;
  for (int r = nd.range_begin; r < r1; ++r) {
    const RowRange rr = t.attn_ranges[r];
    for (int k0 = rr.start; k0 < rr.end; k0 += KT)
      if (!f(k0, min(KT, rr.end - k0), false)) return false;
  }
  const int end = qt.row + qt.n;
  for (int k0 = nd.row_offset; k0 < end; k0 += KT)
    if (!f(k0, min(KT, end - k0), true)) return false;
  return true;
}

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

}  // namespace tck

// ------------------------------------------------------------------------------------------ forward
// Key tiles of a query tile, one at a time in the fixed order of for_key_tiles (for look-ahead).
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

// Asynchronous load of an A x B bf16 tile (rows from rowp(a), nullptr = zeros) into the
// core-matrix layout; `any` is a valid global address used for the zero-filled rows.
template <int A, int B, int NT, class RP>
__device__ __forceinline__ void tile_async(uint8_t* dst, RP rowp, const void* any) {
  constexpr int NCH = A * (B / 8);
#pragma unroll 4
  for (int e = threadIdx.x; e < NCH; e += NT) {
    const int a = e % A, b0 = (e / A) * 8;
    const __nv_bfloat16* p = rowp(a);
    tc::cp_async16(dst + tc::cm_off(a, b0, A), p ? (const void*)(p + b0) : any, p ? 16u : 0u);
  }
}

template <bool SPLIT>
struct AttnFwdSmem {
  static constexpr size_t Qb = size_t(128) * kAttnQK * 2, Kb = size_t(64) * kAttnQK * 2, Vb = size_t(64) * kAttnDV * 2;
  static constexpr size_t Pb = size_t(128) * 64 * 2, X = SPLIT ? 1 : 0;
  static constexpr size_t Q = 0, Ql = Q + Qb, K = Ql + X * Qb, Kl = K + Kb, V = Kl + X * Kb, Vl = V + Vb;
  static constexpr size_t P = Vl + X * Vb;
  static constexpr size_t total = P + 2 * Pb;
  static_assert(total <= 227 * 1024, "shared memory");
};

// Per query tile: O accumulates in TMEM across the key tiles (P V products with accumulate), the
// online softmax keeps a per-row reference maximum that is raised (and O, l rescaled) only when a
// tile's maximum exceeds it by more than 8, so every p = exp(s - m) stays below e^8.  The next key
// tile's K and V are fetched with cp.async while the current tile's softmax and P V run.  Eight
// warps: warp w holds the TMEM lanes (query rows) of sub-partition w % 4 and the column half
// w / 4 (S columns 32 h .. 32 h + 31, O columns 64 h .. 64 h + 63); the two threads of a row combine
// their partial maxima and sums through shared memory, in a fixed order.
constexpr int kAttnFwdThreads = 256;

template <typename Tout, bool SPLIT>
__global__ void __launch_bounds__(kAttnFwdThreads, 1)
    attn_fwd_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ q,
                const __nv_bfloat16* __restrict__ q_lo, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ k_lo, const __nv_bfloat16* __restrict__ v,
                const __nv_bfloat16* __restrict__ v_lo, Tout* __restrict__ o, float* __restrict__ lse,
                int* status) {
  using namespace tck;
  using S = AttnFwdSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, NT = kAttnFwdThreads;
  constexpr float kRaise = 8.f;
  const AttnTile qt = t.attn_qtiles[blockIdx.x];
  const int h = blockIdx.y, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int row = 32 * (w & 3) + lane, half = w >> 2;
  extern __shared__ __align__(1024) uint8_t asmem[];
  uint8_t *sQ = asmem + S::Q, *sQl = asmem + S::Ql, *sK = asmem + S::K, *sKl = asmem + S::Kl, *sV = asmem + S::V,
          *sVl = asmem + S::Vl, *sPh = asmem + S::P, *sPl = sPh + S::Pb;
  __shared__ float red_max[2][128], red_sum[2][128];
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  if (w == 0) tc::tmem_alloc(&tslot, 256);
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  auto qrows = [&](const bf* base) {
    return [=](int a) -> const bf* { return a < qt.n && base ? base + ((size_t)(qt.row + a) * H + h) * DQ : nullptr; };
  };
  auto load_kv = [&](bool is_k, int k0, int nk) {
    if (is_k) {
      tile_async<64, DQ, NT>(sK, [=](int a) -> const bf* { return a < nk ? k + ((size_t)(k0 + a) * H + h) * DQ : nullptr; }, k);
      if constexpr (SPLIT)
        tile_async<64, DQ, NT>(
            sKl, [=](int a) -> const bf* { return a < nk && k_lo ? k_lo + ((size_t)(k0 + a) * H + h) * DQ : nullptr; }, k);
    } else {
      tile_async<64, DV, NT>(sV, [=](int a) -> const bf* { return a < nk ? v + ((size_t)(k0 + a) * H + h) * DV : nullptr; }, v);
      if constexpr (SPLIT)
        tile_async<64, DV, NT>(
            sVl, [=](int a) -> const bf* { return a < nk && v_lo ? v_lo + ((size_t)(k0 + a) * H + h) * DV : nullptr; }, v);
    }
  };
  KeyTileIter<64> it;
  it.init(t, qt);
  int k0 = 0, nk = 0;
  bool own = false;
  bool have = it.next(k0, nk, own);
  tile_async<128, DQ, NT>(sQ, qrows(q), q);
  if constexpr (SPLIT) tile_async<128, DQ, NT>(sQl, qrows(q_lo), q);
  if (have) load_kv(true, k0, nk);
  tc::cp_async_commit();  // group: Q, K_0
  if (have) load_kv(false, k0, nk);
  tc::cp_async_commit();  // group: V_0
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  const uint32_t la = tb + ((uint32_t)(32 * (w & 3)) << 16);
  Sync sy{&bar, 0u, status};
  const int qrow = qt.row + row;
  float m_ref = -INFINITY, l = 0.f;
  bool first = true, ok = true;
  while (have) {
    int k1 = 0, n1 = 0;
    bool own1 = false;
    const bool more = it.next(k1, n1, own1);
    tc::cp_async_wait<1>();  // Q and this tile's K have arrived
    ok = run(sy, [&] {
      mma4(tb, tc::Op{tc::smem_u32(sQ), 128, false}, tc::Op{tc::smem_u32(sQl), 128, false},
           tc::Op{tc::smem_u32(sK), 64, false}, tc::Op{tc::smem_u32(sKl), 64, false}, DQ,
           tc::idesc_bf16(128, 64, false, false), false, !SPLIT, !SPLIT);
    });
    if (!ok) break;
    if (more) load_kv(true, k1, n1);  // K is free once S is in TMEM
    tc::cp_async_commit();
    float s[32];
    tc::tmem_ld32(la + 32 * half, s);
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int c = 32 * half + j;
      const bool valid = row < qt.n && c < nk && (!own || k0 + c <= qrow);
      s[j] = valid ? s[j] * scale : -INFINITY;
      mx = fmaxf(mx, s[j]);
    }
    red_max[half][row] = mx;
    __syncthreads();
    mx = fmaxf(red_max[0][row], red_max[1][row]);
    // raise the reference where the tile's maximum exceeds it by more than kRaise; O (accumulated so
    // far) and l follow.  Both threads of a row take the same decision; TMEM loads and stores are
    // warp-collective, so a warp rescales its 32 rows together when any of them raised.
    const bool raise = mx > m_ref + kRaise;
    const float corr = !raise ? 1.f : (m_ref == -INFINITY ? 0.f : expf(m_ref - mx));
    if (raise) {
      l *= corr;
      m_ref = mx;
    }
    if (!first && __any_sync(0xffffffffu, raise)) {
      for (int c = 0; c < DV / 2; c += 16) {
        float ov[16];
        tc::tmem_ld16(la + 64 + DV / 2 * half + c, ov);
#pragma unroll
        for (int j = 0; j < 16; ++j) ov[j] *= corr;
        tc::tmem_st16(la + 64 + DV / 2 * half + c, ov);
      }
    }
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      s[j] = s[j] == -INFINITY ? 0.f : expf(s[j] - m_ref);
      psum += s[j];
    }
    red_sum[half][row] = psum;
#pragma unroll
    for (int j = 0; j < 32; j += 16) put16<128, true>(sPh, sPl, row, 32 * half + j, s + j);
    __syncthreads();
    l += red_sum[0][row] + red_sum[1][row];
    tc::cp_async_wait<1>();  // this tile's V has arrived
    const bool acc_on = !first;
    ok = run(sy, [&] {
      mma4(tb + 64, tc::Op{tc::smem_u32(sPh), 128, false}, tc::Op{tc::smem_u32(sPl), 128, false},
           tc::Op{tc::smem_u32(sV), 64, true}, tc::Op{tc::smem_u32(sVl), 64, true}, 64,
           tc::idesc_bf16(128, DV, false, true), acc_on, false, !SPLIT);
    });
    if (!ok) break;
    if (more) load_kv(false, k1, n1);  // V is free once P V is done
    tc::cp_async_commit();
    first = false;
    k0 = k1; nk = n1; own = own1; have = more;
  }
  tc::cp_async_wait<0>();
  if (ok) {
    const float inv = 1.f / l;
    Tout* dst = o + ((size_t)qrow * H + h) * DV + DV / 2 * half;
    for (int c = 0; c < DV / 2; c += 16) {
      float ov[16];
      tc::tmem_ld16(la + 64 + DV / 2 * half + c, ov);  // warp-collective: every row takes part
      if (row < qt.n) {
#pragma unroll
        for (int j = 0; j < 16; ++j) ov[j] *= inv;
        st_out16(dst + c, ov);
      }
    }
    if (row < qt.n && half == 0) lse[(size_t)qrow * H + h] = m_ref + logf(l);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (w == 0) tc::tmem_dealloc(tb, 256);
}

// ------------------------------------------------------------------------------------------ backward dQ
// per query tile: delta = rowsum(dO * O) (also written for the dK/dV kernel), then over the key
// tiles P = exp(scale S - lse), dP = dO V^T, dS = P (dP - delta), dQ += dS K; dq = scale dQ.
template <bool SPLIT>
struct AttnDqSmem {
  static constexpr int KT = SPLIT ? 32 : 64;  // key rows per tile
  static constexpr size_t X = SPLIT ? 1 : 0;
  static constexpr size_t Qb = size_t(128) * kAttnQK * 2, Ob = size_t(128) * kAttnDV * 2;
  static constexpr size_t Kb = size_t(KT) * kAttnQK * 2, Vb = size_t(KT) * kAttnDV * 2, Pb = size_t(128) * KT * 2;
  static constexpr size_t Q = 0, Ql = Q + Qb, dO = Ql + X * Qb, dOl = dO + Ob, K = dOl + X * Ob, Kl = K + Kb;
  static constexpr size_t V = Kl + X * Kb, Vl = V + Vb, dS = Vl + X * Vb;
  static constexpr size_t total = dS + 2 * Pb;
  static_assert(total <= 227 * 1024, "shared memory");
};

// Eight warps: warp w holds the query rows of TMEM sub-partition w % 4 and the column half w / 4 of
// each key tile (and of dQ at the end).
constexpr int kAttnDqThreads = 256;

template <typename Tio, bool SPLIT>
__global__ void __launch_bounds__(kAttnDqThreads, 1)
    attn_bwd_dq_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ q_lo, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ k_lo, const __nv_bfloat16* __restrict__ v,
                   const __nv_bfloat16* __restrict__ v_lo, const Tio* __restrict__ o, const float* __restrict__ lse,
                   const __nv_bfloat16* __restrict__ d_o, const __nv_bfloat16* __restrict__ d_o_lo,
                   Tio* __restrict__ dq, float* __restrict__ delta, int* status) {
  using namespace tck;
  using S = AttnDqSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, NT = kAttnDqThreads, KT = S::KT, KH = KT / 2;
  const AttnTile qt = t.attn_qtiles[blockIdx.x];
  const int h = blockIdx.y, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int row = 32 * (w & 3) + lane, half = w >> 2;
  extern __shared__ __align__(1024) uint8_t asmem[];
  uint8_t *sQ = asmem + S::Q, *sQl = asmem + S::Ql, *sO = asmem + S::dO, *sOl = asmem + S::dOl, *sK = asmem + S::K,
          *sKl = asmem + S::Kl, *sV = asmem + S::V, *sVl = asmem + S::Vl, *sDh = asmem + S::dS, *sDl = sDh + S::Pb;
  __shared__ float s_dl[128], s_ls[128];
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  if (w == 0) tc::tmem_alloc(&tslot, 512);
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  auto ident = [](int, int, float x) { return x; };
  auto qrows = [&](const bf* base) {
    return [=](int a) -> const bf* { return a < qt.n && base ? base + ((size_t)(qt.row + a) * H + h) * DQ : nullptr; };
  };
  auto orows = [&](const bf* base) {
    return [=](int a) -> const bf* { return a < qt.n && base ? base + ((size_t)(qt.row + a) * H + h) * DV : nullptr; };
  };
  build_tile_ld<128, DQ, false, bf, NT>(sQ, nullptr, qrows(q), ident);
  build_tile_ld<128, DV, false, bf, NT>(sO, nullptr, orows(d_o), ident);
  if constexpr (SPLIT) {
    build_tile_ld<128, DQ, false, bf, NT>(sQl, nullptr, qrows(q_lo), ident);
    build_tile_ld<128, DV, false, bf, NT>(sOl, nullptr, orows(d_o_lo), ident);
  }
  const int qrow = qt.row + row;
  if (half == 0) {
    float dl = 0.f, ls = 0.f;
    if (row < qt.n) {
      const Tio* orow = o + ((size_t)qrow * H + h) * DV;
      const bf* grow = d_o + ((size_t)qrow * H + h) * DV;
      const bf* glow = SPLIT && d_o_lo ? d_o_lo + ((size_t)qrow * H + h) * DV : nullptr;
      for (int j = 0; j < DV; ++j)
        dl = fmaf(to_f(orow[j]), __bfloat162float(grow[j]) + (glow ? __bfloat162float(glow[j]) : 0.f), dl);
      delta[(size_t)qrow * H + h] = dl;
      ls = lse[(size_t)qrow * H + h];
    }
    s_dl[row] = dl;
    s_ls[row] = ls;
  }
  __syncthreads();
  const float dl = s_dl[row], ls = s_ls[row];
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  const uint32_t la = tb + ((uint32_t)(32 * (w & 3)) << 16);
  Sync sy{&bar, 0u, status};
  // key tiles with one tile of look-ahead: V of the next tile is fetched by cp.async while this tile's
  // dS and dQ products run, K of the next tile once this tile's dQ product has read K
  auto load_k = [&](int k0, int nk) {
    auto rows = [=](const bf* base) {
      return [=](int a) -> const bf* { return a < nk && base ? base + ((size_t)(k0 + a) * H + h) * DQ : nullptr; };
    };
    tile_async<KT, DQ, NT>(sK, rows(k), k);
    if constexpr (SPLIT) tile_async<KT, DQ, NT>(sKl, rows(k_lo), k);
  };
  auto load_v = [&](int k0, int nk) {
    auto rows = [=](const bf* base) {
      return [=](int a) -> const bf* { return a < nk && base ? base + ((size_t)(k0 + a) * H + h) * DV : nullptr; };
    };
    tile_async<KT, DV, NT>(sV, rows(v), v);
    if constexpr (SPLIT) tile_async<KT, DV, NT>(sVl, rows(v_lo), v);
  };
  KeyTileIter<KT> it;
  it.init(t, qt);
  int k0 = 0, nk = 0;
  bool own = false;
  bool have = it.next(k0, nk, own);
  if (have) {
    load_k(k0, nk);
    load_v(k0, nk);
  }
  tc::cp_async_commit();
  bool first = true, ok = true;
  while (have) {
    int k1 = 0, n1 = 0;
    bool own1 = false;
    const bool more = it.next(k1, n1, own1);
    tc::cp_async_wait<0>();  // this tile's K and V have arrived
    ok = run(sy, [&] {
      mma4(tb, tc::Op{tc::smem_u32(sQ), 128, false}, tc::Op{tc::smem_u32(sQl), 128, false},
           tc::Op{tc::smem_u32(sK), KT, false}, tc::Op{tc::smem_u32(sKl), KT, false}, DQ,
           tc::idesc_bf16(128, KT, false, false), false, !SPLIT, !SPLIT);
      mma4(tb + 64, tc::Op{tc::smem_u32(sO), 128, false}, tc::Op{tc::smem_u32(sOl), 128, false},
           tc::Op{tc::smem_u32(sV), KT, false}, tc::Op{tc::smem_u32(sVl), KT, false}, DV,
           tc::idesc_bf16(128, KT, false, false), false, !SPLIT, !SPLIT);
    });
    if (!ok) break;
    if (more) load_v(k1, n1);  // V is free once dP is in TMEM
    tc::cp_async_commit();
    float s[KH], dp[KH];
#pragma unroll
    for (int c = 0; c < KH; c += 16) {
      tc::tmem_ld16(la + KH * half + c, *reinterpret_cast<float(*)[16]>(s + c));
      tc::tmem_ld16(la + 64 + KH * half + c, *reinterpret_cast<float(*)[16]>(dp + c));
    }
#pragma unroll
    for (int j = 0; j < KH; ++j) {
      const int c = KH * half + j;
      const bool valid = row < qt.n && c < nk && (!own || k0 + c <= qrow);
      const float p = valid ? expf(s[j] * scale - ls) : 0.f;
      s[j] = p * (dp[j] - dl);
    }
#pragma unroll
    for (int j = 0; j < KH; j += 16) put16<128, true>(sDh, sDl, row, KH * half + j, s + j);
    const bool acc_on = !first;
    first = false;
    ok = run(sy, [&] {
      mma4(tb + 128, tc::Op{tc::smem_u32(sDh), 128, false}, tc::Op{tc::smem_u32(sDl), 128, false},
           tc::Op{tc::smem_u32(sK), KT, true}, tc::Op{tc::smem_u32(sKl), KT, true}, KT,
           tc::idesc_bf16(128, DQ, false, true), acc_on, false, !SPLIT);
    });
    if (!ok) break;
    if (more) load_k(k1, n1);  // K is free once dQ has read it
    tc::cp_async_commit();
    k0 = k1; nk = n1; own = own1; have = more;
  }
  tc::cp_async_wait<0>();
  if (ok) {
    for (int c = 0; c < DQ / 2; c += 32) {
      float g[32];
      tc::tmem_ld32(la + 128 + DQ / 2 * half + c, g);
      if (row < qt.n) {
#pragma unroll
        for (int j = 0; j < 32; ++j) g[j] *= scale;
        Tio* dst = dq + ((size_t)qrow * H + h) * DQ + DQ / 2 * half + c;
        st_out16(dst, g);
        st_out16(dst + 16, g + 16);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (w == 0) tc::tmem_dealloc(tb, 512);
}

// ------------------------------------------------------------------------------------------ backward dK, dV
// per key tile of node u: query rows [row of the tile, subtree end of u) in tiles of 32 (queries of u
// itself only from the key row on), S^T = K Q^T, dP^T = V dO^T, P^T = exp(scale S^T - lse),
// dS^T = P^T (dP^T - delta); dV += P^T dO, dK += dS^T Q; dk = scale dK.  M = 64 accumulators.
// Q and dO tiles are double-buffered: the next query tile is fetched with cp.async while the current
// one's P, dS and the dV / dK products run.
template <bool SPLIT>
struct AttnDkvSmem {
  static constexpr int QT = 32;  // query rows per tile
  static constexpr size_t X = SPLIT ? 1 : 0;
  static constexpr size_t Kb = size_t(64) * kAttnQK * 2, Vb = size_t(64) * kAttnDV * 2;
  static constexpr size_t Qb = size_t(QT) * kAttnQK * 2, Ob = size_t(QT) * kAttnDV * 2, Pb = size_t(64) * QT * 2;
  static constexpr size_t QO = (1 + X) * (Qb + Ob);  // one query buffer: Q (+lo), dO (+lo)
  static constexpr size_t K = 0, Kl = K + Kb, V = Kl + X * Kb, Vl = V + Vb, Qbuf = Vl + X * Vb;
  static constexpr size_t P = Qbuf + 2 * QO, dS = P + 2 * Pb;
  static constexpr size_t vec = dS + 2 * Pb;  // lse[QT], delta[QT] per buffer
  static constexpr size_t total = vec + 2 * 2 * QT * 4;
  static_assert(total <= 227 * 1024, "shared memory");
};

// Eight warps: warps w and w + 4 share the key rows of TMEM sub-partition w % 4 (M = 64 layout:
// lanes 0..15) and split the columns of every query tile and of dV / dK at the end.
constexpr int kAttnDkvThreads = 256;

template <typename Tio, bool SPLIT>
__global__ void __launch_bounds__(kAttnDkvThreads, 1)
    attn_bwd_dkv_tc(DevTables t, int H, float scale, const __nv_bfloat16* __restrict__ q,
                    const __nv_bfloat16* __restrict__ q_lo, const __nv_bfloat16* __restrict__ k,
                    const __nv_bfloat16* __restrict__ k_lo, const __nv_bfloat16* __restrict__ v,
                    const __nv_bfloat16* __restrict__ v_lo, const float* __restrict__ lse,
                    const __nv_bfloat16* __restrict__ d_o, const __nv_bfloat16* __restrict__ d_o_lo,
                    const float* __restrict__ delta, Tio* __restrict__ dk, Tio* __restrict__ dv, int* status) {
  using namespace tck;
  using S = AttnDkvSmem<SPLIT>;
  using bf = __nv_bfloat16;
  constexpr int DQ = kAttnQK, DV = kAttnDV, NT = kAttnDkvThreads, QT = S::QT, QH = QT / 2;
  const AttnTile kt = t.attn_ktiles[blockIdx.x];
  const AttnNode nd = t.attn_nodes[kt.node];
  const int h = blockIdx.y, tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t asmem[];
  uint8_t *sK = asmem + S::K, *sKl = asmem + S::Kl, *sV = asmem + S::V, *sVl = asmem + S::Vl;
  uint8_t *sPh = asmem + S::P, *sPl = sPh + S::Pb, *sDh = asmem + S::dS, *sDl = sDh + S::Pb;
  float* svec = reinterpret_cast<float*>(asmem + S::vec);  // [buffer][lse QT | delta QT]
  // query buffer b: Q, Q_lo, dO, dO_lo
  auto qbuf = [&](int b, int part) -> uint8_t* {
    uint8_t* base = asmem + S::Qbuf + (size_t)b * S::QO;
    return part == 0 ? base : part == 1 ? base + S::Qb : part == 2 ? base + (1 + S::X) * S::Qb
                                                                   : base + (1 + S::X) * S::Qb + S::Ob;
  };
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  if (w == 0) tc::tmem_alloc(&tslot, 512);
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int k0 = kt.row, nk = kt.n;
  auto krows = [&](const bf* base, int width) {
    return [=](int a) -> const bf* { return a < nk && base ? base + ((size_t)(k0 + a) * H + h) * width : nullptr; };
  };
  tile_async<64, DQ, NT>(sK, krows(k, DQ), k);
  tile_async<64, DV, NT>(sV, krows(v, DV), v);
  if constexpr (SPLIT) {
    tile_async<64, DQ, NT>(sKl, krows(k_lo, DQ), k);
    tile_async<64, DV, NT>(sVl, krows(v_lo, DV), v);
  }
  const int own_end = nd.row_offset + nd.length, q_end = nd.subtree_end;
  // query tile at row q0 into buffer b (rows past q_end are zero)
  auto load_q = [&](int b, int q0) {
    const int nq = min(QT, q_end - q0);
    auto rows = [=](const bf* base, int width) {
      return [=](int a) -> const bf* { return a < nq && base ? base + ((size_t)(q0 + a) * H + h) * width : nullptr; };
    };
    tile_async<QT, DQ, NT>(qbuf(b, 0), rows(q, DQ), q);
    tile_async<QT, DV, NT>(qbuf(b, 2), rows(d_o, DV), d_o);
    if constexpr (SPLIT) {
      tile_async<QT, DQ, NT>(qbuf(b, 1), rows(q_lo, DQ), q);
      tile_async<QT, DV, NT>(qbuf(b, 3), rows(d_o_lo, DV), d_o);
    }
  };
  if (k0 < q_end) load_q(0, k0);
  tc::cp_async_commit();  // group: K, V, query tile 0
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tb = tslot;
  const uint32_t la = tb + ((uint32_t)(32 * (w & 3)) << 16);
  const int r = lane < 16 ? 16 * (w & 3) + lane : -1;  // key row of this thread (M = 64 layout)
  const int half = w >> 2;                                // column half of this warp
  Sync sy{&bar, 0u, status};
  bool ok = true, first = true;
  int b = 0;
  for (int q0 = k0; q0 < q_end && ok; q0 += QT, b ^= 1) {
    const int nq = min(QT, q_end - q0);
    const bool more = q0 + QT < q_end;
    tc::cp_async_wait<0>();  // this query tile (and, the first time, K and V) have arrived
    float* sl = svec + b * 2 * QT;
    float* sd = sl + QT;
    if (tid < QT) {
      sl[tid] = tid < nq ? lse[(size_t)(q0 + tid) * H + h] : 0.f;
      sd[tid] = tid < nq ? delta[(size_t)(q0 + tid) * H + h] : 0.f;
    }
    uint8_t *sQ = qbuf(b, 0), *sQl = qbuf(b, 1), *sO = qbuf(b, 2), *sOl = qbuf(b, 3);
    ok = run(sy, [&] {
      mma4(tb, tc::Op{tc::smem_u32(sK), 64, false}, tc::Op{tc::smem_u32(sKl), 64, false},
           tc::Op{tc::smem_u32(sQ), QT, false}, tc::Op{tc::smem_u32(sQl), QT, false}, DQ,
           tc::idesc_bf16(64, QT, false, false), false, !SPLIT, !SPLIT);
      mma4(tb + 64, tc::Op{tc::smem_u32(sV), 64, false}, tc::Op{tc::smem_u32(sVl), 64, false},
           tc::Op{tc::smem_u32(sO), QT, false}, tc::Op{tc::smem_u32(sOl), QT, false}, DV,
           tc::idesc_bf16(64, QT, false, false), false, !SPLIT, !SPLIT);
    });
    if (!ok) break;
    // the other buffer was last read by the previous tile's dV / dK products, which have completed
    if (more) load_q(b ^ 1, q0 + QT);
    tc::cp_async_commit();
    float s[QH], dp[QH];
    tc::tmem_ld16(la + QH * half, *reinterpret_cast<float(*)[16]>(s));
    tc::tmem_ld16(la + 64 + QH * half, *reinterpret_cast<float(*)[16]>(dp));
    if (r >= 0) {
#pragma unroll
      for (int j = 0; j < QH; ++j) {
        const int c = QH * half + j, qrow = q0 + c;
        const bool valid = r < nk && c < nq && !(qrow < own_end && qrow < k0 + r);
        const float p = valid ? expf(s[j] * scale - sl[c]) : 0.f;
        s[j] = p;
        dp[j] = p * (dp[j] - sd[c]);
      }
      put16<64, true>(sPh, sPl, r, QH * half, s);
      put16<64, true>(sDh, sDl, r, QH * half, dp);
    }
    const bool acc_on = !first;
    first = false;
    ok = run(sy, [&] {
      mma4(tb + 128, tc::Op{tc::smem_u32(sPh), 64, false}, tc::Op{tc::smem_u32(sPl), 64, false},
           tc::Op{tc::smem_u32(sO), QT, true}, tc::Op{tc::smem_u32(sOl), QT, true}, QT,
           tc::idesc_bf16(64, DV, false, true), acc_on, false, !SPLIT);
      mma4(tb + 256, tc::Op{tc::smem_u32(sDh), 64, false}, tc::Op{tc::smem_u32(sDl), 64, false},
           tc::Op{tc::smem_u32(sQ), QT, true}, tc::Op{tc::smem_u32(sQl), QT, true}, QT,
           tc::idesc_bf16(64, DQ, false, true), acc_on, false, !SPLIT);
    });
  }
  tc::cp_async_wait<0>();
  if (ok) {
    for (int c = DV / 2 * half; c < DV / 2 * (half + 1); c += 32) {
      float g[32];
      tc::tmem_ld32(la + 128 + c, g);
      if (r >= 0 && r < nk) {
        Tio* dst = dv + ((size_t)(k0 + r) * H + h) * DV + c;
        if (first) {
#pragma unroll
          for (int j = 0; j < 32; ++j) g[j] = 0.f;
        }
        st_out16(dst, g);
        st_out16(dst + 16, g + 16);
      }
    }
    for (int c = DQ / 2 * half; c < DQ / 2 * (half + 1); c += 32) {
      float g[32];
      tc::tmem_ld32(la + 256 + c, g);
      if (r >= 0 && r < nk) {
#pragma unroll
        for (int j = 0; j < 32; ++j) g[j] = first ? 0.f : g[j] * scale;
        Tio* dst = dk + ((size_t)(k0 + r) * H + h) * DQ + c;
        st_out16(dst, g);
        st_out16(dst + 16, g + 16);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (w == 0) tc::tmem_dealloc(tb, 512);
}

}  // namespace tpc
