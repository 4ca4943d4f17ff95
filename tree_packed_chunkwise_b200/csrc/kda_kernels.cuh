// Chunkwise gated delta-rule (KDA) kernels, tree-packed (fp32 math on CUDA cores).
//
// Per chunk of C rows (chunk-local inclusive cumulative gate G, last valid row G_C):
//   Kbar = k e^G, Khat = k e^{G_C - G}, Qbar = q e^G
//   A = strict_lower(diag(beta) gated(k, k)),  gated(a, b)_ri = sum_c a_rc b_ic e^{G_rc - G_ic}
//   [W | U'] = (I + A)^{-1} [diag(beta) Kbar | diag(beta) V]          (forward substitution)
//   U = U' - W S0,  O = Qbar S0 + lower_incl(gated(q, k)) U,  S_C = Diag(e^{G_C}) S0 + Khat^T U
// gated() is evaluated with one reference row per 16-row sub-block so that no factor
// exceeds e^{range} (range = decay inside one sub-block, checked against kMaxGateRange).
//
// Forward:  prep (all chunks) -> scan (one launch per round) -> out (all chunks)
// Backward: bprep (all chunks) -> bscan (rounds in reverse) -> bdq (all) -> bdkv (all) -> reduce
#pragma once
#include "common.cuh"

namespace tpc {

struct KdaWs {
  int* status;
  float *W, *U, *Khat, *decay, *S0, *slot;                 // forward (kept for the backward)
  float *dU, *dS, *dS0seq, *pdk, *pdG;                     // backward
  float *rdk, *rdv, *rdg, *rdb;                            // replay partials [R][H][D] / [R][H]
  float *tdk, *tdv, *tdg, *tdb;                            // own part of replay-target rows
  float *Mt, *Bc;  // tensor-core path: per-chunk state transition M (bf16 hi/lo operand tile) and B (fp32)
  float *At, *Tm;  // tensor-core path: per-chunk gated key products Atilde and T = (I + diag(beta) Atilde)^{-1}
  float *Pm;       // tensor-core path: per-chunk masked gated products P = lower_incl(gated(q, k))
  // The tensor-core path keeps W, U (U' then U), Pm, S0 and dS as hi/lo bf16 operand tiles (same
  // bytes as fp32), and dU additionally as the tile dUt.
  float *dUt;
};

template <int C, int D>
struct KD {
  static constexpr int LD = D + 1;    // smem row pitch of [C][D] tiles
  static constexpr int LC = C + 1;    // smem row pitch of [C][C] tiles
  static constexpr int CD = C * D;
  static constexpr int DD = D * D;
  static constexpr int NB = C / kSub; // sub-blocks per chunk
  static_assert(C % kSub == 0, "chunk must be a multiple of 16");
};

template <int I, int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (I < N) {
    f(std::integral_constant<int, I>{});
    static_for<I + 1, N>(f);
  }
}

// load rows of a [N, H, D] tensor (head h) for the chunk into smem [C][LD] as fp32; rows >= n -> 0
template <int C, int D, typename T>
__device__ __forceinline__ void load_rows(float* dst, const T* src, const int* rows, int H, int h, int n_valid_from,
                                          int n) {
  constexpr int LD = D + 1;
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    float x = 0.f;
    if (i >= n_valid_from && i < n) x = to_f(src[((size_t)rows[i] * H + h) * D + c]);
    dst[i * LD + c] = x;
  }
}

// G <- inclusive cumulative sum over rows (per channel); rows >= n repeat row n-1.
// Returns via status when a sub-block decays by more than kMaxGateRange.
template <int C, int D>
__device__ __forceinline__ void cumsum_gate(float* G, int n, int* status) {
  constexpr int LD = D + 1;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < C; ++i) {
      if (i < n) acc += G[i * LD + c];
      G[i * LD + c] = acc;
    }
    for (int p = 0; p < C / kSub; ++p) {
      const float range = G[p * kSub * LD + c] - G[(p * kSub + kSub - 1) * LD + c];
      if (!(range <= kMaxGateRange)) set_status(status, kStatusRange);
    }
  }
}

// Z (ld LC) = mask(gated(a, b)) * rowscale (rowscale == nullptr -> 1); a, b, G: [C][LD]
// Fa: [kSub][LD], Fb: [C][LD] scratch.  incl: i <= r, else i < r.
template <int C, int D>
__device__ __forceinline__ void gated_product(float* Z, const float* a, const float* b, const float* G, float* Fa,
                                              float* Fb, bool incl, const float* rowscale) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC;
  static_for<0, K::NB>([&](auto P) {
    constexpr int p = decltype(P)::value;
    constexpr int r0 = p * kSub, IE = r0 + kSub;
    for (int e = threadIdx.x; e < kSub * D; e += blockDim.x) {
      const int r = e / D, c = e % D;
      Fa[r * LD + c] = a[(r0 + r) * LD + c] * expf(G[(r0 + r) * LD + c] - G[r0 * LD + c]);
    }
    for (int e = threadIdx.x; e < IE * D; e += blockDim.x) {
      const int i = e / D, c = e % D;
      Fb[i * LD + c] = b[i * LD + c] * expf(G[r0 * LD + c] - G[i * LD + c]);
    }
    __syncthreads();
    cta_gemm<kSub, IE, D>([&](int r, int c) { return Fa[r * LD + c]; },
                          [&](int c, int i) { return Fb[i * LD + c]; },
                          [&](int r, int i, float v) {
                            const int rr = r0 + r;
                            const bool keep = incl ? (i <= rr) : (i < rr);
                            Z[rr * LC + i] = keep ? v * (rowscale ? rowscale[rr] : 1.f) : 0.f;
                          });
    __syncthreads();
  });
  // columns at or beyond a block's end are zero
  for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
    const int r = e / C, i = e % C;
    if (i >= (r / kSub + 1) * kSub) Z[r * LC + i] = 0.f;
  }
  __syncthreads();
}

// da (ld LDo, rows of the chunk, channels c0..c0+W-1) (+)= rowside adjoint of gated(a, b) for dZ:
//   da_rc = sum_i dZ_ri b_ic e^{G_rc - G_ic}.  Operates on channel window [c0, c0+W) of b and G.
template <int C, int D, int W>
__device__ __forceinline__ void gated_rowside(float* da, int LDo, const float* dZ, const float* b, const float* G,
                                              int c0, float* Fb) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC, LW = W + 1;
  static_for<0, K::NB>([&](auto P) {
    constexpr int p = decltype(P)::value;
    constexpr int r0 = p * kSub, IE = r0 + kSub;
    for (int e = threadIdx.x; e < IE * W; e += blockDim.x) {
      const int i = e / W, c = e % W;
      Fb[i * LW + c] = b[i * LD + c0 + c] * expf(G[r0 * LD + c0 + c] - G[i * LD + c0 + c]);
    }
    __syncthreads();
    cta_gemm<kSub, W, IE>([&](int r, int i) { return dZ[(r0 + r) * LC + i]; },
                          [&](int i, int c) { return Fb[i * LW + c]; },
                          [&](int r, int c, float v) {
                            const int rr = r0 + r;
                            da[rr * LDo + c] += v * expf(G[rr * LD + c0 + c] - G[r0 * LD + c0 + c]);
                          });
    __syncthreads();
  });
}

// db (ld LDo) (+)= colside adjoint: db_ic = sum_r dZ_ri a_rc e^{G_rc - G_ic}, channel window [c0, c0+W).
template <int C, int D, int W>
__device__ __forceinline__ void gated_colside(float* db, int LDo, const float* dZ, const float* a, const float* G,
                                              int c0, float* Fa) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC, LW = W + 1;
  static_for<0, K::NB>([&](auto P) {
    constexpr int p = decltype(P)::value;
    constexpr int r0 = p * kSub, IE = r0 + kSub;
    for (int e = threadIdx.x; e < kSub * W; e += blockDim.x) {
      const int r = e / W, c = e % W;
      Fa[r * LW + c] = a[(r0 + r) * LD + c0 + c] * expf(G[(r0 + r) * LD + c0 + c] - G[r0 * LD + c0 + c]);
    }
    __syncthreads();
    cta_gemm<IE, W, kSub>([&](int i, int r) { return dZ[(r0 + r) * LC + i]; },
                          [&](int r, int c) { return Fa[r * LW + c]; },
                          [&](int i, int c, float v) {
                            db[i * LDo + c] += v * expf(G[r0 * LD + c0 + c] - G[i * LD + c0 + c]);
                          });
    __syncthreads();
  });
}

// ------------------------------------------------------------------------------------------ forward
template <int C, int D>
constexpr size_t fwd_prep_smem() {
  using K = KD<C, D>;
  return sizeof(float) * (2 * C * K::LD + C * (2 * D + 1) + C * K::LC + kSub * K::LD + C * K::LD + C);
}

template <int C, int D, typename Tin>
__global__ void __launch_bounds__(kThreads) kda_fwd_prep(DevTables t, int H, const Tin* __restrict__ k_,
                                                         const Tin* __restrict__ v_, const Tin* __restrict__ g_,
                                                         const Tin* __restrict__ beta_, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC, LX = 2 * D + 1;
  const int ci = blockIdx.x, h = blockIdx.y;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ float sm[];
  float* sk = sm;
  float* sG = sk + C * LD;
  float* sX = sG + C * LD;
  float* sA = sX + C * LX;
  float* sFa = sA + C * LC;
  float* sFb = sFa + kSub * LD;
  float* sb = sFb + C * LD;
  __shared__ int srow[C];
  for (int i = threadIdx.x; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  __syncthreads();
  load_rows<C, D>(sk, k_, srow, H, h, 0, n);
  load_rows<C, D>(sG, g_, srow, H, h, 0, n);
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    sX[i * LX + D + c] = i < n ? to_f(v_[((size_t)srow[i] * H + h) * D + c]) : 0.f;
  }
  for (int i = threadIdx.x; i < C; i += blockDim.x) sb[i] = i < n ? to_f(beta_[(size_t)srow[i] * H + h]) : 0.f;
  __syncthreads();
  cumsum_gate<C, D>(sG, n, ws.status);
  __syncthreads();
  gated_product<C, D>(sA, sk, sk, sG, sFa, sFb, false, sb);
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    sX[i * LX + c] = sb[i] * sk[i * LD + c] * expf(sG[i * LD + c]);
    sX[i * LX + D + c] *= sb[i];
  }
  __syncthreads();
  // (I + A) X = B by forward substitution, one column per thread
  for (int col = threadIdx.x; col < 2 * D; col += blockDim.x) {
    for (int r = 1; r < n; ++r) {
      float acc = sX[r * LX + col];
      for (int i = 0; i < r; ++i) acc = fmaf(-sA[r * LC + i], sX[i * LX + col], acc);
      sX[r * LX + col] = acc;
    }
  }
  __syncthreads();
  const size_t base = ((size_t)ci * H + h);
  float* W = ws.W + base * K::CD;
  float* U = ws.U + base * K::CD;
  float* Kh = ws.Khat + base * K::CD;
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    W[e] = sX[i * LX + c];
    U[e] = sX[i * LX + D + c];
    Kh[e] = sk[i * LD + c] * expf(sG[(n - 1) * LD + c] - sG[i * LD + c]);
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) ws.decay[base * D + c] = expf(sG[(n - 1) * LD + c]);
}

template <int C, int D, int DVT>
constexpr size_t scan_smem() {
  return sizeof(float) * (2 * C * (D + 1) + C * (DVT + 1) + 2 * D * (DVT + 1) + D);
}

// one CTA per (sequence of the round, head, d_v tile): S[:, tile] carried across the chunks
template <int C, int D, int DVT>
__global__ void __launch_bounds__(kThreads) kda_fwd_scan(DevTables t, int seq0, int H, const float* __restrict__ init,
                                                         float* __restrict__ final_state, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LT = DVT + 1;
  const int si = seq0 + blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVT;
  const SeqRec s = t.seqs[si];
  extern __shared__ float sm[];
  float* sW = sm;
  float* sK = sW + C * LD;
  float* sU = sK + C * LD;
  float* sS = sU + C * LT;
  float* sdec = sS + D * LT;
  {
    const float* src = nullptr;
    if (s.import_id >= 0) src = ws.slot + ((size_t)s.import_id * H + h) * K::DD;
    else if (init) src = init + ((size_t)(-(s.import_id + 1)) * H + h) * K::DD;
    for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
      const int c = e / DVT, j = e % DVT;
      sS[c * LT + j] = src ? src[c * D + j0 + j] : 0.f;
    }
  }
  __syncthreads();
  for (int q = 0; q < s.n_chunks; ++q) {
    const int ci = s.chunk_begin + q;
    const size_t base = (size_t)ci * H + h;
    float* S0 = ws.S0 + base * K::DD;
    const float* W = ws.W + base * K::CD;
    const float* Kh = ws.Khat + base * K::CD;
    float* U = ws.U + base * K::CD;
    for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
      const int c = e / DVT, j = e % DVT;
      S0[c * D + j0 + j] = sS[c * LT + j];
    }
    for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
      const int i = e / D, c = e % D;
      sW[i * LD + c] = W[e];
      sK[i * LD + c] = Kh[e];
    }
    for (int e = threadIdx.x; e < C * DVT; e += blockDim.x) {
      const int i = e / DVT, j = e % DVT;
      sU[i * LT + j] = U[i * D + j0 + j];
    }
    for (int c = threadIdx.x; c < D; c += blockDim.x) sdec[c] = ws.decay[base * D + c];
    __syncthreads();
    cta_gemm<C, DVT, D>([&](int r, int c) { return sW[r * LD + c]; }, [&](int c, int j) { return sS[c * LT + j]; },
                        [&](int r, int j, float v) { sU[r * LT + j] -= v; });
    __syncthreads();
    for (int e = threadIdx.x; e < C * DVT; e += blockDim.x) {
      const int i = e / DVT, j = e % DVT;
      U[i * D + j0 + j] = sU[i * LT + j];
    }
    cta_gemm<D, DVT, C>([&](int c, int r) { return sK[r * LD + c]; }, [&](int r, int j) { return sU[r * LT + j]; },
                        [&](int c, int j, float v) { sS[c * LT + j] = fmaf(sdec[c], sS[c * LT + j], v); });
    __syncthreads();
    const int slot = t.chunks[ci].export_slot;
    if (slot >= 0) {
      float* dst = ws.slot + ((size_t)slot * H + h) * K::DD;
      for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
        const int c = e / DVT, j = e % DVT;
        dst[c * D + j0 + j] = sS[c * LT + j];
      }
    }
  }
  if (final_state && s.leaf >= 0) {  // a sequence ending at an internal node has no final state
    float* dst = final_state + ((size_t)s.leaf * H + h) * K::DD;
    for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
      const int c = e / DVT, j = e % DVT;
      dst[c * D + j0 + j] = sS[c * LT + j];
    }
  }
}

template <int C, int D>
constexpr size_t out_smem() {
  using K = KD<C, D>;
  return sizeof(float) * (4 * C * K::LD + C * K::LC + kSub * K::LD + C * K::LD);
}

template <int C, int D, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) kda_fwd_out(DevTables t, int H, const Tin* __restrict__ q_,
                                                        const Tin* __restrict__ k_, const Tin* __restrict__ g_,
                                                        Tout* __restrict__ o_, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC;
  const int ci = blockIdx.x, h = blockIdx.y;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ float sm[];
  float* sq = sm;
  float* sk = sq + C * LD;
  float* sG = sk + C * LD;
  float* sU = sG + C * LD;
  float* sP = sU + C * LD;
  float* sFa = sP + C * LC;
  float* sFb = sFa + kSub * LD;
  __shared__ int srow[C];
  for (int i = threadIdx.x; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  __syncthreads();
  load_rows<C, D>(sq, q_, srow, H, h, 0, n);
  load_rows<C, D>(sk, k_, srow, H, h, 0, n);
  load_rows<C, D>(sG, g_, srow, H, h, 0, n);
  const size_t base = (size_t)ci * H + h;
  const float* U = ws.U + base * K::CD;
  const float* S0 = ws.S0 + base * K::DD;
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) sU[(e / D) * LD + e % D] = U[e];
  __syncthreads();
  cumsum_gate<C, D>(sG, n, nullptr);
  __syncthreads();
  gated_product<C, D>(sP, sq, sk, sG, sFa, sFb, true, nullptr);
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    sq[i * LD + c] *= expf(sG[i * LD + c]);
  }
  __syncthreads();
  cta_gemm<C, D, D + C>(
      [&](int r, int kk) { return kk < D ? sq[r * LD + kk] : sP[r * LC + kk - D]; },
      [&](int kk, int j) { return kk < D ? S0[kk * D + j] : sU[(kk - D) * LD + j]; },
      [&](int r, int j, float v) {
        if (r >= ch.n_replay && r < n) o_[((size_t)srow[r] * H + h) * D + j] = from_f<Tout>(v);
      });
}

// ----------------------------------------------------------------------------------------- backward
template <int C, int D>
constexpr size_t bprep_smem() {
  using K = KD<C, D>;
  return sizeof(float) * (4 * C * K::LD + C * K::LC + kSub * K::LD + C * K::LD);
}

// dU0 = P^T dO  and  X = Qbar^T dO - W^T dU0  (the state-independent parts of the reverse scan)
template <int C, int D, typename Tin>
__global__ void __launch_bounds__(kThreads) kda_bwd_prep(DevTables t, int H, const Tin* __restrict__ q_,
                                                         const Tin* __restrict__ k_, const Tin* __restrict__ g_,
                                                         const Tin* __restrict__ do_, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC;
  const int ci = blockIdx.x, h = blockIdx.y;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ float sm[];
  float* sq = sm;
  float* sk = sq + C * LD;
  float* sG = sk + C * LD;
  float* sdO = sG + C * LD;
  float* sP = sdO + C * LD;
  float* sFa = sP + C * LC;
  float* sFb = sFa + kSub * LD;
  __shared__ int srow[C];
  for (int i = threadIdx.x; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  __syncthreads();
  load_rows<C, D>(sq, q_, srow, H, h, 0, n);
  load_rows<C, D>(sk, k_, srow, H, h, 0, n);
  load_rows<C, D>(sG, g_, srow, H, h, 0, n);
  load_rows<C, D>(sdO, do_, srow, H, h, ch.n_replay, n);  // replayed rows have no output
  __syncthreads();
  cumsum_gate<C, D>(sG, n, nullptr);
  __syncthreads();
  gated_product<C, D>(sP, sq, sk, sG, sFa, sFb, true, nullptr);
  const size_t base = (size_t)ci * H + h;
  float* dU = ws.dU + base * K::CD;
  float* sdU = sFb;  // Fb is free now
  cta_gemm<C, D, C>([&](int i, int r) { return sP[r * LC + i]; }, [&](int r, int j) { return sdO[r * LD + j]; },
                    [&](int i, int j, float v) {
                      sdU[i * LD + j] = v;
                      dU[i * D + j] = v;
                    });
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    sq[i * LD + c] *= expf(sG[i * LD + c]);
  }
  __syncthreads();
  const float* W = ws.W + base * K::CD;
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) sk[(e / D) * LD + e % D] = W[e];  // sk <- W
  __syncthreads();
  float* X = ws.dS + base * K::DD;
  cta_gemm<D, D, 2 * C>(
      [&](int c, int kk) { return kk < C ? sq[kk * LD + c] : sk[(kk - C) * LD + c]; },
      [&](int kk, int j) { return kk < C ? sdO[kk * LD + j] : -sdU[(kk - C) * LD + j]; },
      [&](int c, int j, float v) { X[c * D + j] = v; });
}

// reverse scan over the chunks of one sequence: dS (gradient of the state at a chunk end)
template <int C, int D, int DVT>
__global__ void __launch_bounds__(kThreads) kda_bwd_scan(DevTables t, int seq0, int H, const float* __restrict__ d_final,
                                                         KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LT = DVT + 1;
  const int si = seq0 + blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVT;
  const SeqRec s = t.seqs[si];
  extern __shared__ float sm[];
  float* sW = sm;
  float* sK = sW + C * LD;
  float* sY = sK + C * LD;
  float* sdS = sY + C * LT;
  float* sX = sdS + D * LT;
  float* sdec = sX + D * LT;
  for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
    const int c = e / DVT, j = e % DVT;
    sdS[c * LT + j] = (d_final && s.leaf >= 0) ? d_final[((size_t)s.leaf * H + h) * K::DD + c * D + j0 + j] : 0.f;
  }
  __syncthreads();
  for (int q = s.n_chunks - 1; q >= 0; --q) {
    const int ci = s.chunk_begin + q;
    const size_t base = (size_t)ci * H + h;
    const int slot = t.chunks[ci].export_slot;
    if (slot >= 0) {  // consumers' gradients of this boundary state, in a fixed order
      const SlotRec sr = t.slots[slot];
      for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
        const int c = e / DVT, j = e % DVT;
        float acc = sdS[c * LT + j];
        for (int m = 0; m < sr.n_cons; ++m) {
          const int cs = t.slot_cons[sr.cons_begin + m];
          acc += ws.dS0seq[((size_t)cs * H + h) * K::DD + c * D + j0 + j];
        }
        sdS[c * LT + j] = acc;
      }
    }
    const float* W = ws.W + base * K::CD;
    const float* Kh = ws.Khat + base * K::CD;
    float* dU = ws.dU + base * K::CD;
    float* dSg = ws.dS + base * K::DD;
    for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
      const int i = e / D, c = e % D;
      sW[i * LD + c] = W[e];
      sK[i * LD + c] = Kh[e];
    }
    for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
      const int c = e / DVT, j = e % DVT;
      sX[c * LT + j] = dSg[c * D + j0 + j];
    }
    for (int c = threadIdx.x; c < D; c += blockDim.x) sdec[c] = ws.decay[base * D + c];
    __syncthreads();
    cta_gemm<C, DVT, D>([&](int r, int c) { return sK[r * LD + c]; }, [&](int c, int j) { return sdS[c * LT + j]; },
                        [&](int r, int j, float v) { sY[r * LT + j] = v; });
    for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
      const int c = e / DVT, j = e % DVT;
      dSg[c * D + j0 + j] = sdS[c * LT + j];  // gradient at the chunk end, for the chunk kernels
    }
    __syncthreads();
    for (int e = threadIdx.x; e < C * DVT; e += blockDim.x) {
      const int i = e / DVT, j = e % DVT;
      dU[i * D + j0 + j] += sY[i * LT + j];
    }
    cta_gemm<D, DVT, C>([&](int c, int r) { return sW[r * LD + c]; }, [&](int r, int j) { return sY[r * LT + j]; },
                        [&](int c, int j, float v) {
                          sdS[c * LT + j] = fmaf(sdec[c], sdS[c * LT + j], sX[c * LT + j] - v);
                        });
    __syncthreads();
  }
  float* dst = ws.dS0seq + ((size_t)si * H + h) * K::DD;
  for (int e = threadIdx.x; e < D * DVT; e += blockDim.x) {
    const int c = e / DVT, j = e % DVT;
    dst[c * D + j0 + j] = sdS[c * LT + j];
  }
}

template <int C, int D>
constexpr size_t bdq_smem() {
  using K = KD<C, D>;
  return sizeof(float) * (6 * C * K::LD + C * K::LC + kSub * K::LD);
}

// dq (final) and the parts of dk, dG that involve P, S0 and dS_end:
//   dP = lower_incl(dO U^T);  dq = e^G (dO S0^T) + rowside(dP, k)
//   pdk = e^{G_C - G} (U dS_end^T) + colside(dP, q);  pdG = q dq - k pdk
//   pdG[n-1] += sum_i Khat_i (U dS_end^T)_i + e^{G_C} rowsum(dS_end * S0)
template <int C, int D, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) kda_bwd_dq(DevTables t, int H, const Tin* __restrict__ q_,
                                                       const Tin* __restrict__ k_, const Tin* __restrict__ g_,
                                                       const Tin* __restrict__ do_, Tout* __restrict__ dq_, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC;
  const int ci = blockIdx.x, h = blockIdx.y;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ float sm[];
  float* B0 = sm;
  float* B1 = B0 + C * LD;
  float* B2 = B1 + C * LD;
  float* B3 = B2 + C * LD;
  float* B4 = B3 + C * LD;
  float* B5 = B4 + C * LD;
  float* sdP = B5 + C * LD;
  float* sFa = sdP + C * LC;
  __shared__ int srow[C];
  __shared__ float sgc[D];
  for (int i = threadIdx.x; i < C; i += blockDim.x) srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
  __syncthreads();
  const size_t base = (size_t)ci * H + h;
  const float* S0 = ws.S0 + base * K::DD;
  const float* dSe = ws.dS + base * K::DD;
  const float* U = ws.U + base * K::CD;
  load_rows<C, D>(B0, do_, srow, H, h, ch.n_replay, n);
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) B1[(e / D) * LD + e % D] = U[e];
  __syncthreads();
  cta_gemm<C, C, D>([&](int r, int j) { return B0[r * LD + j]; }, [&](int j, int i) { return B1[i * LD + j]; },
                    [&](int r, int i, float v) { sdP[r * LC + i] = (i <= r) ? v : 0.f; });
  cta_gemm<C, D, D>([&](int r, int j) { return B0[r * LD + j]; }, [&](int j, int c) { return S0[c * D + j]; },
                    [&](int r, int c, float v) { B2[r * LD + c] = v; });  // Tq = dO S0^T
  cta_gemm<C, D, D>([&](int r, int j) { return B1[r * LD + j]; }, [&](int j, int c) { return dSe[c * D + j]; },
                    [&](int r, int c, float v) { B3[r * LD + c] = v; });  // T1 = U dS_end^T
  __syncthreads();
  load_rows<C, D>(B0, k_, srow, H, h, 0, n);
  load_rows<C, D>(B1, q_, srow, H, h, 0, n);
  load_rows<C, D>(B4, g_, srow, H, h, 0, n);
  __syncthreads();
  cumsum_gate<C, D>(B4, n, nullptr);
  __syncthreads();
  const float* sk = B0;
  const float* sq = B1;
  float* sdq = B2;
  float* spdk = B3;
  const float* sG = B4;
  // dq = e^G Tq ; pdk = e^{G_C - G} T1 ; dG_C partial
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    sdq[i * LD + c] *= expf(sG[i * LD + c]);
    spdk[i * LD + c] *= expf(sG[(n - 1) * LD + c] - sG[i * LD + c]);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < n; ++i) acc = fmaf(sk[i * LD + c], spdk[i * LD + c], acc);
    float acc2 = 0.f;
    for (int j = 0; j < D; ++j) acc2 = fmaf(dSe[c * D + j], S0[c * D + j], acc2);
    sgc[c] = acc + expf(sG[(n - 1) * LD + c]) * acc2;
  }
  gated_rowside<C, D, D>(sdq, LD, sdP, sk, sG, 0, B5);
  gated_colside<C, D, D>(spdk, LD, sdP, sq, sG, 0, sFa);
  float* pdk = ws.pdk + base * K::CD;
  float* pdG = ws.pdG + base * K::CD;
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) {
    const int i = e / D, c = e % D;
    const float dqv = sdq[i * LD + c];
    float dG = sq[i * LD + c] * dqv - sk[i * LD + c] * spdk[i * LD + c];
    if (i == n - 1) dG += sgc[c];
    pdk[e] = spdk[i * LD + c];
    pdG[e] = dG;
    if (i >= ch.n_replay && i < n) dq_[((size_t)srow[i] * H + h) * D + c] = from_f<Tout>(dqv);
  }
}

template <int C, int D>
constexpr size_t bdkv_smem() {
  using K = KD<C, D>;
  return sizeof(float) * (3 * C * K::LD + 2 * C * K::LC + kSub * K::LD + C * K::LD + 2 * C * 33 + 2 * C);
}

// The WY part of the backward, channel tile by channel tile (32 channels):
//   X = [W | U'] = (I + A)^{-1} [beta Kbar | beta V]  (recomputed),  dX = [-dU S0^T | dU]
//   dB = (I + A)^{-T} dX,  dA = -strict_lower(dB X^T)
//   dk += e^G beta dB_k + rowside(beta dA, k) + colside(beta dA, k);  dv = beta dB_v
//   dG += Kbar beta dB_k + k (rowside - colside);  dbeta = rowsum(dB_k Kbar + dB_v v + dA Atilde)
// then dg = reverse cumsum of dG; replayed rows go to the replay partials.
template <int C, int D, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) kda_bwd_dkv(DevTables t, int H, const Tin* __restrict__ k_,
                                                        const Tin* __restrict__ v_, const Tin* __restrict__ g_,
                                                        const Tin* __restrict__ beta_, Tout* __restrict__ dk_,
                                                        Tout* __restrict__ dv_, float* __restrict__ dg_,
                                                        float* __restrict__ dbeta_, KdaWs ws) {
  using K = KD<C, D>;
  constexpr int LD = K::LD, LC = K::LC;
  constexpr int TW = (D < 32) ? D : 32, LT = TW + 1;
  const int ci = blockIdx.x, h = blockIdx.y;
  const ChunkRec ch = t.chunks[ci];
  const int n = ch.n_rows;
  extern __shared__ float sm[];
  float* sk = sm;
  float* sG = sk + C * LD;
  float* sdU = sG + C * LD;
  float* sAt = sdU + C * LD;  // Atilde (without beta)
  float* sdA = sAt + C * LC;
  float* sFa = sdA + C * LC;
  float* sFb = sFa + kSub * LD;
  float* sXt = sFb + C * LD;   // [C][33] tile of X
  float* sBt = sXt + C * 33;   // [C][33] tile of dX / dB
  float* sb = sBt + C * 33;
  float* sdb = sb + C;
  __shared__ int srow[C];
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    srow[i] = i < n ? chunk_row(ch, t.replay_rows, i) : 0;
    sb[i] = i < n ? to_f(beta_[(size_t)(i < n ? chunk_row(ch, t.replay_rows, i) : 0) * H + h]) : 0.f;
    sdb[i] = 0.f;
  }
  __syncthreads();
  const size_t base = (size_t)ci * H + h;
  const float* S0 = ws.S0 + base * K::DD;
  const float* dUg = ws.dU + base * K::CD;
  float* pdk = ws.pdk + base * K::CD;
  float* pdG = ws.pdG + base * K::CD;
  load_rows<C, D>(sk, k_, srow, H, h, 0, n);
  load_rows<C, D>(sG, g_, srow, H, h, 0, n);
  for (int e = threadIdx.x; e < C * D; e += blockDim.x) sdU[(e / D) * LD + e % D] = dUg[e];
  for (int e = threadIdx.x; e < C * C; e += blockDim.x) sdA[(e / C) * LC + e % C] = 0.f;
  __syncthreads();
  cumsum_gate<C, D>(sG, n, nullptr);
  __syncthreads();
  gated_product<C, D>(sAt, sk, sk, sG, sFa, sFb, false, nullptr);
  // two passes over channel tiles: first the key half (W, dW), then the value half (U', dU)
  for (int half = 0; half < 2; ++half) {
    for (int c0 = 0; c0 < D; c0 += TW) {
      // X tile (right-hand side, then solved) and dX tile
      for (int e = threadIdx.x; e < C * TW; e += blockDim.x) {
        const int i = e / TW, c = e % TW;
        float x;
        if (half == 0) x = sb[i] * sk[i * LD + c0 + c] * expf(sG[i * LD + c0 + c]);
        else x = i < n ? sb[i] * to_f(v_[((size_t)srow[i] * H + h) * D + c0 + c]) : 0.f;
        sXt[i * LT + c] = x;
        if (half == 1) sBt[i * LT + c] = sdU[i * LD + c0 + c];
      }
      if (half == 0) {
        // dW tile = -dU S0^T restricted to channels c0..c0+TW
        cta_gemm<C, TW, D>([&](int r, int j) { return sdU[r * LD + j]; },
                           [&](int j, int c) { return S0[(c0 + c) * D + j]; },
                           [&](int r, int c, float v) { sBt[r * LT + c] = -v; });
      }
      __syncthreads();
      for (int col = threadIdx.x; col < TW; col += blockDim.x) {
        for (int r = 1; r < n; ++r) {  // forward substitution (I + A) X = B
          float acc = sXt[r * LT + col];
          for (int i = 0; i < r; ++i) acc = fmaf(-sb[r] * sAt[r * LC + i], sXt[i * LT + col], acc);
          sXt[r * LT + col] = acc;
        }
        for (int r = n - 2; r >= 0; --r) {  // backward substitution (I + A)^T dB = dX
          float acc = sBt[r * LT + col];
          for (int i = r + 1; i < n; ++i) acc = fmaf(-sb[i] * sAt[i * LC + r], sBt[i * LT + col], acc);
          sBt[r * LT + col] = acc;
        }
      }
      __syncthreads();
      cta_gemm<C, C, TW>([&](int r, int c) { return sBt[r * LT + c]; }, [&](int c, int i) { return sXt[i * LT + c]; },
                         [&](int r, int i, float v) {
                           if (i < r) sdA[r * LC + i] -= v;
                         });
      // per-row dbeta and per-element contributions
      if (half == 0) {
        for (int e = threadIdx.x; e < C * TW; e += blockDim.x) {
          const int i = e / TW, c = e % TW;
          const float kbar = sk[i * LD + c0 + c] * expf(sG[i * LD + c0 + c]);
          const float bdb = sb[i] * sBt[i * LT + c];
          const size_t gi = (size_t)i * D + c0 + c;
          pdk[gi] += expf(sG[i * LD + c0 + c]) * bdb;
          pdG[gi] += kbar * bdb;
        }
      } else {
        for (int e = threadIdx.x; e < C * TW; e += blockDim.x) {
          const int i = e / TW, c = e % TW;
          if (i >= n) continue;
          const float val = sb[i] * sBt[i * LT + c];
          if (i < ch.n_replay) {
            ws.rdv[((size_t)(ch.replay_base + i) * H + h) * D + c0 + c] = val;
          } else {
            const int tg = t.row_tgt[srow[i]];
            if (tg >= 0) ws.tdv[((size_t)tg * H + h) * D + c0 + c] = val;
            else dv_[((size_t)srow[i] * H + h) * D + c0 + c] = from_f<Tout>(val);
          }
        }
      }
      for (int i = threadIdx.x; i < C; i += blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < TW; ++c) {
          const float other = half == 0 ? sk[i * LD + c0 + c] * expf(sG[i * LD + c0 + c])
                                        : (i < n ? to_f(v_[((size_t)srow[i] * H + h) * D + c0 + c]) : 0.f);
          acc = fmaf(sBt[i * LT + c], other, acc);
        }
        sdb[i] += acc;
      }
      __syncthreads();
    }
  }
  // dAtilde = beta * dA ; dbeta += rowsum(dA * Atilde)
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < i; ++j) acc = fmaf(sdA[i * LC + j], sAt[i * LC + j], acc);
    sdb[i] += acc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < C * C; e += blockDim.x) sdA[(e / C) * LC + e % C] *= sb[e / C];
  __syncthreads();
  // rowside / colside of dAtilde w.r.t. k, per channel tile, into tiles then global partials
  for (int c0 = 0; c0 < D; c0 += TW) {
    for (int e = threadIdx.x; e < C * TW; e += blockDim.x) {
      sXt[(e / TW) * LT + e % TW] = 0.f;
      sBt[(e / TW) * LT + e % TW] = 0.f;
    }
    __syncthreads();
    gated_rowside<C, D, TW>(sXt, LT, sdA, sk, sG, c0, sFb);
    gated_colside<C, D, TW>(sBt, LT, sdA, sk, sG, c0, sFa);
    for (int e = threadIdx.x; e < C * TW; e += blockDim.x) {
      const int i = e / TW, c = e % TW;
      const size_t gi = (size_t)i * D + c0 + c;
      const float rs = sXt[i * LT + c], cs = sBt[i * LT + c];
      pdk[gi] += rs + cs;
      pdG[gi] += sk[i * LD + c0 + c] * (rs - cs);
    }
    __syncthreads();
  }
  // dg = reverse cumulative sum of dG; write dk, dg, dbeta
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int i = n - 1; i >= 0; --i) {
      acc += pdG[(size_t)i * D + c];
      const float dkv = pdk[(size_t)i * D + c];
      if (i < ch.n_replay) {
        const size_t ri = ((size_t)(ch.replay_base + i) * H + h) * D + c;
        ws.rdk[ri] = dkv;
        ws.rdg[ri] = acc;
      } else {
        const int tg = t.row_tgt[srow[i]];
        if (tg >= 0) {
          ws.tdk[((size_t)tg * H + h) * D + c] = dkv;
          ws.tdg[((size_t)tg * H + h) * D + c] = acc;
        } else {
          dk_[((size_t)srow[i] * H + h) * D + c] = from_f<Tout>(dkv);
          dg_[((size_t)srow[i] * H + h) * D + c] = acc;
        }
      }
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    if (i < ch.n_replay) {
      ws.rdb[(size_t)(ch.replay_base + i) * H + h] = sdb[i];
    } else {
      const int tg = t.row_tgt[srow[i]];
      if (tg >= 0) ws.tdb[(size_t)tg * H + h] = sdb[i];
      else dbeta_[(size_t)srow[i] * H + h] = sdb[i];
    }
  }
}

// rows that are replayed somewhere: own gradient + replay partials, in ascending replay index
template <int D, typename Tout>
__global__ void kda_replay_reduce(DevTables t, int H, Tout* __restrict__ dk_, Tout* __restrict__ dv_,
                                  float* __restrict__ dg_, float* __restrict__ dbeta_, KdaWs ws) {
  const int tg = blockIdx.x, h = blockIdx.y;
  const int row = t.tgt_row[tg];
  const int p0 = t.tgt_begin[tg], p1 = t.tgt_begin[tg + 1];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const size_t o = ((size_t)tg * H + h) * D + c;
    float a = ws.tdk[o], b = ws.tdv[o], g = ws.tdg[o];
    for (int p = p0; p < p1; ++p) {
      const size_t r = ((size_t)t.tgt_parts[p] * H + h) * D + c;
      a += ws.rdk[r];
      b += ws.rdv[r];
      g += ws.rdg[r];
    }
    const size_t d = ((size_t)row * H + h) * D + c;
    dk_[d] = from_f<Tout>(a);
    dv_[d] = from_f<Tout>(b);
    dg_[d] = g;
  }
  if (threadIdx.x == 0) {
    float b = ws.tdb[(size_t)tg * H + h];
    for (int p = p0; p < p1; ++p) b += ws.rdb[(size_t)t.tgt_parts[p] * H + h];
    dbeta_[(size_t)row * H + h] = b;
  }
}

// d_init[root] = sum over the sequences that start from that root's initial state (fixed order)
template <int D>
__global__ void kda_init_reduce(DevTables t, int H, float* __restrict__ d_init, KdaWs ws) {
  const int r = blockIdx.x, h = blockIdx.y;
  const int b0 = t.root_cons_begin[r], b1 = t.root_cons_begin[r + 1];
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    float acc = 0.f;
    for (int m = b0; m < b1; ++m) acc += ws.dS0seq[((size_t)t.root_cons[m] * H + h) * D * D + e];
    d_init[((size_t)r * H + h) * D * D + e] = acc;
  }
}

}  // namespace tpc
