// Wall attention prefill backward: the gradients of o (and optionally lse)
// with respect to q, k, v, g, g_scalar and the sink (Wall Attention README,
// intro formula and "Usage / Training-Prefill"; its "code structure" section
// names the backward kernel).
//
// With p = exp(x - lse) and delta = sum_c dO[i,c] o[i,c] - dlse[i], the
// softmax Jacobian gives dS(i,j) = p(i,j) (dO[i].v[j] - delta[i]).  The decay
// of the score splits over the prepass anchors exactly as in the forward,
//   exp(G[i] - G[j]) = exp(G[i] - AQ) exp(AQ - AK) exp(AK - G[j]),
// so every product below is a dense contraction of the anchored operands
// (qh, kh) with one channel vector c = exp(AQ - AK) per (query, key) tile:
//   dq[i]   = scale exp(G[i] - AQ)  o  sum_j dS(i,j) (kh[j] c)
//   dk_h[j] = scale exp(AK - G[j])  o  sum_i dS(i,j) (qh[i] c)
//   dv_h[j] = sum_i p(i,j) dO[i]
// The per-row factors are applied after the contraction ("post" kernels),
// which also form dG = q o dq - k o dk_h and dGs = sum_j dS(i,j) - sum_i dS(i,j),
// and turn them into dg and dg_scalar by a reverse prefix sum restarting at
// every document end (G and Gs are inclusive prefix sums of g and g_scalar).
//
// Passes: the forward prepass (anchored operands, block sums, gate prefixes),
// bwd_pre (delta, lse in log2 units, sink terms), a key-block kernel (dk_h,
// dv_h accumulators), a query-block kernel (dq accumulator), then the post
// kernels and the reductions over the query heads of each KV group.  This file
// holds the CUDA-core (fp32 FMA) contraction kernels, used for fp32 inputs, and
// every pass around the contraction; the bf16 tensor-core contraction kernels
// live in wall_bwd_tc.cu and write the same accumulators.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

constexpr int SB = 64;  // rows per tile of the CUDA-core contraction kernels

__device__ __forceinline__ int row_lo(const int* rowlo, int window, int t) {
  if (rowlo != nullptr) return rowlo[t];
  if (window > 0) return t - window + 1 > 0 ? t - window + 1 : 0;
  return 0;
}

// Gate prefix of row t in log2 units: Gs[t] * log2(e).
__device__ __forceinline__ float gate_row(const float* ssl, const float* ssa, int bh, int NB,
                                          int t) {
  return ssa[(static_cast<size_t>(bh) * NB + t / kBlockRows) * 4] -
         ssl[static_cast<size_t>(bh) * NB * kBlockRows + t];
}

// ------------------------------------------------------------------ bwd_pre
// VD/8 lanes per (b, t, hq) row (a warp covers 32*8/VD rows), each lane one
// 8-channel chunk of o and dO.  Per (batch * head) rows of stride TP = NB*128
// (16-byte aligned slices for bulk copies):
//   rowt  = Gs[t] log2(e) - lse[t] log2(e)   (query-side constant of log2 p)
//   colt  = Gs[t] log2(e)                    (key side; with g_scalar only)
//   delta = dO[t].o[t] - dlse[t]
// and psd (stride T): the row's sink term p_sink (dlse - dO.o) of dL/dsink.
template <typename Tin, int VD, bool HAS_GS>
__global__ void __launch_bounds__(256) bwd_pre_kernel(
    const Tin* __restrict__ o, const Tin* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ dlse, const float* __restrict__ sink, const float* __restrict__ ssl,
    const float* __restrict__ ssa, int B, int T, int HQ, int NB, float* __restrict__ rowt,
    float* __restrict__ colt, float* __restrict__ delta, float* __restrict__ psd) {
  constexpr int LPR = VD / 8;  // lanes per row
  const int lane = threadIdx.x & 31, l = lane % LPR;
  const long long r = ((static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5) * (32 / LPR) +
                      lane / LPR;
  const bool row_ok = r < static_cast<long long>(B) * T * HQ;
  float acc = 0.f;
  if (row_ok) {
    float a[8], d[8];
    load8(o + r * VD + l * 8, a);
    load8(dout + r * VD + l * 8, d);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(a[e], d[e], acc);
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row_ok && l == 0) {
    const int hq = static_cast<int>(r % HQ);
    const long long bt = r / HQ;
    const int t = static_cast<int>(bt % T), b = static_cast<int>(bt / T);
    const int bh = b * HQ + hq;
    const size_t i = static_cast<size_t>(bh) * NB * kBlockRows + t;
    const float l2 = lse[r] * kLog2e;
    const float dl = dlse != nullptr ? dlse[r] : 0.f;
    const float gt = HAS_GS ? gate_row(ssl, ssa, bh, NB, t) : 0.f;
    rowt[i] = gt - l2;
    if (HAS_GS) colt[i] = gt;
    delta[i] = acc - dl;
    if (psd != nullptr)
      psd[static_cast<size_t>(bh) * T + t] =
          sink != nullptr ? ex2_approx(sink[hq] * kLog2e - l2) * (dl - acc) : 0.f;
  }
}

// ------------------------------------------------------------------ CUDA-core contractions
// Tile products shared by both kernels: a thread (ty, tx) of the 16 x 16 grid
// owns rows ty*4..ty*4+3 (queries) and columns tx*4..tx*4+3 (keys) of the
// 64 x 64 score tile.  A is row-major [64][D] (query side), BT is the key
// side transposed, [D][64].
template <int D>
__device__ __forceinline__ void tile_product(const float* __restrict__ A,
                                             const float* __restrict__ BT, int ty, int tx,
                                             float (&s)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) s[a][c] = 0.f;
#pragma unroll 2
  for (int n = 0; n < D; n += 4) {
    float4 av[4], bv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) av[a] = *reinterpret_cast<const float4*>(A + (ty * 4 + a) * D + n);
#pragma unroll
    for (int u = 0; u < 4; ++u) bv[u] = *reinterpret_cast<const float4*>(BT + (n + u) * SB + tx * 4);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float x[4] = {av[a].x, av[a].y, av[a].z, av[a].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        s[a][0] = fmaf(x[u], bv[u].x, s[a][0]);
        s[a][1] = fmaf(x[u], bv[u].y, s[a][1]);
        s[a][2] = fmaf(x[u], bv[u].z, s[a][2]);
        s[a][3] = fmaf(x[u], bv[u].w, s[a][3]);
      }
    }
  }
}

// p and dS of one thread's 4 x 4 patch.  s: q.k of the anchored operands;
// row terms (gate - lse, log2 units), delta and first admitted key per row in
// shared memory; key-side gate per column.
template <bool HAS_GS>
__device__ __forceinline__ void probs_and_grads(float (&s)[4][4], float (&dp)[4][4],
                                                const float* sRow, const float* sDel,
                                                const int* sLo, const float* sCol, int q0, int j0,
                                                int T, int ty, int tx, float sc) {
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = ty * 4 + a, i = q0 + r;
    const float rowt = sRow[r], del = sDel[r];
    const int lo = sLo[r];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      float x = fmaf(s[a][c], sc, rowt);
      if (HAS_GS) x -= sCol[tx * 4 + c];
      const bool ok = i < T && j <= i && j >= lo;
      const float p = ok ? ex2_approx(x) : 0.f;
      s[a][c] = p;
      dp[a][c] = p * (dp[a][c] - del);
    }
  }
}

// Per query row of the tile at q0: gate - lse (log2), delta, first admitted key.
__device__ __forceinline__ void load_row_terms(int tid, int q0, int T, size_t rbase,
                                               const float* rowt, const float* delta,
                                               const int* rowlo, int window, float* sRow,
                                               float* sDel, int* sLo) {
  if (tid < SB) {
    const int t = q0 + tid;
    const bool ok = t < T;
    sRow[tid] = ok ? rowt[rbase + t] : 0.f;
    sDel[tid] = ok ? delta[rbase + t] : 0.f;
    sLo[tid] = ok ? row_lo(rowlo, window, t) : 0x7fffffff;
  }
}

// Key-block kernel: one CTA per (64-key block, batch * query head); loops over
// the query tiles that admit any of its keys and accumulates
//   accK[j] = sum_i dS(i,j) (qh[i] c),  dvh[j] = sum_i p(i,j) dO[i],
//   rsA[j]  = sum_i dS(i,j).
template <typename Tin, int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(256) bwd_dkdv_simt_kernel(
    const Tin* __restrict__ qh, const Tin* __restrict__ kh, const Tin* __restrict__ v,
    const Tin* __restrict__ dout, const float* __restrict__ AQ, const float* __restrict__ AK,
    const float* __restrict__ rowt, const float* __restrict__ colt,
    const float* __restrict__ delta, const int* __restrict__ rowlo, int window, int B, int T,
    int HQ, int H, int NB, float sc, float* __restrict__ accK, float* __restrict__ dvh,
    float* __restrict__ rsA) {
  constexpr int KC = KD / 16, VC = VD / 16;
  extern __shared__ float sm[];
  float* sKT = sm;               // [KD][SB] anchored key block, transposed
  float* sVT = sKT + KD * SB;    // [VD][SB]
  float* sQ = sVT + VD * SB;     // [SB][KD] anchored query tile times c
  float* sDO = sQ + SB * KD;     // [SB][VD]
  float* sP = sDO + SB * VD;     // [SB][SB] (query, key)
  float* sDS = sP + SB * SB;     // [SB][SB]
  float* sCv = sDS + SB * SB;    // [KD]
  float* sRow = sCv + KD;        // [SB]
  float* sDel = sRow + SB;       // [SB]
  float* sCol = sDel + SB;       // [SB]
  int* sLo = reinterpret_cast<int*>(sCol + SB);  // [SB]
  __shared__ int s_qhi;

  const int BHQ = B * HQ;
  const int kb = static_cast<int>(blockIdx.x / BHQ);  // early key blocks (most work) first
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  const int j0 = kb * SB, kblk = j0 / kBlockRows;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  for (int e = tid; e < SB * KD; e += 256) {
    const int r = e / KD, n = e % KD, t = j0 + r;
    sKT[n * SB + r] = t < T ? load1(kh + (static_cast<size_t>(bh) * T + t) * KD + n) : 0.f;
  }
  for (int e = tid; e < SB * VD; e += 256) {
    const int r = e / VD, c = e % VD, t = j0 + r;
    sVT[c * SB + r] =
        t < T ? load1(v + ((static_cast<size_t>(b) * T + t) * H + kvh) * VD + c) : 0.f;
  }
  const size_t rbase = static_cast<size_t>(bh) * NB * kBlockRows;
  if (HAS_GS && tid < SB) sCol[tid] = j0 + tid < T ? colt[rbase + j0 + tid] : 0.f;
  if (tid == 0) {
    // last query row that admits a key of this block (first admitted key is
    // non-decreasing in the row)
    const int jmax = min(j0 + SB - 1, T - 1);
    int lo = jmax, hi = T - 1;
    if (rowlo != nullptr || window > 0) {
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (row_lo(rowlo, window, mid) <= jmax) lo = mid; else hi = mid - 1;
      }
    } else {
      lo = T - 1;
    }
    s_qhi = lo;
  }
  __syncthreads();
  const int qb_hi = s_qhi / SB;

  float dk[4][KC], dv[4][VC], rs[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    rs[a] = 0.f;
#pragma unroll
    for (int m = 0; m < KC; ++m) dk[a][m] = 0.f;
#pragma unroll
    for (int m = 0; m < VC; ++m) dv[a][m] = 0.f;
  }

  for (int qb = kb; qb <= qb_hi; ++qb) {
    const int q0 = qb * SB, ablk = 2 * (q0 / (2 * kBlockRows));
    if (tid < KD)
      sCv[tid] = ex2_approx((AQ[(static_cast<size_t>(bh) * NB + ablk) * KD + tid] -
                             AK[(static_cast<size_t>(bh) * NB + kblk) * KD + tid]) * kLog2e);
    load_row_terms(tid, q0, T, rbase, rowt, delta, rowlo, window, sRow, sDel, sLo);
    __syncthreads();
    for (int e = tid; e < SB * KD; e += 256) {
      const int r = e / KD, n = e % KD, t = q0 + r;
      sQ[e] = t < T ? load1(qh + (static_cast<size_t>(bh) * T + t) * KD + n) * sCv[n] : 0.f;
    }
    for (int e = tid; e < SB * VD; e += 256) {
      const int r = e / VD, c = e % VD, t = q0 + r;
      sDO[e] = t < T ? load1(dout + ((static_cast<size_t>(b) * T + t) * HQ + hq) * VD + c) : 0.f;
    }
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_product<KD>(sQ, sKT, ty, tx, s);
    tile_product<VD>(sDO, sVT, ty, tx, dp);
    probs_and_grads<HAS_GS>(s, dp, sRow, sDel, sLo, sCol, q0, j0, T, ty, tx, sc);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      *reinterpret_cast<float4*>(sP + (ty * 4 + a) * SB + tx * 4) =
          make_float4(s[a][0], s[a][1], s[a][2], s[a][3]);
      *reinterpret_cast<float4*>(sDS + (ty * 4 + a) * SB + tx * 4) =
          make_float4(dp[a][0], dp[a][1], dp[a][2], dp[a][3]);
    }
    __syncthreads();
    // this thread's keys ty*4.., channels tx*KC.., values tx*VC..
#pragma unroll 2
    for (int r = 0; r < SB; ++r) {
      const float4 p4 = *reinterpret_cast<const float4*>(sP + r * SB + ty * 4);
      const float4 d4 = *reinterpret_cast<const float4*>(sDS + r * SB + ty * 4);
      const float pa[4] = {p4.x, p4.y, p4.z, p4.w};
      const float da[4] = {d4.x, d4.y, d4.z, d4.w};
      float qv[KC], ov[VC];
#pragma unroll
      for (int m = 0; m < KC; m += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(sQ + r * KD + tx * KC + m);
        qv[m] = t4.x; qv[m + 1] = t4.y; qv[m + 2] = t4.z; qv[m + 3] = t4.w;
      }
#pragma unroll
      for (int m = 0; m < VC; m += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(sDO + r * VD + tx * VC + m);
        ov[m] = t4.x; ov[m + 1] = t4.y; ov[m + 2] = t4.z; ov[m + 3] = t4.w;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        rs[a] += da[a];
#pragma unroll
        for (int m = 0; m < KC; ++m) dk[a][m] = fmaf(da[a], qv[m], dk[a][m]);
#pragma unroll
        for (int m = 0; m < VC; ++m) dv[a][m] = fmaf(pa[a], ov[m], dv[a][m]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int j = j0 + ty * 4 + a;
    if (j >= T) continue;
    const size_t row = static_cast<size_t>(bh) * T + j;
#pragma unroll
    for (int m = 0; m < KC; m += 4)
      *reinterpret_cast<float4*>(accK + row * KD + tx * KC + m) =
          make_float4(dk[a][m], dk[a][m + 1], dk[a][m + 2], dk[a][m + 3]);
#pragma unroll
    for (int m = 0; m < VC; m += 4)
      *reinterpret_cast<float4*>(dvh + row * VD + tx * VC + m) =
          make_float4(dv[a][m], dv[a][m + 1], dv[a][m + 2], dv[a][m + 3]);
    if (tx == 0) rsA[row] = rs[a];
  }
}

// Query-block kernel: one CTA per (64-row query block, batch * query head);
// loops over the admitted key tiles and accumulates
//   accQ[i] = sum_j dS(i,j) (kh[j] c),  rsB[i] = sum_j dS(i,j).
template <typename Tin, int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(256) bwd_dq_simt_kernel(
    const Tin* __restrict__ qh, const Tin* __restrict__ kh, const Tin* __restrict__ v,
    const Tin* __restrict__ dout, const float* __restrict__ AQ, const float* __restrict__ AK,
    const float* __restrict__ rowt, const float* __restrict__ colt,
    const float* __restrict__ delta, const int* __restrict__ rowlo, int window, int B, int T,
    int HQ, int H, int NB, float sc, float* __restrict__ accQ, float* __restrict__ rsB) {
  constexpr int KC = KD / 16;
  extern __shared__ float sm[];
  float* sQ = sm;                // [SB][KD] anchored query tile
  float* sDO = sQ + SB * KD;     // [SB][VD]
  float* sKT = sDO + SB * VD;    // [KD][SB] anchored key tile times c, transposed
  float* sK = sKT + KD * SB;     // [SB][KD] the same, row-major
  float* sVT = sK + SB * KD;     // [VD][SB]
  float* sDST = sVT + VD * SB;   // [SB][SB] dS transposed (key, query)
  float* sCv = sDST + SB * SB;   // [KD]
  float* sRow = sCv + KD;        // [SB]
  float* sDel = sRow + SB;       // [SB]
  float* sCol = sDel + SB;       // [SB]
  int* sLo = reinterpret_cast<int*>(sCol + SB);  // [SB]
  __shared__ int s_lo;

  const int nqb = (T + SB - 1) / SB;
  const int BHQ = B * HQ;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x / BHQ);  // long rows first
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  const int q0 = qb * SB, ablk = 2 * (q0 / (2 * kBlockRows));
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  const size_t rbase = static_cast<size_t>(bh) * NB * kBlockRows;
  if (tid == 0) s_lo = row_lo(rowlo, window, q0);  // rows' first keys are non-decreasing
  load_row_terms(tid, q0, T, rbase, rowt, delta, rowlo, window, sRow, sDel, sLo);
  for (int e = tid; e < SB * KD; e += 256) {
    const int r = e / KD, n = e % KD, t = q0 + r;
    sQ[e] = t < T ? load1(qh + (static_cast<size_t>(bh) * T + t) * KD + n) : 0.f;
  }
  for (int e = tid; e < SB * VD; e += 256) {
    const int r = e / VD, c = e % VD, t = q0 + r;
    sDO[e] = t < T ? load1(dout + ((static_cast<size_t>(b) * T + t) * HQ + hq) * VD + c) : 0.f;
  }
  __syncthreads();
  const int kt_hi = min(q0 + SB - 1, T - 1) / SB;
  const int kt_lo = s_lo / SB;

  float dq[4][KC], rs[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    rs[a] = 0.f;
#pragma unroll
    for (int m = 0; m < KC; ++m) dq[a][m] = 0.f;
  }

  for (int kt = kt_hi; kt >= kt_lo; --kt) {
    const int j0 = kt * SB, kblk = j0 / kBlockRows;
    if (tid < KD)
      sCv[tid] = ex2_approx((AQ[(static_cast<size_t>(bh) * NB + ablk) * KD + tid] -
                             AK[(static_cast<size_t>(bh) * NB + kblk) * KD + tid]) * kLog2e);
    if (HAS_GS && tid < SB) sCol[tid] = j0 + tid < T ? colt[rbase + j0 + tid] : 0.f;
    __syncthreads();
    for (int e = tid; e < SB * KD; e += 256) {
      const int r = e / KD, n = e % KD, t = j0 + r;
      const float x =
          t < T ? load1(kh + (static_cast<size_t>(bh) * T + t) * KD + n) * sCv[n] : 0.f;
      sK[e] = x;
      sKT[n * SB + r] = x;
    }
    for (int e = tid; e < SB * VD; e += 256) {
      const int r = e / VD, c = e % VD, t = j0 + r;
      sVT[c * SB + r] =
          t < T ? load1(v + ((static_cast<size_t>(b) * T + t) * H + kvh) * VD + c) : 0.f;
    }
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_product<KD>(sQ, sKT, ty, tx, s);
    tile_product<VD>(sDO, sVT, ty, tx, dp);
    probs_and_grads<HAS_GS>(s, dp, sRow, sDel, sLo, sCol, q0, j0, T, ty, tx, sc);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int a = 0; a < 4; ++a) rs[a] += dp[a][c];
      *reinterpret_cast<float4*>(sDST + (tx * 4 + c) * SB + ty * 4) =
          make_float4(dp[0][c], dp[1][c], dp[2][c], dp[3][c]);
    }
    __syncthreads();
#pragma unroll 2
    for (int j = 0; j < SB; ++j) {
      const float4 d4 = *reinterpret_cast<const float4*>(sDST + j * SB + ty * 4);
      const float da[4] = {d4.x, d4.y, d4.z, d4.w};
      float kv[KC];
#pragma unroll
      for (int m = 0; m < KC; m += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(sK + j * KD + tx * KC + m);
        kv[m] = t4.x; kv[m + 1] = t4.y; kv[m + 2] = t4.z; kv[m + 3] = t4.w;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < KC; ++m) dq[a][m] = fmaf(da[a], kv[m], dq[a][m]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) rs[a] += __shfl_xor_sync(0xffffffffu, rs[a], off);
    const int i = q0 + ty * 4 + a;
    if (i >= T) continue;
    const size_t row = static_cast<size_t>(bh) * T + i;
#pragma unroll
    for (int m = 0; m < KC; m += 4)
      *reinterpret_cast<float4*>(accQ + row * KD + tx * KC + m) =
          make_float4(dq[a][m], dq[a][m + 1], dq[a][m + 2], dq[a][m + 3]);
    if (tx == 0) rsB[row] = rs[a];
  }
}

// ------------------------------------------------------------------ post passes
// Bit u of `mask` (u = 1..127): a document starts at row b0 + u.
__device__ __forceinline__ void doc_start_mask(const int32_t* __restrict__ cu, int nseq, int b0,
                                               int b1, uint32_t* mask) {
  if (threadIdx.x < 4) mask[threadIdx.x] = 0u;
  __syncthreads();
  if (cu != nullptr && threadIdx.x == 0) {
    int lo = 0, hi = nseq;  // first d with cu[d] > b0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (cu[mid] > b0) hi = mid; else lo = mid + 1;
    }
    for (int d = lo; d < nseq && cu[d] < b1; ++d) {
      const int u = cu[d] - b0;
      mask[u >> 5] |= 1u << (u & 31);
    }
  }
  __syncthreads();
}

__device__ __forceinline__ bool bit_of(const uint32_t* mask, int u) {
  return (mask[u >> 5] >> (u & 31)) & 1u;
}

// Two consecutive elements (bf16: one 4-byte access; f32: one 8-byte access).
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(bf16_lo(u), bf16_hi(u));
}
__device__ __forceinline__ float2 load2(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, float2 f) {
  *reinterpret_cast<uint32_t*>(p) = pack_bf16(f.x, f.y);
}
__device__ __forceinline__ void store2(float* p, float2 f) { *reinterpret_cast<float2*>(p) = f; }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }

// The post passes split a 128-row block over 8 warps of 16 rows; a lane owns
// two adjacent channels of a 64-channel group.
constexpr int kPostRows = 16;
constexpr int kPostWarps = kBlockRows / kPostRows;
constexpr int kPostThreads = kPostWarps * 32 + 32;  // + one warp for the scalar channels

// The first document start inside the block (row > b0), or b1.
__device__ __forceinline__ int first_doc_start(const uint32_t* mask, int b0, int b1) {
#pragma unroll
  for (int w = 0; w < 4; ++w)
    if (mask[w] != 0u) return min(b1, b0 + 32 * w + __ffs(static_cast<int>(mask[w])) - 1);
  return b1;
}

// One CTA per (128-row block, batch * KV head, 64-channel group).  For every
// query head of the KV group, the block-local prefix L of g is rebuilt (each
// warp's segment sum through shared memory, then a walk down its 16 rows):
//   G[t] - AQ = L[t] (+ the first half's block sum in an odd block),
//   AK - G[t] = (block sum) - L[t].
// Writes dq (final), dG = q dq - k dk_h (over accQ) and the block's "head": the
// sum of dG from the block's first row up to the first document start inside
// the block.  dk and dv are the sums of dk_h = scale e^{AK-G} accK and of dv_h
// over the group's query heads, formed in registers and written once.  The
// last warp (channel group 0) does the gate channel (dGs = rsB - rsA, over
// rsB) and the block's sink sums.
template <typename Tin, int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(kPostThreads, 2) bwd_post_local_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ g,
    const float* __restrict__ bsum, const int32_t* __restrict__ cu, int nseq, int T, int HQ, int H,
    int NB, float scale, float* __restrict__ accQ, const float* __restrict__ accK,
    const float* __restrict__ dvh, const float* __restrict__ rsA, float* __restrict__ rsB,
    const float* __restrict__ psd, Tin* __restrict__ dq, Tin* __restrict__ dk,
    Tin* __restrict__ dv, float* __restrict__ head, float* __restrict__ sinkblk) {
  __shared__ uint32_t mask[4];
  __shared__ float2 ssum[2][kPostWarps][32];
  __shared__ float2 hred[2][kPostWarps][32];
  const int blk = blockIdx.x, z = blockIdx.z;
  const int b = blockIdx.y / H, kvh = blockIdx.y % H, grp = HQ / H;
  const int b0 = blk * kBlockRows, b1 = min(T, b0 + kBlockRows);
  doc_start_mask(cu, nseq, b0, b1, mask);
  const int fds = first_doc_start(mask, b0, b1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < kPostWarps) {
    const int u0 = b0 + warp * kPostRows;
    const int nrow = max(0, min(kPostRows, b1 - u0));
    const int n = z * 64 + 2 * lane;
    if (z * 64 < KD) {
      float2 dks[kPostRows];
#pragma unroll
      for (int r = 0; r < kPostRows; ++r) dks[r] = make_float2(0.f, 0.f);
      for (int m = 0; m < grp; ++m) {
        const int hq = kvh * grp + m, bh = b * HQ + hq;
        const Tin* grow = g + (static_cast<size_t>(b) * T * HQ + hq) * KD + n;  // row stride HQ*KD
        const size_t rs = static_cast<size_t>(HQ) * KD;
        float2 sg = make_float2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kPostRows; ++r)
          if (r < nrow) sg = add2(sg, load2(grow + (u0 + r) * rs));
        ssum[m & 1][warp][lane] = sg;
        named_bar_sync(1, kPostWarps * 32);
        float2 L = make_float2(0.f, 0.f);
        for (int w = 0; w < warp; ++w) L = add2(L, ssum[m & 1][w][lane]);
        const size_t bb = static_cast<size_t>(bh) * NB + blk;
        const float2 tot = load2(bsum + bb * KD + n);
        const float2 qoff = (blk & 1) ? load2(bsum + (bb - 1) * KD + n) : make_float2(0.f, 0.f);
        float2 hs = make_float2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kPostRows; ++r) {
          if (r < nrow) {
            const int u = u0 + r;
            const size_t iq = ((static_cast<size_t>(b) * T + u) * HQ + hq) * KD + n;
            const size_t ik = ((static_cast<size_t>(b) * T + u) * H + kvh) * KD + n;
            const size_t ia = (static_cast<size_t>(bh) * T + u) * KD + n;
            L = add2(L, load2(g + iq));
            const float2 aq = load2(accQ + ia), ak = load2(accK + ia);
            const float2 dqv = make_float2(scale * ex2_approx((qoff.x + L.x) * kLog2e) * aq.x,
                                           scale * ex2_approx((qoff.y + L.y) * kLog2e) * aq.y);
            const float2 dkv = make_float2(scale * ex2_approx((tot.x - L.x) * kLog2e) * ak.x,
                                           scale * ex2_approx((tot.y - L.y) * kLog2e) * ak.y);
            store2(dq + iq, dqv);
            const float2 qv = load2(q + iq), kv = load2(k + ik);
            const float2 dG = make_float2(qv.x * dqv.x - kv.x * dkv.x, qv.y * dqv.y - kv.y * dkv.y);
            store2(accQ + ia, dG);
            dks[r] = add2(dks[r], dkv);
            if (u < fds) hs = add2(hs, dG);
          }
        }
        hred[m & 1][warp][lane] = hs;
        named_bar_sync(1, kPostWarps * 32);
        if (warp == 0) {
          float2 h = make_float2(0.f, 0.f);
#pragma unroll
          for (int w = 0; w < kPostWarps; ++w) h = add2(h, hred[m & 1][w][lane]);
          // rows of head are KD + 1 floats: an odd row starts off an 8-byte boundary
          float* hp = head + (static_cast<size_t>(bh) * NB + blk) * (KD + 1) + n;
          hp[0] = h.x;
          hp[1] = h.y;
        }
      }
#pragma unroll
      for (int r = 0; r < kPostRows; ++r)
        if (r < nrow)
          store2(dk + ((static_cast<size_t>(b) * T + u0 + r) * H + kvh) * KD + n, dks[r]);
    }
    if (z * 64 < VD) {
#pragma unroll 4
      for (int r = 0; r < kPostRows; ++r) {
        if (r < nrow) {
          const int u = u0 + r;
          float2 s = make_float2(0.f, 0.f);
          for (int m = 0; m < grp; ++m)
            s = add2(s, load2(dvh + ((static_cast<size_t>(b) * HQ + kvh * grp + m) * T + u) * VD + n));
          store2(dv + ((static_cast<size_t>(b) * T + u) * H + kvh) * VD + n, s);
        }
      }
    }
  } else if (z == 0) {
    for (int m = 0; m < grp; ++m) {
      const int bh = b * HQ + kvh * grp + m;
      float hs = 0.f, ss = 0.f;
      for (int u = b0 + lane; u < b1; u += 32) {
        const size_t i = static_cast<size_t>(bh) * T + u;
        if (HAS_GS) {
          const float d = rsB[i] - rsA[i];
          rsB[i] = d;
          if (u < fds) hs += d;
        }
        if (psd != nullptr) ss += psd[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        hs += __shfl_xor_sync(0xffffffffu, hs, off);
        ss += __shfl_xor_sync(0xffffffffu, ss, off);
      }
      if (lane == 0) {
        head[(static_cast<size_t>(bh) * NB + blk) * (KD + 1) + KD] = hs;
        if (psd != nullptr) sinkblk[static_cast<size_t>(bh) * NB + blk] = ss;
      }
    }
  }
}

// One row of the fixed-group post pass: the row's loads for all GS heads, then
// dq, dG (over accQ) and the group's dk.
template <typename Tin, int KD, int GS>
__device__ __forceinline__ void post_row(int r, bool in_head, const Tin* __restrict__ q,
                                         const Tin* __restrict__ k, const Tin* __restrict__ g,
                                         float* __restrict__ accQ, const float* __restrict__ accK,
                                         Tin* __restrict__ dq, Tin* __restrict__ dk, size_t iq0,
                                         size_t ia0, size_t ik0, int sq, int sk, size_t sh,
                                         float scale, float2 (&L)[GS], const float2 (&tot)[GS],
                                         const float2 (&qoff)[GS], float2 (&hs)[GS]) {
  const float2 kv = load2(k + ik0 + r * sk);
  float2 dks = make_float2(0.f, 0.f);
#pragma unroll
  for (int m = 0; m < GS; ++m) {
    const size_t iq = iq0 + r * sq + m * KD, ia = ia0 + r * KD + m * sh;
    L[m] = add2(L[m], load2(g + iq));
    const float2 aq = load2(accQ + ia), ak = load2(accK + ia), qv = load2(q + iq);
    const float2 dqv = make_float2(scale * ex2_approx((qoff[m].x + L[m].x) * kLog2e) * aq.x,
                                   scale * ex2_approx((qoff[m].y + L[m].y) * kLog2e) * aq.y);
    const float2 dkv = make_float2(scale * ex2_approx((tot[m].x - L[m].x) * kLog2e) * ak.x,
                                   scale * ex2_approx((tot[m].y - L[m].y) * kLog2e) * ak.y);
    store2(dq + iq, dqv);
    const float2 dG = make_float2(qv.x * dqv.x - kv.x * dkv.x, qv.y * dqv.y - kv.y * dkv.y);
    store2(accQ + ia, dG);
    dks = add2(dks, dkv);
    if (in_head) hs[m] = add2(hs[m], dG);
  }
  store2(dk + ik0 + r * sk, dks);
}

// The same pass for a group of GS query heads known at compile time: rows
// outer, heads inner, so every row issues the group's loads together and the
// per-head prefix state stays in registers; all heads' segment offsets are
// found before the walk (one barrier), the head sums after it (one more).
template <typename Tin, int KD, int VD, bool HAS_GS, int GS>
__global__ void __launch_bounds__(kPostThreads, GS <= 4 ? 2 : 1) bwd_post_local_group_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ g,
    const float* __restrict__ bsum, const int32_t* __restrict__ cu, int nseq, int T, int HQ, int H,
    int NB, float scale, float* __restrict__ accQ, const float* __restrict__ accK,
    const float* __restrict__ dvh, const float* __restrict__ rsA, float* __restrict__ rsB,
    const float* __restrict__ psd, Tin* __restrict__ dq, Tin* __restrict__ dk,
    Tin* __restrict__ dv, float* __restrict__ head, float* __restrict__ sinkblk) {
  __shared__ uint32_t mask[4];
  __shared__ float2 red[GS][kPostWarps][32];
  const int blk = blockIdx.x, z = blockIdx.z;
  const int b = blockIdx.y / H, kvh = blockIdx.y % H;
  const int b0 = blk * kBlockRows, b1 = min(T, b0 + kBlockRows);
  doc_start_mask(cu, nseq, b0, b1, mask);
  const int fds = first_doc_start(mask, b0, b1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < kPostWarps) {
    const int u0 = b0 + warp * kPostRows;
    const int nrow = max(0, min(kPostRows, b1 - u0));
    const int n = z * 64 + 2 * lane;
    const int hq0 = kvh * GS, bh0 = b * HQ + hq0;
    if (z * 64 < KD) {
      // row u0 of head hq0; head m is + m*KD (q, g, dq) or + m*T*KD (accQ, accK)
      const size_t iq0 = ((static_cast<size_t>(b) * T + u0) * HQ + hq0) * KD + n;
      const size_t ia0 = (static_cast<size_t>(bh0) * T + u0) * KD + n;
      const size_t ik0 = ((static_cast<size_t>(b) * T + u0) * H + kvh) * KD + n;
      const int sq = HQ * KD, sk = H * KD;      // row strides
      const size_t sh = static_cast<size_t>(T) * KD;  // head stride of accQ / accK
      float2 L[GS];
#pragma unroll
      for (int m = 0; m < GS; ++m) L[m] = make_float2(0.f, 0.f);
      if (nrow == kPostRows) {
#pragma unroll
        for (int r = 0; r < kPostRows; ++r)
#pragma unroll
          for (int m = 0; m < GS; ++m) L[m] = add2(L[m], load2(g + iq0 + r * sq + m * KD));
      } else {
        for (int r = 0; r < nrow; ++r)
#pragma unroll
          for (int m = 0; m < GS; ++m) L[m] = add2(L[m], load2(g + iq0 + r * sq + m * KD));
      }
#pragma unroll
      for (int m = 0; m < GS; ++m) red[m][warp][lane] = L[m];
      named_bar_sync(1, kPostWarps * 32);
      float2 tot[GS], qoff[GS], hs[GS];
#pragma unroll
      for (int m = 0; m < GS; ++m) {
        L[m] = make_float2(0.f, 0.f);
        for (int w = 0; w < warp; ++w) L[m] = add2(L[m], red[m][w][lane]);
        const size_t bb = static_cast<size_t>(bh0 + m) * NB + blk;
        tot[m] = load2(bsum + bb * KD + n);
        qoff[m] = (blk & 1) ? load2(bsum + (bb - 1) * KD + n) : make_float2(0.f, 0.f);
        hs[m] = make_float2(0.f, 0.f);
      }
      named_bar_sync(1, kPostWarps * 32);  // red is reused for the head sums
      if (nrow == kPostRows) {  // no row past T: a guard-free walk the compiler can pipeline
        constexpr int kUnroll = GS <= 2 ? 4 : 2;
#pragma unroll kUnroll
        for (int r = 0; r < kPostRows; ++r)
          post_row<Tin, KD, GS>(r, u0 + r < fds, q, k, g, accQ, accK, dq, dk, iq0, ia0, ik0, sq, sk,
                                sh, scale, L, tot, qoff, hs);
      } else {
        for (int r = 0; r < nrow; ++r)
          post_row<Tin, KD, GS>(r, u0 + r < fds, q, k, g, accQ, accK, dq, dk, iq0, ia0, ik0, sq, sk,
                                sh, scale, L, tot, qoff, hs);
      }
#pragma unroll
      for (int m = 0; m < GS; ++m) red[m][warp][lane] = hs[m];
      named_bar_sync(1, kPostWarps * 32);
      if (warp < GS) {  // warp m sums head m's partial sums
        float2 h = make_float2(0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kPostWarps; ++w) h = add2(h, red[warp][w][lane]);
        // rows of head are KD + 1 floats: an odd row starts off an 8-byte boundary
        float* hp = head + (static_cast<size_t>(bh0 + warp) * NB + blk) * (KD + 1) + n;
        hp[0] = h.x;
        hp[1] = h.y;
      }
    }
    if (z * 64 < VD) {
      const size_t iv0 = (static_cast<size_t>(bh0) * T + u0) * VD + n;
      const size_t io0 = ((static_cast<size_t>(b) * T + u0) * H + kvh) * VD + n;
      const size_t shv = static_cast<size_t>(T) * VD;
#pragma unroll 4
      for (int r = 0; r < kPostRows; ++r) {
        if (r < nrow) {
          float2 s = make_float2(0.f, 0.f);
#pragma unroll
          for (int m = 0; m < GS; ++m) s = add2(s, load2(dvh + iv0 + r * VD + m * shv));
          store2(dv + io0 + r * (H * VD), s);
        }
      }
    }
  } else if (z == 0) {
#pragma unroll 1
    for (int m = 0; m < GS; ++m) {
      const int bh = b * HQ + kvh * GS + m;
      float hsg = 0.f, ss = 0.f;
      for (int u = b0 + lane; u < b1; u += 32) {
        const size_t i = static_cast<size_t>(bh) * T + u;
        if (HAS_GS) {
          const float d = rsB[i] - rsA[i];
          rsB[i] = d;
          if (u < fds) hsg += d;
        }
        if (psd != nullptr) ss += psd[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        hsg += __shfl_xor_sync(0xffffffffu, hsg, off);
        ss += __shfl_xor_sync(0xffffffffu, ss, off);
      }
      if (lane == 0) {
        head[(static_cast<size_t>(bh) * NB + blk) * (KD + 1) + KD] = hsg;
        if (psd != nullptr) sinkblk[static_cast<size_t>(bh) * NB + blk] = ss;
      }
    }
  }
}

// One thread per (batch * query head, channel) (channel KD: the gate): walks
// the blocks from the last, producing the carry into each block = the sum of
// dG over the later rows of the document that holds the block's last row.
template <int KD>
__global__ void __launch_bounds__(KD + 32) bwd_post_scan_kernel(
    const float* __restrict__ head, const int32_t* __restrict__ cu, int nseq, int T, int NB,
    float* __restrict__ carry) {
  const int bh = blockIdx.x, n = threadIdx.x;
  if (n > KD) return;
  float c = 0.f;
  for (int blk = NB - 1; blk >= 0; --blk) {
    const size_t i = (static_cast<size_t>(bh) * NB + blk) * (KD + 1) + n;
    carry[i] = c;
    const int b0 = blk * kBlockRows, b1 = min(T, b0 + kBlockRows);
    bool start_b0 = blk == 0, inner = false;
    if (cu != nullptr) {
      int lo = 0, hi = nseq;  // first d with cu[d] >= b0
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] >= b0) hi = mid; else lo = mid + 1;
      }
      start_b0 = cu[lo] == b0;
      const int e = start_b0 ? lo + 1 : lo;
      inner = e < nseq && cu[e] < b1;
    }
    c = start_b0 ? 0.f : head[i] + (inner ? 0.f : c);
  }
}

// One CTA per (128-row block, batch * query head, 64-channel group): the reverse
// prefix sums inside each document, dg[u] = sum of dG over rows u..(document
// end - 1).  Each warp publishes its rows' sum up to its first document start
// and whether one starts there; the carry into a warp is the block's carry
// passed back through the later warps (cut at the first of them that holds a
// document start).  The last warp (channel group 0) does the gate channel.
template <typename Tin, int KD, bool HAS_GS>
__global__ void __launch_bounds__(kPostThreads) bwd_post_final_kernel(
    const float* __restrict__ dG, const float* __restrict__ dGs, const float* __restrict__ carry,
    const int32_t* __restrict__ cu, int nseq, int T, int HQ, int NB, Tin* __restrict__ dg,
    Tin* __restrict__ dgs) {
  __shared__ uint32_t mask[4];
  __shared__ float2 hsum[kPostWarps][32];
  __shared__ int hstart[kPostWarps];
  const int blk = blockIdx.x, bh = blockIdx.y, z = blockIdx.z;
  const int b = bh / HQ, hq = bh % HQ;
  const int b0 = blk * kBlockRows, b1 = min(T, b0 + kBlockRows);
  doc_start_mask(cu, nseq, b0, b1, mask);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t cbase = (static_cast<size_t>(bh) * NB + blk) * (KD + 1);
  if (warp < kPostWarps) {
    const int u0 = b0 + warp * kPostRows;
    const int nrow = max(0, min(kPostRows, b1 - u0));
    const int n = z * 64 + 2 * lane;
    // bit r: a document starts at row u0 + r (never at b0 itself)
    const uint32_t bits = (mask[warp >> 1] >> ((warp & 1) * kPostRows)) & 0xffffu;
    float2 x[kPostRows];
#pragma unroll
    for (int r = 0; r < kPostRows; ++r)
      x[r] = r < nrow ? load2(dG + (static_cast<size_t>(bh) * T + u0 + r) * KD + n)
                      : make_float2(0.f, 0.f);
    const int first = bits != 0u ? __ffs(static_cast<int>(bits)) - 1 : kPostRows;
    float2 h = make_float2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kPostRows; ++r)
      if (r < first) h = add2(h, x[r]);
    hsum[warp][lane] = h;
    if (lane == 0) hstart[warp] = bits != 0u;
    named_bar_sync(1, kPostWarps * 32);
    float2 acc = make_float2(carry[cbase + n], carry[cbase + n + 1]);  // rows of KD + 1 floats
    for (int w = kPostWarps - 1; w > warp; --w)
      acc = hstart[w] ? hsum[w][lane] : add2(hsum[w][lane], acc);
#pragma unroll
    for (int r = kPostRows - 1; r >= 0; --r) {
      if (r < nrow) {
        acc = add2(acc, x[r]);
        store2(dg + ((static_cast<size_t>(b) * T + u0 + r) * HQ + hq) * KD + n, acc);
      }
      if ((bits >> r) & 1u) acc = make_float2(0.f, 0.f);
    }
  } else if (HAS_GS && z == 0 && lane == 0) {
    float acc = carry[cbase + KD];
    for (int u = b1 - 1; u >= b0; --u) {
      acc += dGs[static_cast<size_t>(bh) * T + u];
      store1(dgs + (static_cast<size_t>(b) * T + u) * HQ + hq, acc);
      if (u > b0 && bit_of(mask, u - b0)) acc = 0.f;
    }
  }
}

// dsink[hq] = sum over batch and blocks of the per-block sink sums (fixed order).
__global__ void __launch_bounds__(256) bwd_sink_sum_kernel(const float* __restrict__ sinkblk,
                                                           int B, int HQ, int NB,
                                                           float* __restrict__ dsink) {
  __shared__ float red[256];
  const int hq = blockIdx.x, tid = threadIdx.x;
  float s = 0.f;
  for (int i = tid; i < B * NB; i += 256) {
    const int b = i / NB, blk = i % NB;
    s += sinkblk[(static_cast<size_t>(b) * HQ + hq) * NB + blk];
  }
  red[tid] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (tid < w) red[tid] += red[tid + w];
    __syncthreads();
  }
  if (tid == 0) dsink[hq] = red[0];
}

// ------------------------------------------------------------------ launches
void record(void* ev, cudaStream_t st) {
  if (ev != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

template <typename Tin, int KD, int VD, bool HAS_GS>
cudaError_t contract_simt(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw,
                          cudaStream_t st) {
  const FwdArgs& f = a.f;
  const int* rowlo = f.cu_seqlens ? fw.rowlo : nullptr;
  const float sc = f.scale * kLog2e;
  const int nb = (f.T + SB - 1) / SB;
  const unsigned grid = static_cast<unsigned>(nb) * f.B * f.HQ;
  record(a.ev[0], st);
  cudaError_t e;
  {
    auto kern = bwd_dkdv_simt_kernel<Tin, KD, VD, HAS_GS>;
    const int smem = (2 * KD * SB + 2 * VD * SB + 2 * SB * SB + KD + 4 * SB) * 4;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 256, smem, st>>>(
        static_cast<const Tin*>(fw.qh), static_cast<const Tin*>(fw.kh),
        static_cast<const Tin*>(f.v), static_cast<const Tin*>(a.dout), fw.AQ, fw.AK, bw.rowt,
        bw.colt, bw.delta, rowlo, f.window, f.B, f.T, f.HQ, f.H, f.NB, sc, bw.accK, bw.dvh, bw.rsA);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  record(a.ev[1], st);
  {
    auto kern = bwd_dq_simt_kernel<Tin, KD, VD, HAS_GS>;
    const int smem = (3 * KD * SB + 2 * VD * SB + SB * SB + KD + 4 * SB) * 4;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 256, smem, st>>>(
        static_cast<const Tin*>(fw.qh), static_cast<const Tin*>(fw.kh),
        static_cast<const Tin*>(f.v), static_cast<const Tin*>(a.dout), fw.AQ, fw.AK, bw.rowt,
        bw.colt, bw.delta, rowlo, f.window, f.B, f.T, f.HQ, f.H, f.NB, sc, bw.accQ, bw.rsB);
    e = cudaGetLastError();
  }
  record(a.ev[2], st);
  return e;
}

template <typename Tin, int KD, int VD, bool HAS_GS>
cudaError_t launch_post_local(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw,
                              cudaStream_t st) {
  const FwdArgs& f = a.f;
  const dim3 grid(f.NB, f.B * f.H, (KD > VD ? KD : VD) / 64);  // 64-channel groups
  auto go = [&](auto kern) {
    kern<<<grid, kPostThreads, 0, st>>>(
        static_cast<const Tin*>(f.q), static_cast<const Tin*>(f.k), static_cast<const Tin*>(f.g),
        fw.bsum, f.cu_seqlens, f.num_seqs, f.T, f.HQ, f.H, f.NB, f.scale, bw.accQ, bw.accK,
        bw.dvh, bw.rsA, bw.rsB, f.sink ? bw.psd : nullptr, static_cast<Tin*>(a.dq),
        static_cast<Tin*>(a.dk), static_cast<Tin*>(a.dv), bw.head, bw.sinkblk);
    return cudaGetLastError();
  };
  switch (f.HQ / f.H) {  // query heads per KV head
    case 1: return go(bwd_post_local_group_kernel<Tin, KD, VD, HAS_GS, 1>);
    case 2: return go(bwd_post_local_group_kernel<Tin, KD, VD, HAS_GS, 2>);
    case 4: return go(bwd_post_local_group_kernel<Tin, KD, VD, HAS_GS, 4>);
    case 8: return go(bwd_post_local_group_kernel<Tin, KD, VD, HAS_GS, 8>);
    default: return go(bwd_post_local_kernel<Tin, KD, VD, HAS_GS>);
  }
}

template <typename Tin, int KD, int VD, bool HAS_GS>
cudaError_t bwd_impl(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw, cudaStream_t st) {
  const FwdArgs& f = a.f;
  const int BHQ = f.B * f.HQ;
  const long long rows = static_cast<long long>(f.B) * f.T * f.HQ;
  const long long pre_warps = (rows + 32 / (VD / 8) - 1) / (32 / (VD / 8));
  bwd_pre_kernel<Tin, VD, HAS_GS><<<static_cast<unsigned>((pre_warps * 32 + 255) / 256), 256, 0, st>>>(
      static_cast<const Tin*>(f.o), static_cast<const Tin*>(a.dout), f.lse, a.dlse, f.sink, fw.ssl,
      fw.ssa, f.B, f.T, f.HQ, f.NB, bw.rowt, bw.colt, bw.delta, f.sink ? bw.psd : nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // bf16: tensor-core contraction kernels; fp32: exact CUDA-core kernels
  e = sizeof(Tin) == 2 ? launch_bwd_tc(a, fw, bw, st) : contract_simt<Tin, KD, VD, HAS_GS>(a, fw, bw, st);
  if (e != cudaSuccess) return e;
  if ((e = launch_post_local<Tin, KD, VD, HAS_GS>(a, fw, bw, st)) != cudaSuccess) return e;
  bwd_post_scan_kernel<KD><<<BHQ, KD + 32, 0, st>>>(bw.head, f.cu_seqlens, f.num_seqs, f.T, f.NB,
                                                     bw.carry);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_post_final_kernel<Tin, KD, HAS_GS><<<dim3(f.NB, BHQ, KD / 64), kPostThreads, 0, st>>>(
      bw.accQ, bw.rsB, bw.carry, f.cu_seqlens, f.num_seqs, f.T, f.HQ, f.NB,
      static_cast<Tin*>(a.dg), static_cast<Tin*>(a.dg_scalar));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (f.sink != nullptr) {
    bwd_sink_sum_kernel<<<f.HQ, 256, 0, st>>>(bw.sinkblk, f.B, f.HQ, f.NB, a.dsink);
    e = cudaGetLastError();
  }
  return e;
}

template <typename Tin>
cudaError_t bwd_dispatch(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw,
                         cudaStream_t st) {
  const bool gs = a.f.g_scalar != nullptr;
#define WALL_BWD(KD_, VD_)                                                        \
  if (a.f.K == KD_ && a.f.V == VD_)                                               \
    return gs ? bwd_impl<Tin, KD_, VD_, true>(a, fw, bw, st)                      \
              : bwd_impl<Tin, KD_, VD_, false>(a, fw, bw, st);
  WALL_BWD(64, 64)
  WALL_BWD(64, 128)
  WALL_BWD(128, 64)
  WALL_BWD(128, 128)
#undef WALL_BWD
  return cudaErrorInvalidValue;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw, bool bf16,
                       cudaStream_t st) {
  return bf16 ? bwd_dispatch<__nv_bfloat16>(a, fw, bw, st) : bwd_dispatch<float>(a, fw, bw, st);
}

size_t bwd_workspace_layout(int B, int T, int HQ, int K, int V, bool bf16, FwdWork* fw,
                            BwdWork* bw, char* base) {
  size_t off = align256(fwd_workspace_layout(B, T, HQ, K, bf16, fw, base));
  const size_t BHQ = static_cast<size_t>(B) * HQ;
  const size_t NB = (static_cast<size_t>(T) + kBlockRows - 1) / kBlockRows;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return base ? reinterpret_cast<float*>(base + o) : nullptr;
  };
  BwdWork tmp;
  BwdWork* p = bw ? bw : &tmp;
  p->rowt = take(BHQ * NB * kBlockRows * 4);
  p->colt = take(BHQ * NB * kBlockRows * 4);
  p->delta = take(BHQ * NB * kBlockRows * 4);
  p->psd = take(BHQ * T * 4);
  p->rsA = take(BHQ * T * 4);
  p->rsB = take(BHQ * T * 4);
  p->accQ = take(BHQ * T * K * 4);
  p->accK = take(BHQ * T * K * 4);
  p->dvh = take(BHQ * T * V * 4);
  p->head = take(BHQ * NB * (K + 1) * 4);
  p->carry = take(BHQ * NB * (K + 1) * 4);
  p->sinkblk = take(BHQ * NB * 4);
  return off;
}

}  // namespace wall
