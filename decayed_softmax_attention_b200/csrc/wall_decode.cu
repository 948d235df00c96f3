// Wall attention single-step decode (Wall Attention README, "Decode") over the
// pre-rescaled cache that wall_cache.cu builds:
//   x_j = scale * sum_n q[n] k_tilde[j,n] exp2(p_curr[n] - R_{j/C}[n])
// (+ (PS_t - PS_j) ln 2 with the scalar gate's cache, the forward's Gs_t - Gs_j)
//
// The decode is a GEMV-like pass that streams k_tilde and v from HBM once.
// Grid = (split, KV head, batch); one CTA serves the HQ/H query heads that
// share a KV head, so each v row is read once for the whole group.  Inside a
// warp, lane l covers a contiguous slice of the group's concatenated k_tilde
// row (16-byte vector loads); per-head dot products are reduced with warp
// shuffles.  Each CTA writes (o, max, sum) partials per head; a combine pass
// merges the splits (warp-shuffle reductions) and adds the sink.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// ----------------------------------------------------------------- vector loads
template <typename T, int N>
__device__ __forceinline__ void load_n(const T* p, float* f);

template <int N>
__device__ __forceinline__ void load_n_bf16(const __nv_bfloat16* p, float* f) {
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 8) load8(p + i, f + i);
  } else if constexpr (N == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  } else {
    static_assert(N == 2, "unsupported vector width");
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf16_lo(u); f[1] = bf16_hi(u);
  }
}
template <int N>
__device__ __forceinline__ void load_n_f32(const float* p, float* f) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 u = *reinterpret_cast<const float4*>(p + i);
      f[i] = u.x; f[i + 1] = u.y; f[i + 2] = u.z; f[i + 3] = u.w;
    }
  } else {
    static_assert(N == 2, "unsupported vector width");
    const float2 u = *reinterpret_cast<const float2*>(p);
    f[0] = u.x; f[1] = u.y;
  }
}
template <typename T, int N>
__device__ __forceinline__ void load_n(const T* p, float* f) {
  if constexpr (sizeof(T) == 2) load_n_bf16<N>(reinterpret_cast<const __nv_bfloat16*>(p), f);
  else load_n_f32<N>(reinterpret_cast<const float*>(p), f);
}

__device__ __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store1(float* p, float x) { *p = x; }
// x rounded as store1 would store it to p's type
__device__ __forceinline__ float as_stored(const __nv_bfloat16*, float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
__device__ __forceinline__ float as_stored(const float*, float x) { return x; }
// N consecutive values in as few stores as their alignment allows (the address
// is aligned to the whole piece: 8 bytes, or N * sizeof(T) when smaller)
template <typename T, int N>
__device__ __forceinline__ void store_n(T* p, const float* f) {
  if constexpr (sizeof(T) == 2 && N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      uint2 u;
      u.x = pack_bf16(f[i], f[i + 1]);
      u.y = pack_bf16(f[i + 2], f[i + 3]);
      *reinterpret_cast<uint2*>(p + i) = u;
    }
  } else if constexpr (sizeof(T) == 2 && N % 2 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 2) *reinterpret_cast<uint32_t*>(p + i) = pack_bf16(f[i], f[i + 1]);
  } else if constexpr (sizeof(T) == 4 && N % 2 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 2) *reinterpret_cast<float2*>(p + i) = make_float2(f[i], f[i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) store1(p + i, f[i]);
  }
}

// ----------------------------------------------------------------- split-KV decode
// Rows of one (batch, KV head) are streamed through a ring of shared-memory
// stages by TMA: per stage SR rows of the group's k_tilde ([SR][G][K]), of v
// ([SR][V]) and the anchor vectors of their chunk ([G][K] fp32).  The tensor
// maps end at T_kv, so rows past the cache length arrive as zeros (and are
// masked).  One producer thread issues the copies; NW consumer warps split
// each stage's rows.  Bytes in flight = stages x stage size, independent of
// registers.
template <typename T, int KD, int VD, int G>
struct DecCfg {
  static constexpr int GK = G * KD;
  static constexpr int ESZ = static_cast<int>(sizeof(T));
  static constexpr int SR0 = 32768 / (GK * ESZ);
  static constexpr int SR = SR0 > 32 ? 32 : (SR0 < 8 ? 8 : SR0);  // rows per stage
  static constexpr int NW = 4;                                     // consumer warps
  static constexpr int RPW = SR / NW;                              // rows per warp per stage
  static constexpr int K_BYTES = SR * GK * ESZ;
  static constexpr int V_BYTES = SR * VD * ESZ;
  static constexpr int R_BYTES = GK * 4;
  // scalar-gate rows of the stage ([SR][GB] fp32: the group's heads, padded to a
  // 16-byte TMA box row), reserved in every stage, loaded only by the gated decode
  static constexpr int GB = G >= 4 ? G : 4;
  static constexpr int GT_BYTES = SR * GB * 4;
  static constexpr int LOAD_BYTES = K_BYTES + V_BYTES + R_BYTES;
  static constexpr int STAGE = LOAD_BYTES + GT_BYTES;
  static constexpr int MERGE = (NW + 1) * G * (VD + 2) * 4;  // + the fused step's new row
  static constexpr int NS0 = (225280 - MERGE) / STAGE;
  static constexpr int NS = NS0 > 4 ? 4 : NS0;                     // stages in the ring
  static constexpr int OFF_BAR = NS * STAGE;
  static constexpr int OFF_MERGE = OFF_BAR + 2 * NS * 8 + 16;
  static constexpr int SMEM = OFF_MERGE + MERGE + 128;
  static_assert(NS >= 2, "decode stage does not fit");
  static_assert(SR % NW == 0, "rows per stage must split over the consumer warps");
};

// FUSED: the step's new token (row T_b - 1 of each batch row) is not in the
// cache yet.  The stream stops before it; in the CTA whose split holds that
// row, one extra warp forms it from k_new, g_new and p_prev exactly as the
// append does (P = p_prev + g log2 e, a new chunk anchor or the stored one,
// k_tilde rounded to the cache dtype), scores it, and writes the row, its
// value, a new anchor and P_last back to the cache, all while the other warps
// stream; its (score, 1, value row) joins the CTA's merge as one more partial.
// No other CTA reads that row, that anchor or P_last, so one launch both
// appends and attends.
template <typename T, int KD, int VD, int G, bool PAGED, bool GATE, bool FUSED>
__global__ void __launch_bounds__((DecCfg<T, KD, VD, G>::NW + 2) * 32) decode_split_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __grid_constant__ CUtensorMap tmG, int gtma, const T* __restrict__ q, const float* __restrict__ p_curr, const float* __restrict__ r_cache,
    int T_kv, int HQ, int C, int cps, int nsplit, float sc, float* __restrict__ part,
    int* err, uint64_t wait_ns, int fault, const int* __restrict__ seqlens, PageMap pm,
    const float* __restrict__ gs_cache, const float* __restrict__ gs_curr, DecodeFuse fu) {
  using D = DecCfg<T, KD, VD, G>;
  constexpr int LPH = 32 / G;    // lanes per query head
  constexpr int CPL = KD / LPH;  // k_tilde channels per lane
  constexpr int VPL = VD / 32;   // v channels per lane
  extern __shared__ __align__(128) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + D::OFF_BAR);
  uint64_t* empty = full + D::NS;
  int* abort_flag = reinterpret_cast<int*>(dsm + D::OFF_BAR + 2 * D::NS * 8);
  float* sm_ml = reinterpret_cast<float*>(dsm + D::OFF_MERGE);       // [NW + 1][G][2]
  float* sm_o = sm_ml + (D::NW + 1) * G * 2;                         // [NW + 1][G][VD]

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // rows of this batch row's cache: all T_kv, or its own length (clamped to
  // [1, T_kv]); splits past the end of a shorter row hold no rows
  const int T_b = seqlens ? max(1, min(seqlens[b], T_kv)) : T_kv;
  const int nchunks = (T_b + C - 1) / C;
  const int ncap = (pm.cap + C - 1) / C;  // anchor chunks per batch row (dense caches)
  const int ck0 = s * cps;
  const int ck1 = min(ck0 + cps, nchunks);
  const int row_begin = ck0 * C;
  const int row_end = min(ck1 * C, T_b);
  const int t_new = T_b - 1;                                // FUSED: the appended row
  const int s_end = FUSED ? min(row_end, t_new) : row_end;  // rows streamed from the cache
  const int nst = s_end > row_begin ? (s_end - row_begin + D::SR - 1) / D::SR : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < D::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], D::NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, err, wait_ns};

  if (warp == D::NW) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const int slot = i % D::NS;
        if (i >= D::NS && !mbar_wait(&empty[slot], ((i / D::NS) - 1) & 1, wc)) break;
        const int row0 = row_begin + i * D::SR;
        uint8_t* st = dsm + slot * D::STAGE;
        if (!(fault == 2 && i == 0)) {  // testing hook: starve the consumers
          // a stage never straddles a cache block: it starts on a chunk
          // boundary plus a multiple of SR, and SR divides C divides the block
          const int trow = PAGED ? static_cast<int>(pm.row(b, row0)) : row0;
          const int tb = PAGED ? 0 : b;
          const size_t rslot = PAGED ? pm.chunk(b, row0, C)
                                     : static_cast<size_t>(b) * ncap + row0 / C;
          const bool gload = GATE && gtma;
          mbar_arrive_expect_tx(&full[slot], D::LOAD_BYTES + (gload ? D::GT_BYTES : 0));
          tma_load_4d(st, &tmK, &full[slot], 0, h * G, trow, tb);
          tma_load_4d(st + D::K_BYTES, &tmV, &full[slot], 0, h, trow, tb);
          bulk_load(st + D::K_BYTES + D::V_BYTES, r_cache + (rslot * HQ + h * G) * KD,
                    D::R_BYTES, &full[slot]);
          if (gload)
            tma_load_3d(st + D::LOAD_BYTES, &tmG, &full[slot], (h * G / D::GB) * D::GB, trow, tb);
        }
        issued = i + 1;
      }
      for (int i = issued > D::NS ? issued - D::NS : 0; i < issued; ++i)
        if (!(fault == 2 && i == 0)) mbar_drain(&full[i % D::NS], (i / D::NS) & 1, wait_ns);
    }
  } else {
    // ------------------------------------------------------------- consumers
    // A lane's channels of its head come in 16-byte pieces that interleave with
    // the other lanes of the head: piece j of lane l starts at channel
    // (l + LPH j) PC, so a quarter-warp's loads cover contiguous bytes.
    constexpr int PC0 = 16 / static_cast<int>(sizeof(T));
    constexpr int PC = PC0 < CPL ? PC0 : CPL;
    const int hl = lane / LPH;
    const int hq = h * G + hl;
    const int chan0 = hl * KD + (lane % LPH) * PC;  // piece j: chan0 + j * LPH * PC
    float qv[CPL], pc[CPL], qt[CPL];
#pragma unroll
    for (int j = 0; j < CPL / PC; ++j) {
      const size_t off = (static_cast<size_t>(b) * HQ + h * G) * KD + chan0 + j * LPH * PC;
      load_n<T, PC>(q + off, qv + j * PC);
      if (FUSED) {  // P of the new row, as the append forms it
        float gn[PC], pp[PC];
        load_n<T, PC>(static_cast<const T*>(fu.g_new) + off, gn);
        if (t_new > 0) load_n<float, PC>(p_curr + off, pp);
#pragma unroll
        for (int e = 0; e < PC; ++e) pc[j * PC + e] = fmaf(gn[e], kLog2e, t_new > 0 ? pp[e] : 0.f);
      } else {
        load_n<float, PC>(p_curr + off, pc + j * PC);
      }
    }
#pragma unroll
    for (int e = 0; e < CPL; ++e) qv[e] *= sc;
    if (FUSED && warp == D::NW + 1) {
      // ---- the fused step's new row, formed by a warp of its own while the
      // other warps stream the cache: its score and value enter the CTA's merge
      // as one more partial (max = its score, sum = 1, o = its value row)
      const bool mine = t_new >= row_begin && t_new < row_end;
      float d = -INFINITY;
      float vn[VPL];
#pragma unroll
      for (int c = 0; c < VPL; ++c) vn[c] = 0.f;
      if (mine) {
        const bool fresh = t_new % C == 0;  // the row opens a chunk: its anchor is its own P
        const size_t rslot = PAGED ? pm.chunk(b, t_new, C) : static_cast<size_t>(b) * ncap + t_new / C;
        float* ra = fu.r_cache + (rslot * HQ + h * G) * KD;
        const size_t prow = PAGED ? pm.row(b, t_new) : static_cast<size_t>(b) * pm.cap + t_new;
        T* kw = static_cast<T*>(fu.k_tilde) + (prow * HQ + h * G) * KD;
        const int kofs = chan0 - hl * KD;  // this lane's first channel within its head
        T* vw = static_cast<T*>(fu.v) + (prow * gridDim.y + h) * VD + lane * VPL;
        load_n<T, VPL>(static_cast<const T*>(fu.v_new) + (static_cast<size_t>(b) * gridDim.y + h) * VD +
                           lane * VPL, vn);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < CPL / PC; ++j) {
          float R[PC], kn[PC];
          if (fresh) {
#pragma unroll
            for (int e = 0; e < PC; ++e) R[e] = pc[j * PC + e];
          } else {
            load_n<float, PC>(ra + chan0 + j * LPH * PC, R);
          }
          load_n<T, PC>(static_cast<const T*>(fu.k_new) + (static_cast<size_t>(b) * gridDim.y + h) * KD +
                            kofs + j * LPH * PC, kn);
          float kt[PC];
#pragma unroll
          for (int e = 0; e < PC; ++e) {
            const int n = j * PC + e;
            if (!fresh && R[e] - pc[n] > kCacheRangeLog2) atomicOr(err, kDevErrRange);
            kt[e] = as_stored(kw, fresh ? kn[e] : kn[e] * ex2_approx(R[e] - pc[n]));  // as the cache holds it
            acc = fmaf(qv[n] * exp2f(pc[n] - R[e]), kt[e], acc);
          }
          // whole 16-byte pieces (a lane's piece is PC contiguous channels)
          store_n<T, PC>(kw + chan0 + j * LPH * PC, kt);
          if (fresh) store_n<float, PC>(ra + chan0 + j * LPH * PC, pc + j * PC);
          store_n<float, PC>(fu.p_last + (static_cast<size_t>(b) * HQ + h * G) * KD + chan0 + j * LPH * PC,
                             pc + j * PC);
        }
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        d = acc;
#pragma unroll
        for (int c = 0; c < VPL; ++c) vn[c] = as_stored(vw, vn[c]);
        store_n<T, VPL>(vw, vn);
        if (GATE && lane % LPH == 0) {  // the new row's gate prefix PS (its own term is 0)
          const size_t gi = static_cast<size_t>(b) * HQ + hq;
          const float ps = fmaf(load1(static_cast<const T*>(fu.gs_new) + gi), kLog2e,
                                t_new > 0 ? fu.gs_prev[gi] : 0.f);
          const_cast<float*>(gs_cache)[prow * HQ + hq] = ps;
          fu.gs_last[gi] = ps;
        }
      }
      if (lane % LPH == 0) {
        sm_ml[(D::NW * G + hl) * 2] = d;
        sm_ml[(D::NW * G + hl) * 2 + 1] = 1.f;
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int c = 0; c < VPL; ++c) sm_o[(D::NW * G + hh) * VD + lane * VPL + c] = vn[c];
    } else {
    // scalar gate: the logit gains PS(current row) - PS(row j), exp2 units
    // (fused: PS of the new row, from the previous row's PS and the token's g_scalar)
    float gcur = 0.f;
    if (GATE && FUSED) {
      const size_t i = static_cast<size_t>(b) * HQ + hq;
      gcur = fmaf(load1(static_cast<const T*>(fu.gs_new) + i), kLog2e,
                  t_new > 0 ? fu.gs_prev[i] : 0.f);
    } else if (GATE) {
      gcur = gs_curr[static_cast<size_t>(b) * HQ + hq];
    }
    float m = -INFINITY, l = 0.f;
    float o[G][VPL];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int c = 0; c < VPL; ++c) o[hh][c] = 0.f;
    int cur_chunk = -1;
    // scalar gate: this lane's head, the warp's rows of a stage, loaded one stage ahead
    float gnext[D::RPW];
    auto gate_load = [&](int i, float* dst) {
      const int rb = row_begin + i * D::SR, r0 = warp * D::RPW;
      const size_t prow0 = PAGED ? pm.row(b, rb) : static_cast<size_t>(b) * pm.cap + rb;
#pragma unroll
      for (int rr = 0; rr < D::RPW; ++rr)
        dst[rr] = rb + r0 + rr < row_end ? gs_cache[(prow0 + r0 + rr) * HQ + hq] : 0.f;
    };
    if (GATE && !gtma && nst > 0) gate_load(0, gnext);
    const int gcol = hq - (h * G / D::GB) * D::GB;  // this head's column of a staged gate row
    for (int i = 0; i < nst; ++i) {
      const int slot = i % D::NS;
      const bool got = mbar_wait(&full[slot], (i / D::NS) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint8_t* st = dsm + slot * D::STAGE;
      const int row0 = row_begin + i * D::SR;
      if (row0 / C != cur_chunk) {
        cur_chunk = row0 / C;
        float R[CPL];
        const float* sr = reinterpret_cast<const float*>(st + D::K_BYTES + D::V_BYTES);
#pragma unroll
        for (int j = 0; j < CPL / PC; ++j) load_n<float, PC>(sr + chan0 + j * LPH * PC, R + j * PC);
#pragma unroll
        for (int e = 0; e < CPL; ++e) qt[e] = qv[e] * exp2f(pc[e] - R[e]);
      }
      const int r0 = warp * D::RPW;
      float sres[D::RPW], vv[D::RPW][VPL], gsv[D::RPW];
      if (GATE && gtma) {  // staged with the stage's rows by the producer
        const float* sg = reinterpret_cast<const float*>(st + D::LOAD_BYTES);
#pragma unroll
        for (int rr = 0; rr < D::RPW; ++rr) gsv[rr] = sg[(r0 + rr) * D::GB + gcol];
      } else if (GATE) {
        // (a stage lies in one block of a paged cache, see the producer)
#pragma unroll
        for (int rr = 0; rr < D::RPW; ++rr) gsv[rr] = gnext[rr];
        if (i + 1 < nst) gate_load(i + 1, gnext);
      }
#pragma unroll
      for (int rr = 0; rr < D::RPW; ++rr) {
        float kf[CPL];
#pragma unroll
        for (int j = 0; j < CPL / PC; ++j)
          load_n<T, PC>(reinterpret_cast<const T*>(st) + (r0 + rr) * D::GK + chan0 + j * LPH * PC,
                        kf + j * PC);
        load_n<T, VPL>(reinterpret_cast<const T*>(st + D::K_BYTES) + (r0 + rr) * VD + lane * VPL,
                       vv[rr]);
        if ((PAGED || FUSED || seqlens != nullptr) && row0 + r0 + rr >= s_end) {
          // past the streamed rows: a row past a shorter batch row's length, a
          // paged block, or the row the fused append is about to write may hold
          // anything there (its weight is 0, but 0 x NaN is not); past T_kv of
          // a dense cache the tensor map already reads zeros
#pragma unroll
          for (int c = 0; c < VPL; ++c) vv[rr][c] = 0.f;
        }
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < CPL; ++e) d = fmaf(qt[e], kf[e], d);
        sres[rr] = d;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
      for (int rr = 0; rr < D::RPW; ++rr) {
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1)
          sres[rr] += __shfl_xor_sync(0xffffffffu, sres[rr], off);
        if (GATE) sres[rr] += gcur - gsv[rr];
        if (row0 + r0 + rr >= s_end) sres[rr] = -INFINITY;
      }
      float mloc = sres[0];
#pragma unroll
      for (int rr = 1; rr < D::RPW; ++rr) mloc = fmaxf(mloc, sres[rr]);
      const float mn = fmaxf(m, mloc);
      if (mn == -INFINITY) continue;  // every row of this warp's slice is past the end
      const float alpha = exp2f(m - mn);
      float pr[D::RPW], rs = 0.f;
#pragma unroll
      for (int rr = 0; rr < D::RPW; ++rr) {
        pr[rr] = exp2f(sres[rr] - mn);
        rs += pr[rr];
      }
      l = l * alpha + rs;
      m = mn;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float ah = __shfl_sync(0xffffffffu, alpha, hh * LPH);
#pragma unroll
        for (int c = 0; c < VPL; ++c) o[hh][c] *= ah;
#pragma unroll
        for (int rr = 0; rr < D::RPW; ++rr) {
          const float ph = __shfl_sync(0xffffffffu, pr[rr], hh * LPH);
#pragma unroll
          for (int c = 0; c < VPL; ++c) o[hh][c] = fmaf(ph, vv[rr][c], o[hh][c]);
        }
      }
    }
    if (lane % LPH == 0) {
      sm_ml[(warp * G + hl) * 2] = m;
      sm_ml[(warp * G + hl) * 2 + 1] = l;
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int c = 0; c < VPL; ++c) sm_o[(warp * G + hh) * VD + lane * VPL + c] = o[hh][c];
    }
  }
  __syncthreads();
  constexpr int NPART = D::NW + (FUSED ? 1 : 0);  // partials to merge
  // merge the consumer warps of this CTA into one partial per query head
  for (int e = threadIdx.x; e < G * (VD + 2); e += blockDim.x) {
    const int hh = e / (VD + 2), c = e % (VD + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NPART; ++w) M = fmaxf(M, sm_ml[(w * G + hh) * 2]);
    float val;
    if (M == -INFINITY) {
      val = (c == VD) ? -INFINITY : 0.f;
    } else if (c == VD) {
      val = M;
    } else {
      val = 0.f;
#pragma unroll
      for (int w = 0; w < NPART; ++w) {
        const float mw = sm_ml[(w * G + hh) * 2];
        if (mw == -INFINITY) continue;
        const float wt = exp2f(mw - M);
        val += wt * (c == VD + 1 ? sm_ml[(w * G + hh) * 2 + 1] : sm_o[(w * G + hh) * VD + c]);
      }
    }
    part[((static_cast<size_t>(b) * HQ + h * G + hh) * nsplit + s) * (VD + 2) + c] = val;
  }
}

// One warp per (batch, query head): merge the split partials, add the sink.
template <typename T, int VD>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part,
                                                             int nsplit, int nbh, int HQ,
                                                             const float* __restrict__ sink,
                                                             T* __restrict__ o,
                                                             float* __restrict__ lse) {
  constexpr int VPL = VD / 32;
  const int bhq = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bhq >= nbh) return;
  const float* pp = part + static_cast<size_t>(bhq) * nsplit * (VD + 2);
  float M = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, pp[s * (VD + 2) + VD]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float sink2 = sink ? sink[bhq % HQ] * kLog2e : -INFINITY;
  M = fmaxf(M, sink2);
  float Z = 0.f;
  for (int s = lane; s < nsplit; s += 32) {
    const float ms = pp[s * (VD + 2) + VD];
    if (ms != -INFINITY) Z += exp2f(ms - M) * pp[s * (VD + 2) + VD + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, off);
  if (sink) Z += exp2f(sink2 - M);
  float acc[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) acc[c] = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = pp[s * (VD + 2) + VD];
    if (ms == -INFINITY) continue;
    const float wt = exp2f(ms - M);
#pragma unroll
    for (int c = 0; c < VPL; ++c) acc[c] = fmaf(wt, pp[s * (VD + 2) + lane * VPL + c], acc[c]);
  }
  const float inv = 1.f / Z;
#pragma unroll
  for (int c = 0; c < VPL; ++c) store1(o + static_cast<size_t>(bhq) * VD + lane * VPL + c, acc[c] * inv);
  if (lse != nullptr && lane == 0) lse[bhq] = (M + log2f(Z)) * kLn2;
}

// The SIMT split pass (fp32 caches, 16-head groups; bf16 with smaller groups
// runs on the tensor cores, wall_split_mma.cu).
template <typename T, int KD, int VD, int G>
cudaError_t decode_split_simt(const DecodeArgs& a, cudaStream_t st) {
  using D = DecCfg<T, KD, VD, G>;
  const CUtensorMapDataType tdt =
      sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap tmK, tmV;
  // dense: [B, cap, ...] with rows limited to T_kv; paged: the pool as one
  // batch row of nblk * bs rows
  const bool paged = a.pm.paged();
  const cuuint64_t rows = paged ? static_cast<cuuint64_t>(a.pm.nblk) * a.pm.bs
                                : static_cast<cuuint64_t>(a.T_kv);
  const cuuint64_t rstride = paged ? rows : static_cast<cuuint64_t>(a.cap);
  const cuuint64_t nb = paged ? 1 : static_cast<cuuint64_t>(a.B);
  {  // k_tilde
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.HQ), rows,
                                nb};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(KD) * sizeof(T),
                                   static_cast<cuuint64_t>(a.HQ) * KD * sizeof(T),
                                   rstride * a.HQ * KD * sizeof(T)};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(KD), static_cast<cuuint32_t>(G),
                               static_cast<cuuint32_t>(D::SR), 1};
    if (!encode_tiled(&tmK, tdt, 4, a.k_tilde, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  {  // v
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(a.H), rows,
                                nb};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(VD) * sizeof(T),
                                   static_cast<cuuint64_t>(a.H) * VD * sizeof(T),
                                   rstride * a.H * VD * sizeof(T)};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(VD), 1, static_cast<cuuint32_t>(D::SR), 1};
    if (!encode_tiled(&tmV, tdt, 4, a.v, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  const bool gate = a.gs_cache != nullptr;
  const bool fused = a.fuse.k_new != nullptr;
  if (gate && fused && a.fuse.gs_new == nullptr) return cudaErrorInvalidValue;
  // scalar-gate rows through the stage ring when a gate-cache row is a whole number
  // of 16-byte pieces (HQ % 4 == 0); otherwise each lane loads its rows itself
  CUtensorMap tmG = tmK;
  int gtma = 0;
  if (gate && a.HQ % 4 == 0) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.HQ), rows, nb};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.HQ) * 4,
                                   rstride * a.HQ * 4};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(D::GB), static_cast<cuuint32_t>(D::SR), 1};
    if (!encode_tiled(&tmG, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.gs_cache, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    gtma = 1;
  }
  auto kern = fused ? (paged ? (gate ? decode_split_kernel<T, KD, VD, G, true, true, true>
                                     : decode_split_kernel<T, KD, VD, G, true, false, true>)
                             : (gate ? decode_split_kernel<T, KD, VD, G, false, true, true>
                                     : decode_split_kernel<T, KD, VD, G, false, false, true>))
              : paged ? (gate ? decode_split_kernel<T, KD, VD, G, true, true, false>
                              : decode_split_kernel<T, KD, VD, G, true, false, false>)
                      : (gate ? decode_split_kernel<T, KD, VD, G, false, true, false>
                              : decode_split_kernel<T, KD, VD, G, false, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM);
  if (e != cudaSuccess) return e;
  const int nchunks = (a.T_kv + a.chunk - 1) / a.chunk;
  const int cps = (nchunks + a.nsplit - 1) / a.nsplit;
  dim3 grid(a.nsplit, a.H, a.B);
  kern<<<grid, (D::NW + (fused ? 2 : 1)) * 32, D::SMEM, st>>>(
      tmK, tmV, tmG, gtma, static_cast<const T*>(a.q), a.p_curr, a.r_cache, a.T_kv, a.HQ, a.chunk,
      cps, a.nsplit, a.scale * kLog2e, a.part, a.err, a.wait_ns, a.fault, a.seqlens, a.pm,
      a.gs_cache, a.gs_curr, a.fuse);
  return cudaGetLastError();
}

template <typename T, int KD, int VD, int G>
cudaError_t decode_impl(const DecodeArgs& a, cudaStream_t st) {
  cudaError_t e;
  if constexpr (sizeof(T) == 2 && G <= 8) {
    e = launch_decode_mma<KD, VD, G>(a, st);
  } else {
    e = decode_split_simt<T, KD, VD, G>(a, st);
  }
  if (e != cudaSuccess) return e;
  if (a.mid_event != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.mid_event), st);
  const int nbh = a.B * a.HQ;
  decode_combine_kernel<T, VD><<<(nbh + 3) / 4, 128, 0, st>>>(a.part, a.nsplit, nbh, a.HQ, a.sink,
                                                             static_cast<T*>(a.o), a.lse);
  return cudaGetLastError();
}

template <typename T, int KD, int VD>
cudaError_t decode_by_group(const DecodeArgs& a, cudaStream_t st) {
  switch (a.HQ / a.H) {
    case 1: return decode_impl<T, KD, VD, 1>(a, st);
    case 2: return decode_impl<T, KD, VD, 2>(a, st);
    case 4: return decode_impl<T, KD, VD, 4>(a, st);
    case 8: return decode_impl<T, KD, VD, 8>(a, st);
    case 16: return decode_impl<T, KD, VD, 16>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t decode_by_dims(const DecodeArgs& a, cudaStream_t st) {
  if (a.K == 64 && a.V == 64) return decode_by_group<T, 64, 64>(a, st);
  if (a.K == 64 && a.V == 128) return decode_by_group<T, 64, 128>(a, st);
  if (a.K == 128 && a.V == 64) return decode_by_group<T, 128, 64>(a, st);
  if (a.K == 128 && a.V == 128) return decode_by_group<T, 128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_supported(int K, int V, int group) {
  const bool kv = (K == 64 || K == 128) && (V == 64 || V == 128);
  const bool g = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
  return kv && g;
}

// Upper bound on the split count (sizes the workspace): enough CTAs for several
// full waves over the SMs, never more splits than chunks.  Non-decreasing in T_kv.
int decode_max_splits(int B, int T_kv, int HQ, int H, int chunk) {
  (void)HQ;
  const long nchunks = (static_cast<long>(T_kv) + chunk - 1) / chunk;
  const long target = 148L * 16;
  const long groups = static_cast<long>(B) * H;
  long ns = (target + groups - 1) / groups;
  if (ns < 1) ns = 1;
  if (ns > nchunks) ns = nchunks;
  return static_cast<int>(ns);
}

// Splits actually launched (ctas_per_sm CTAs of the split pass are resident on
// an SM): the count up to the bound whose CTAs fill the last wave best,
// preferring fewer splits; chunks are dealt out evenly so no split is empty.
int decode_num_splits(int B, int T_kv, int HQ, int H, int chunk, int ctas_per_sm) {
  const int ns_max = decode_max_splits(B, T_kv, HQ, H, chunk);
  const int nchunks = (T_kv + chunk - 1) / chunk;
  const long groups = static_cast<long>(B) * H;
  const long sms = 148L * (ctas_per_sm > 0 ? ctas_per_sm : 1);
  int best = 1;
  double best_eff = -1.0;
  for (int ns = 1; ns <= ns_max; ++ns) {
    const int cps = (nchunks + ns - 1) / ns;
    const int used = (nchunks + cps - 1) / cps;
    const long ctas = groups * used;
    const long waves = (ctas + sms - 1) / sms;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * sms);
    const double score = eff * (ctas >= sms ? 1.0 : static_cast<double>(ctas) / sms);
    if (score > best_eff + 0.02) {
      best_eff = score;
      best = used;
    }
  }
  return best;
}

size_t decode_workspace_bytes(int B, int HQ, int V, int nsplit) {
  return static_cast<size_t>(B) * HQ * nsplit * (V + 2) * sizeof(float);
}

cudaError_t launch_decode_combine(const float* part, int nsplit, int nbh, int HQ,
                                  const float* sink, void* o, float* lse, int V, bool bf16,
                                  cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((nbh + 3) / 4);
  if (V != 64 && V != 128) return cudaErrorInvalidValue;
  if (bf16) {
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
    if (V == 64)
      decode_combine_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(part, nsplit, nbh, HQ, sink, ob, lse);
    else
      decode_combine_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(part, nsplit, nbh, HQ, sink, ob, lse);
  } else {
    float* of = static_cast<float*>(o);
    if (V == 64)
      decode_combine_kernel<float, 64><<<grid, 128, 0, st>>>(part, nsplit, nbh, HQ, sink, of, lse);
    else
      decode_combine_kernel<float, 128><<<grid, 128, 0, st>>>(part, nsplit, nbh, HQ, sink, of, lse);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? decode_by_dims<__nv_bfloat16>(a, st) : decode_by_dims<float>(a, st);
}

}  // namespace wall
