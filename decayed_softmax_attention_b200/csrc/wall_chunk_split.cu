// Wall attention for a chunk of a few new tokens per sequence (multi-token
// decode, e.g. speculative verification) against the decode cache, in the
// split-KV style of the single-token decode (wall_decode.cu); longer chunks go
// to the tensor-core query tiles of wall_chunk_tc.cu.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// N consecutive elements as floats (N = 2, 4 or a multiple of 8).
template <int N>
__device__ __forceinline__ void load_n(const __nv_bfloat16* p, float* f) {
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 8) load8(p + i, f + i);
  } else if constexpr (N == 4) {
    load4(p, f);
  } else {
    static_assert(N == 2, "unsupported vector width");
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf16_lo(u); f[1] = bf16_hi(u);
  }
}
template <int N>
__device__ __forceinline__ void load_n(const float* p, float* f) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) load4(p + i, f + i);
  } else {
    static_assert(N == 2, "unsupported vector width");
    const float2 u = *reinterpret_cast<const float2*>(p);
    f[0] = u.x; f[1] = u.y;
  }
}
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

// ----------------------------------------------------------------- few-token chunks
// A chunk of M new tokens per sequence (multi-token decode, e.g. speculative
// verification) attends the cache the decode's way when M is small: a
// 128-row tensor-core query tile would be nearly all padding, while the work
// is a stream of the cache with a few dot products per row.  Grid =
// (split x token group, KV head, batch); one CTA streams its rows' k_tilde
// and v once for the G query heads and MQ = 16 / G tokens of its group.
// The queries arrive anchored, qh_i = q_i exp2(P_i - AQ) with AQ = P just
// before the chunk, so token i's score of cache row j is
//   scale * sum_n qh_i[n] exp2(AQ[n] - R_{j/C}[n]) k_tilde[j, n]
// — the single-token decode's formula with p_curr = AQ (Wall Attention README,
// "Decode"), masked to j <= t0 + i (and the window).
//
// Per group of RB rows a warp forms NV = MQ * RB scores per head, split over
// the head's LPH lanes; a butterfly reduce-scatter leaves each lane the full
// sums of NV / LPH of them (instead of every lane reducing all NV), the owner
// lanes run the online softmax for their token, and the probabilities reach
// the value accumulators through shared memory (each lane holds V / 32
// channels of o for every head and token).  Per-lane state: queries
// MQ * CPL = KD / 2 floats, accumulators MQ * G * VD / 32 = VD / 2 floats.
//
// fp32 caches take the same pass for chunks of any length (there is no fp32
// tensor-core tile): each CTA then stops at its token group's last causal row
// and starts at its first token's window, and reads the anchor AQ of the
// group's 256-row query block.
template <int KD, int VD, int G, int ES>
struct MultiCfg {
  static constexpr int MQ = 16 / G;  // tokens per CTA
  static constexpr int LPH = 32 / G;
  static constexpr int CPL = KD / LPH;
  static constexpr int VPL = VD / 32;
  static constexpr int GK = G * KD;
  static constexpr int SR0 = 32768 / (GK * ES);
  static constexpr int SR = SR0 > 32 ? 32 : (SR0 < 8 ? 8 : SR0);  // rows per stage
  static constexpr int NW = 8;                                     // consumer warps
  static constexpr int RPW = SR / NW;                              // rows per warp per stage
  static constexpr int RB = RPW < G ? RPW : G;                     // rows per softmax group
  static constexpr int NV = MQ * RB;                               // scores per head per group
  static constexpr int NO = NV >= LPH ? NV / LPH : 1;              // sums a lane owns
  static constexpr int REP = NV >= LPH ? 1 : LPH / NV;             // lanes holding each sum
  static constexpr int TSPAN = RB / NO;                            // owners per token
  static constexpr int K_BYTES = SR * GK * ES;
  static constexpr int V_BYTES = SR * VD * ES;
  static constexpr int R_BYTES = GK * 4;
  static constexpr int STAGE = K_BYTES + V_BYTES + R_BYTES;
  static constexpr int NS0 = 172032 / STAGE;
  static constexpr int NS = NS0 > 4 ? 4 : NS0;  // stages in the ring
  static constexpr int RING = NS * STAGE;
  static constexpr int MERGE = NW * MQ * G * (VD + 2) * 4;  // overlays the ring after the loop
  static constexpr int BODY = RING > MERGE ? RING : MERGE;
  static constexpr int OFF_Q = BODY;                       // [MQ][CPL][32] fp32, scaled queries
  static constexpr int OFF_AQ = OFF_Q + MQ * GK * 4;       // [CPL][32] fp32 (GK = 32 CPL)
  static constexpr int OFF_P = OFF_AQ + GK * 4;            // [NW][RB + 1][MQ * G] fp32
  static constexpr int OFF_BAR = OFF_P + NW * (RB + 1) * MQ * G * 4;
  static constexpr int SMEM = OFF_BAR + 2 * NS * 8 + 16 + 128;
  static_assert(NS >= 2, "stage does not fit");
  static_assert(SR % NW == 0 && RPW % RB == 0, "rows must split over warps and groups");
  static_assert(NO <= RB && RB % NO == 0, "a lane's sums must belong to one token");
  static_assert(CPL % 2 == 0 && MQ * G % 4 == 0, "packed fp32 pairs");
};

// Sum N values over aligned groups of W lanes (partners xor W/2 .. 1) and
// scatter the sums: lane l (mod W) ends with max(1, N / W) of them, starting at
// index l * (N / W) (N >= W) or l / (W / N) (N < W, each sum held by W / N
// lanes).  Each step sends the half a lane gives away and adds the partner's
// copy of the half it keeps.
template <int N, int W>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
  if constexpr (W > 1) {
    if constexpr (N >= 2) {
      constexpr int HALF = N / 2;
      const bool up = (lane & (W / 2)) != 0;
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const float send = up ? v[i] : v[HALF + i];
        const float keep = up ? v[HALF + i] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, W / 2);
      }
      reduce_scatter<HALF, W / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], W / 2);
      reduce_scatter<1, W / 2>(v, lane);
    }
  }
}

template <int KD, int VD, int G, typename T>
__global__ void __launch_bounds__((MultiCfg<KD, VD, G, sizeof(T)>::NW + 1) * 32, 1)
    chunk_split_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const T* __restrict__ qh,
                       const float* __restrict__ AQ, const float* __restrict__ r_cache, int t0,
                       int M, int HQ, int C, int cap, int window, int ck_lo, int cps, int nsplit,
                       int ntg, float sc, float* __restrict__ part, int* err, uint64_t wait_ns,
                       const int* __restrict__ wide, int fault,
                       const float* __restrict__ gs_cache) {
  using D = MultiCfg<KD, VD, G, sizeof(T)>;
  constexpr int MQ = D::MQ, LPH = D::LPH, CPL = D::CPL, VPL = D::VPL, RB = D::RB, NV = D::NV;
  constexpr int NO = D::NO, REP = D::REP, MG = MQ * G;
  // channels per k_tilde load; a lane's pieces interleave with the other lanes
  // of its head (piece j of lane l starts at channel (l + LPH j) PC), so each
  // quarter-warp's 16-byte loads cover 128 contiguous bytes (no bank conflicts)
  constexpr int PW = 16 / static_cast<int>(sizeof(T));
  constexpr int PC = CPL < PW ? CPL : PW;
  extern __shared__ __align__(128) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + D::OFF_BAR);
  uint64_t* empty = full + D::NS;
  int* abort_flag = reinterpret_cast<int*>(dsm + D::OFF_BAR + 2 * D::NS * 8);
  float* sQ = reinterpret_cast<float*>(dsm + D::OFF_Q);
  float* sAQ = reinterpret_cast<float*>(dsm + D::OFF_AQ);

  const int s = blockIdx.x / ntg, tg = blockIdx.x % ntg, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T_b = t0 + M;  // cache rows after the chunk's append
  const int nchunks = (T_b + C - 1) / C;
  const int ncap = (cap + C - 1) / C;
  const int ck0 = ck_lo + s * cps;
  const int ck1 = min(ck0 + cps, nchunks);
  const int m0 = tg * MQ;  // first token of this CTA's group
  const int qb = m0 >> 8;  // its 256-row query block (MQ divides 256)
  // rows the group can see: up to its last token's row, from its first token's
  // window on (chunk-aligned, so every stage stays inside one anchor chunk)
  const int lo_g = window > 0 ? max(0, t0 + m0 + 1 - window) / C * C : 0;
  const int row_begin = max(ck0 * C, lo_g);
  const int row_end = min(min(ck1 * C, T_b), t0 + min(m0 + MQ, M));
  const int nst = row_end > row_begin ? (row_end - row_begin + D::SR - 1) / D::SR : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < D::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], D::NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the group's queries (scaled, fp32; zero past the chunk's last token) and AQ,
  // lane-major: element e of lane L's channels at [e][L] (queries [m][e][L]), so the
  // warp's loads of one element are 32 consecutive words (no bank conflicts)
  for (int idx = threadIdx.x; idx < MQ * CPL * 32; idx += (D::NW + 1) * 32) {
    const int L = idx & 31, m = (idx >> 5) / CPL, e = (idx >> 5) % CPL;
    const int n = (L % LPH) * PC + (e / PC) * LPH * PC + e % PC;  // channel within the head
    const size_t bh = static_cast<size_t>(b) * HQ + h * G + L / LPH;
    sQ[idx] = m0 + m < M ? sc * to_f32(qh[(bh * M + m0 + m) * KD + n]) : 0.f;
  }
  const int NQB = (M + 255) >> 8;
  for (int idx = threadIdx.x; idx < CPL * 32; idx += (D::NW + 1) * 32) {
    const int L = idx & 31, e = idx >> 5;
    const int n = (L % LPH) * PC + (e / PC) * LPH * PC + e % PC;
    sAQ[idx] = AQ[((static_cast<size_t>(b) * HQ + h * G + L / LPH) * NQB + qb) * KD + n];
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
        if (!(fault == 7 && i == 0)) {  // testing hook: starve the consumers
          mbar_arrive_expect_tx(&full[slot], D::STAGE);
          tma_load_4d(st, &tmK, &full[slot], 0, h * G, row0, b);
          tma_load_4d(st + D::K_BYTES, &tmV, &full[slot], 0, h, row0, b);
          bulk_load(st + D::K_BYTES + D::V_BYTES,
                    r_cache + ((static_cast<size_t>(b) * ncap + row0 / C) * HQ + h * G) * KD,
                    D::R_BYTES, &full[slot]);
        }
        issued = i + 1;
      }
      for (int i = issued > D::NS ? issued - D::NS : 0; i < issued; ++i)
        if (!(fault == 7 && i == 0)) mbar_drain(&full[i % D::NS], (i / D::NS) & 1, wait_ns);
    }
  }
  float mrun = -INFINITY, lpart = 0.f;  // the owned token's running max, partial sum
  // o of (token, head) pairs k = 2 kp, 2 kp + 1 (index m * G + hh), this lane's channels
  float2 o2[MG / 2][VPL];
#pragma unroll
  for (int kp = 0; kp < MG / 2; ++kp)
#pragma unroll
    for (int c = 0; c < VPL; ++c) o2[kp][c] = make_float2(0.f, 0.f);
  const int hl = lane / LPH, l = lane % LPH;
  const int chan0 = hl * KD + l * PC;  // channel of piece j: chan0 + j * LPH * PC
  // Strong decay inside the group's 256-row query block: this head's rows of
  // that block are left to the diagonal kernel (masked here, factors kept finite).
  const int qrow0 = t0 + (qb << 8);  // cache row of the block's first token
  const bool wide_h = wide[(static_cast<size_t>(b) * HQ + h * G + hl) * NQB + qb] != 0;
  const int row_cap = wide_h ? qrow0 - 1 : 0x7fffffff;
  const int base = NV >= LPH ? l * NO : l / REP;  // first owned score index (token-major)
  const int m_own = base / RB;                    // this lane's token
  if (warp < D::NW) {
    // ------------------------------------------------------------- consumers
    // scalar gate: the logit gains PS(token's row) - PS(key row), log2 units
    const size_t gsb = static_cast<size_t>(b) * cap;
    const int ghq = h * G + hl;
    const float gs_tok = (gs_cache != nullptr && m0 + m_own < M)
                             ? gs_cache[(gsb + t0 + m0 + m_own) * HQ + ghq] : 0.f;
    float* pb = reinterpret_cast<float*>(dsm + D::OFF_P) + warp * (RB + 1) * MG;  // [RB][MG]
    float* ab = pb + RB * MG;                                                     // [MG]
    float2 qt2[MQ][CPL / 2];
    int cur_chunk = -1;
    const int mg_own = m0 + m_own;
    for (int i = 0; i < nst; ++i) {
      const int slot = i % D::NS;
      const bool got = mbar_wait(&full[slot], (i / D::NS) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint8_t* st = dsm + slot * D::STAGE;
      const int row0 = row_begin + i * D::SR;
      if (row0 / C != cur_chunk) {  // q_t = q exp2(AQ - R_c) for this chunk's anchor
        cur_chunk = row0 / C;
        const float* R = reinterpret_cast<const float*>(st + D::K_BYTES + D::V_BYTES);
#pragma unroll
        for (int e = 0; e < CPL; e += 2) {
          const int n = chan0 + (e / PC) * LPH * PC + e % PC;
          const float2 r2 = *reinterpret_cast<const float2*>(R + n);
          const bool own = wide_h && cur_chunk * C >= qrow0;
          const float2 f = own ? make_float2(0.f, 0.f)
                               : make_float2(exp2f(sAQ[e * 32 + lane] - r2.x),
                                             exp2f(sAQ[(e + 1) * 32 + lane] - r2.y));
#pragma unroll
          for (int m = 0; m < MQ; ++m)
            qt2[m][e / 2] = __fmul2_rn(
                make_float2(sQ[(m * CPL + e) * 32 + lane], sQ[(m * CPL + e + 1) * 32 + lane]), f);
        }
      }
      const T* sk = reinterpret_cast<const T*>(st);
      const T* sv = reinterpret_cast<const T*>(st + D::K_BYTES);
#pragma unroll 1
      for (int gq = 0; gq < D::RPW / RB; ++gq) {
        const int rg0 = warp * D::RPW + gq * RB;  // first row of the group within the stage
        float v[NV];
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
          float2 acc[MQ];
#pragma unroll
          for (int m = 0; m < MQ; ++m) acc[m] = make_float2(0.f, 0.f);
#pragma unroll
          for (int e0 = 0; e0 < CPL; e0 += PC) {
            float kf[PC];
            load_n<PC>(sk + (rg0 + rb) * D::GK + chan0 + (e0 / PC) * LPH * PC, kf);
#pragma unroll
            for (int e = 0; e < PC; e += 2)
#pragma unroll
              for (int m = 0; m < MQ; ++m)
                acc[m] = __ffma2_rn(qt2[m][(e0 + e) / 2], make_float2(kf[e], kf[e + 1]), acc[m]);
          }
#pragma unroll
          for (int m = 0; m < MQ; ++m) v[m * RB + rb] = acc[m].x + acc[m].y;
        }
        reduce_scatter<NV, LPH>(v, lane);
        // owned sums: token m_own, rows rb = base % RB + j; mask, then online softmax
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NO; ++j) {
          const int row = row0 + rg0 + (base % RB) + j;
          const bool ok = mg_own < M && row < row_end && row <= t0 + mg_own && row <= row_cap &&
                          (window == 0 || t0 + mg_own - row < window);
          const float gterm = (gs_cache != nullptr && ok) ? gs_tok - gs_cache[(gsb + row) * HQ + ghq]
                                                          : 0.f;
          v[j] = ok ? v[j] + gterm : -INFINITY;
          mx = fmaxf(mx, v[j]);
        }
#pragma unroll
        for (int off = REP; off < REP * D::TSPAN; off <<= 1)
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mn = fmaxf(mrun, mx);
        const bool grow = mn > mrun;
        const float alpha = grow ? exp2f(mrun - mn) : 1.f;
        float ps = 0.f;
#pragma unroll
        for (int j = 0; j < NO; ++j) {
          const float p = mn == -INFINITY ? 0.f : exp2f(v[j] - mn);
          pb[((base % RB) + j) * MG + m_own * G + hl] = p;
          ps += p;
        }
        lpart = lpart * alpha + ps;
        mrun = mn;
        ab[m_own * G + hl] = alpha;
        const bool any_grow = __any_sync(0xffffffffu, grow);
        __syncwarp();
        if (any_grow) {
#pragma unroll
          for (int k = 0; k < MG; k += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(ab + k);
#pragma unroll
            for (int c = 0; c < VPL; ++c) {
              o2[k / 2][c] = __fmul2_rn(o2[k / 2][c], make_float2(a4.x, a4.y));
              o2[k / 2 + 1][c] = __fmul2_rn(o2[k / 2 + 1][c], make_float2(a4.z, a4.w));
            }
          }
        }
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
          float vf[VPL];
          load_n<VPL>(sv + (rg0 + rb) * VD + lane * VPL, vf);
#pragma unroll
          for (int k = 0; k < MG; k += 4) {
            const float4 p4 = *reinterpret_cast<const float4*>(pb + rb * MG + k);
#pragma unroll
            for (int c = 0; c < VPL; ++c) {
              const float2 vd = make_float2(vf[c], vf[c]);
              o2[k / 2][c] = __ffma2_rn(make_float2(p4.x, p4.y), vd, o2[k / 2][c]);
              o2[k / 2 + 1][c] = __ffma2_rn(make_float2(p4.z, p4.w), vd, o2[k / 2 + 1][c]);
            }
          }
        }
        __syncwarp();  // before the next group's writes to pb / ab
      }
      if (lane == 0) mbar_arrive(&empty[slot]);  // the stage is no longer read
    }
    // each token's sum over its owner lanes (replicas hold the same partial)
#pragma unroll
    for (int off = REP; off < REP * D::TSPAN; off <<= 1)
      lpart += __shfl_xor_sync(0xffffffffu, lpart, off);
  }
  __syncthreads();  // the ring is free: the merge area overlays it
  float* sm_ml = reinterpret_cast<float*>(dsm);  // [NW][MG][2]
  float* sm_o = sm_ml + D::NW * MG * 2;          // [NW][MG][VD]
  if (warp < D::NW) {
    if (l % (REP * D::TSPAN) == 0) {
      sm_ml[(warp * MG + m_own * G + hl) * 2] = mrun;
      sm_ml[(warp * MG + m_own * G + hl) * 2 + 1] = lpart;
    }
#pragma unroll
    for (int kp = 0; kp < MG / 2; ++kp)
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        sm_o[(warp * MG + 2 * kp) * VD + lane * VPL + c] = o2[kp][c].x;
        sm_o[(warp * MG + 2 * kp + 1) * VD + lane * VPL + c] = o2[kp][c].y;
      }
  }
  __syncthreads();
  // merge the consumer warps into one partial per (token, query head)
  for (int e = threadIdx.x; e < MG * (VD + 2); e += (D::NW + 1) * 32) {
    const int k = e / (VD + 2), c = e % (VD + 2);
    const int m = k / G, hh = k % G;
    if (m0 + m >= M) continue;
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < D::NW; ++w) Mx = fmaxf(Mx, sm_ml[(w * MG + k) * 2]);
    float val;
    if (Mx == -INFINITY) {
      val = (c == VD) ? -INFINITY : 0.f;
    } else if (c == VD) {
      val = Mx;
    } else {
      val = 0.f;
#pragma unroll
      for (int w = 0; w < D::NW; ++w) {
        const float mw = sm_ml[(w * MG + k) * 2];
        if (mw == -INFINITY) continue;
        const float wt = exp2f(mw - Mx);
        val += wt * (c == VD + 1 ? sm_ml[(w * MG + k) * 2 + 1] : sm_o[(w * MG + k) * VD + c]);
      }
    }
    const size_t row = (static_cast<size_t>(b) * M + m0 + m) * HQ + h * G + hh;
    part[(row * nsplit + s) * (VD + 2) + c] = val;
  }
}

// Splits per (token group, KV head, batch row): the decode's bound with every
// token group counted as a batch row of its own.
int chunk_max_splits(int B, int M, int cap, int HQ, int H, int chunk) {
  const int ntg = (M + 16 / (HQ / H) - 1) / (16 / (HQ / H));
  const long groups = static_cast<long>(B) * ntg;
  return decode_max_splits(groups > 0x7fffffffL ? 0x7fffffff : static_cast<int>(groups), cap, HQ,
                           H, chunk);
}

template <int KD, int VD, int G, typename T>
cudaError_t chunk_split_impl(const ChunkArgs& a, const void* qh, const float* AQ, const int* wide,
                             float* lse, float* part, cudaStream_t st) {
  using D = MultiCfg<KD, VD, G, sizeof(T)>;
  constexpr CUtensorMapDataType TD =
      sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  constexpr cuuint64_t ES = sizeof(T);
  const int T_b = a.t0 + a.M;
  // chunks wholly before the first token's window are skipped
  const int lo = a.window > 0 ? (a.t0 + 1 - a.window > 0 ? a.t0 + 1 - a.window : 0) : 0;
  const int ck_lo = lo / a.chunk;
  const int nch = (T_b + a.chunk - 1) / a.chunk - ck_lo;
  const int ntg = (a.M + D::MQ - 1) / D::MQ;
  int ns = decode_num_splits(a.B * ntg, nch * a.chunk, a.HQ, a.H, a.chunk,
                             decode_ctas_per_sm(KD, VD, G, sizeof(T) == 2));
  const int ns_cap = chunk_max_splits(a.B, a.M, a.cap, a.HQ, a.H, a.chunk);
  if (ns > ns_cap) ns = ns_cap;
  const int cps = (nch + ns - 1) / ns;
  const int nsplit = (nch + cps - 1) / cps;
  cudaError_t e;
  if constexpr (sizeof(T) == 2 && G <= 8) {
    e = launch_chunk_mma<KD, VD, G>(a, qh, AQ, wide, part, ck_lo, cps, nsplit, ntg, st);
  } else {
    CUtensorMap tmK, tmV;
    // the maps end at the chunk's last row: rows past it arrive as zeros
    const cuuint64_t rows = static_cast<cuuint64_t>(a.t0) + a.M;
    {
      const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.HQ), rows,
                                  static_cast<cuuint64_t>(a.B)};
      const cuuint64_t strides[3] = {static_cast<cuuint64_t>(KD) * ES,
                                     static_cast<cuuint64_t>(a.HQ) * KD * ES,
                                     static_cast<cuuint64_t>(a.cap) * a.HQ * KD * ES};
      const cuuint32_t box[4] = {static_cast<cuuint32_t>(KD), static_cast<cuuint32_t>(G),
                                 static_cast<cuuint32_t>(D::SR), 1};
      if (!encode_tiled(&tmK, TD, 4, a.k_tilde, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    }
    {
      const cuuint64_t dims[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(a.H), rows,
                                  static_cast<cuuint64_t>(a.B)};
      const cuuint64_t strides[3] = {static_cast<cuuint64_t>(VD) * ES,
                                     static_cast<cuuint64_t>(a.H) * VD * ES,
                                     static_cast<cuuint64_t>(a.cap) * a.H * VD * ES};
      const cuuint32_t box[4] = {static_cast<cuuint32_t>(VD), 1, static_cast<cuuint32_t>(D::SR), 1};
      if (!encode_tiled(&tmV, TD, 4, a.v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    }
    auto kern = chunk_split_kernel<KD, VD, G, T>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit * ntg, a.H, a.B);
    if (a.ev_mid != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_mid), st);
    kern<<<grid, (D::NW + 1) * 32, D::SMEM, st>>>(
        tmK, tmV, static_cast<const T*>(qh), AQ, a.r_cache, a.t0, a.M, a.HQ, a.chunk, a.cap,
        a.window, ck_lo, cps, nsplit, ntg, a.scale * kLog2e, part, a.err, a.wait_ns, wide,
        a.fault, a.gs_cache);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  return launch_decode_combine(part, nsplit, a.B * a.M * a.HQ, a.HQ, a.sink, a.o, lse, VD,
                               sizeof(T) == 2, st);
}

template <int KD, int VD, typename T>
cudaError_t chunk_split_by_group(const ChunkArgs& a, const void* qh, const float* AQ,
                                 const int* wide, float* lse, float* part, cudaStream_t st) {
  switch (a.HQ / a.H) {
    case 1: return chunk_split_impl<KD, VD, 1, T>(a, qh, AQ, wide, lse, part, st);
    case 2: return chunk_split_impl<KD, VD, 2, T>(a, qh, AQ, wide, lse, part, st);
    case 4: return chunk_split_impl<KD, VD, 4, T>(a, qh, AQ, wide, lse, part, st);
    case 8: return chunk_split_impl<KD, VD, 8, T>(a, qh, AQ, wide, lse, part, st);
    case 16: return chunk_split_impl<KD, VD, 16, T>(a, qh, AQ, wide, lse, part, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t chunk_split_by_dims(const ChunkArgs& a, const void* qh, const float* AQ,
                                const int* wide, float* lse, float* part, cudaStream_t st) {
  if (a.K == 64 && a.V == 64) return chunk_split_by_group<64, 64, T>(a, qh, AQ, wide, lse, part, st);
  if (a.K == 64 && a.V == 128) return chunk_split_by_group<64, 128, T>(a, qh, AQ, wide, lse, part, st);
  if (a.K == 128 && a.V == 64) return chunk_split_by_group<128, 64, T>(a, qh, AQ, wide, lse, part, st);
  if (a.K == 128 && a.V == 128) return chunk_split_by_group<128, 128, T>(a, qh, AQ, wide, lse, part, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool chunk_split_applies(int M, int HQ, int H, bool bf16) {
  const int g = HQ / H;
  const bool pow2 = g == 1 || g == 2 || g == 4 || g == 8 || g == 16;
  return pow2 && M >= 1 && (!bf16 || M <= 2 * (16 / g));
}

size_t chunk_split_part_bytes(int B, int M, int cap, int HQ, int H, int V, int chunk) {
  return static_cast<size_t>(B) * M * HQ * chunk_max_splits(B, M, cap, HQ, H, chunk) * (V + 2) *
         sizeof(float);
}

cudaError_t launch_chunk_split(const ChunkArgs& a, const void* qh, const float* AQ,
                               const int* wide, float* lse, float* part, cudaStream_t st) {
  return a.bf16 ? chunk_split_by_dims<__nv_bfloat16>(a, qh, AQ, wide, lse, part, st)
                : chunk_split_by_dims<float>(a, qh, AQ, wide, lse, part, st);
}

}  // namespace wall
