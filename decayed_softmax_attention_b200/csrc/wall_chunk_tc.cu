// Wall attention over a cached prefix for a chunk of new tokens (chunked
// prefill / multi-token decode), bf16, on the tcgen05 tensor cores of sm_100a.
//
// The M new queries of a chunk at positions t0 .. t0 + M - 1 attend the
// decode cache (Wall Attention README, "Decode": k_tilde = k exp2(R_c - P),
// one anchor R_c per chunk of C rows) over rows 0 .. t0 + i (causal, optional
// window and sink), after the chunk's own keys were appended to it.  Per
// (256-row query block, cache tile of 128 rows):
//   S = Qh * diag(c_r) * Kt^T,  Qh = q exp2(P_i - AQ),  c_r = exp2(AQ - R_c(r))
// with AQ = P just before the query block; c depends on the key row's chunk
// (128 / C vectors per tile).  Same pipeline as the prefill kernel: warp 0
// TMA producer (query tiles once; cache k_tilde / v tiles and their anchor
// vectors through 2-stage rings), warp 1 MMA issuer (PV_A(j-1), QK_A(j),
// PV_B(j-1), QK_B(j)), warp 2 TMEM owner, warpgroups 1/2 online softmax of
// query tiles A/B, warpgroup 3 rescales each key tile in shared memory.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

struct ChunkParams {
  const float* AQ;       // [B*HQ][NQB][KD] log2 units: P just before each 256-row query block
  const float* r_cache;  // [B, ncap, HQ, KD] anchors (log2 units)
  const float* sink;
  const int* wide;  // [B*HQ][NQB]: the block's own rows are left to the diagonal kernel
  int window;
  int B, M, t0, HQ, H, cap, NQB;
  float sc;  // scale * log2(e)
  __nv_bfloat16* o;  // [B, M, HQ, VD]
  float* lse;        // [B, M, HQ]
  int* err;
  uint64_t wait_ns;
  int fault;  // testing hook: 6 = the producer skips its first key tile
  const float* gs_cache;  // scalar gate: PS per (cache row, query head), log2 units, or null
};

template <int KD, int VD, int CH>
struct ChCfg {
  static constexpr int BM = 128, BN = 128, NQ = 2;
  static constexpr int KS = 2, VS = 2;
  static constexpr int NRC = BN / CH;  // anchor chunks per key tile
  static constexpr int QBOX = KD / 64, VBOX = VD / 64;
  static constexpr int Q_BYTES = BM * KD * 2;
  static constexpr int K_BYTES = BN * KD * 2;
  static constexpr int V_BYTES = BN * VD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_AQ = OFF_V + VS * V_BYTES;
  static constexpr int OFF_R = OFF_AQ + KD * 4;                // [KS][NRC][KD]
  static constexpr int OFF_C = OFF_R + KS * NRC * KD * 4;      // [2][NRC][KD]
  static constexpr int OFF_GS = OFF_C + 2 * NRC * KD * 4;         // [2 tiles][2][BN] fp32
  static constexpr int OFF_BAR = OFF_GS + 2 * 2 * BN * 4;
  // qfull, kfull[KS], kready[KS], kempty[KS], vfull[VS], vempty[VS], sfull[2], pfull[2],
  // ofinal, mdrain
  static constexpr int NBAR = 1 + 3 * KS + 2 * VS + 2 + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_USED = OFF_MISC + 64;
  // at least 116 KB so that a second CTA never shares the SM (all 512 TMEM columns each)
  static constexpr int SMEM_ALLOC = (SMEM_USED + 1024) > 118784 ? (SMEM_USED + 1024) : 118784;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_O = 256;  // + 128 * tile
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, VD, 0, 1);
};

// Scale the 8 bf16 of one 16-byte chunk by c[0..7], with c split into a bf16
// head and a bf16 tail (chi + clo == c to ~16 bits): x*clo is formed first and
// x*chi + x*clo is rounded once, so the result carries a single bf16 rounding.
__device__ __forceinline__ uint4 scale_chunk(uint4 u, const __nv_bfloat162* chi,
                                             const __nv_bfloat162* clo) {
  uint4 r;
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&u);
  __nv_bfloat162* y = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = __hfma2(x[i], chi[i], __hmul2(x[i], clo[i]));
  return r;
}

__device__ __forceinline__ bool bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Keeps the compiler from touching registers filled by tcgen05.ld before the
// matching tcgen05.wait::ld.
__device__ __forceinline__ void reg_fence32(float* r) {
  asm volatile(""
               : "+f"(r[0]), "+f"(r[1]), "+f"(r[2]), "+f"(r[3]), "+f"(r[4]), "+f"(r[5]),
                 "+f"(r[6]), "+f"(r[7]), "+f"(r[8]), "+f"(r[9]), "+f"(r[10]), "+f"(r[11]),
                 "+f"(r[12]), "+f"(r[13]), "+f"(r[14]), "+f"(r[15]), "+f"(r[16]), "+f"(r[17]),
                 "+f"(r[18]), "+f"(r[19]), "+f"(r[20]), "+f"(r[21]), "+f"(r[22]), "+f"(r[23]),
                 "+f"(r[24]), "+f"(r[25]), "+f"(r[26]), "+f"(r[27]), "+f"(r[28]), "+f"(r[29]),
                 "+f"(r[30]), "+f"(r[31]));
}
template <int KD, int VD, int CH, bool GS>
__global__ void __launch_bounds__(512, 1)
    wall_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const ChunkParams p) {
  using C = ChCfg<KD, VD, CH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* sAQ = reinterpret_cast<float*>(smem + C::OFF_AQ);
  float* sR = reinterpret_cast<float*>(smem + C::OFF_R);
  float* sC = reinterpret_cast<float*>(smem + C::OFF_C);
  float* sGS = reinterpret_cast<float*>(smem + C::OFF_GS);  // [query tile][2][BN] gate prefixes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;
  uint64_t* kready = kfull + C::KS;
  uint64_t* kempty = kready + C::KS;
  uint64_t* vfull = kempty + C::KS;
  uint64_t* vempty = vfull + C::VS;
  uint64_t* sfull = vempty + C::VS;
  uint64_t* pfull = sfull + 2;
  uint64_t* ofinal = pfull + 2;
  uint64_t* mdrain = ofinal + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* sched_lo = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);  // [2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2;
  const int BHQ = p.B * p.HQ;
  const int qblk = p.NQB - 1 - static_cast<int>(blockIdx.x / BHQ);
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
  const int q0 = qblk * 2 * C::BM;            // first chunk row of the block
  const bool has_b = q0 + C::BM < p.M;
  const int ncap = (p.cap + CH - 1) / CH;
  const int last_chunk = (p.t0 + p.M - 1) / CH;  // chunk of the last cache row in use

  if (tid == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < C::KS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kready[s], 128);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < C::VS; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sfull[x], 1);
      mbar_init(&pfull[x], 128);
    }
    mbar_init(ofinal, 1);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    sched_lo[0] = 0x7fffffff;
    sched_lo[1] = 0x7fffffff;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();

  // Admitted cache rows per query row (absolute position t0 + i): [lo, t0 + i].
  const bool is_softmax = (wg == 1 || wg == 2);
  const int X = wg - 1;  // query tile of a softmax warpgroup
  const int row = tid - 128 * wg;
  const int ci = q0 + C::BM * X + row;        // chunk row
  const int gi = p.t0 + ci;                   // absolute position
  const bool row_ok = is_softmax && ci < p.M;
  int my_lo = 0;
  if (row_ok) {
    if (p.window > 0) my_lo = gi - p.window + 1 > 0 ? gi - p.window + 1 : 0;
    atomicMin(&sched_lo[X], my_lo);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // key-tile ranges (tile index kt = cache row / 128) of query tiles A and B; a
  // wide block (strong decay inside it) stops before its own first row abs0
  const bool wide = p.wide[static_cast<size_t>(bh) * p.NQB + qblk] != 0;
  const int abs0 = p.t0 + q0;
  const int wide_hi = abs0 > 0 ? (abs0 - 1) / C::BN : -1;
  const int ktA_hi = wide ? wide_hi : (p.t0 + min(q0 + C::BM, p.M) - 1) / C::BN;
  const int ktB_hi = wide ? wide_hi : has_b ? (p.t0 + min(q0 + 2 * C::BM, p.M) - 1) / C::BN : ktA_hi;
  const int ktA_lo = sched_lo[0] / C::BN;
  const int ktB_lo = has_b ? sched_lo[1] / C::BN : ktB_hi + 1;
  const int kt_hi = has_b ? ktB_hi : ktA_hi;
  const int kt_lo = has_b ? min(ktA_lo, ktB_lo) : ktA_lo;
  const int nt = kt_hi - kt_lo + 1;  // visit order j = 0..nt-1 is kt = kt_hi - j
  const int jfA = kt_hi - ktA_hi, jlA = kt_hi - ktA_lo;
  const int jfB = has_b ? kt_hi - ktB_hi : 0, jlB = has_b ? kt_hi - ktB_lo : -1;
  const WaitCtl wc{abort_flag, p.err, p.wait_ns};

  if (wg == 0) {
    reg_dealloc<80>();
    if (warp == 0 && lane == 0) {
      // ----------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int nk = 0, nv = 0;
      mbar_arrive_expect_tx(qfull, (has_b ? 2 : 1) * C::Q_BYTES + KD * 4);
      for (int bx = 0; bx < C::QBOX; ++bx) {
        tma_load_3d(sQ + bx * 16384, &tmQ, qfull, bx * 64, q0, bh);
        if (has_b) tma_load_3d(sQ + C::Q_BYTES + bx * 16384, &tmQ, qfull, bx * 64, q0 + C::BM, bh);
      }
      bulk_load(sAQ, p.AQ + (static_cast<size_t>(bh) * p.NQB + qblk) * KD, KD * 4, qfull);
      for (int j = 0; j < nt; ++j) {
        const int kt = kt_hi - j;
        const int ks = j % C::KS;
        if (j >= C::KS && !mbar_wait(&kempty[ks], ((j / C::KS) - 1) & 1, wc)) break;
        if (!(p.fault == 6 && j == 0)) {  // testing hook: starve the consumers
          mbar_arrive_expect_tx(&kfull[ks], C::K_BYTES + C::NRC * KD * 4);
          for (int bx = 0; bx < C::QBOX; ++bx)
            tma_load_4d(sK + ks * C::K_BYTES + bx * 16384, &tmK, &kfull[ks], bx * 64, hq,
                        kt * C::BN, b);
          for (int c = 0; c < C::NRC; ++c) {
            // anchors of the tile's chunks; a chunk past the last row in use (its rows
            // arrive as zeros and are masked) reads that row's anchor instead
            const int ck = min(kt * C::NRC + c, last_chunk);
            bulk_load(sR + (ks * C::NRC + c) * KD,
                      p.r_cache + ((static_cast<size_t>(b) * ncap + ck) * p.HQ + hq) * KD,
                      KD * 4, &kfull[ks]);
          }
        }
        nk = j + 1;
        const int vs = j % C::VS;
        if (j >= C::VS && !mbar_wait(&vempty[vs], ((j / C::VS) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&vfull[vs], C::V_BYTES);
        for (int bx = 0; bx < C::VBOX; ++bx)
          tma_load_4d(sV + vs * C::V_BYTES + bx * 16384, &tmV, &vfull[vs], bx * 64, kvh,
                      kt * C::BN, b);
        nv = j + 1;
      }
      mbar_drain(qfull, 0, p.wait_ns);
      for (int j = nk > C::KS ? nk - C::KS : 0; j < nk; ++j)
        if (!(p.fault == 6 && j == 0)) mbar_drain(&kfull[j % C::KS], (j / C::KS) & 1, p.wait_ns);
      for (int j = nv > C::VS ? nv - C::VS : 0; j < nv; ++j)
        mbar_drain(&vfull[j % C::VS], (j / C::VS) & 1, p.wait_ns);
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(qfull, 0, wc);
      tc_fence_after();
      const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = sw128_desc(smem_u32(sV), 16384, 1024);
      bool pendA = false, pendB = false;
      bool vseen = false;
      int vrem_prev = 0;
      auto issue_pv = [&](int x, int jj) -> bool {
        const int cnt = jj - (x == 0 ? jfA : jfB), vs = jj % C::VS;
        if (!mbar_wait(&pfull[x], cnt & 1, wc)) return false;
        if ((x == 0 || !vseen) && !mbar_wait(&vfull[vs], (jj / C::VS) & 1, wc)) return false;
        vseen = true;
        tc_fence_after();
        const uint64_t dV = dV0 + static_cast<uint64_t>(vs * (C::V_BYTES >> 4));
        const uint32_t dO = tmem_base + C::COL_O + 128 * x, aP = tmem_base + C::COL_S + 128 * x;
        umma_ts(dO, aP, dV, C::IDESC_PV, cnt > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < C::BN / 16; ++kk)
          umma_ts(dO, aP + kk * 8, dV + static_cast<uint64_t>((kk * 2048) >> 4), C::IDESC_PV, 1u);
        if (--vrem_prev == 0) umma_commit(&vempty[vs]);
        return true;
      };
      auto issue_qk = [&](int x, int ks) {
        const uint32_t dS = tmem_base + C::COL_S + 128 * x;
        const uint64_t dA = dQ0 + static_cast<uint64_t>(x * (C::Q_BYTES >> 4));
        const uint64_t dB = dK0 + static_cast<uint64_t>(ks * (C::K_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          umma_ss(dS, dA + koff, dB + koff, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sfull[x]);
      };
      for (int j = 0; ok && j < nt; ++j) {
        const int ks = j % C::KS;
        int vrem_cur = 0;
        vseen = false;
        if (!mbar_wait(&kready[ks], (j / C::KS) & 1, wc)) { ok = false; break; }
        if (pendA) {
          if (!issue_pv(0, j - 1)) { ok = false; break; }
          pendA = false;
        }
        tc_fence_after();
        if (j >= jfA && j <= jlA) {
          issue_qk(0, ks);
          pendA = true;
          ++vrem_cur;
        }
        if (pendB) {
          if (!issue_pv(1, j - 1)) { ok = false; break; }
          pendB = false;
        }
        if (j >= jfB && j <= jlB) {
          issue_qk(1, ks);
          pendB = true;
          ++vrem_cur;
        }
        umma_commit(&kempty[ks]);
        if (vrem_cur == 0) umma_commit(&vempty[j % C::VS]);
        vrem_prev = vrem_cur;
      }
      if (ok && pendA) ok = issue_pv(0, nt - 1);
      if (ok && pendB) ok = issue_pv(1, nt - 1);
      if (ok) umma_commit(ofinal);
      umma_commit(mdrain);
      mbar_drain(mdrain, 0, p.wait_ns);
    }
  } else if (is_softmax) {
    // ------------------------------------------------------------- softmax + epilogue
    reg_alloc<192>();
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = C::COL_S + 128 * X, colO = C::COL_O + 128 * X;
    const int lo = row_ok ? my_lo : 0;
    const int hi = row_ok ? (wide ? min(gi, abs0 - 1) : gi) : -1;
    const float2 sc2 = make_float2(p.sc, p.sc);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int jf = X == 0 ? jfA : jfB, jl = X == 0 ? jlA : jlB;
    // Scalar gate: the logit gains PS(query row) - PS(key row) (log2 units).  Thread r
    // of the warpgroup loads key row kt * BN + r of each tile, one tile ahead; the
    // warpgroup shares the tile's 128 values through shared memory.
    const size_t gsb = static_cast<size_t>(b) * p.cap;  // first gate row of this batch row
    const int nrows = p.t0 + p.M;                       // gate rows written so far
    auto gate_row = [&](int r) -> float {
      return (r >= 0 && r < nrows) ? p.gs_cache[(gsb + r) * p.HQ + hq] : 0.f;
    };
    const float gs_row = (GS && row_ok) ? gate_row(gi) : 0.f;
    float gs_next = (GS && jl >= jf) ? gate_row((kt_hi - jf) * C::BN + row) : 0.f;
    for (int j = jf; j <= jl; ++j) {
      const int cnt = j - jf;
      const int kt = kt_hi - j;
      float* gsl = sGS + (X * 2 + (cnt & 1)) * C::BN;
      if (GS) {
        gsl[row] = gs_next;
        if (j < jl) gs_next = gate_row((kt - 1) * C::BN + row);
      }
      const bool got = mbar_wait(&sfull[X], cnt & 1, wc);
      // gated: one decision for the whole warpgroup (the barrier also publishes gsl)
      if (GS ? bar_or(2 + X, 128, !got) : !__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[C::BN];
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) tmem_ld32(lane_base + colS + c, s + c);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) reg_fence32(s + c);
      const int j0 = kt * C::BN;
      const bool partial = !__all_sync(0xffffffffu, lo <= j0 && hi >= j0 + C::BN - 1);
      if (partial) {
#pragma unroll
        for (int jj = 0; jj < C::BN; ++jj) {
          const int jg = j0 + jj;
          if (jg < lo || jg > hi) s[jj] = -INFINITY;
        }
      }
      if (GS) {  // s <- s * sc - PS(key row); the row's PS joins through off below
#pragma unroll
        for (int jj = 0; jj < C::BN; jj += 4) {
          const float4 g4 = *reinterpret_cast<const float4*>(gsl + jj);
          const float2 a = ffma2(make_float2(s[jj], s[jj + 1]), sc2, make_float2(-g4.x, -g4.y));
          const float2 c = ffma2(make_float2(s[jj + 2], s[jj + 3]), sc2, make_float2(-g4.z, -g4.w));
          s[jj] = a.x; s[jj + 1] = a.y; s[jj + 2] = c.x; s[jj + 3] = c.y;
        }
      }
      float mx0 = s[0], mx1 = s[1];
#pragma unroll
      for (int jj = 2; jj < C::BN; jj += 4) {
        mx0 = fmax3(mx0, s[jj], s[jj + 1]);
        mx1 = fmax3(mx1, s[jj + 2], s[jj + 3]);
      }
      const float mt = GS ? fmaxf(mx0, mx1) + gs_row : fmaxf(mx0, mx1) * p.sc;
      const bool need = mt > m_used + 8.f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_used - mt);
        l *= alpha;
        m_used = mt;
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      const float2 off = make_float2(gs_row - base, gs_row - base);
      const float2 mul = GS ? make_float2(1.f, 1.f) : sc2;  // (gated scores are already scaled)
      float2 rs = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int jj = 0; jj < 32; jj += 2) {
          const float2 t = ffma2(make_float2(s[c + jj], s[c + jj + 1]), mul, off);
          const float2 pv = make_float2(ex2_approx(t.x), ex2_approx(t.y));
          rs = fadd2(rs, pv);
          pk[jj >> 1] = pack_bf16(pv.x, pv.y);
        }
        tmem_st16(lane_base + colS + (c >> 1), pk);
      }
      l += rs.x + rs.y;
      if (cnt > 0 && __any_sync(0xffffffffu, need)) {
        // PV_X(j-1) was issued before QK_X(j), so it is complete: rescale O_X now.
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < VD; c += 32) {
          float ov[32];
          tmem_ld32(lane_base + colO + c, ov);
          tmem_wait_ld();
          reg_fence32(ov);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 t = fmul2(make_float2(ov[e], ov[e + 1]), a2);
            ov[e] = t.x;
            ov[e + 1] = t.y;
          }
          tmem_st32(lane_base + colO + c, reinterpret_cast<uint32_t*>(ov));
        }
        tmem_wait_st();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pfull[X]);
    }
    if (ok && jl >= jf) {
      const bool got = mbar_wait(ofinal, 0, wc);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok && jl >= jf) {
      tc_fence_after();
      float Z = l;
      if (p.sink != nullptr && m_used != -INFINITY) Z += ex2_approx(p.sink[hq] * kLog2e - m_used);
      const float inv = 1.f / Z;
      __nv_bfloat16* orow =
          p.o + ((static_cast<size_t>(b) * p.M + (row_ok ? ci : 0)) * p.HQ + hq) * VD;
#pragma unroll 1
      for (int c = 0; c < VD; c += 32) {
        float ov[32];
        tmem_ld32(lane_base + colO + c, ov);
        tmem_wait_ld();
        reg_fence32(ov);
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 u;
            u.x = pack_bf16(ov[e] * inv, ov[e + 1] * inv);
            u.y = pack_bf16(ov[e + 2] * inv, ov[e + 3] * inv);
            u.z = pack_bf16(ov[e + 4] * inv, ov[e + 5] * inv);
            u.w = pack_bf16(ov[e + 6] * inv, ov[e + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c + e) = u;
          }
        }
      }
      if (row_ok && p.lse != nullptr)
        p.lse[(static_cast<size_t>(b) * p.M + ci) * p.HQ + hq] = (m_used + log2f(Z)) * kLn2;
    }
  } else {
    // ------------------------------------------------------------- key-tile rescale
    // Row r of a key tile belongs to anchor chunk r / CH; its channels are
    // multiplied by c = exp2(AQ - R_chunk) (all log2 units).
    reg_dealloc<48>();
    const int r = tid - 384;
    bool ok = mbar_wait(qfull, 0, wc);
    ok = !bar_or(1, 128, !ok);
    constexpr int CPR = KD / 8;        // 16-byte chunks per key row
    constexpr int RSTEP = 128 / CPR;   // rows between this thread's chunks
    static_assert(CH % RSTEP == 0, "a thread's rows must map to anchor chunks statically");
    const int L = r % CPR, box = L >> 3, c16 = L & 7;
    const int row0 = r / CPR;          // < RSTEP, so row0 + m RSTEP lies in chunk m RSTEP / CH
    const uint32_t phys = static_cast<uint32_t>((c16 ^ (row0 & 7)) << 4);
    for (int j = 0; ok && j < nt; ++j) {
      const int ks = j % C::KS;
      const bool got = mbar_wait(&kfull[ks], (j / C::KS) & 1, wc);
      float* cb = sC + (j & 1) * C::NRC * KD;
      if (got && r < KD) {
        const int kt = kt_hi - j;
#pragma unroll
        for (int c = 0; c < C::NRC; ++c)  // a wide block's own chunks: masked, kept finite
          cb[c * KD + r] = (wide && kt * C::BN + c * CH >= abs0)
                               ? 0.f
                               : ex2_approx(sAQ[r] - sR[(ks * C::NRC + c) * KD + r]);
      }
      if (bar_or(1, 128, !got || *abort_flag != 0)) break;
      uint8_t* tile = sK + ks * C::K_BYTES + box * 16384;
#pragma unroll
      for (int ck = 0; ck < C::NRC; ++ck) {
        __nv_bfloat162 chi[4], clo[4];
        {
          const float* cv0 = cb + ck * KD + box * 64 + c16 * 8;
          const float4 c0 = *reinterpret_cast<const float4*>(cv0);
          const float4 c1 = *reinterpret_cast<const float4*>(cv0 + 4);
          const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            chi[i] = __floats2bfloat162_rn(cv[2 * i], cv[2 * i + 1]);
            const float2 h = __bfloat1622float2(chi[i]);
            clo[i] = __floats2bfloat162_rn(cv[2 * i] - h.x, cv[2 * i + 1] - h.y);
          }
        }
        // this thread's rows in chunk ck: m in [ck CH / RSTEP, (ck + 1) CH / RSTEP)
#pragma unroll
        for (int m = ck * (CH / RSTEP); m < (ck + 1) * (CH / RSTEP); ++m) {
          uint4* ptr = reinterpret_cast<uint4*>(tile + (row0 + m * RSTEP) * 128 + phys);
          *ptr = scale_chunk(*ptr, chi, clo);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&kready[ks]);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// The chunk's query side: P_i = P_prev + prefix of g * log2(e) over the chunk;
// per 256-row query block AQ = P just before the block and
// qh_i = q_i exp2(P_i - AQ) (a block-local prefix, so the exponent stays
// bounded).  One CTA per (256-row block, batch * head); thread (channel group
// of 4, row group of RPG rows).  Pass 1 sums g per block; pass 2 adds the
// earlier blocks' sums to P_prev (AQ), scans the row groups in shared memory
// and writes qh.
template <int KD>
struct ChunkPrepCfg {
  static constexpr int CG = KD / 4;        // channel groups of 4
  static constexpr int RG = 256 / CG;      // row groups
  static constexpr int RPG = 256 / RG;     // rows per row group
};

template <int KD, typename T>
__device__ __forceinline__ void chunk_rowgroup_sum(const T* gb, size_t rstep, int r0, int r1,
                                                   float* acc) {
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    float gv[4];
    load4(gb + r * rstep, gv);
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] = fmaf(gv[c], kLog2e, acc[c]);
  }
}

template <int KD, typename T>
__global__ void __launch_bounds__(256) chunk_sum_kernel(const T* __restrict__ g, int M, int HQ,
                                                        int NQB, float* __restrict__ bsum) {
  using PC = ChunkPrepCfg<KD>;
  __shared__ float tot[PC::RG][KD];
  const int blk = blockIdx.x, bh = blockIdx.y, b = bh / HQ, hq = bh % HQ;
  const int cg = threadIdx.x % PC::CG, rg = threadIdx.x / PC::CG;
  const int r0 = blk * 256 + rg * PC::RPG, r1 = min(M, r0 + PC::RPG);
  const size_t rstep = static_cast<size_t>(HQ) * KD;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  chunk_rowgroup_sum<KD>(g + (static_cast<size_t>(b) * M * HQ + hq) * KD + cg * 4, rstep, r0, r1,
                         acc);
#pragma unroll
  for (int c = 0; c < 4; ++c) tot[rg][cg * 4 + c] = acc[c];
  __syncthreads();
  if (threadIdx.x < KD) {
    float sum = 0.f;
    for (int r = 0; r < PC::RG; ++r) sum += tot[r][threadIdx.x];
    bsum[(static_cast<size_t>(bh) * NQB + blk) * KD + threadIdx.x] = sum;
  }
}

// qh is written in the input's type (bf16 feeds the tensor-core tiles, fp32
// the exact split pass).
template <int KD, typename T>
__global__ void __launch_bounds__(256) chunk_apply_kernel(
    const T* __restrict__ q, const T* __restrict__ g, const float* __restrict__ p_prev,
    const float* __restrict__ bsum, int M, int t0, int HQ, int NQB, T* __restrict__ qh,
    float* __restrict__ AQ, int* __restrict__ wide) {
  using PC = ChunkPrepCfg<KD>;
  __shared__ float tot[PC::RG][KD];
  __shared__ int s_span;  // largest |P_i - AQ| of the block (float bits), log2 units
  if (threadIdx.x == 0) s_span = 0;
  const int blk = blockIdx.x, bh = blockIdx.y, b = bh / HQ, hq = bh % HQ;
  const int cg = threadIdx.x % PC::CG, rg = threadIdx.x / PC::CG;
  const int r0 = blk * 256 + rg * PC::RPG, r1 = min(M, r0 + PC::RPG);
  const size_t rstep = static_cast<size_t>(HQ) * KD;
  const T* gb = g + (static_cast<size_t>(b) * M * HQ + hq) * KD + cg * 4;
  const T* qb = q + (static_cast<size_t>(b) * M * HQ + hq) * KD + cg * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  chunk_rowgroup_sum<KD>(gb, rstep, r0, r1, acc);
#pragma unroll
  for (int c = 0; c < 4; ++c) tot[rg][cg * 4 + c] = acc[c];
  __syncthreads();
  if (rg == 0) {  // AQ = P_prev + the earlier blocks' sums
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = cg * 4 + c;
      float aq = (t0 > 0 && p_prev) ? p_prev[static_cast<size_t>(bh) * KD + n] : 0.f;
      for (int k = 0; k < blk; ++k) aq += bsum[(static_cast<size_t>(bh) * NQB + k) * KD + n];
      AQ[(static_cast<size_t>(bh) * NQB + blk) * KD + n] = aq;
    }
  }
  float loc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float pre = 0.f;
    for (int r = 0; r < rg; ++r) pre += tot[r][cg * 4 + c];
    loc[c] = pre;
  }
  T* ob = qh + static_cast<size_t>(bh) * M * KD + cg * 4;
  float span = 0.f;
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    float gv[4], qv[4], o4[4];
    load4(gb + r * rstep, gv);
    load4(qb + r * rstep, qv);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      loc[c] = fmaf(gv[c], kLog2e, loc[c]);
      span = fmaxf(span, fabsf(loc[c]));
      o4[c] = qv[c] * ex2_approx(loc[c]);
    }
    store4(ob + static_cast<size_t>(r) * KD, o4);
  }
  // The block's own cache chunks carry anchors P at rows inside it, so the
  // factor exp2(AQ - R_c) spans the same range as the query factor.
  if (span > 0.f) atomicMax(&s_span, __float_as_int(span));
  __syncthreads();
  if (threadIdx.x == 0)
    wide[static_cast<size_t>(bh) * NQB + blk] =
        __int_as_float(s_span) > kPrefillSpanNats * kLog2e ? 1 : 0;
}

template <int KD, int VD, int CH>
cudaError_t chunk_impl(const ChunkArgs& a, void* qh, float* AQ, const int* wide, float* lse,
                       cudaStream_t st) {
  using C = ChCfg<KD, VD, CH>;
  const int BHQ = a.B * a.HQ;
  const int NQB = (a.M + 255) / 256;
  CUtensorMap tmQ, tmK, tmV;
  {  // anchored chunk queries [B*HQ][M][K]
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.M),
                                static_cast<cuuint64_t>(BHQ)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(KD) * 2,
                                   static_cast<cuuint64_t>(a.M) * KD * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!encode_tiled(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, qh, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {  // cache k_tilde / v: the maps end at the chunk's last row, so rows past it
     // (never written, may hold anything) arrive as zeros
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint64_t rows = static_cast<cuuint64_t>(a.t0) + a.M;
    const cuuint64_t kd[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.HQ), rows,
                              static_cast<cuuint64_t>(a.B)};
    const cuuint64_t ks[3] = {static_cast<cuuint64_t>(KD) * 2,
                              static_cast<cuuint64_t>(a.HQ) * KD * 2,
                              static_cast<cuuint64_t>(a.cap) * a.HQ * KD * 2};
    const cuuint64_t vd[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(a.H), rows,
                              static_cast<cuuint64_t>(a.B)};
    const cuuint64_t vs[3] = {static_cast<cuuint64_t>(VD) * 2,
                              static_cast<cuuint64_t>(a.H) * VD * 2,
                              static_cast<cuuint64_t>(a.cap) * a.H * VD * 2};
    if (!encode_tiled(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k_tilde, kd, ks, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tiled(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v_cache, vd, vs, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  auto kern = a.gs_cache != nullptr ? wall_chunk_tc_kernel<KD, VD, CH, true>
                                    : wall_chunk_tc_kernel<KD, VD, CH, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  ChunkParams p;
  p.AQ = AQ;
  p.r_cache = a.r_cache;
  p.sink = a.sink;
  p.wide = wide;
  p.window = a.window;
  p.B = a.B;
  p.M = a.M;
  p.t0 = a.t0;
  p.HQ = a.HQ;
  p.H = a.H;
  p.cap = a.cap;
  p.NQB = NQB;
  p.sc = a.scale * kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = lse;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.fault = a.fault;
  p.gs_cache = a.gs_cache;
  const unsigned grid = static_cast<unsigned>(NQB) * BHQ;
  if (a.ev_mid != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_mid), st);
  kern<<<grid, 512, C::SMEM_ALLOC, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

template <int KD, int VD>
cudaError_t chunk_by_c(const ChunkArgs& a, void* qh, float* AQ, const int* wide, float* lse,
                       cudaStream_t st) {
  switch (a.chunk) {
    case 32: return chunk_impl<KD, VD, 32>(a, qh, AQ, wide, lse, st);
    case 64: return chunk_impl<KD, VD, 64>(a, qh, AQ, wide, lse, st);
    case 128: return chunk_impl<KD, VD, 128>(a, qh, AQ, wide, lse, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t align256c(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t chunk_workspace_bytes(int B, int M, int cap, int HQ, int H, int K, int V, int chunk,
                             bool bf16) {
  const size_t BHQ = static_cast<size_t>(B) * HQ;
  const size_t NQB = (static_cast<size_t>(M) + 255) / 256;
  const size_t es = bf16 ? 2 : 4;
  const size_t prep = align256c(BHQ * M * K * es) + 2 * align256c(BHQ * NQB * K * 4) +
                      align256c(BHQ * NQB * 4) + align256c(BHQ * M * 4);
  return prep + (chunk_split_applies(M, HQ, H, bf16)
                     ? align256c(chunk_split_part_bytes(B, M, cap, HQ, H, V, chunk))
                     : 0);
}

template <int KD, typename T>
cudaError_t chunk_prep(const ChunkArgs& a, void* qh, float* AQ, float* bsum, int* wide,
                       cudaStream_t st) {
  const int NQB = (a.M + 255) / 256;
  const dim3 grid(NQB, a.B * a.HQ);
  const T* g = static_cast<const T*>(a.g_new);
  if (NQB > 1) {
    chunk_sum_kernel<KD, T><<<grid, 256, 0, st>>>(g, a.M, a.HQ, NQB, bsum);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  chunk_apply_kernel<KD, T><<<grid, 256, 0, st>>>(static_cast<const T*>(a.q), g, a.p_prev, bsum,
                                                  a.M, a.t0, a.HQ, NQB, static_cast<T*>(qh), AQ,
                                                  wide);
  return cudaGetLastError();
}

cudaError_t launch_chunk(const ChunkArgs& a, cudaStream_t st) {
  char* ws = static_cast<char*>(a.workspace);
  const size_t BHQ = static_cast<size_t>(a.B) * a.HQ;
  const size_t NQB = (static_cast<size_t>(a.M) + 255) / 256;
  void* qh = ws;
  char* cur = ws + align256c(BHQ * a.M * a.K * (a.bf16 ? 2 : 4));
  float* AQ = reinterpret_cast<float*>(cur);
  cur += align256c(BHQ * NQB * a.K * 4);
  float* bsum = reinterpret_cast<float*>(cur);
  cur += align256c(BHQ * NQB * a.K * 4);
  int* wide = reinterpret_cast<int*>(cur);
  cur += align256c(BHQ * NQB * 4);
  float* lse = a.lse != nullptr ? a.lse : reinterpret_cast<float*>(cur);
  cur += align256c(BHQ * a.M * 4);
  // 1. the chunk's queries, anchored (reads p_prev before the append below
  //    overwrites p_last, which may be the same buffer)
  cudaError_t e;
  if (a.bf16)
    e = a.K == 64 ? chunk_prep<64, __nv_bfloat16>(a, qh, AQ, bsum, wide, st)
                  : chunk_prep<128, __nv_bfloat16>(a, qh, AQ, bsum, wide, st);
  else
    e = a.K == 64 ? chunk_prep<64, float>(a, qh, AQ, bsum, wide, st)
                  : chunk_prep<128, float>(a, qh, AQ, bsum, wide, st);
  if (e != cudaSuccess) return e;
  // 2. the chunk's keys join the cache (rows t0 .. t0 + M - 1)
  CacheArgs c;
  c.k_new = a.k_new; c.g_new = a.g_new; c.p_prev = a.t0 > 0 ? a.p_prev : nullptr;
  c.B = a.B; c.t_start = a.t0; c.T_new = a.M; c.cap = a.cap; c.HQ = a.HQ; c.H = a.H; c.K = a.K;
  c.chunk = a.chunk; c.k_tilde = a.k_tilde; c.r_cache = a.r_cache; c.p_last = a.p_last;
  c.err = a.err; c.wait_ns = a.wait_ns; c.fault = 0;
  c.pm.cap = a.cap;
  e = launch_cache_build(c, a.bf16, st);
  if (e != cudaSuccess) return e;
  if (a.gs_new != nullptr) {  // the chunk's gate prefixes join the gate cache
    GateArgs ga;
    ga.gs_new = a.gs_new; ga.gs_prev = a.t0 > 0 ? a.gs_prev : nullptr; ga.t_pos = nullptr;
    ga.B = a.B; ga.t_start = a.t0; ga.T_new = a.M; ga.HQ = a.HQ;
    ga.gcache = a.gs_cache; ga.gs_last = a.gs_last;
    ga.pm.cap = a.cap;
    e = launch_gate_cache(ga, a.bf16, st);
    if (e != cudaSuccess) return e;
  }
  // 3. the chunk's queries attend the cache: a few tokens per sequence (and
  //    fp32 chunks of any length) the decode's way, longer bf16 chunks in
  //    128-row tensor-core query tiles
  if (chunk_split_applies(a.M, a.HQ, a.H, a.bf16)) {
    e = launch_chunk_split(a, qh, AQ, wide, lse, reinterpret_cast<float*>(cur), st);
  } else if (!a.bf16) {
    return cudaErrorInvalidValue;
  } else if (a.K == 64 && a.V == 64) {
    e = chunk_by_c<64, 64>(a, qh, AQ, wide, lse, st);
  } else if (a.K == 64 && a.V == 128) {
    e = chunk_by_c<64, 128>(a, qh, AQ, wide, lse, st);
  } else if (a.K == 128 && a.V == 64) {
    e = chunk_by_c<128, 64>(a, qh, AQ, wide, lse, st);
  } else if (a.K == 128 && a.V == 128) {
    e = chunk_by_c<128, 128>(a, qh, AQ, wide, lse, st);
  } else {
    return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  // 4. wide blocks (strong decay inside a 256-row query block): the chunk's own
  //    pairs there, exactly, merged with the result for the rows before
  DiagParams d;
  d.q = a.q; d.k = a.k_new; d.g = a.g_new; d.gs = a.gs_new; d.v = a.v_cache;
  d.sink = a.sink; d.rowlo = nullptr; d.wide = wide; d.window = a.window;
  d.B = a.B; d.Tb = a.M; d.HQ = a.HQ; d.H = a.H; d.NQB = static_cast<int>(NQB);
  d.vT = a.cap; d.voff = a.t0; d.pos0 = a.t0;
  d.scale = a.scale; d.o = a.o; d.lse = lse;
  return launch_diag(d, a.bf16, a.K, a.V, st);
}

}  // namespace wall
