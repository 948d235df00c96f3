// Wall attention prefill forward, bf16, on the 5th-generation tensor cores
// (tcgen05 + TMEM) of sm_100a.
//
// One CTA computes a 256-row query block (two 128-row tiles, A and B) of one
// (batch, query head).  The score of the Wall Attention README intro,
//   x(i,j) = scale * sum_n q[i,n] k[j,n] exp(G[i,n] - G[j,n]) + Gs[i] - Gs[j],
// becomes a dense contraction per (query block, key tile) pair:
//   S = Qh * diag(c) * Kh^T,  c[n] = exp(AQ[n] - AK[n])
// where Qh/Kh are the anchored operands of the prepass (query anchor per
// 256-row block, key anchor per 128-row block), so one rescaled key tile
// serves both query tiles.  The rescale warpgroup multiplies each key tile by
// c in shared memory (in place), the MMA warp issues S_X = Qh_X * Kt^T into
// TMEM, each softmax warpgroup (one query row per thread, read straight from
// its TMEM lane) runs the online softmax in the exp2 domain and writes P
// (bf16) back into TMEM over S_X, and the MMA warp accumulates O_X += P_X * V
// with P taken from TMEM.  This is the streaming (FlashAttention-style)
// softmax the README names; the decay factor never leaves the tile.
//
// Warp roles (512 threads): warpgroup 0 = warp 0 TMA producer, warp 1 MMA
// issuer, warp 2 TMEM allocator; warpgroups 1 and 2 = softmax + epilogue of
// query tiles A and B; warpgroup 3 = key-tile rescale.  Registers are
// re-balanced at start (setmaxnreg): softmax warpgroups 192, warpgroup 0 80,
// rescale 48 (sum 512 per thread slot = the 65536 registers of the launch).
//
// MMA issue order per key tile j: PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j), so
// one softmax warpgroup works while the tensor core serves the other (the
// rescaled key tile is waited for before PV_A(j-1), so PV_A and QK_A issue back
// to back: the MMA issue queue is only a few instructions deep), and
// "S_X(j) complete" implies "PV_X(j-1) complete" (tcgen05 ops of one thread
// run in issue order): a softmax warpgroup may rescale O_X as soon as it has
// read S_X(j).  Key tiles are visited from the diagonal backwards so the row
// maximum is found early; O is rescaled only when a row maximum grows by more
// than 2^8 (exact: the final normalisation uses the same stale maximum).
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

struct TcParams {
  const float* AQ;
  const float* AK;
  const float* ssl;
  const float* ssa;
  const float* sink;
  const int* rowlo;
  const int* wide;  // per (batch*head, 256-row query block): own key tiles left to the diagonal kernel
  int window;
  int B, T, HQ, H, NB;
  float sc;  // scale * log2(e)
  __nv_bfloat16* o;
  float* lse;
  int* err;
  uint64_t wait_ns;
  int fault;
};

template <int KD, int VD>
struct TcCfg {
  static constexpr int BM = 128, BN = 128, NQ = 2;
  static constexpr int KS = 2, VS = 2;
  static constexpr int QBOX = KD / 64, VBOX = VD / 64;
  static constexpr int Q_BYTES = BM * KD * 2;
  static constexpr int K_BYTES = BN * KD * 2;
  static constexpr int V_BYTES = BN * VD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_AQ = OFF_V + VS * V_BYTES;
  static constexpr int OFF_AK = OFF_AQ + KD * 4;
  static constexpr int OFF_C = OFF_AK + KS * KD * 4;
  // gate channels of the QK contraction (one 16-channel K slice, 32-byte
  // swizzle): query side constant (1, 1, 0, ...), key side per stage
  static constexpr int GX_BYTES = BM * 32;
  static constexpr int OFF_QX = (OFF_C + 2 * KD * 4 + 1023) / 1024 * 1024;
  static constexpr int OFF_KX = OFF_QX + GX_BYTES;
  static constexpr int OFF_BAR = OFF_KX + KS * GX_BYTES;
  // qfull, kfull[KS], kready[KS], kempty[KS], vfull[VS], vempty[VS], sfull[2], pfull[2],
  // ofinal, mdrain
  static constexpr int NBAR = 1 + 3 * KS + 2 * VS + 2 + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_USED = OFF_MISC + 64;
  // At least 116 KB so that a second CTA never shares the SM (each CTA takes
  // all 512 TMEM columns).
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
template <int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(512, 1)
    wall_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmKX, const TcParams p) {
  using C = TcCfg<KD, VD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* sAQ = reinterpret_cast<float*>(smem + C::OFF_AQ);
  float* sAK = reinterpret_cast<float*>(smem + C::OFF_AK);
  float* sC = reinterpret_cast<float*>(smem + C::OFF_C);
  uint8_t* sQX = smem + C::OFF_QX;
  uint8_t* sKX = smem + C::OFF_KX;
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
  const int NQB = (p.NB + 1) / 2;
  const int qblk = NQB - 1 - static_cast<int>(blockIdx.x / BHQ);
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
  const int q0 = qblk * 2 * C::BM;
  const bool has_b = q0 + C::BM < p.T;
  // issued first: the load's latency hides behind the set-up below
  const int wide_flag = __ldg(p.wide + static_cast<size_t>(bh) * NQB + qblk);

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
  if (HAS_GS && tid >= 128 && tid < 256) {
    // query-side gate channels (1, 1, 0, ..., 0) per row, 32-byte swizzled
    const int r = tid - 128;
    const int half = (r >> 2) & 1;  // where the logical first 16 bytes land
    *reinterpret_cast<uint4*>(sQX + r * 32 + half * 16) = make_uint4(0x3F803F80u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(sQX + r * 32 + (half ^ 1) * 16) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  __syncthreads();

  // Admitted key range per query row: [lo_i, i] (causal, window, document).
  const bool is_softmax = (wg == 1 || wg == 2);
  const int X = wg - 1;  // query tile of a softmax warpgroup
  const int row = tid - 128 * wg;
  const int gi = q0 + C::BM * X + row;
  const bool row_ok = is_softmax && gi < p.T;
  int my_lo = 0;
  if (row_ok) {
    if (p.rowlo != nullptr) {
      my_lo = p.rowlo[gi];
    } else if (p.window > 0) {
      my_lo = gi - p.window + 1 > 0 ? gi - p.window + 1 : 0;
    }
    atomicMin(&sched_lo[X], my_lo);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // key-tile ranges (tile index kt = key row / 128) of query tiles A and B; a
  // wide block (strong decay inside it) stops before its own two key tiles
  const bool wide = wide_flag != 0;
  const int ktA_hi = wide ? 2 * qblk - 1 : 2 * qblk, ktB_hi = wide ? 2 * qblk - 1 : 2 * qblk + 1;
  const int ktA_lo = sched_lo[0] / C::BN;
  const int ktB_lo = has_b ? sched_lo[1] / C::BN : ktB_hi + 1;
  const int kt_hi = has_b ? ktB_hi : ktA_hi;
  const int kt_lo = has_b ? min(ktA_lo, ktB_lo) : ktA_lo;
  const int nt = kt_hi - kt_lo + 1;  // visit order j = 0..nt-1 is kt = kt_hi - j
  // visit indices of the first/last key tile of each query tile (B may have none)
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
      int nk = 0, nv = 0;  // key / value tiles whose copies were issued
      mbar_arrive_expect_tx(qfull, (has_b ? 2 : 1) * C::Q_BYTES + KD * 4);
      for (int bx = 0; bx < C::QBOX; ++bx) {
        tma_load_3d(sQ + bx * 16384, &tmQ, qfull, bx * 64, q0, bh);
        if (has_b) tma_load_3d(sQ + C::Q_BYTES + bx * 16384, &tmQ, qfull, bx * 64, q0 + C::BM, bh);
      }
      bulk_load(sAQ, p.AQ + (static_cast<size_t>(bh) * p.NB + 2 * qblk) * KD, KD * 4, qfull);
      for (int j = 0; j < nt; ++j) {
        const int kt = kt_hi - j;
        const int ks = j % C::KS;
        if (j >= C::KS && !mbar_wait(&kempty[ks], ((j / C::KS) - 1) & 1, wc)) break;
        if (!(p.fault == 1 && j == 0)) {
          mbar_arrive_expect_tx(&kfull[ks], C::K_BYTES + KD * 4 + (HAS_GS ? C::GX_BYTES : 0));
          for (int bx = 0; bx < C::QBOX; ++bx)
            tma_load_3d(sK + ks * C::K_BYTES + bx * 16384, &tmK, &kfull[ks], bx * 64, kt * C::BN, bh);
          if (HAS_GS) tma_load_3d(sKX + ks * C::GX_BYTES, &tmKX, &kfull[ks], 0, kt * C::BN, bh);
          bulk_load(sAK + ks * KD, p.AK + (static_cast<size_t>(bh) * p.NB + kt) * KD, KD * 4,
                    &kfull[ks]);
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
      // Every copy issued must land before the CTA may exit: the last KS (VS)
      // tiles issued are the only ones a consumer may not have waited for.
      mbar_drain(qfull, 0, p.wait_ns);
      for (int j = nk > C::KS ? nk - C::KS : 0; j < nk; ++j)
        if (!(p.fault == 1 && j == 0)) mbar_drain(&kfull[j % C::KS], (j / C::KS) & 1, p.wait_ns);
      for (int j = nv > C::VS ? nv - C::VS : 0; j < nv; ++j)
        mbar_drain(&vfull[j % C::VS], (j / C::VS) & 1, p.wait_ns);
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(qfull, 0, wc);
      tc_fence_after();
      // Descriptors of every operand stage, built once: a K step only adds a
      // constant to the start-address field, so each MMA costs one add per operand.
      const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = sw128_desc(smem_u32(sV), 16384, 1024);
      const uint64_t dQX = HAS_GS ? sw32_desc(smem_u32(sQX), 256) : 0;
      const uint64_t dKX0 = HAS_GS ? sw32_desc(smem_u32(sKX), 256) : 0;
      // Only the previous key tile's P*V products can be pending at tile j.
      bool pendA = false, pendB = false;
      bool vseen = false;  // V stage of the previous tile already waited for
      int vrem_prev = 0;  // P*V reads still to issue for the previous tile's V stage
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
      auto issue_qk = [&](int x, int j, int ks) {
        const uint32_t dS = tmem_base + C::COL_S + 128 * x;
        const uint64_t dA = dQ0 + static_cast<uint64_t>(x * (C::Q_BYTES >> 4));
        const uint64_t dB = dK0 + static_cast<uint64_t>(ks * (C::K_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          umma_ss(dS, dA + koff, dB + koff, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        if (HAS_GS) {
          // + key-side gate term: (1, 1, 0..) x (hi, lo, 0..) over one more K slice
          umma_ss(dS, dQX, dKX0 + static_cast<uint64_t>(ks * (C::GX_BYTES >> 4)), C::IDESC_QK, 1u);
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
          issue_qk(0, j, ks);
          pendA = true;
          ++vrem_cur;
        }
        if (pendB) {
          if (!issue_pv(1, j - 1)) { ok = false; break; }
          pendB = false;
        }
        if (j >= jfB && j <= jlB) {
          issue_qk(1, j, ks);
          pendB = true;
          ++vrem_cur;
        }
        umma_commit(&kempty[ks]);
        if (vrem_cur == 0) umma_commit(&vempty[j % C::VS]);  // no P*V reads this tile
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
    const int hi = row_ok ? gi : 0x7fffffff;
    float rowA = 0.f;
    if (HAS_GS && row_ok) {
      rowA = p.ssa[(static_cast<size_t>(bh) * p.NB + gi / C::BM) * 4] -
             p.ssl[static_cast<size_t>(bh) * p.NB * C::BM + gi];
    }
    const float2 sc2 = make_float2(p.sc, p.sc);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const int jf = X == 0 ? jfA : jfB, jl = X == 0 ? jlA : jlB;
    // gate prefix before the key tile (log2 units), fetched one tile ahead
    float colA_next = 0.f;
    if (HAS_GS && jl >= jf) colA_next = p.ssa[(static_cast<size_t>(bh) * p.NB + (kt_hi - jf)) * 4];
    for (int j = jf; j <= jl; ++j) {
      const int cnt = j - jf;
      const int kt = kt_hi - j;
      const float colA = colA_next;
      if (HAS_GS && j < jl) colA_next = p.ssa[(static_cast<size_t>(bh) * p.NB + (kt - 1)) * 4];
      const bool got = mbar_wait(&sfull[X], cnt & 1, wc);
      if (!__all_sync(0xffffffffu, got)) {
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

      // S already holds scale^-1 * (key-side gate term) for gated inputs; the
      // row side joins through w.
      const int j0 = kt * C::BN;
      const float w = HAS_GS ? rowA - colA : 0.f;
      const bool partial = !__all_sync(0xffffffffu, lo <= j0 && hi >= j0 + C::BN - 1);
      if (partial) {
#pragma unroll
        for (int jj = 0; jj < C::BN; ++jj) {
          const int jg = j0 + jj;
          if (jg < lo || jg > hi) s[jj] = -INFINITY;
        }
      }
      float mx0 = s[0], mx1 = s[1];
#pragma unroll
      for (int jj = 2; jj < C::BN; jj += 4) {
        mx0 = fmax3(mx0, s[jj], s[jj + 1]);
        mx1 = fmax3(mx1, s[jj + 2], s[jj + 3]);
      }
      const float mt = fmaxf(mx0, mx1) * p.sc + w;
      const bool need = mt > m_used + 8.f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_used - mt);
        l *= alpha;
        m_used = mt;
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      const float2 off = make_float2(w - base, w - base);
      float2 rs = make_float2(0.f, 0.f);
      // P in 32-column chunks: each chunk's scores die once its 16 packed
      // bf16x2 columns are stored over S (the chunk's own, already-read columns).
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int jj = 0; jj < 32; jj += 2) {
          const float2 t = ffma2(make_float2(s[c + jj], s[c + jj + 1]), sc2, off);
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
          p.o + ((static_cast<size_t>(b) * p.T + (row_ok ? gi : 0)) * p.HQ + hq) * VD;
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
        p.lse[(static_cast<size_t>(b) * p.T + gi) * p.HQ + hq] = (m_used + log2f(Z)) * kLn2;
    }
  } else {
    // ------------------------------------------------------------- key-tile rescale
    reg_dealloc<48>();
    const int r = tid - 384;
    bool ok = mbar_wait(qfull, 0, wc);
    ok = !bar_or(1, 128, !ok);
    constexpr int CPR = KD / 8;        // 16-byte chunks per key row
    constexpr int RSTEP = 128 / CPR;   // rows between this thread's chunks
    const int L = r % CPR, box = L >> 3, c16 = L & 7;
    const int row0 = r / CPR;
    const uint32_t phys = static_cast<uint32_t>((c16 ^ (row0 & 7)) << 4);
    for (int j = 0; ok && j < nt; ++j) {
      const int ks = j % C::KS;
      const bool got = mbar_wait(&kfull[ks], (j / C::KS) & 1, wc);
      float* cb = sC + (j & 1) * KD;
      if (got && r < KD) cb[r] = ex2_approx((sAQ[r] - sAK[ks * KD + r]) * kLog2e);
      if (bar_or(1, 128, !got || *abort_flag != 0)) break;
      __nv_bfloat162 chi[4], clo[4];
      {
        const float4 c0 = *reinterpret_cast<const float4*>(cb + box * 64 + c16 * 8);
        const float4 c1 = *reinterpret_cast<const float4*>(cb + box * 64 + c16 * 8 + 4);
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          chi[i] = __floats2bfloat162_rn(cv[2 * i], cv[2 * i + 1]);
          const float2 h = __bfloat1622float2(chi[i]);
          clo[i] = __floats2bfloat162_rn(cv[2 * i] - h.x, cv[2 * i + 1] - h.y);
        }
      }
      uint8_t* tile = sK + ks * C::K_BYTES + box * 16384;
#pragma unroll 4
      for (int m = 0; m < CPR; ++m) {
        uint4* ptr = reinterpret_cast<uint4*>(tile + (row0 + m * RSTEP) * 128 + phys);
        *ptr = scale_chunk(*ptr, chi, clo);
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

template <int KD, int VD, bool HAS_GS>
cudaError_t tc_impl(const FwdArgs& a, const FwdWork& w, const CUtensorMap& tmQ,
                    const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKX,
                    cudaStream_t st) {
  using C = TcCfg<KD, VD>;
  auto kern = wall_fwd_tc_kernel<KD, VD, HAS_GS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.AQ = w.AQ;
  p.AK = w.AK;
  p.ssl = w.ssl;
  p.ssa = w.ssa;
  p.sink = a.sink;
  p.rowlo = a.cu_seqlens ? w.rowlo : nullptr;
  p.wide = w.wide;
  p.window = a.window;
  p.B = a.B;
  p.T = a.T;
  p.HQ = a.HQ;
  p.H = a.H;
  p.NB = a.NB;
  p.sc = a.scale * kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse != nullptr ? a.lse : w.lse_ws;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.fault = a.fault;
  const unsigned grid = static_cast<unsigned>((a.NB + 1) / 2) * a.B * a.HQ;
  kern<<<grid, 512, C::SMEM_ALLOC, st>>>(tmQ, tmK, tmV, tmKX, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs& a, const FwdWork& w, const CUtensorMap& tmQ,
                          const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKX,
                          cudaStream_t st) {
  const bool gs = a.g_scalar != nullptr;
#define WALL_TC(KD_, VD_)                                                      \
  if (a.K == KD_ && a.V == VD_)                                                \
    return gs ? tc_impl<KD_, VD_, true>(a, w, tmQ, tmK, tmV, tmKX, st)         \
              : tc_impl<KD_, VD_, false>(a, w, tmQ, tmK, tmV, tmKX, st);
  WALL_TC(64, 64)
  WALL_TC(64, 128)
  WALL_TC(128, 64)
  WALL_TC(128, 128)
#undef WALL_TC
  return cudaErrorInvalidValue;
}

}  // namespace wall
