// Wall attention prefill forward, bf16, on the 5th-generation tensor cores
// (tcgen05 + TMEM) of sm_100a.
//
// One CTA computes a 128-row query block of one (batch, query head).  The
// score of the Wall Attention README intro,
//   x(i,j) = scale * sum_n q[i,n] k[j,n] exp(G[i,n] - G[j,n]) + Gs[i] - Gs[j],
// becomes a dense contraction per (query block, key tile) pair:
//   S = Qh * diag(c) * Kh^T,  c[n] = exp(AQ[n] - AK[n])
// where Qh/Kh are the anchored operands written by the prepass.  The rescale
// warpgroup multiplies each key tile by c in shared memory (in place), the MMA
// warp issues S = Qh * Kt^T into TMEM, the softmax warpgroup (one query row
// per thread, read straight from its TMEM lane) runs the online softmax in the
// exp2 domain and writes P (bf16) back into TMEM over S, and the MMA warp
// accumulates O += P * V with P taken from TMEM.  This is the streaming
// (FlashAttention-style) softmax the README names; the decay factor never
// leaves the tile.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warps 4-7 softmax + epilogue, warps 8-11 key rescale.
// Key tiles are visited from the diagonal backwards so the running maximum is
// found early; O is rescaled only when a row maximum grows by more than 2^8
// (exact: the final normalisation uses the same stale maximum).
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
  static constexpr int BM = 128, BN = 128;
  static constexpr int KS = 3, VS = 2;
  static constexpr int QBOX = KD / 64, VBOX = VD / 64;
  static constexpr int Q_BYTES = BM * KD * 2;
  static constexpr int K_BYTES = BN * KD * 2;
  static constexpr int V_BYTES = BN * VD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * K_BYTES;
  static constexpr int OFF_AQ = OFF_V + VS * V_BYTES;
  static constexpr int OFF_AK = OFF_AQ + KD * 4;
  static constexpr int OFF_COL = OFF_AK + KS * KD * 4;
  static constexpr int OFF_COLA = OFF_COL + VS * BN * 4;
  static constexpr int OFF_C = OFF_COLA + VS * 16;
  static constexpr int OFF_BAR = OFF_C + 2 * KD * 4;
  // qfull, kfull[KS], kready[KS], kempty[KS], vfull[VS], vempty[VS], sfull[2], pfull[2],
  // odone, ofinal, mdrain
  static constexpr int NBAR = 1 + 3 * KS + 2 * VS + 2 + 2 + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_USED = OFF_MISC + 64;
  // At least 116 KB so that a second CTA never shares the SM (each CTA takes
  // all 512 TMEM columns).
  static constexpr int SMEM_ALLOC =
      (SMEM_USED + 1024) > 118784 ? (SMEM_USED + 1024) : 118784;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_O = 256;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, VD, 0, 1);
};

// Pack the 8 bf16 of one 16-byte chunk, scaled by c[0..7].
__device__ __forceinline__ uint4 scale_chunk(uint4 u, const float* c) {
  uint4 r;
  r.x = pack_bf16(bf16_lo(u.x) * c[0], bf16_hi(u.x) * c[1]);
  r.y = pack_bf16(bf16_lo(u.y) * c[2], bf16_hi(u.y) * c[3]);
  r.z = pack_bf16(bf16_lo(u.z) * c[4], bf16_hi(u.z) * c[5]);
  r.w = pack_bf16(bf16_lo(u.w) * c[6], bf16_hi(u.w) * c[7]);
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
// matching tcgen05.wait::ld (and from recycling tcgen05.st sources early).
__device__ __forceinline__ void reg_fence32(float* r) {
  asm volatile(""
               : "+f"(r[0]), "+f"(r[1]), "+f"(r[2]), "+f"(r[3]), "+f"(r[4]), "+f"(r[5]),
                 "+f"(r[6]), "+f"(r[7]), "+f"(r[8]), "+f"(r[9]), "+f"(r[10]), "+f"(r[11]),
                 "+f"(r[12]), "+f"(r[13]), "+f"(r[14]), "+f"(r[15]), "+f"(r[16]), "+f"(r[17]),
                 "+f"(r[18]), "+f"(r[19]), "+f"(r[20]), "+f"(r[21]), "+f"(r[22]), "+f"(r[23]),
                 "+f"(r[24]), "+f"(r[25]), "+f"(r[26]), "+f"(r[27]), "+f"(r[28]), "+f"(r[29]),
                 "+f"(r[30]), "+f"(r[31]));
}
__device__ __forceinline__ void reg_fence32u(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]));
}

template <int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(384, 1)
    wall_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcParams p) {
  using C = TcCfg<KD, VD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* sAQ = reinterpret_cast<float*>(smem + C::OFF_AQ);
  float* sAK = reinterpret_cast<float*>(smem + C::OFF_AK);
  float* sCol = reinterpret_cast<float*>(smem + C::OFF_COL);
  float* sColA = reinterpret_cast<float*>(smem + C::OFF_COLA);
  float* sC = reinterpret_cast<float*>(smem + C::OFF_C);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;
  uint64_t* kready = kfull + C::KS;
  uint64_t* kempty = kready + C::KS;
  uint64_t* vfull = kempty + C::KS;
  uint64_t* vempty = vfull + C::VS;
  uint64_t* sfull = vempty + C::VS;
  uint64_t* pfull = sfull + 2;
  uint64_t* odone = pfull + 2;
  uint64_t* ofinal = odone + 1;
  uint64_t* mdrain = ofinal + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* sched_lo = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BHQ = p.B * p.HQ;
  const int qb = p.NB - 1 - static_cast<int>(blockIdx.x / BHQ);
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
  const int q0 = qb * C::BM;

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&pfull[s], 128);
    }
    mbar_init(odone, 1);
    mbar_init(ofinal, 1);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    *sched_lo = 0x7fffffff;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();

  // Admitted key range per query row: [lo_i, i] (causal, window, document).
  int my_lo = 0;
  const bool is_softmax = (warp >= 4 && warp < 8);
  const int row = tid - 128;
  const int gi = q0 + row;
  const bool row_ok = is_softmax && gi < p.T;
  if (row_ok) {
    if (p.rowlo != nullptr) {
      my_lo = p.rowlo[gi];
    } else if (p.window > 0) {
      my_lo = gi - p.window + 1 > 0 ? gi - p.window + 1 : 0;
    }
    atomicMin(sched_lo, my_lo);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int lo_all = *sched_lo;
  const int kt_hi = qb;
  const int kt_lo = lo_all == 0x7fffffff ? kt_hi : (lo_all / C::BN);
  const int nt = kt_hi - kt_lo + 1;
  const WaitCtl wc{abort_flag, p.err, p.wait_ns};

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int last_k[C::KS], last_v[C::VS];
      for (int s = 0; s < C::KS; ++s) last_k[s] = -1;
      for (int s = 0; s < C::VS; ++s) last_v[s] = -1;
      mbar_arrive_expect_tx(qfull, C::Q_BYTES + KD * 4);
      for (int bx = 0; bx < C::QBOX; ++bx) tma_load_3d(sQ + bx * 16384, &tmQ, qfull, bx * 64, q0, bh);
      bulk_load(sAQ, p.AQ + (static_cast<size_t>(bh) * p.NB + qb) * KD, KD * 4, qfull);
      for (int n = 0; n < nt; ++n) {
        const int kt = kt_hi - n;
        const int ks = n % C::KS;
        if (n >= C::KS && !mbar_wait(&kempty[ks], ((n / C::KS) - 1) & 1, wc)) break;
        if (!(p.fault == 1 && n == 0)) {
          mbar_arrive_expect_tx(&kfull[ks], C::K_BYTES + KD * 4);
          for (int bx = 0; bx < C::QBOX; ++bx)
            tma_load_3d(sK + ks * C::K_BYTES + bx * 16384, &tmK, &kfull[ks], bx * 64, kt * C::BN, bh);
          bulk_load(sAK + ks * KD, p.AK + (static_cast<size_t>(bh) * p.NB + kt) * KD, KD * 4,
                    &kfull[ks]);
          last_k[ks] = n;
        }
        const int vs = n % C::VS;
        if (n >= C::VS && !mbar_wait(&vempty[vs], ((n / C::VS) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&vfull[vs], C::V_BYTES + (HAS_GS ? C::BN * 4 + 16 : 0));
        for (int bx = 0; bx < C::VBOX; ++bx)
          tma_load_4d(sV + vs * C::V_BYTES + bx * 16384, &tmV, &vfull[vs], bx * 64, kvh,
                      kt * C::BN, b);
        if (HAS_GS) {
          bulk_load(sCol + vs * C::BN,
                    p.ssl + static_cast<size_t>(bh) * p.NB * C::BN + static_cast<size_t>(kt) * C::BN,
                    C::BN * 4, &vfull[vs]);
          bulk_load(sColA + vs * 4, p.ssa + (static_cast<size_t>(bh) * p.NB + kt) * 4, 16,
                    &vfull[vs]);
        }
        last_v[vs] = n;
      }
      // Every copy issued must land before the CTA may exit.
      mbar_drain(qfull, 0, p.wait_ns);
      for (int s = 0; s < C::KS; ++s)
        if (last_k[s] >= 0) mbar_drain(&kfull[s], (last_k[s] / C::KS) & 1, p.wait_ns);
      for (int s = 0; s < C::VS; ++s)
        if (last_v[s] >= 0) mbar_drain(&vfull[s], (last_v[s] / C::VS) & 1, p.wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, wc);
      tc_fence_after();
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      auto issue_pv = [&](int m) -> bool {
        const int pb = m & 1, vs = m % C::VS;
        if (!mbar_wait(&pfull[pb], (m >> 1) & 1, wc)) return false;
        if (!mbar_wait(&vfull[vs], (m / C::VS) & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(sVa + vs * C::V_BYTES + kk * 2048, 16384, 1024);
          umma_ts(tmem_base + C::COL_O, tmem_base + C::COL_S0 + pb * 128 + kk * 8, bdesc,
                  C::IDESC_PV, (m > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&vempty[vs]);
        umma_commit(odone);
        return true;
      };
      for (int n = 0; ok && n < nt; ++n) {
        const int ks = n % C::KS;
        if (!mbar_wait(&kready[ks], (n / C::KS) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dS = tmem_base + C::COL_S0 + (n & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t adesc = sw128_desc(sQa + koff, 16, 1024);
          const uint64_t bdesc = sw128_desc(sKa + ks * C::K_BYTES + koff, 16, 1024);
          umma_ss(dS, adesc, bdesc, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&kempty[ks]);
        umma_commit(&sfull[n & 1]);
        if (n > 0 && !issue_pv(n - 1)) ok = false;
      }
      if (ok && nt > 0) ok = issue_pv(nt - 1);
      if (ok) umma_commit(ofinal);
      umma_commit(mdrain);
      mbar_drain(mdrain, 0, p.wait_ns);
    }
  } else if (is_softmax) {
    // ------------------------------------------------------------- softmax + epilogue
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int lo = row_ok ? my_lo : 0;
    const int hi = row_ok ? gi : 0x7fffffff;
    float rowA = 0.f;
    if (HAS_GS) {
      rowA = p.ssa[(static_cast<size_t>(bh) * p.NB + qb) * 4] +
             p.ssl[static_cast<size_t>(bh) * p.NB * C::BM + gi];
    }
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      const int kt = kt_hi - n, sb = n & 1, vs = n % C::VS;
      bool got = mbar_wait(&sfull[sb], (n >> 1) & 1, wc);
      if (HAS_GS && got) got = mbar_wait(&vfull[vs], (n / C::VS) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[C::BN];
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) tmem_ld32(lane_base + C::COL_S0 + sb * 128 + c, s + c);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < C::BN; c += 32) reg_fence32(s + c);

      const int j0 = kt * C::BN;
      float w = 0.f;
      if (HAS_GS) {
        const float* col = sCol + vs * C::BN;
        w = rowA - sColA[vs * 4];
#pragma unroll
        for (int j = 0; j < C::BN; j += 4) {
          const float4 cv = *reinterpret_cast<const float4*>(col + j);
          s[j] = fmaf(s[j], p.sc, -cv.x);
          s[j + 1] = fmaf(s[j + 1], p.sc, -cv.y);
          s[j + 2] = fmaf(s[j + 2], p.sc, -cv.z);
          s[j + 3] = fmaf(s[j + 3], p.sc, -cv.w);
        }
      }
      const bool partial = !__all_sync(0xffffffffu, lo <= j0 && hi >= j0 + C::BN - 1);
      if (partial) {
#pragma unroll
        for (int j = 0; j < C::BN; ++j) {
          const int jg = j0 + j;
          if (jg < lo || jg > hi) s[j] = -INFINITY;
        }
      }
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < C::BN; ++j) mt = fmaxf(mt, s[j]);
      mt = HAS_GS ? mt + w : mt * p.sc;
      const bool need = mt > m_used + 8.f;
      float alpha = 1.f;
      if (need) {
        alpha = ex2_approx(m_used - mt);
        l *= alpha;
        m_used = mt;
      }
      if (n > 0 && __any_sync(0xffffffffu, need)) {
        const bool g2 = mbar_wait(odone, (n - 1) & 1, wc);
        if (!__all_sync(0xffffffffu, g2)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < VD; c += 32) {
          float ov[32];
          tmem_ld32(lane_base + C::COL_O + c, ov);
          tmem_wait_ld();
          reg_fence32(ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] *= alpha;
          tmem_st32(lane_base + C::COL_O + c, reinterpret_cast<uint32_t*>(ov));
          tmem_wait_st();
          reg_fence32(ov);
        }
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[C::BN / 2];
      float rs = 0.f;
      if (HAS_GS) {
        const float off = w - base;
#pragma unroll
        for (int j = 0; j < C::BN; j += 2) {
          const float p0 = ex2_approx(s[j] + off), p1 = ex2_approx(s[j + 1] + off);
          rs += p0 + p1;
          pk[j >> 1] = pack_bf16(p0, p1);
        }
      } else {
        const float off = -base;
#pragma unroll
        for (int j = 0; j < C::BN; j += 2) {
          const float p0 = ex2_approx(fmaf(s[j], p.sc, off));
          const float p1 = ex2_approx(fmaf(s[j + 1], p.sc, off));
          rs += p0 + p1;
          pk[j >> 1] = pack_bf16(p0, p1);
        }
      }
      l += rs;
      tmem_st32(lane_base + C::COL_S0 + sb * 128, pk);
      tmem_st32(lane_base + C::COL_S0 + sb * 128 + 32, pk + 32);
      tmem_wait_st();
      reg_fence32u(pk);
      reg_fence32u(pk + 32);
      tc_fence_before();
      mbar_arrive(&pfull[sb]);
    }
    if (ok) {
      const bool got = mbar_wait(ofinal, 0, wc);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after();
      float Z = l;
      if (p.sink != nullptr && m_used != -INFINITY) Z += ex2_approx(p.sink[hq] * kLog2e - m_used);
      const float inv = 1.f / Z;
      __nv_bfloat16* orow =
          p.o + ((static_cast<size_t>(b) * p.T + (row_ok ? gi : 0)) * p.HQ + hq) * VD;
#pragma unroll 1
      for (int c = 0; c < VD; c += 32) {
        float ov[32];
        tmem_ld32(lane_base + C::COL_O + c, ov);
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
  } else if (warp >= 8) {
    // ------------------------------------------------------------- key-tile rescale
    const int r = tid - 256;
    bool ok = mbar_wait(qfull, 0, wc);
    ok = !bar_or(1, 128, !ok);
    constexpr int CPR = KD / 8;        // 16-byte chunks per key row
    constexpr int RSTEP = 128 / CPR;   // rows between this thread's chunks
    const int L = r % CPR, box = L >> 3, c16 = L & 7;
    const int row0 = r / CPR;
    const uint32_t phys = static_cast<uint32_t>((c16 ^ (row0 & 7)) << 4);
    for (int n = 0; ok && n < nt; ++n) {
      const int ks = n % C::KS;
      const bool got = mbar_wait(&kfull[ks], (n / C::KS) & 1, wc);
      float* cb = sC + (n & 1) * KD;
      if (got && r < KD) cb[r] = ex2_approx((sAQ[r] - sAK[ks * KD + r]) * kLog2e);
      if (bar_or(1, 128, !got || *abort_flag != 0)) break;
      float cv[8];
      const float4 c0 = *reinterpret_cast<const float4*>(cb + box * 64 + c16 * 8);
      const float4 c1 = *reinterpret_cast<const float4*>(cb + box * 64 + c16 * 8 + 4);
      cv[0] = c0.x; cv[1] = c0.y; cv[2] = c0.z; cv[3] = c0.w;
      cv[4] = c1.x; cv[5] = c1.y; cv[6] = c1.z; cv[7] = c1.w;
      uint8_t* tile = sK + ks * C::K_BYTES + box * 16384;
#pragma unroll 4
      for (int m = 0; m < CPR; ++m) {
        uint4* ptr = reinterpret_cast<uint4*>(tile + (row0 + m * RSTEP) * 128 + phys);
        *ptr = scale_chunk(*ptr, cv);
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
                    const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t st) {
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
  p.window = a.window;
  p.B = a.B;
  p.T = a.T;
  p.HQ = a.HQ;
  p.H = a.H;
  p.NB = a.NB;
  p.sc = a.scale * kLog2e;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.fault = a.fault;
  const unsigned grid = static_cast<unsigned>(a.NB) * a.B * a.HQ;
  kern<<<grid, 384, C::SMEM_ALLOC, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs& a, const FwdWork& w, const CUtensorMap& tmQ,
                          const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t st) {
  const bool gs = a.g_scalar != nullptr;
#define WALL_TC(KD_, VD_)                                                      \
  if (a.K == KD_ && a.V == VD_)                                                \
    return gs ? tc_impl<KD_, VD_, true>(a, w, tmQ, tmK, tmV, st)               \
              : tc_impl<KD_, VD_, false>(a, w, tmQ, tmK, tmV, st);
  WALL_TC(64, 64)
  WALL_TC(64, 128)
  WALL_TC(128, 64)
  WALL_TC(128, 128)
#undef WALL_TC
  return cudaErrorInvalidValue;
}

}  // namespace wall
