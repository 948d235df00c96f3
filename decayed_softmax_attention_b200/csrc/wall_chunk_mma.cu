// Few-token chunks against the decode cache (multi-token decode, e.g.
// speculative verification) on the tensor cores: the split-KV pass of
// wall_chunk_split.cu with its dot products moved from packed fp32 FMAs to
// warp-level bf16 MMAs (m16n8k16, fp32 accumulate).  bf16 caches, groups of
// 1, 2, 4 or 8 query heads per KV head; fp32 and 16-head groups keep the
// SIMT pass.
//
// A CTA (split, token group, KV head, batch row) is one producer warp that
// streams 16-row stages of the cache (each query head's k_tilde rows and the
// v rows, 128-byte swizzled TMA tiles) plus the anchors R_c of every anchor
// chunk it enters, and one consumer warp.  The consumer's 16 MMA rows are
// the (token, head) pairs of its group, row r = token * G + head, so the
// score tile of a stage is a 16 x 16 block:
//   S[r, j] = sum_n qt[r, n] k_tilde[j, head(r), n],
//   qt[r, n] = scale log2(e) qh[r, n] 2^(AQ[head(r), n] - R_c[head(r), n])
// (the decode's formula, Wall Attention README "Decode"; qh and AQ as in the
// chunk's query prep).  k_tilde differs per query head, so the consumer runs
// one MMA chain per head over all 16 rows and keeps, for each of its rows,
// the chain of that row's head (a G-fold redundancy that costs nothing
// against the bytes each row streams).  The online softmax runs on the
// accumulator fragments (each row held by 4 lanes), and P, converted to bf16,
// is already in the A-operand layout of the P * V products.  The running
// maximum is raised only when a row maximum grows by more than 2^8 (exact:
// o and l share the stale maximum).  Partials (o, max, sum) go to the same
// layout as the SIMT pass, so the decode's combine finishes both.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

template <int KD, int VD, int G>
struct MmaCfg {
  static constexpr int MQ = 16 / G;  // tokens per CTA: 16 (token, head) rows
  static constexpr int BR = 16;      // cache rows per stage
  static constexpr int KB = BR * 128;  // one 64-channel half of 16 rows (128-byte swizzle)
  static constexpr int KH = KD / 64, VH = VD / 64;
  static constexpr int K_BYTES = G * KH * KB;
  static constexpr int V_BYTES = VH * KB;
  static constexpr int STAGE = K_BYTES + V_BYTES;  // a multiple of 1024
  // two stages in flight per consumer warp for G >= 4 keep four CTAs (four consumer
  // warps) on an SM for G = 4
  static constexpr int NS = G >= 4 ? 2 : 4;
  static constexpr int R_BYTES = G * KD * 4;
  static constexpr int QS = KD + 8;  // bf16 row stride of the staged queries (bank spread)
  static constexpr int FS = KD + 4;  // fp32 row stride of the per-chunk query factors
  static constexpr int OFF_R = NS * STAGE;             // [2][G][KD] fp32 anchors R_c
  static constexpr int OFF_Q = OFF_R + 2 * R_BYTES;    // [16][QS] bf16 anchored queries
  static constexpr int OFF_AQ = OFF_Q + 16 * QS * 2;   // [G][KD] fp32
  static constexpr int OFF_F = OFF_AQ + G * KD * 4;    // [G][FS] fp32 factors of a chunk
  static constexpr int OFF_BAR = OFF_F + G * FS * 4;
  static constexpr int SMEM = OFF_BAR + (2 * NS + 4) * 8 + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;  // the base is aligned to 1024 at run time
  static_assert(STAGE % 1024 == 0, "swizzled TMA tiles need 1024-byte alignment");
  static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D = A * B + D, A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, channel) in a run of 128-byte-swizzled 64-channel
// halves of `rows` rows each (the layout a SWIZZLE_128B TMA tile lands in).
__device__ __forceinline__ uint32_t swz(int row, int ch, int half_bytes) {
  const int x = ch >> 6, c16 = (ch & 63) >> 3;
  return x * half_bytes + row * 128 + ((c16 ^ (row & 7)) << 4);
}

template <int KD, int VD, int G>
__global__ void __launch_bounds__(64, 1) chunk_mma_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16* __restrict__ qh, const float* __restrict__ AQ,
    const float* __restrict__ r_cache, int t0, int M, int HQ, int C, int cap, int window,
    int ck_lo, int cps, int nsplit, int ntg, float sc, float* __restrict__ part, int* err,
    uint64_t wait_ns, const int* __restrict__ wide, int fault, const float* __restrict__ gs_cache) {
  using D = MmaCfg<KD, VD, G>;
  constexpr int MQ = D::MQ;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + D::OFF_BAR);
  uint64_t* empty = full + D::NS;
  uint64_t* rfull = empty + D::NS;
  uint64_t* rempty = rfull + 2;
  int* abort_flag = reinterpret_cast<int*>(rempty + 2);
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(dsm + D::OFF_Q);
  float* sAQ = reinterpret_cast<float*>(dsm + D::OFF_AQ);
  float* sF = reinterpret_cast<float*>(dsm + D::OFF_F);

  const int s = blockIdx.x / ntg, tg = blockIdx.x % ntg, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T_b = t0 + M;  // cache rows after the chunk's append
  const int nchunks = (T_b + C - 1) / C;
  const int ncap = (cap + C - 1) / C;
  const int ck0 = ck_lo + s * cps;
  const int ck1 = min(ck0 + cps, nchunks);
  const int m0 = tg * MQ;  // first token of this CTA's group
  const int qb = m0 >> 8;  // its 256-row query block
  const int NQB = (M + 255) >> 8;
  // rows the group can see (chunk-aligned start: a stage never straddles an anchor chunk)
  const int lo_g = window > 0 ? max(0, t0 + m0 + 1 - window) / C * C : 0;
  const int row_begin = max(ck0 * C, lo_g);
  const int row_end = min(min(ck1 * C, T_b), t0 + min(m0 + MQ, M));
  const int nst = row_end > row_begin ? (row_end - row_begin + D::BR - 1) / D::BR : 0;
  const int qrow0 = t0 + (qb << 8);  // cache row of the query block's first token

  if (threadIdx.x == 0) {
    for (int i = 0; i < D::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the group's anchored queries (zero past the chunk's last token) and AQ
  for (int idx = threadIdx.x; idx < 16 * KD; idx += 64) {
    const int r = idx / KD, n = idx % KD, m = r / G, hh = r % G;
    const size_t bh = static_cast<size_t>(b) * HQ + h * G + hh;
    sQ[r * D::QS + n] = m0 + m < M ? qh[(bh * M + m0 + m) * KD + n] : __float2bfloat16(0.f);
  }
  for (int idx = threadIdx.x; idx < G * KD; idx += 64) {
    const int hh = idx / KD, n = idx % KD;
    sAQ[idx] = AQ[((static_cast<size_t>(b) * HQ + h * G + hh) * NQB + qb) * KD + n];
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, err, wait_ns};

  if (warp == 1) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0, rissued = 0;
      for (int i = 0; i < nst; ++i) {
        const int row0 = row_begin + i * D::BR;
        if (i == 0 || row0 % C == 0) {  // a new anchor chunk: its R_c rows
          const int ci = row0 / C - row_begin / C, rs = ci & 1;
          if (ci >= 2 && !mbar_wait(&rempty[rs], ((ci >> 1) - 1) & 1, wc)) break;
          mbar_arrive_expect_tx(&rfull[rs], D::R_BYTES);
          bulk_load(dsm + D::OFF_R + rs * D::R_BYTES,
                    r_cache + ((static_cast<size_t>(b) * ncap + row0 / C) * HQ + h * G) * KD,
                    D::R_BYTES, &rfull[rs]);
          rissued = ci + 1;
        }
        const int slot = i % D::NS;
        if (i >= D::NS && !mbar_wait(&empty[slot], ((i / D::NS) - 1) & 1, wc)) break;
        uint8_t* st = dsm + slot * D::STAGE;
        if (!(fault == 7 && i == 0)) {  // testing hook: starve the consumer
          mbar_arrive_expect_tx(&full[slot], D::STAGE);
#pragma unroll
          for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int x = 0; x < D::KH; ++x)
              tma_load_4d(st + (hh * D::KH + x) * D::KB, &tmK, &full[slot], x * 64, h * G + hh,
                          row0, b);
#pragma unroll
          for (int x = 0; x < D::VH; ++x)
            tma_load_4d(st + D::K_BYTES + x * D::KB, &tmV, &full[slot], x * 64, h, row0, b);
        }
        issued = i + 1;
      }
      // every copy issued lands before the CTA may exit
      for (int i = issued > D::NS ? issued - D::NS : 0; i < issued; ++i)
        if (!(fault == 7 && i == 0)) mbar_drain(&full[i % D::NS], (i / D::NS) & 1, wait_ns);
      for (int ci = rissued > 2 ? rissued - 2 : 0; ci < rissued; ++ci)
        mbar_drain(&rfull[ci & 1], (ci >> 1) & 1, wait_ns);
    }
    return;
  }

  // --------------------------------------------------------------- consumer
  const int r1 = lane >> 2, hh = r1 % G;  // rows r1 and r1 + 8 (same head: G divides 8)
  const int mt1 = r1 / G, mt2 = (r1 + 8) / G;  // their tokens within the group
  const int kq = (lane & 3) * 2;  // first of the lane's two key / channel columns
  const int tok1 = t0 + m0 + mt1, tok2 = t0 + m0 + mt2;  // their cache rows
  const bool ok1 = m0 + mt1 < M, ok2 = m0 + mt2 < M;
  const int ghq = h * G + hh;
  unsigned wide_mask = 0;  // heads of the group whose query block is wide
#pragma unroll
  for (int g = 0; g < G; ++g)
    if (wide[(static_cast<size_t>(b) * HQ + h * G + g) * NQB + qb] != 0) wide_mask |= 1u << g;
  // strong decay inside the query block: its own rows are left to the diagonal kernel.
  // Key j is visible to the lane's rows iff wlo <= j <= lim (per row).
  const int row_cap = (wide_mask >> hh) & 1 ? qrow0 - 1 : 0x7fffffff;
  const int lim1 = ok1 ? min(min(tok1, row_cap), row_end - 1) : -1;
  const int lim2 = ok2 ? min(min(tok2, row_cap), row_end - 1) : -1;
  const int wlo1 = window > 0 ? tok1 - window + 1 : 0;
  const int wlo2 = window > 0 ? tok2 - window + 1 : 0;
  const size_t gsb = static_cast<size_t>(b) * cap;
  const float gs1 = (gs_cache != nullptr && ok1) ? gs_cache[(gsb + tok1) * HQ + ghq] : 0.f;
  const float gs2 = (gs_cache != nullptr && ok2) ? gs_cache[(gsb + tok2) * HQ + ghq] : 0.f;
  // ldmatrix lane roles: matrix lane / 8, its row lane % 8; the lane's byte offsets in a
  // stage: k_tilde (keys 0-7 / 8-15 by lm >> 1, channels +0 / +8 by lm & 1) per 16-channel
  // step, v (keys by lm & 1, channels by lm >> 1) per 16-channel step
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t sbase = smem_u32(dsm);
  uint32_t koff[KD / 16], voff[VD / 16];
#pragma unroll
  for (int ks = 0; ks < KD / 16; ++ks)
    koff[ks] = swz((lm >> 1) * 8 + lr, ks * 16 + (lm & 1) * 8, D::KB);
#pragma unroll
  for (int n2 = 0; n2 < VD / 16; ++n2)
    voff[n2] = D::K_BYTES + swz((lm & 1) * 8 + lr, n2 * 16 + (lm >> 1) * 8, D::KB);

  float o[VD / 8][4];
#pragma unroll
  for (int nt = 0; nt < VD / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float mrun1 = -INFINITY, mrun2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  uint32_t qa[KD / 16][4];
#pragma unroll
  for (int ks = 0; ks < KD / 16; ++ks) qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;

  for (int i = 0; i < nst; ++i) {
    const int row0 = row_begin + i * D::BR;
    if (i == 0 || row0 % C == 0) {
      // a new anchor chunk: factors sc 2^(AQ - R_c) per (head, channel), then the
      // A fragments qt of the lane's rows
      const int ci = row0 / C - row_begin / C, rs = ci & 1;
      const bool got = mbar_wait(&rfull[rs], (ci >> 1) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) break;
      const float* R = reinterpret_cast<const float*>(dsm + D::OFF_R + rs * D::R_BYTES);
      const bool own_chunk = row0 >= qrow0;  // the chunk lies in the query block
#pragma unroll
      for (int idx = lane; idx < G * KD; idx += 32) {
        const int fh = idx / KD, n = idx % KD;
        const bool own = own_chunk && ((wide_mask >> fh) & 1);
        sF[fh * D::FS + n] = own ? 0.f : sc * exp2f(sAQ[idx] - R[idx]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[rs]);
      const float* F = sF + hh * D::FS;
      const __nv_bfloat16* q1 = sQ + r1 * D::QS;
      const __nv_bfloat16* q2 = sQ + (r1 + 8) * D::QS;
#pragma unroll
      for (int ks = 0; ks < KD / 16; ++ks) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int n = ks * 16 + kq + hi * 8;
          const float2 f = *reinterpret_cast<const float2*>(F + n);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q1 + n));
          const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q2 + n));
          qa[ks][hi * 2] = pack_bf16(a.x * f.x, a.y * f.y);
          qa[ks][hi * 2 + 1] = pack_bf16(c.x * f.x, c.y * f.y);
        }
      }
      __syncwarp();  // sF is rewritten at the next chunk
    }
    const int slot = i % D::NS;
    const bool got = mbar_wait(&full[slot], (i / D::NS) & 1, wc);
    if (!__all_sync(0xffffffffu, got)) break;
    const uint32_t st = sbase + slot * D::STAGE;

    // S = qt * k_tilde^T, one chain per head; the lane keeps its rows' head
    float sv[2][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < KD / 16; ++ks) {
        // matrices: keys 0-7 / 8-15 (lm >> 1) x channels +0 / +8 (lm & 1)
        uint32_t bk[4];
        ldsm_x4(st + g * D::KH * D::KB + koff[ks], bk);
        mma_bf16(c[0], qa[ks], bk[0], bk[1]);
        mma_bf16(c[1], qa[ks], bk[2], bk[3]);
      }
      if (g == hh) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sv[nt][e] = c[nt][e];
      }
    }
    // mask (causal per token, window, the stage's end, wide rows) and the gate term
    float mx1 = -INFINITY, mx2 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = row0 + nt * 8 + kq + e;
        const bool k1 = j <= lim1 && j >= wlo1;
        const bool k2 = j <= lim2 && j >= wlo2;
        float gj = 0.f;
        if (gs_cache != nullptr && (k1 || k2)) gj = gs_cache[(gsb + j) * HQ + ghq];
        sv[nt][e] = k1 ? sv[nt][e] + (gs1 - gj) : -INFINITY;
        sv[nt][2 + e] = k2 ? sv[nt][2 + e] + (gs2 - gj) : -INFINITY;
        mx1 = fmaxf(mx1, sv[nt][e]);
        mx2 = fmaxf(mx2, sv[nt][2 + e]);
      }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      mx2 = fmaxf(mx2, __shfl_xor_sync(0xffffffffu, mx2, off));
    }
    const bool g1 = mx1 > mrun1 + 8.f || (mrun1 == -INFINITY && mx1 > -INFINITY);
    const bool g2 = mx2 > mrun2 + 8.f || (mrun2 == -INFINITY && mx2 > -INFINITY);
    if (__any_sync(0xffffffffu, g1 || g2)) {
      const float n1 = g1 ? mx1 : mrun1, n2 = g2 ? mx2 : mrun2;
      const float a1 = g1 ? (mrun1 == -INFINITY ? 0.f : exp2f(mrun1 - n1)) : 1.f;
      const float a2 = g2 ? (mrun2 == -INFINITY ? 0.f : exp2f(mrun2 - n2)) : 1.f;
#pragma unroll
      for (int nt = 0; nt < VD / 8; ++nt) {
        o[nt][0] *= a1; o[nt][1] *= a1;
        o[nt][2] *= a2; o[nt][3] *= a2;
      }
      l1 *= a1;
      l2 *= a2;
      mrun1 = n1;
      mrun2 = n2;
    }
    // P (bf16) in the A layout of P * V: (row r1, keys 0-7), (r1 + 8, 0-7), (r1, 8-15), (r1 + 8, 8-15)
    uint32_t pa[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float p0 = mrun1 == -INFINITY ? 0.f : ex2_approx(sv[nt][0] - mrun1);
      const float p1 = mrun1 == -INFINITY ? 0.f : ex2_approx(sv[nt][1] - mrun1);
      const float p2 = mrun2 == -INFINITY ? 0.f : ex2_approx(sv[nt][2] - mrun2);
      const float p3 = mrun2 == -INFINITY ? 0.f : ex2_approx(sv[nt][3] - mrun2);
      l1 += p0 + p1;
      l2 += p2 + p3;
      pa[nt * 2] = pack_bf16(p0, p1);
      pa[nt * 2 + 1] = pack_bf16(p2, p3);
    }
    // O += P * V: matrices keys 0-7 / 8-15 (lm & 1) x channels +0 / +8 (lm >> 1)
#pragma unroll
    for (int n2 = 0; n2 < VD / 16; ++n2) {
      uint32_t bv[4];
      ldsm_x4_t(st + voff[n2], bv);
      mma_bf16(o[2 * n2], pa, bv[0], bv[1]);
      mma_bf16(o[2 * n2 + 1], pa, bv[2], bv[3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);  // the stage is no longer read
  }

  // partials: o relative to the running maximum, the maximum, the sum (4 lanes a row)
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    l2 += __shfl_xor_sync(0xffffffffu, l2, off);
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int mt = half ? mt2 : mt1;
    if (m0 + mt >= M) continue;
    const float mr = half ? mrun2 : mrun1, lr_ = half ? l2 : l1;
    const size_t row = (static_cast<size_t>(b) * M + m0 + mt) * HQ + ghq;
    float* dst = part + (row * nsplit + s) * (VD + 2);
#pragma unroll
    for (int nt = 0; nt < VD / 8; ++nt) {
      const float2 v = mr == -INFINITY ? make_float2(0.f, 0.f)
                                       : make_float2(o[nt][half * 2], o[nt][half * 2 + 1]);
      *reinterpret_cast<float2*>(dst + nt * 8 + kq) = v;
    }
    if ((lane & 3) == 0) {
      dst[VD] = mr;
      dst[VD + 1] = mr == -INFINITY ? 0.f : lr_;
    }
  }
}

}  // namespace

template <int KD, int VD, int G>
cudaError_t launch_chunk_mma(const ChunkArgs& a, const void* qh, const float* AQ, const int* wide,
                             float* part, int ck_lo, int cps, int nsplit, int ntg,
                             cudaStream_t st) {
  using D = MmaCfg<KD, VD, G>;
  CUtensorMap tmK, tmV;
  // the maps end at the chunk's last row: rows past it arrive as zeros
  const cuuint64_t rows = static_cast<cuuint64_t>(a.t0) + a.M;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.HQ), rows,
                                static_cast<cuuint64_t>(a.B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(KD) * 2,
                                   static_cast<cuuint64_t>(a.HQ) * KD * 2,
                                   static_cast<cuuint64_t>(a.cap) * a.HQ * KD * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(D::BR), 1};
    if (!encode_tiled(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k_tilde, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(a.H), rows,
                                static_cast<cuuint64_t>(a.B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(VD) * 2,
                                   static_cast<cuuint64_t>(a.H) * VD * 2,
                                   static_cast<cuuint64_t>(a.cap) * a.H * VD * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(D::BR), 1};
    if (!encode_tiled(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v_cache, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  auto kern = chunk_mma_kernel<KD, VD, G>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(nsplit * ntg, a.H, a.B);
  if (a.ev_mid != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_mid), st);
  kern<<<grid, 64, D::SMEM_ALLOC, st>>>(
      tmK, tmV, static_cast<const __nv_bfloat16*>(qh), AQ, a.r_cache, a.t0, a.M, a.HQ, a.chunk,
      a.cap, a.window, ck_lo, cps, nsplit, ntg, a.scale * kLog2e, part, a.err, a.wait_ns, wide,
      a.fault, a.gs_cache);
  return cudaGetLastError();
}

#define WALL_CHUNK_MMA(KD, VD, G)                                                              \
  template cudaError_t launch_chunk_mma<KD, VD, G>(const ChunkArgs&, const void*, const float*, \
                                                   const int*, float*, int, int, int, int,     \
                                                   cudaStream_t);
#define WALL_CHUNK_MMA_G(KD, VD) \
  WALL_CHUNK_MMA(KD, VD, 1) WALL_CHUNK_MMA(KD, VD, 2) WALL_CHUNK_MMA(KD, VD, 4) WALL_CHUNK_MMA(KD, VD, 8)
WALL_CHUNK_MMA_G(64, 64)
WALL_CHUNK_MMA_G(64, 128)
WALL_CHUNK_MMA_G(128, 64)
WALL_CHUNK_MMA_G(128, 128)

}  // namespace wall
