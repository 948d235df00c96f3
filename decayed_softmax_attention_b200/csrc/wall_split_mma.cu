// The split-KV pass over the decode cache on the tensor cores, for the
// single-token decode (Wall Attention README, "Decode"; dense or paged cache,
// per-row lengths, scalar gate, the fused append of the step's token) and for
// chunks of a few new tokens (multi-token decode, e.g. speculative
// verification): the dot products of the SIMT passes (wall_decode.cu,
// wall_chunk_split.cu) as warp-level bf16 MMAs (m16n8k16, fp32 accumulate).
// bf16 caches, groups of 1, 2, 4 or 8 query heads per KV head; fp32 and
// 16-head groups keep the SIMT passes.
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
// layout as the SIMT passes, so the decode's combine finishes both.
//
// Decode: the one token is row T_b - 1 of its batch row, its queries q and
// p_curr take the places of qh and AQ (qt = scale q 2^(p_curr - R_c)), and
// only the MMA rows of token 0 are real.  Rows of a stage past the rows in
// use (a shorter batch row, the rest of a paged block, the row a fused step
// is about to write) may hold anything: their scores are masked and their v
// rows zeroed in shared memory before P * V (0 x NaN is not 0).  The fused
// step's new row is formed by a third warp exactly as the append forms it
// (P = p_prev + g log2 e, a fresh chunk anchor or the stored one, k_tilde
// rounded to the cache dtype), written to the cache, scored, and merged into
// the consumer's partial of the CTA whose split holds it.
#include <atomic>

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
  static constexpr int OFF_NEW = OFF_F + G * FS * 4;   // fused step: [G] scores, [VD] v row
  static constexpr int OFF_BAR = (OFF_NEW + (G + VD) * 4 + 15) / 16 * 16;
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


struct MmaParams {
  const __nv_bfloat16* qh;  // chunk: anchored queries [B*HQ][M][K]; decode: q [B][HQ][K]
  const float* AQ;          // chunk: [B*HQ][NQB][K]; decode: p_curr [B][HQ][K] (fused: p_prev)
  const float* r_cache;
  const int* wide;          // [B*HQ][NQB] wide query blocks (null: none)
  const float* gs_cache;    // scalar-gate cache (null: no gate)
  const float* gs_curr;     // decode: PS of the current row [B][HQ] (null: the cache's row)
  const int* seqlens;       // decode: rows of each batch row (null: t0 + M for all)
  float* part;
  int* err;
  uint64_t wait_ns;
  int t0, M, T_kv, HQ, C, window, ck_lo, cps, nsplit, ntg;
  int skip_first;           // testing hook: the producer skips its first stage
  float sc;                 // scale * log2(e)
  PageMap pm;               // paged cache (pm.bt set) or dense (pm.cap = cap)
  DecodeFuse fu;            // FUSED: the step's new token
};

template <int KD, int VD, int G, bool PAGED, bool FUSED>
__global__ void __launch_bounds__(64, 1)
    split_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const MmaParams p) {
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
  float* sNew = reinterpret_cast<float*>(dsm + D::OFF_NEW);

  const int s = blockIdx.x / p.ntg, tg = blockIdx.x % p.ntg, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HQ = p.HQ, C = p.C, M = p.M;
  // this batch row's rows after the new tokens: T_b; its tokens sit at t0b .. T_b - 1
  const int T_b = p.seqlens ? max(M, min(p.seqlens[b], p.T_kv)) : p.t0 + M;
  const int t0b = T_b - M;
  const int nchunks = (T_b + C - 1) / C;
  const int ncap = (p.pm.cap + C - 1) / C;  // anchor chunks per batch row (dense caches)
  // per-row lengths: each split takes an even share of its own row's chunks (a shorter
  // row gives every split less work instead of leaving the last splits empty)
  const int cps = p.seqlens ? (nchunks - p.ck_lo + p.nsplit - 1) / p.nsplit : p.cps;
  const int ck0 = p.ck_lo + s * cps;
  const int ck1 = min(ck0 + cps, nchunks);
  const int m0 = tg * MQ;  // first token of this CTA's group
  const int qb = m0 >> 8;  // its 256-row query block
  const int NQB = (M + 255) >> 8;
  // rows the group can see (chunk-aligned start: a stage never straddles an anchor chunk)
  const int lo_g = p.window > 0 ? max(0, t0b + m0 + 1 - p.window) / C * C : 0;
  const int row_begin = max(ck0 * C, lo_g);
  const int row_end = min(min(ck1 * C, T_b), t0b + min(m0 + MQ, M));
  const int t_new = T_b - 1;  // FUSED: the row the step appends
  const bool mine = FUSED && t_new >= row_begin && t_new < row_end;
  const int s_end = FUSED ? min(row_end, t_new) : row_end;  // rows streamed from the cache
  const int nst = s_end > row_begin ? (s_end - row_begin + D::BR - 1) / D::BR : 0;
  const int qrow0 = t0b + (qb << 8);  // cache row of the query block's first token
  const size_t bhq0 = static_cast<size_t>(b) * HQ + h * G;  // the group's first query head

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
  // the group's (anchored) queries, zero past the last token, and AQ: the fused step's
  // P of the new row, p_prev + g log2 e, as the append forms it
  for (int idx = threadIdx.x; idx < 16 * KD; idx += blockDim.x) {
    const int r = idx / KD, n = idx % KD, m = r / G, hh = r % G;
    sQ[r * D::QS + n] =
        m0 + m < M ? p.qh[((bhq0 + hh) * M + m0 + m) * KD + n] : __float2bfloat16(0.f);
  }
  for (int idx = threadIdx.x; idx < G * KD; idx += blockDim.x) {
    const int hh = idx / KD, n = idx % KD;
    const size_t at = ((bhq0 + hh) * NQB + qb) * KD + n;
    if (FUSED) {
      const float gn = load1(static_cast<const __nv_bfloat16*>(p.fu.g_new) + at);
      sAQ[idx] = fmaf(gn, kLog2e, t_new > 0 ? p.AQ[at] : 0.f);
    } else {
      sAQ[idx] = p.AQ[at];
    }
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, p.err, p.wait_ns};

  if (warp == 1) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0, rissued = 0;
      // a stage never straddles a paged block: it starts on a chunk boundary plus a
      // multiple of 16 rows, and 16 divides C divides the block; the block lookup of
      // the next stage is issued a stage ahead
      int trow_next = PAGED && nst > 0 ? static_cast<int>(p.pm.row(b, row_begin)) : 0;
      for (int i = 0; i < nst; ++i) {
        const int row0 = row_begin + i * D::BR;
        const int trow = PAGED ? trow_next : row0;
        if (PAGED && i + 1 < nst) trow_next = static_cast<int>(p.pm.row(b, row0 + D::BR));
        const int tb = PAGED ? 0 : b;
        if (i == 0 || row0 % C == 0) {  // a new anchor chunk: its R_c rows
          const int ci = row0 / C - row_begin / C, rs = ci & 1;
          if (ci >= 2 && !mbar_wait(&rempty[rs], ((ci >> 1) - 1) & 1, wc)) break;
          // paged: chunk slots follow the pool's rows (the block size is a multiple of C)
          const size_t rslot = PAGED ? static_cast<size_t>(trow / C)
                                     : static_cast<size_t>(b) * ncap + row0 / C;
          mbar_arrive_expect_tx(&rfull[rs], D::R_BYTES);
          bulk_load(dsm + D::OFF_R + rs * D::R_BYTES, p.r_cache + (rslot * HQ + h * G) * KD,
                    D::R_BYTES, &rfull[rs]);
          rissued = ci + 1;
        }
        const int slot = i % D::NS;
        if (i >= D::NS && !mbar_wait(&empty[slot], ((i / D::NS) - 1) & 1, wc)) break;
        uint8_t* st = dsm + slot * D::STAGE;
        if (!(p.skip_first && i == 0)) {  // testing hook: starve the consumer
          mbar_arrive_expect_tx(&full[slot], D::STAGE);
#pragma unroll
          for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int x = 0; x < D::KH; ++x)
              tma_load_4d(st + (hh * D::KH + x) * D::KB, &tmK, &full[slot], x * 64, h * G + hh,
                          trow, tb);
#pragma unroll
          for (int x = 0; x < D::VH; ++x)
            tma_load_4d(st + D::K_BYTES + x * D::KB, &tmV, &full[slot], x * 64, h, trow, tb);
        }
        issued = i + 1;
      }
      // every copy issued lands before the CTA may exit
      for (int i = issued > D::NS ? issued - D::NS : 0; i < issued; ++i)
        if (!(p.skip_first && i == 0)) mbar_drain(&full[i % D::NS], (i / D::NS) & 1, p.wait_ns);
      for (int ci = rissued > 2 ? rissued - 2 : 0; ci < rissued; ++ci)
        mbar_drain(&rfull[ci & 1], (ci >> 1) & 1, p.wait_ns);
    }
    return;
  }

  // --------------------------------------------------------------- consumer
  const int r1 = lane >> 2, hh = r1 % G;  // rows r1 and r1 + 8 (same head: G divides 8)
  const int mt1 = r1 / G, mt2 = (r1 + 8) / G;  // their tokens within the group
  const int kq = (lane & 3) * 2;  // first of the lane's two key / channel columns
  const int tok1 = t0b + m0 + mt1, tok2 = t0b + m0 + mt2;  // their cache rows
  const bool ok1 = m0 + mt1 < M, ok2 = m0 + mt2 < M;
  const int ghq = h * G + hh;
  unsigned wide_mask = 0;  // heads of the group whose query block is wide
  if (p.wide != nullptr) {
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (p.wide[(bhq0 + g) * NQB + qb] != 0) wide_mask |= 1u << g;
  }
  // strong decay inside the query block: its own rows are left to the diagonal kernel.
  // Key j is visible to the lane's rows iff wlo <= j <= lim (per row); rows from s_end
  // on are not streamed
  const int row_cap = (wide_mask >> hh) & 1 ? qrow0 - 1 : 0x7fffffff;
  const int lim1 = ok1 ? min(min(tok1, row_cap), s_end - 1) : -1;
  const int lim2 = ok2 ? min(min(tok2, row_cap), s_end - 1) : -1;
  const int wlo1 = p.window > 0 ? tok1 - p.window + 1 : 0;
  const int wlo2 = p.window > 0 ? tok2 - p.window + 1 : 0;
  // scalar gate: the logit gains PS(token's row) - PS(key row), log2 units
  const float* gsc = p.gs_cache;
  auto gs_row = [&](int j) -> size_t {
    return PAGED ? p.pm.row(b, j) : static_cast<size_t>(b) * p.pm.cap + j;
  };
  float gs1 = 0.f, gs2 = 0.f;
  if (gsc != nullptr) {
    if (FUSED) {
      const size_t gi = bhq0 + hh;
      gs1 = fmaf(load1(static_cast<const __nv_bfloat16*>(p.fu.gs_new) + gi), kLog2e,
                 t_new > 0 ? p.fu.gs_prev[gi] : 0.f);
    } else if (p.gs_curr != nullptr) {
      gs1 = p.gs_curr[bhq0 + hh];
    } else {
      if (ok1) gs1 = gsc[gs_row(tok1) * HQ + ghq];
      if (ok2) gs2 = gsc[gs_row(tok2) * HQ + ghq];
    }
  }
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

  if (FUSED && mine) {
    // ---- the fused step's new row (batch row b, KV head h, its G query heads), formed
    // before the stream (the producer is already filling the ring): lane-strided over
    // (head, channel), k_tilde as the cache stores it; its scores and value row wait
    // in shared memory for the merge at the end
    const bool fresh = t_new % C == 0;  // the row opens a chunk: its anchor is its own P
    const size_t prow = PAGED ? p.pm.row(b, t_new) : static_cast<size_t>(b) * p.pm.cap + t_new;
    const size_t rslot = PAGED ? prow / C : static_cast<size_t>(b) * ncap + t_new / C;
    float* ra = p.fu.r_cache + (rslot * HQ + h * G) * KD;
    __nv_bfloat16* kw = static_cast<__nv_bfloat16*>(p.fu.k_tilde) + (prow * HQ + h * G) * KD;
    const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(p.fu.k_new) +
                              (static_cast<size_t>(b) * gridDim.y + h) * KD;
    float dsum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      dsum[g] = 0.f;
#pragma unroll
      for (int n = lane; n < KD; n += 32) {
        const float pc = sAQ[g * KD + n];
        const float R = fresh ? pc : ra[g * KD + n];
        if (!fresh && R - pc > kCacheRangeLog2) atomicOr(p.err, kDevErrRange);
        const float kf = __bfloat162float(kn[n]);
        const __nv_bfloat16 kt = __float2bfloat16_rn(fresh ? kf : kf * ex2_approx(R - pc));
        kw[g * KD + n] = kt;
        const float qv = __bfloat162float(sQ[g * D::QS + n]);  // MMA row g: token 0, head g
        dsum[g] = fmaf(qv * p.sc * exp2f(pc - R), __bfloat162float(kt), dsum[g]);
        p.fu.p_last[(bhq0 + g) * KD + n] = pc;
      }
    }
    if (fresh)
      for (int idx = lane; idx < G * KD; idx += 32) ra[idx] = sAQ[idx];
    const __nv_bfloat16* vn = static_cast<const __nv_bfloat16*>(p.fu.v_new) +
                              (static_cast<size_t>(b) * gridDim.y + h) * VD;
    __nv_bfloat16* vw = static_cast<__nv_bfloat16*>(p.fu.v) + (prow * gridDim.y + h) * VD;
    for (int c = lane; c < VD; c += 32) {
      const __nv_bfloat16 x = vn[c];
      vw[c] = x;
      sNew[G + c] = __bfloat162float(x);
    }
    if (gsc != nullptr && lane < G) {  // the new row's gate prefix PS (its own term is 0)
      const_cast<float*>(gsc)[prow * HQ + h * G + lane] = fmaf(
          load1(static_cast<const __nv_bfloat16*>(p.fu.gs_new) + bhq0 + lane), kLog2e,
          t_new > 0 ? p.fu.gs_prev[bhq0 + lane] : 0.f);
      p.fu.gs_last[bhq0 + lane] = gsc[prow * HQ + h * G + lane];
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum[g] += __shfl_xor_sync(0xffffffffu, dsum[g], off);
      if (lane == 0) sNew[g] = dsum[g];
    }
    __syncwarp();
  }

  float o[VD / 8][4];
#pragma unroll
  for (int nt = 0; nt < VD / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float mrun1 = -INFINITY, mrun2 = -INFINITY, l1 = 0.f, l2 = 0.f;
  uint32_t qa[KD / 16][4];
#pragma unroll
  for (int ks = 0; ks < KD / 16; ++ks) qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;
  // gate prefixes of the lane's 4 keys of a stage (keys nt * 8 + kq + e), fetched a stage
  // ahead; a stage lies in one paged block, so one lookup serves its rows
  float gnext[4] = {0.f, 0.f, 0.f, 0.f};
  auto gate_fetch = [&](int row0, float* dst) {
    const size_t prow0 = gs_row(row0);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int jo = (q4 >> 1) * 8 + kq + (q4 & 1);
      dst[q4] = row0 + jo < s_end ? gsc[(prow0 + jo) * HQ + ghq] : 0.f;
    }
  };
  if (gsc != nullptr && nst > 0) gate_fetch(row_begin, gnext);

  for (int i = 0; i < nst; ++i) {
    const int row0 = row_begin + i * D::BR;
    float gk[4] = {gnext[0], gnext[1], gnext[2], gnext[3]};
    if (gsc != nullptr && i + 1 < nst) gate_fetch(row0 + D::BR, gnext);
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
        sF[fh * D::FS + n] = own ? 0.f : p.sc * exp2f(sAQ[idx] - R[idx]);
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
    if (row0 + D::BR > s_end) {
      // rows from s_end on may hold anything: zero their v rows (both halves)
      uint8_t* sv0 = dsm + slot * D::STAGE + D::K_BYTES;
      const int first = s_end - row0;  // >= 1
      for (int idx = lane; idx < (D::BR - first) * 8 * D::VH; idx += 32) {
        const int rr = first + idx / (8 * D::VH), rest = idx % (8 * D::VH);
        *reinterpret_cast<uint4*>(sv0 + (rest >> 3) * D::KB + rr * 128 + (rest & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();  // ordered before the slot's next TMA fill
      __syncwarp();
    }

    // S = qt * k_tilde^T, one chain per head; the lane keeps its rows' head
    float sv[2][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < KD / 16; ++ks) {
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
    // mask (causal per token, window, the streamed rows, wide rows) and the gate term
    float mx1 = -INFINITY, mx2 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = row0 + nt * 8 + kq + e;
        const bool k1 = j <= lim1 && j >= wlo1;
        const bool k2 = j <= lim2 && j >= wlo2;
        const float gj = gk[nt * 2 + e];
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
  if (FUSED && mine) {
    // the new row (score d, sum 1, value v) joins the partial of token 0's rows
    if (mt1 == 0) {
      const float d = sNew[hh];
      {
        const float mn = fmaxf(mrun1, d);
        const float a = mrun1 == -INFINITY ? 0.f : exp2f(mrun1 - mn);
        const float w = exp2f(d - mn);
#pragma unroll
        for (int nt = 0; nt < VD / 8; ++nt) {
          o[nt][0] = fmaf(o[nt][0], a, w * sNew[G + nt * 8 + kq]);
          o[nt][1] = fmaf(o[nt][1], a, w * sNew[G + nt * 8 + kq + 1]);
        }
        l1 = fmaf(l1, a, w);
        mrun1 = mn;
      }
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int mt = half ? mt2 : mt1;
    if (m0 + mt >= M) continue;
    const float mr = half ? mrun2 : mrun1, lr_ = half ? l2 : l1;
    const size_t row = (static_cast<size_t>(b) * M + m0 + mt) * HQ + ghq;
    float* dst = p.part + (row * p.nsplit + s) * (VD + 2);
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

namespace {

// k_tilde and v tile maps: 64-channel halves of 16 rows, 128-byte swizzle.  Dense caches:
// [B, rows, ...] with row stride cap; a paged pool: one batch row of nblk * bs rows.
template <int KD, int VD>
bool mma_maps(CUtensorMap* tmK, CUtensorMap* tmV, const void* k_tilde, const void* v, int HQ,
              int H, cuuint64_t rows, cuuint64_t rstride, cuuint64_t nb) {
  const cuuint32_t box[4] = {64, 1, 16, 1};
  const cuuint64_t kd[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(HQ), rows, nb};
  const cuuint64_t ks[3] = {static_cast<cuuint64_t>(KD) * 2,
                            static_cast<cuuint64_t>(HQ) * KD * 2, rstride * HQ * KD * 2};
  const cuuint64_t vd[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(H), rows, nb};
  const cuuint64_t vs[3] = {static_cast<cuuint64_t>(VD) * 2, static_cast<cuuint64_t>(H) * VD * 2,
                            rstride * H * VD * 2};
  return encode_tiled(tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k_tilde, kd, ks, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tiled(tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v, vd, vs, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int KD, int VD, int G, bool PAGED, bool FUSED>
cudaError_t run_split_mma(const CUtensorMap& tmK, const CUtensorMap& tmV, const MmaParams& p,
                          dim3 grid, cudaStream_t st) {
  using D = MmaCfg<KD, VD, G>;
  auto kern = split_mma_kernel<KD, VD, G, PAGED, FUSED>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  kern<<<grid, 64, D::SMEM_ALLOC, st>>>(tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

template <int KD, int VD, int G>
cudaError_t launch_chunk_mma(const ChunkArgs& a, const void* qh, const float* AQ, const int* wide,
                             float* part, int ck_lo, int cps, int nsplit, int ntg,
                             cudaStream_t st) {
  CUtensorMap tmK, tmV;
  // the maps end at the chunk's last row: rows past it arrive as zeros
  if (!mma_maps<KD, VD>(&tmK, &tmV, a.k_tilde, a.v_cache, a.HQ, a.H,
                        static_cast<cuuint64_t>(a.t0) + a.M, static_cast<cuuint64_t>(a.cap),
                        static_cast<cuuint64_t>(a.B)))
    return cudaErrorInvalidValue;
  MmaParams p{};
  p.qh = static_cast<const __nv_bfloat16*>(qh);
  p.AQ = AQ;
  p.r_cache = a.r_cache;
  p.wide = wide;
  p.gs_cache = a.gs_cache;
  p.part = part;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.t0 = a.t0; p.M = a.M; p.T_kv = a.t0 + a.M; p.HQ = a.HQ; p.C = a.chunk; p.window = a.window;
  p.ck_lo = ck_lo; p.cps = cps; p.nsplit = nsplit; p.ntg = ntg;
  p.skip_first = a.fault == 7 ? 1 : 0;
  p.sc = a.scale * kLog2e;
  p.pm.cap = a.cap;
  if (a.ev_mid != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_mid), st);
  return run_split_mma<KD, VD, G, false, false>(tmK, tmV, p, dim3(nsplit * ntg, a.H, a.B), st);
}

template <int KD, int VD, int G>
cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t st) {
  const bool paged = a.pm.paged();
  const bool fused = a.fuse.k_new != nullptr;
  if (a.gs_cache != nullptr && fused && a.fuse.gs_new == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tmK, tmV;
  // dense: [B, cap, ...] with rows limited to T_kv; paged: the pool as one batch row
  const cuuint64_t rows = paged ? static_cast<cuuint64_t>(a.pm.nblk) * a.pm.bs
                                : static_cast<cuuint64_t>(a.T_kv);
  if (!mma_maps<KD, VD>(&tmK, &tmV, a.k_tilde, a.v, a.HQ, a.H, rows,
                        paged ? rows : static_cast<cuuint64_t>(a.cap),
                        paged ? 1 : static_cast<cuuint64_t>(a.B)))
    return cudaErrorInvalidValue;
  MmaParams p{};
  p.qh = static_cast<const __nv_bfloat16*>(a.q);
  p.AQ = a.p_curr;
  p.r_cache = a.r_cache;
  p.gs_cache = a.gs_cache;
  p.gs_curr = a.gs_curr;
  p.seqlens = a.seqlens;
  p.part = a.part;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.t0 = a.T_kv - 1; p.M = 1; p.T_kv = a.T_kv; p.HQ = a.HQ; p.C = a.chunk; p.window = 0;
  const int nchunks = (a.T_kv + a.chunk - 1) / a.chunk;
  p.ck_lo = 0; p.cps = (nchunks + a.nsplit - 1) / a.nsplit; p.nsplit = a.nsplit; p.ntg = 1;
  p.skip_first = a.fault == 2 ? 1 : 0;
  p.sc = a.scale * kLog2e;
  p.pm = a.pm;
  p.fu = a.fuse;
  const dim3 grid(a.nsplit, a.H, a.B);
  if (paged)
    return fused ? run_split_mma<KD, VD, G, true, true>(tmK, tmV, p, grid, st)
                 : run_split_mma<KD, VD, G, true, false>(tmK, tmV, p, grid, st);
  return fused ? run_split_mma<KD, VD, G, false, true>(tmK, tmV, p, grid, st)
               : run_split_mma<KD, VD, G, false, false>(tmK, tmV, p, grid, st);
}

namespace {
template <int KD, int VD, int G>
int mma_ctas_per_sm() {
  static std::atomic<int> cached{0};
  const int v = cached.load();
  if (v > 0) return v;
  using D = MmaCfg<KD, VD, G>;
  auto kern = split_mma_kernel<KD, VD, G, false, false>;
  int n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM_ALLOC) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 64, D::SMEM_ALLOC) != cudaSuccess ||
      n < 1)
    n = 1;
  cached.store(n);
  return n;
}
template <int KD, int VD>
int mma_ctas_by_group(int group) {
  switch (group) {
    case 1: return mma_ctas_per_sm<KD, VD, 1>();
    case 2: return mma_ctas_per_sm<KD, VD, 2>();
    case 4: return mma_ctas_per_sm<KD, VD, 4>();
    case 8: return mma_ctas_per_sm<KD, VD, 8>();
    default: return 1;
  }
}
}  // namespace

int decode_ctas_per_sm(int K, int V, int group, bool bf16) {
  if (!bf16) return 1;
  if (K == 64 && V == 64) return mma_ctas_by_group<64, 64>(group);
  if (K == 64 && V == 128) return mma_ctas_by_group<64, 128>(group);
  if (K == 128 && V == 64) return mma_ctas_by_group<128, 64>(group);
  if (K == 128 && V == 128) return mma_ctas_by_group<128, 128>(group);
  return 1;
}

#define WALL_SPLIT_MMA(KD, VD, G)                                                               \
  template cudaError_t launch_chunk_mma<KD, VD, G>(const ChunkArgs&, const void*, const float*, \
                                                   const int*, float*, int, int, int, int,     \
                                                   cudaStream_t);                              \
  template cudaError_t launch_decode_mma<KD, VD, G>(const DecodeArgs&, cudaStream_t);
#define WALL_SPLIT_MMA_G(KD, VD) \
  WALL_SPLIT_MMA(KD, VD, 1) WALL_SPLIT_MMA(KD, VD, 2) WALL_SPLIT_MMA(KD, VD, 4) WALL_SPLIT_MMA(KD, VD, 8)
WALL_SPLIT_MMA_G(64, 64)
WALL_SPLIT_MMA_G(64, 128)
WALL_SPLIT_MMA_G(128, 64)
WALL_SPLIT_MMA_G(128, 128)

}  // namespace wall
