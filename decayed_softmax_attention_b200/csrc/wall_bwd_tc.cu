// Wall attention prefill backward, bf16, on the tcgen05 tensor cores (sm_100a):
// the two contraction kernels of the backward (Wall Attention README, intro
// formula; the gradient passes around them are in wall_bwd.cu).
//
// Both kernels recompute the score tile from the anchored operands of the
// forward prepass with one channel vector c = exp(AQ - AK) per (query tile,
// key tile) pair, exactly as the forward does, take p = exp2(x - lse) with the
// forward's lse, and form dS = p (dP - delta), dP = dO V^T:
//
// Key-block kernel (one CTA per 128-key tile of one batch * query head; loops
// over the query tiles that admit its keys):
//   S^T = Kh (Qh c)^T,  dP^T = V dO^T            (tcgen05, both operands in SMEM)
//   dV += P^T dO,       dK += dS^T (Qh c)        (P^T, dS^T read from TMEM)
// TMEM: S^T | dP^T | dV | dK = 4 x 128 columns; P^T (dS^T) are stored as packed
// bf16 over the S^T (dP^T) columns (each elementwise half inside the columns it
// read itself).  MMA issue order per query tile i:
//   dV(i), S(i+1), dK(i), dP(i+1)
// so the elementwise warpgroup's two passes (P from S; dS from dP) overlap
// the tensor core, and every TMEM overwrite follows, in issue order, the MMA
// that read the old contents (tcgen05 ops of one thread run in order).
//
// Query-block kernel (one CTA per 128-row query tile; loops over the admitted
// key tiles, diagonal first):
//   S = Qh (Kh c)^T,  dP = dO V^T,  dQ += dS (Kh c)
// TMEM: S0 | S1 | dP | dQ; S is double-buffered so S(j+1) is computed while
// the elementwise warpgroup works on tile j.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator; warpgroups 1 and 2 = elementwise + epilogue, one TMEM lane =
// one row per thread, warpgroup 1 on the tile's columns 0-63 and warpgroup 2 on
// 64-127 (two warps per SM sub-partition hide each other's MUFU and TMEM
// latencies); warpgroup 3 multiplies each streamed Qh (key-block kernel) or Kh
// (query-block kernel) tile by c in shared memory.  Registers are re-split at
// start (setmaxnreg): 88 / 168 / 168 / 88 in the key-block kernel, 88 / 176 /
// 176 / 72 in the query-block kernel (each sums to 512 = 4 x the 128 of the
// launch).  The elementwise passes run on fp32 pairs (.f32x2 fma / mul / add):
// P stays in registers as fp32 between the two passes, and the per-column
// vectors are read 4 at a time as broadcast 16-byte loads.  Every wait is
// bounded (device error word + CTA abort flag), copies in flight are drained
// and TMEM is freed before exit.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

struct BtcParams {
  const float* AQ;     // [bh][NB][KD] prepass anchors
  const float* AK;
  const float* rowt;   // [bh][TP] Gs log2e - lse log2e
  const float* colt;   // [bh][TP] Gs log2e (g_scalar only)
  const float* delta;  // [bh][TP]
  const int* rowlo;    // [TP] first admitted key (packed documents) or null
  int window;
  int B, T, HQ, H, NB;
  float sc;            // scale * log2(e)
  float* acc;          // key-block: dK accumulator; query-block: dQ accumulator [bh][T][KD]
  float* dvh;          // key-block: dV [bh][T][VD]
  float* rs;           // row sums of dS: rsA (per key) / rsB (per query) [bh][T]
  int* err;
  uint64_t wait_ns;
  int fault;           // testing hook: 4 = key-block producer skips its first query tile,
                       // 5 = query-block producer skips its first key tile
};

template <int KD, int VD>
struct BtcCfg {
  static constexpr int BM = 128;
  static constexpr int KB = BM * KD * 2;  // one 128-row bf16 tile of KD channels
  static constexpr int VB = BM * VD * 2;
  static constexpr int KBOX = KD / 64, VBOX = VD / 64;
  static constexpr int VEC = 128 * 4;     // one per-row fp32 vector of a tile
  // key-block kernel
  static constexpr int A_K = 0;
  static constexpr int A_V = A_K + KB;
  static constexpr int A_Q = A_V + VB;           // 2 stages
  static constexpr int A_DO = A_Q + 2 * KB;      // 2 stages
  static constexpr int A_AQ = A_DO + 2 * VB;     // 2 x KD fp32
  static constexpr int A_ROWT = A_AQ + 2 * KD * 4;
  static constexpr int A_DEL = A_ROWT + 2 * VEC;
  static constexpr int A_LO = A_DEL + 2 * VEC;
  static constexpr int A_AK = A_LO + 2 * VEC;    // KD fp32
  static constexpr int A_COLT = A_AK + KD * 4;   // 128 fp32
  static constexpr int A_C = A_COLT + VEC;       // 2 x KD fp32
  static constexpr int A_BAR = A_C + 2 * KD * 4;
  // kvfull, qfull[2], qready[2], qempty[2], sfull, dpfull, pready, dsready, final, mdrain
  static constexpr int A_NBAR = 1 + 2 + 2 + 2 + 6 + 2;  // + qready_hi[2]
  static constexpr int A_MISC = A_BAR + A_NBAR * 8;
  static constexpr int A_RS = A_MISC + 64;       // 128 fp32
  // at least 116 KB so that a second CTA never shares the SM (each takes all of TMEM)
  static constexpr int A_SMEM = (A_RS + VEC + 1024) > 118784 ? (A_RS + VEC + 1024) : 118784;
  // query-block kernel
  static constexpr int KS = 3;                   // streamed key tiles
  static constexpr int B_Q = 0;
  static constexpr int B_DO = B_Q + KB;
  static constexpr int B_K = B_DO + VB;          // KS stages
  static constexpr int B_V = B_K + KS * KB;      // 1 stage
  static constexpr int B_AQ = B_V + VB;          // KD fp32
  static constexpr int B_ROWT = B_AQ + KD * 4;
  static constexpr int B_DEL = B_ROWT + VEC;
  static constexpr int B_AK = B_DEL + VEC;       // KS x KD fp32
  static constexpr int B_COLT = B_AK + KS * KD * 4;  // KS x 128 fp32
  static constexpr int B_LO = B_COLT + KS * VEC;     // KS x 128 int (unused without packing)
  static constexpr int B_C = B_LO + KS * VEC;        // 2 x KD fp32
  static constexpr int B_BAR = B_C + 2 * KD * 4;
  // qfull, kfull[KS], kready[KS], kempty[KS], vfull, vempty, sfull[2], dpfull, dsready, final, mdrain
  static constexpr int B_NBAR = 1 + 3 * KS + 2 + 2 + 4;
  static constexpr int B_MISC = B_BAR + B_NBAR * 8;
  static constexpr int B_RS = B_MISC + 64;       // 128 fp32
  static constexpr int B_SMEM = (B_RS + VEC + 1024) > 118784 ? (B_RS + VEC + 1024) : 118784;
  static constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t IDESC_NK = idesc_bf16_f32(128, KD, 0, 1);  // N = KD, B MN-major
  static constexpr uint32_t IDESC_NV = idesc_bf16_f32(128, VD, 0, 1);  // N = VD, B MN-major
};

// K-step offset (16 bf16 channels) inside a K-major 128-byte-swizzled tile
// made of 64-channel boxes of 16 KB: descriptor units of 16 bytes.
__device__ __forceinline__ uint64_t kmaj_step(int kk) {
  return static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
}
// TMEM column of K-step kk (16 rows) of a packed-bf16 operand written by the
// two elementwise halves: half h stores its 64 values of a row as 32 packed
// columns at 64 h .. 64 h + 31 (inside the columns it read itself).
__device__ __forceinline__ uint32_t packed_col(int kk) { return kk * 8 + (kk >= 4 ? 32 : 0); }
// TMEM column where half cb/64 stores the packed chunk starting at column c.
__device__ __forceinline__ uint32_t packed_dst(int c, int cb) { return cb + ((c - cb) >> 1); }

// K-step offset (16 rows) inside an MN-major tile: 16 rows of 128 bytes.
__device__ __forceinline__ uint64_t mnmaj_step(int kk) {
  return static_cast<uint64_t>((kk * 2048) >> 4);
}

// Scale the 8 bf16 of one 16-byte chunk by c[0..7] (c split into a bf16 head
// and tail so the product carries a single bf16 rounding).
__device__ __forceinline__ uint4 scale8(uint4 u, const __nv_bfloat162* chi,
                                        const __nv_bfloat162* clo) {
  uint4 r;
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&u);
  __nv_bfloat162* y = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = __hfma2(x[i], chi[i], __hmul2(x[i], clo[i]));
  return r;
}

// OR of `pred` over the `nthreads` threads of named barrier `id`.
__device__ __forceinline__ bool bar_any(int id, int nthreads, bool pred) {
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
__device__ __forceinline__ void fence_regs32(float* r) {
  asm volatile(""
               : "+f"(r[0]), "+f"(r[1]), "+f"(r[2]), "+f"(r[3]), "+f"(r[4]), "+f"(r[5]),
                 "+f"(r[6]), "+f"(r[7]), "+f"(r[8]), "+f"(r[9]), "+f"(r[10]), "+f"(r[11]),
                 "+f"(r[12]), "+f"(r[13]), "+f"(r[14]), "+f"(r[15]), "+f"(r[16]), "+f"(r[17]),
                 "+f"(r[18]), "+f"(r[19]), "+f"(r[20]), "+f"(r[21]), "+f"(r[22]), "+f"(r[23]),
                 "+f"(r[24]), "+f"(r[25]), "+f"(r[26]), "+f"(r[27]), "+f"(r[28]), "+f"(r[29]),
                 "+f"(r[30]), "+f"(r[31]));
}

// Multiplies one 128-row tile of KD bf16 channels (128-byte swizzle, boxes of
// 64 channels) by c[KD] in place; 128 threads, r = thread index.  BATCH chunks
// are loaded before any is scaled and stored (the query-block kernel's key
// tiles; the key-block kernel rescales its query tiles box by box instead).
template <int KD, int BATCH>
__device__ __forceinline__ void rescale_tile(uint8_t* tile, const float* c, int r) {
  constexpr int CPR = KD / 8;       // 16-byte chunks per row
  constexpr int RSTEP = 128 / CPR;  // rows between a thread's chunks
  const int L = r % CPR, box = L >> 3, c16 = L & 7;
  const int row0 = r / CPR;
  __nv_bfloat162 chi[4], clo[4];
  {
    const float4 c0 = *reinterpret_cast<const float4*>(c + box * 64 + c16 * 8);
    const float4 c1 = *reinterpret_cast<const float4*>(c + box * 64 + c16 * 8 + 4);
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      chi[i] = __floats2bfloat162_rn(cv[2 * i], cv[2 * i + 1]);
      const float2 h = __bfloat1622float2(chi[i]);
      clo[i] = __floats2bfloat162_rn(cv[2 * i] - h.x, cv[2 * i + 1] - h.y);
    }
  }
  uint8_t* base = tile + box * 16384;
#pragma unroll(BATCH == 1 ? 4 : CPR / BATCH)
  for (int m0 = 0; m0 < CPR; m0 += BATCH) {
    uint4* ptr[BATCH];
    uint4 v[BATCH];
#pragma unroll
    for (int m = 0; m < BATCH; ++m) {
      const int row = row0 + (m0 + m) * RSTEP;
      // 128-byte swizzle: the 16-byte chunk index is XORed with the row's index mod 8
      ptr[m] = reinterpret_cast<uint4*>(base + row * 128 + ((c16 ^ (row & 7)) << 4));
      v[m] = *ptr[m];
    }
#pragma unroll
    for (int m = 0; m < BATCH; ++m) *ptr[m] = scale8(v[m], chi, clo);
  }
}

// Multiplies one 64-channel box (128 rows x 8 chunks of 16 bytes, 128-byte
// swizzle) of a tile by c[box*64 ..] in place; 128 threads, r = thread index:
// chunk r & 7 of rows (r >> 3) + 16 m, all 8 loaded before any is stored.
__device__ __forceinline__ void rescale_box(uint8_t* tile, const float* c, int r, int box) {
  const int c16 = r & 7, row0 = r >> 3;
  __nv_bfloat162 chi[4], clo[4];
  {
    const float4 c0 = *reinterpret_cast<const float4*>(c + box * 64 + c16 * 8);
    const float4 c1 = *reinterpret_cast<const float4*>(c + box * 64 + c16 * 8 + 4);
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      chi[i] = __floats2bfloat162_rn(cv[2 * i], cv[2 * i + 1]);
      const float2 h = __bfloat1622float2(chi[i]);
      clo[i] = __floats2bfloat162_rn(cv[2 * i] - h.x, cv[2 * i + 1] - h.y);
    }
  }
  uint8_t* base = tile + box * 16384;
  uint4* ptr[8];
  uint4 v[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int row = row0 + 16 * m;
    ptr[m] = reinterpret_cast<uint4*>(base + row * 128 + ((c16 ^ (row & 7)) << 4));
    v[m] = *ptr[m];
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) *ptr[m] = scale8(v[m], chi, clo);
}

__device__ __forceinline__ int first_key(const int* lo_tab, int window, int t) {
  if (lo_tab != nullptr) return lo_tab[t];
  if (window > 0) return t - window + 1 > 0 ? t - window + 1 : 0;
  return 0;
}

// ============================================================== key-block kernel
template <int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(512, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDO, const BtcParams p) {
  using C = BtcCfg<KD, VD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem + C::A_K;
  uint8_t* sV = smem + C::A_V;
  uint8_t* sQ = smem + C::A_Q;
  uint8_t* sDO = smem + C::A_DO;
  float* sAQ = reinterpret_cast<float*>(smem + C::A_AQ);
  float* sRowt = reinterpret_cast<float*>(smem + C::A_ROWT);
  float* sDel = reinterpret_cast<float*>(smem + C::A_DEL);
  int* sLo = reinterpret_cast<int*>(smem + C::A_LO);
  float* sAK = reinterpret_cast<float*>(smem + C::A_AK);
  float* sColt = reinterpret_cast<float*>(smem + C::A_COLT);
  float* sC = reinterpret_cast<float*>(smem + C::A_C);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::A_BAR);
  uint64_t* kvfull = bars;
  uint64_t* qfull = bars + 1;
  uint64_t* qready = bars + 3;
  uint64_t* qempty = bars + 5;
  uint64_t* sfull = bars + 7;
  uint64_t* dpfull = bars + 8;
  uint64_t* pready = bars + 9;
  uint64_t* dsready = bars + 10;
  uint64_t* final_bar = bars + 11;
  uint64_t* mdrain = bars + 12;
  uint64_t* qready_hi = bars + 13;  // [2]: channels 64.. of the stage rescaled
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::A_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::A_MISC + 4);
  int* s_qhi = reinterpret_cast<int*>(smem + C::A_MISC + 8);
  float* sRs = reinterpret_cast<float*>(smem + C::A_RS);  // [128] second half's row sums

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  const int BHQ = p.B * p.HQ;
  const int kt = static_cast<int>(blockIdx.x / BHQ);  // early key tiles (most query tiles) first
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
  const int j0 = kt * 128;
  const size_t TP = static_cast<size_t>(p.NB) * 128;
  const int* lo_tab = p.rowlo;

  if (tid == 0) {
    mbar_init(kvfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qready[s], 128);
      mbar_init(&qready_hi[s], 128);
      mbar_init(&qempty[s], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(dpfull, 1);
    mbar_init(pready, 256);
    mbar_init(dsready, 256);
    mbar_init(final_bar, 1);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    // last query row admitting a key of this tile (first admitted key grows with the row)
    const int jmax = min(j0 + 127, p.T - 1);
    int lo = jmax, hi = p.T - 1;
    if (lo_tab != nullptr || p.window > 0) {
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_key(lo_tab, p.window, mid) <= jmax) lo = mid; else hi = mid - 1;
      }
    } else {
      lo = p.T - 1;
    }
    *s_qhi = lo;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int it_lo = kt;                 // query tiles kt .. s_qhi / 128
  const int nt = *s_qhi / 128 - it_lo + 1;
  const WaitCtl wc{abort_flag, p.err, p.wait_ns};
  constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 384;

  if (wg == 0) {
    reg_dealloc<88>();
    if (warp == 0 && lane == 0) {
      // ----------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(kvfull, C::KB + C::VB + KD * 4 + (HAS_GS ? C::VEC : 0));
      for (int bx = 0; bx < C::KBOX; ++bx)
        tma_load_3d(sK + bx * 16384, &tmK, kvfull, bx * 64, j0, bh);
      for (int bx = 0; bx < C::VBOX; ++bx)
        tma_load_4d(sV + bx * 16384, &tmV, kvfull, bx * 64, kvh, j0, b);
      bulk_load(sAK, p.AK + (static_cast<size_t>(bh) * p.NB + kt) * KD, KD * 4, kvfull);
      if (HAS_GS) bulk_load(sColt, p.colt + bh * TP + j0, C::VEC, kvfull);
      int nq = 0;
      for (int it = 0; it < nt; ++it) {
        const int s = it & 1;
        if (it >= 2 && !mbar_wait(&qempty[s], ((it >> 1) - 1) & 1, wc)) break;
        const int q0 = (it_lo + it) * 128;
        if (!(p.fault == 4 && it == 0)) {
          const uint32_t bytes = C::KB + C::VB + KD * 4 + 2 * C::VEC + (lo_tab ? C::VEC : 0);
          mbar_arrive_expect_tx(&qfull[s], bytes);
          for (int bx = 0; bx < C::KBOX; ++bx)
            tma_load_3d(sQ + s * C::KB + bx * 16384, &tmQ, &qfull[s], bx * 64, q0, bh);
          for (int bx = 0; bx < C::VBOX; ++bx)
            tma_load_4d(sDO + s * C::VB + bx * 16384, &tmDO, &qfull[s], bx * 64, hq, q0, b);
          bulk_load(sAQ + s * KD, p.AQ + (static_cast<size_t>(bh) * p.NB + 2 * (q0 / 256)) * KD,
                    KD * 4, &qfull[s]);
          bulk_load(sRowt + s * 128, p.rowt + bh * TP + q0, C::VEC, &qfull[s]);
          bulk_load(sDel + s * 128, p.delta + bh * TP + q0, C::VEC, &qfull[s]);
          if (lo_tab) bulk_load(sLo + s * 128, lo_tab + q0, C::VEC, &qfull[s]);
        }
        nq = it + 1;
      }
      mbar_drain(kvfull, 0, p.wait_ns);
      for (int it = nq > 2 ? nq - 2 : 0; it < nq; ++it)
        if (!(p.fault == 4 && it == 0)) mbar_drain(&qfull[it & 1], (it >> 1) & 1, p.wait_ns);
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(kvfull, 0, wc);
      tc_fence_after();
      const uint64_t dKa = sw128_desc(smem_u32(sK), 16, 1024);       // A of S^T (K-major)
      const uint64_t dVa = sw128_desc(smem_u32(sV), 16, 1024);       // A of dP^T (K-major)
      const uint64_t dQk = sw128_desc(smem_u32(sQ), 16, 1024);       // B of S^T (K-major)
      const uint64_t dOk = sw128_desc(smem_u32(sDO), 16, 1024);      // B of dP^T (K-major)
      const uint64_t dQm = sw128_desc(smem_u32(sQ), 16384, 1024);    // B of dK (MN-major)
      const uint64_t dOm = sw128_desc(smem_u32(sDO), 16384, 1024);   // B of dV (MN-major)
      const uint32_t tS = tmem_base + COL_S, tDP = tmem_base + COL_DP;
      const uint32_t tDV = tmem_base + COL_DV, tDK = tmem_base + COL_DK;
      // S^T over the first 64 channels once they are rescaled (the caller waits
      // on qready), the rest after qready_hi
      auto issue_s = [&](int it) -> bool {
        const uint64_t qo = static_cast<uint64_t>((it & 1) * (C::KB >> 4));
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          if (kk == 4) {
            if (!mbar_wait(&qready_hi[it & 1], (it >> 1) & 1, wc)) return false;
            tc_fence_after();
          }
          umma_ss(tS, dKa + kmaj_step(kk), dQk + qo + kmaj_step(kk), C::IDESC_SS, kk > 0 ? 1u : 0u);
        }
        umma_commit(sfull);
        return true;
      };
      auto issue_dp = [&](int it) {
        const uint64_t oo = static_cast<uint64_t>((it & 1) * (C::VB >> 4));
#pragma unroll
        for (int kk = 0; kk < VD / 16; ++kk)
          umma_ss(tDP, dVa + kmaj_step(kk), dOk + oo + kmaj_step(kk), C::IDESC_SS, kk > 0 ? 1u : 0u);
        umma_commit(dpfull);
      };
      if (ok) ok = mbar_wait(&qready[0], 0, wc);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
        if (ok) issue_dp(0);
      }
      for (int it = 0; ok && it < nt; ++it) {
        const int s = it & 1;
        if (!mbar_wait(pready, it & 1, wc)) { ok = false; break; }
        tc_fence_after();
        {  // dV += P^T dO  (P^T: 128 keys x 128 queries, bf16 in TMEM)
          const uint64_t oo = static_cast<uint64_t>(s * (C::VB >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tDV, tS + packed_col(kk), dOm + oo + mnmaj_step(kk), C::IDESC_NV,
                    (it > 0 || kk > 0) ? 1u : 0u);
        }
        if (it + 1 < nt) {
          if (!mbar_wait(&qready[(it + 1) & 1], ((it + 1) >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          if (!issue_s(it + 1)) { ok = false; break; }
        }
        if (!mbar_wait(dsready, it & 1, wc)) { ok = false; break; }
        tc_fence_after();
        {  // dK += dS^T (Qh c)
          const uint64_t qo = static_cast<uint64_t>(s * (C::KB >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tDK, tDP + packed_col(kk), dQm + qo + mnmaj_step(kk), C::IDESC_NK,
                    (it > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&qempty[s]);
        }
        if (it + 1 < nt) issue_dp(it + 1);
      }
      if (ok) umma_commit(final_bar);
      umma_commit(mdrain);
      mbar_drain(mdrain, 0, p.wait_ns);
    }
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------- elementwise + epilogue
    // warpgroup wg handles the query columns [64 (wg - 1), 64 wg) of every tile
    reg_alloc<168>();
    const int hc = wg - 1, cb = 64 * hc;
    const int r = tid - 128 * wg;            // key row within the tile = TMEM lane
    const int j = j0 + r;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = mbar_wait(kvfull, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    const float colj = (HAS_GS && ok) ? sColt[r] : 0.f;
    const float2 ncol2 = make_float2(-colj, -colj), sc2 = make_float2(p.sc, p.sc);
    const float2 neg1 = make_float2(-1.f, -1.f);
    float2 rs2 = make_float2(0.f, 0.f);
    for (int it = 0; ok && it < nt; ++it) {
      const int s = it & 1;
      const int q0 = (it_lo + it) * 128;
      const float* rowt = sRowt + s * 128;
      const float* del = sDel + s * 128;
      const int* lo = sLo + s * 128;
      // the per-query vectors of this stage (landed with the tile's copies)
      bool got = mbar_wait(&qfull[s], (it >> 1) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      // the whole tile admitted: every query after every key, inside the window/document
      const int qlast = q0 + 127;
      const bool full = q0 >= j0 + 127 && qlast < p.T &&
                        (lo_tab ? lo[127] : first_key(nullptr, p.window, qlast)) <= j0;
      got = mbar_wait(sfull, it & 1, wc);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      // pass 1: P^T = exp2(S^T sc + rowt - colt) over the admitted (query, key)
      // pairs; fp32 pairs stay in registers for pass 2, bf16 pairs go to TMEM
      float2 pf[32];
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_S + cb + c, x);
        tmem_wait_ld();
        fence_regs32(x);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 r4 = *reinterpret_cast<const float4*>(rowt + cb + c + e);
          const float2 y0 = ffma2(make_float2(x[e], x[e + 1]), sc2,
                                  fadd2(make_float2(r4.x, r4.y), ncol2));  // rowt - colt
          const float2 y1 = ffma2(make_float2(x[e + 2], x[e + 3]), sc2,
                                  fadd2(make_float2(r4.z, r4.w), ncol2));
          pf[(c + e) >> 1] = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
          pf[(c + e + 2) >> 1] = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
        }
        if (!full) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = q0 + cb + c + e;
            int2 l2 = make_int2(0, 0);
            if (lo_tab) l2 = *reinterpret_cast<const int2*>(lo + cb + c + e);
            const int f0 = lo_tab ? l2.x : first_key(nullptr, p.window, q);
            const int f1 = lo_tab ? l2.y : first_key(nullptr, p.window, q + 1);
            if (!(q < p.T && q >= j && f0 <= j)) pf[(c + e) >> 1].x = 0.f;
            if (!(q + 1 < p.T && q + 1 >= j && f1 <= j)) pf[(c + e) >> 1].y = 0.f;
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(pf[(c >> 1) + e].x, pf[(c >> 1) + e].y);
        tmem_st16(lane_base + COL_S + packed_dst(cb + c, cb), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pready);
      // pass 2: dS^T = P^T (dP^T - delta), over dP^T's columns; row sums for dGs
      got = mbar_wait(dpfull, it & 1, wc);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_DP + cb + c, x);
        tmem_wait_ld();
        fence_regs32(x);
        // query columns past T: delta there is not defined (padding); taken as 0
        // there, where p = 0 and dP = 0 (dO's rows past T are zero-filled)
        const int nvalid = full ? 32 : p.T - (q0 + cb + c);
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 d4 = *reinterpret_cast<const float4*>(del + cb + c + e);
          if (e + 3 >= nvalid) {
            if (e >= nvalid) d4.x = 0.f;
            if (e + 1 >= nvalid) d4.y = 0.f;
            if (e + 2 >= nvalid) d4.z = 0.f;
            d4.w = 0.f;
          }
          const float2 d0 = fmul2(pf[(c + e) >> 1],
                                  ffma2(make_float2(d4.x, d4.y), neg1, make_float2(x[e], x[e + 1])));
          const float2 d1 = fmul2(pf[(c + e + 2) >> 1],
                                  ffma2(make_float2(d4.z, d4.w), neg1, make_float2(x[e + 2], x[e + 3])));
          rs2 = fadd2(rs2, fadd2(d0, d1));
          dk[e >> 1] = pack_bf16(d0.x, d0.y);
          dk[(e >> 1) + 1] = pack_bf16(d1.x, d1.y);
        }
        tmem_st16(lane_base + COL_DP + packed_dst(cb + c, cb), dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(dsready);
    }
    // the two halves' row sums: the second half's go through shared memory
    float rsum = rs2.x + rs2.y;
    if (hc == 1) sRs[r] = rsum;
    named_bar_sync(2, 256);
    if (hc == 0) rsum += sRs[r];
    if (ok) {
      const bool got = mbar_wait(final_bar, 0, wc);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after();
      const bool row_ok = j < p.T;
      float* krow = p.acc + (static_cast<size_t>(bh) * p.T + (row_ok ? j : 0)) * KD;
      float* vrow = p.dvh + (static_cast<size_t>(bh) * p.T + (row_ok ? j : 0)) * VD;
#pragma unroll 1
      for (int c = hc * (KD / 2); c < (hc + 1) * (KD / 2); c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_DK + c, x);
        tmem_wait_ld();
        fence_regs32(x);
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(krow + c + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
#pragma unroll 1
      for (int c = hc * (VD / 2); c < (hc + 1) * (VD / 2); c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_DV + c, x);
        tmem_wait_ld();
        fence_regs32(x);
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(vrow + c + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
      if (row_ok && hc == 0) p.rs[static_cast<size_t>(bh) * p.T + j] = rsum;
    }
  } else {
    // ------------------------------------------------------------- query-tile rescale (by c)
    reg_dealloc<88>();
    const int r = tid - 384;
    bool ok = mbar_wait(kvfull, 0, wc);
    ok = !bar_any(1, 128, !ok);
    for (int it = 0; ok && it < nt; ++it) {
      const int s = it & 1;
      const bool got = mbar_wait(&qfull[s], (it >> 1) & 1, wc);
      float* cb = sC + s * KD;
      if (got && r < KD) cb[r] = ex2_approx((sAQ[s * KD + r] - sAK[r]) * kLog2e);
      if (bar_any(1, 128, !got || *abort_flag != 0)) break;
      rescale_box(sQ + s * C::KB, cb, r, 0);
      fence_proxy_async_smem();
      mbar_arrive(&qready[s]);
      if (KD > 64) rescale_box(sQ + s * C::KB, cb, r, 1);
      fence_proxy_async_smem();
      mbar_arrive(&qready_hi[s]);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ============================================================== query-block kernel
template <int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(512, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmDO, const BtcParams p) {
  using C = BtcCfg<KD, VD>;
  constexpr int KS = C::KS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::B_Q;
  uint8_t* sDO = smem + C::B_DO;
  uint8_t* sK = smem + C::B_K;
  uint8_t* sV = smem + C::B_V;
  float* sAQ = reinterpret_cast<float*>(smem + C::B_AQ);
  float* sRowt = reinterpret_cast<float*>(smem + C::B_ROWT);
  float* sDel = reinterpret_cast<float*>(smem + C::B_DEL);
  float* sAK = reinterpret_cast<float*>(smem + C::B_AK);
  float* sColt = reinterpret_cast<float*>(smem + C::B_COLT);
  float* sC = reinterpret_cast<float*>(smem + C::B_C);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::B_BAR);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;
  uint64_t* kready = kfull + KS;
  uint64_t* kempty = kready + KS;
  uint64_t* vfull = kempty + KS;
  uint64_t* vempty = vfull + 1;
  uint64_t* sfull = vempty + 1;  // [2]
  uint64_t* dpfull = sfull + 2;
  uint64_t* dsready = dpfull + 1;
  uint64_t* final_bar = dsready + 1;
  uint64_t* mdrain = final_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::B_MISC);
  int* abort_flag = reinterpret_cast<int*>(smem + C::B_MISC + 4);
  int* s_lo = reinterpret_cast<int*>(smem + C::B_MISC + 8);
  float* sRs = reinterpret_cast<float*>(smem + C::B_RS);  // [128] second half's row sums

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  const int BHQ = p.B * p.HQ;
  const int nqt = (p.T + 127) / 128;
  const int qt = nqt - 1 - static_cast<int>(blockIdx.x / BHQ);  // long rows first
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
  const int q0 = qt * 128;
  const size_t TP = static_cast<size_t>(p.NB) * 128;
  const int* lo_tab = p.rowlo;

  if (tid == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kready[s], 128);
      mbar_init(&kempty[s], 1);
    }
    mbar_init(vfull, 1);
    mbar_init(vempty, 1);
    mbar_init(&sfull[0], 1);
    mbar_init(&sfull[1], 1);
    mbar_init(dpfull, 1);
    mbar_init(dsready, 256);
    mbar_init(final_bar, 1);
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    *s_lo = first_key(lo_tab, p.window, q0);  // smallest first key of the tile's rows
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kt_hi = qt, kt_lo = *s_lo / 128;
  const int nt = kt_hi - kt_lo + 1;  // visit jt = 0..nt-1 is key tile kt_hi - jt
  const WaitCtl wc{abort_flag, p.err, p.wait_ns};
  constexpr uint32_t COL_S = 0, COL_DP = 256, COL_DQ = 384;

  if (wg == 0) {
    reg_dealloc<88>();
    if (warp == 0 && lane == 0) {
      // ----------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(qfull, C::KB + C::VB + KD * 4 + 2 * C::VEC);
      for (int bx = 0; bx < C::KBOX; ++bx) tma_load_3d(sQ + bx * 16384, &tmQ, qfull, bx * 64, q0, bh);
      for (int bx = 0; bx < C::VBOX; ++bx)
        tma_load_4d(sDO + bx * 16384, &tmDO, qfull, bx * 64, hq, q0, b);
      bulk_load(sAQ, p.AQ + (static_cast<size_t>(bh) * p.NB + 2 * (q0 / 256)) * KD, KD * 4, qfull);
      bulk_load(sRowt, p.rowt + bh * TP + q0, C::VEC, qfull);
      bulk_load(sDel, p.delta + bh * TP + q0, C::VEC, qfull);
      int nk = 0, nv = 0;
      for (int jt = 0; jt < nt; ++jt) {
        const int kt = kt_hi - jt, ks = jt % KS;
        if (jt >= KS && !mbar_wait(&kempty[ks], ((jt / KS) - 1) & 1, wc)) break;
        if (!(p.fault == 5 && jt == 0)) {
          mbar_arrive_expect_tx(&kfull[ks], C::KB + KD * 4 + (HAS_GS ? C::VEC : 0));
          for (int bx = 0; bx < C::KBOX; ++bx)
            tma_load_3d(sK + ks * C::KB + bx * 16384, &tmK, &kfull[ks], bx * 64, kt * 128, bh);
          bulk_load(sAK + ks * KD, p.AK + (static_cast<size_t>(bh) * p.NB + kt) * KD, KD * 4,
                    &kfull[ks]);
          if (HAS_GS) bulk_load(sColt + ks * 128, p.colt + bh * TP + kt * 128, C::VEC, &kfull[ks]);
        }
        nk = jt + 1;
        if (jt >= 1 && !mbar_wait(vempty, (jt - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(vfull, C::VB);
        for (int bx = 0; bx < C::VBOX; ++bx)
          tma_load_4d(sV + bx * 16384, &tmV, vfull, bx * 64, kvh, kt * 128, b);
        nv = jt + 1;
      }
      mbar_drain(qfull, 0, p.wait_ns);
      for (int jt = nk > KS ? nk - KS : 0; jt < nk; ++jt)
        if (!(p.fault == 5 && jt == 0)) mbar_drain(&kfull[jt % KS], (jt / KS) & 1, p.wait_ns);
      if (nv > 0) mbar_drain(vfull, (nv - 1) & 1, p.wait_ns);
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      bool ok = mbar_wait(qfull, 0, wc);
      tc_fence_after();
      const uint64_t dQa = sw128_desc(smem_u32(sQ), 16, 1024);      // A of S (K-major)
      const uint64_t dOa = sw128_desc(smem_u32(sDO), 16, 1024);     // A of dP (K-major)
      const uint64_t dKk = sw128_desc(smem_u32(sK), 16, 1024);      // B of S (K-major)
      const uint64_t dVk = sw128_desc(smem_u32(sV), 16, 1024);      // B of dP (K-major)
      const uint64_t dKm = sw128_desc(smem_u32(sK), 16384, 1024);   // B of dQ (MN-major)
      const uint32_t tDP = tmem_base + COL_DP, tDQ = tmem_base + COL_DQ;
      auto issue_s = [&](int jt) -> bool {
        const int ks = jt % KS;
        if (!mbar_wait(&kready[ks], (jt / KS) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t tS = tmem_base + COL_S + 128 * (jt & 1);
        const uint64_t ko = static_cast<uint64_t>(ks * (C::KB >> 4));
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk)
          umma_ss(tS, dQa + kmaj_step(kk), dKk + ko + kmaj_step(kk), C::IDESC_SS, kk > 0 ? 1u : 0u);
        umma_commit(&sfull[jt & 1]);
        return true;
      };
      auto issue_dp = [&](int jt) -> bool {
        if (!mbar_wait(vfull, jt & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < VD / 16; ++kk)
          umma_ss(tDP, dOa + kmaj_step(kk), dVk + kmaj_step(kk), C::IDESC_SS, kk > 0 ? 1u : 0u);
        umma_commit(dpfull);
        umma_commit(vempty);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok) ok = issue_dp(0);
      if (ok && nt > 1) ok = issue_s(1);
      for (int jt = 0; ok && jt < nt; ++jt) {
        if (!mbar_wait(dsready, jt & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const int ks = jt % KS;
        const uint64_t ko = static_cast<uint64_t>(ks * (C::KB >> 4));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ += dS (Kh c): dS 128 queries x 128 keys in TMEM
          umma_ts(tDQ, tDP + packed_col(kk), dKm + ko + mnmaj_step(kk), C::IDESC_NK,
                  (jt > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&kempty[ks]);
        if (jt + 1 < nt && !issue_dp(jt + 1)) { ok = false; break; }
        if (jt + 2 < nt && !issue_s(jt + 2)) { ok = false; break; }
      }
      if (ok) umma_commit(final_bar);
      umma_commit(mdrain);
      mbar_drain(mdrain, 0, p.wait_ns);
    }
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------- elementwise + epilogue
    // warpgroup wg handles the key columns [64 (wg - 1), 64 wg) of every tile
    reg_alloc<176>();
    const int hc = wg - 1, cb = 64 * hc;
    const int r = tid - 128 * wg;  // query row within the tile = TMEM lane
    const int t = q0 + r;
    const bool row_ok = t < p.T;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int lo_t = row_ok ? first_key(lo_tab, p.window, t) : 0x7fffffff;
    const int lo_last = first_key(lo_tab, p.window, min(q0 + 127, p.T - 1));
    bool ok = mbar_wait(qfull, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    const float rowt = ok ? sRowt[r] : 0.f, del = ok ? sDel[r] : 0.f;
    const float2 rowt2 = make_float2(rowt, rowt), del2 = make_float2(del, del);
    const float2 sc2 = make_float2(p.sc, p.sc), neg1 = make_float2(-1.f, -1.f);
    float2 rs2 = make_float2(0.f, 0.f);
    for (int jt = 0; ok && jt < nt; ++jt) {
      const int ks = jt % KS, k0 = (kt_hi - jt) * 128;
      const float* colt = sColt + ks * 128;
      const bool full = q0 + 127 < p.T && k0 + 127 <= q0 && lo_last <= k0;
      bool got = mbar_wait(&kfull[ks], (jt / KS) & 1, wc);  // key-side vectors of this stage
      got = got && mbar_wait(&sfull[jt & 1], (jt >> 1) & 1, wc);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const uint32_t colS = COL_S + 128 * (jt & 1);
      // pass 1: p = exp2(S sc + rowt - colt), kept in registers as fp32 pairs
      // (fma(colt, -1, rowt) is the rounded difference rowt - colt)
      float2 pf[32];
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float x[32];
        tmem_ld32(lane_base + colS + cb + c, x);
        tmem_wait_ld();
        fence_regs32(x);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float2 off0 = rowt2, off1 = rowt2;
          if (HAS_GS) {
            const float4 c4 = *reinterpret_cast<const float4*>(colt + cb + c + e);
            off0 = ffma2(make_float2(c4.x, c4.y), neg1, rowt2);
            off1 = ffma2(make_float2(c4.z, c4.w), neg1, rowt2);
          }
          const float2 y0 = ffma2(make_float2(x[e], x[e + 1]), sc2, off0);
          const float2 y1 = ffma2(make_float2(x[e + 2], x[e + 3]), sc2, off1);
          pf[(c + e) >> 1] = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
          pf[(c + e + 2) >> 1] = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
        }
        if (!full) {  // keys after the row, before its first key, or past T: p = 0
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int key = k0 + cb + c + e;
            if (key > t || key < lo_t) pf[(c + e) >> 1].x = 0.f;
            if (key + 1 > t || key + 1 < lo_t) pf[(c + e) >> 1].y = 0.f;
          }
        }
      }
      // pass 2: dS = p (dP - delta) over dP's columns; row sums for dGs.  A row
      // past T has p = 0 and feeds only its own dQ row and row sum, never stored.
      got = mbar_wait(dpfull, jt & 1, wc);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_DP + cb + c, x);
        tmem_wait_ld();
        fence_regs32(x);
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 dd = ffma2(del2, neg1, make_float2(x[e], x[e + 1]));  // dP - delta
          const float2 d = fmul2(pf[(c + e) >> 1], dd);
          rs2 = fadd2(rs2, d);
          dk[e >> 1] = pack_bf16(d.x, d.y);
        }
        tmem_st16(lane_base + COL_DP + packed_dst(cb + c, cb), dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(dsready);
    }
    // the two halves' row sums: the second half's go through shared memory
    float rsum = rs2.x + rs2.y;
    if (hc == 1) sRs[r] = rsum;
    named_bar_sync(2, 256);
    if (hc == 0) rsum += sRs[r];
    if (ok) {
      const bool got = mbar_wait(final_bar, 0, wc);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after();
      float* qrow = p.acc + (static_cast<size_t>(bh) * p.T + (row_ok ? t : 0)) * KD;
#pragma unroll 1
      for (int c = hc * (KD / 2); c < (hc + 1) * (KD / 2); c += 32) {
        float x[32];
        tmem_ld32(lane_base + COL_DQ + c, x);
        tmem_wait_ld();
        fence_regs32(x);
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(qrow + c + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
      if (row_ok && hc == 0) p.rs[static_cast<size_t>(bh) * p.T + t] = rsum;
    }
  } else {
    // ------------------------------------------------------------- key-tile rescale (by c)
    reg_dealloc<72>();  // 88 + 2 x 176 + 72 = 512 registers per thread-quad
    const int r = tid - 384;
    bool ok = mbar_wait(qfull, 0, wc);
    ok = !bar_any(1, 128, !ok);
    for (int jt = 0; ok && jt < nt; ++jt) {
      const int ks = jt % KS;
      const bool got = mbar_wait(&kfull[ks], (jt / KS) & 1, wc);
      float* cb = sC + (jt & 1) * KD;
      if (got && r < KD) cb[r] = ex2_approx((sAQ[r] - sAK[ks * KD + r]) * kLog2e);
      if (bar_any(1, 128, !got || *abort_flag != 0)) break;
      rescale_tile<KD, 4>(sK + ks * C::KB, cb, r);
      fence_proxy_async_smem();
      mbar_arrive(&kready[ks]);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ launch
void record_event(void* ev, cudaStream_t st) {
  if (ev != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

template <int KD, int VD, bool HAS_GS>
cudaError_t btc_impl(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw, cudaStream_t st) {
  using C = BtcCfg<KD, VD>;
  const FwdArgs& f = a.f;
  const int BHQ = f.B * f.HQ;
  CUtensorMap tmQ, tmK, tmV, tmDO;
  {  // anchored q / k: [B*HQ][T][K], 64-channel x 128-row boxes, 128-byte swizzle
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(f.T),
                                static_cast<cuuint64_t>(BHQ)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(KD) * 2,
                                   static_cast<cuuint64_t>(f.T) * KD * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!encode_tiled(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, fw.qh, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tiled(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, fw.kh, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {  // v [B, T, H, V] and dO [B, T, HQ, V]: 64-channel x 128-row boxes
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint64_t vd[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(f.H),
                              static_cast<cuuint64_t>(f.T), static_cast<cuuint64_t>(f.B)};
    const cuuint64_t vs[3] = {static_cast<cuuint64_t>(VD) * 2,
                              static_cast<cuuint64_t>(f.H) * VD * 2,
                              static_cast<cuuint64_t>(f.T) * f.H * VD * 2};
    const cuuint64_t od[4] = {static_cast<cuuint64_t>(VD), static_cast<cuuint64_t>(f.HQ),
                              static_cast<cuuint64_t>(f.T), static_cast<cuuint64_t>(f.B)};
    const cuuint64_t os[3] = {static_cast<cuuint64_t>(VD) * 2,
                              static_cast<cuuint64_t>(f.HQ) * VD * 2,
                              static_cast<cuuint64_t>(f.T) * f.HQ * VD * 2};
    if (!encode_tiled(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, f.v, vd, vs, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tiled(&tmDO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.dout, od, os, box,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  BtcParams p;
  p.AQ = fw.AQ;
  p.AK = fw.AK;
  p.rowt = bw.rowt;
  p.colt = bw.colt;
  p.delta = bw.delta;
  p.rowlo = f.cu_seqlens ? fw.rowlo : nullptr;
  p.window = f.window;
  p.B = f.B;
  p.T = f.T;
  p.HQ = f.HQ;
  p.H = f.H;
  p.NB = f.NB;
  p.sc = f.scale * kLog2e;
  p.err = f.err;
  p.wait_ns = f.wait_ns;
  p.fault = f.fault;
  const unsigned grid = static_cast<unsigned>(f.NB) * BHQ;

  auto kA = bwd_dkdv_tc_kernel<KD, VD, HAS_GS>;
  cudaError_t e = cudaFuncSetAttribute(kA, cudaFuncAttributeMaxDynamicSharedMemorySize, C::A_SMEM);
  if (e != cudaSuccess) return e;
  auto kB = bwd_dq_tc_kernel<KD, VD, HAS_GS>;
  e = cudaFuncSetAttribute(kB, cudaFuncAttributeMaxDynamicSharedMemorySize, C::B_SMEM);
  if (e != cudaSuccess) return e;

  record_event(a.ev[0], st);
  p.acc = bw.accK;
  p.dvh = bw.dvh;
  p.rs = bw.rsA;
  kA<<<grid, 512, C::A_SMEM, st>>>(tmQ, tmK, tmV, tmDO, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  record_event(a.ev[1], st);
  p.acc = bw.accQ;
  p.dvh = nullptr;
  p.rs = bw.rsB;
  kB<<<grid, 512, C::B_SMEM, st>>>(tmQ, tmK, tmV, tmDO, p);
  e = cudaGetLastError();
  record_event(a.ev[2], st);
  return e;
}

}  // namespace

cudaError_t launch_bwd_tc(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw,
                          cudaStream_t st) {
  const bool gs = a.f.g_scalar != nullptr;
#define WALL_BTC(KD_, VD_)                                                       \
  if (a.f.K == KD_ && a.f.V == VD_)                                              \
    return gs ? btc_impl<KD_, VD_, true>(a, fw, bw, st)                          \
              : btc_impl<KD_, VD_, false>(a, fw, bw, st);
  WALL_BTC(64, 64)
  WALL_BTC(64, 128)
  WALL_BTC(128, 64)
  WALL_BTC(128, 128)
#undef WALL_BTC
  return cudaErrorInvalidValue;
}

}  // namespace wall
