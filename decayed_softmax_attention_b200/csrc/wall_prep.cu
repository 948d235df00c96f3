// Prefill prepass of Wall attention (Wall Attention README, "Usage" shapes;
// the decay of the intro formula folded into anchored operands).
//
// The score's per-channel factor exp(G[i,n] - G[j,n]) splits exactly as
//   exp(G[i] - AQ) * exp(AQ - AK) * exp(AK - G[j])
// for any anchors AQ, AK.  With AQ = G just before the query's 256-row block
// and AK = G at the last row of the key's 128-row block, the first and last
// factors are folded once into qh and kh here, and the middle one (one vector
// per (query block, key block) pair) is applied to each key tile inside the
// main kernel.  For a key block that ends before the query block starts, and
// a decay g <= 0, all three factors are at most 1: they can only underflow,
// and only where the true product is smaller still, so those tiles are exact
// for any decay strength.  Inside the query block (its own two key tiles) the
// query factor shrinks while exp(AQ - AK) grows, each spanning up to 256 rows
// of accumulated decay; a block where that span exceeds kPrefillSpanNats in
// any channel is flagged "wide", the attention kernels skip its own key tiles
// and the diagonal kernel (wall_fwd_diag.cu) evaluates those pairs exactly.
// Prefix sums run over the whole row; with packed documents only differences
// inside a document are ever used, so they equal the per-document sums of the
// definition.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// bar.red.or over `nthreads` threads of named barrier `id`: a barrier whose
// result (any thread's predicate) every participant sees.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
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

// One CTA per (256-row query block, batch*query head); each half of the CTA
// (128 threads) owns one 128-row key block.  Thread layout per half: CG
// channel groups of 8 channels x RG row groups of RPG consecutive rows.
// Key operands are anchored per 128-row block (AK = G at the block's last
// row); query operands per 256-row block (AQ = G just before the block), so
// the two 128-row query tiles of one prefill CTA share one anchor.
//
// Pass 1 sums g over each thread's rows; after one barrier every thread knows
// the prefix before its rows and carries, per channel, the query exponent
// qa = (G_t - AQ) log2(e) (advanced by one fma per row) and the constant
// (AK - AQ) log2(e), so the key exponent (AK - G_t) log2(e) is one subtraction.
// Pass 2 reads g again (from L2: the CTA read it a few microseconds earlier)
// with q and k and writes qh and kh.  The arithmetic runs on packed fp32 pairs;
// KT (the decode cache is emitted too) is a template flag so the plain prefill
// carries no cache work.  Four CTAs per SM (64 registers a thread) for the
// plain bf16 prefill.

template <typename Tin, int KD, bool KT>
__global__ void __launch_bounds__(256, KT ? (KD == 64 ? 2 : 3) : (sizeof(Tin) == 4 ? 3 : 4))
    prep_local_kernel(
    const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ g,
    const Tin* __restrict__ gs, const int32_t* __restrict__ cu, int nseq, int window, int T,
    int HQ, int H, int NB, Tin* __restrict__ qh, Tin* __restrict__ kh, float* __restrict__ bsum,
    float* __restrict__ ssl, float* __restrict__ ssb, __nv_bfloat16* __restrict__ kx,
    float inv_scale, int* __restrict__ rowlo, Tin* __restrict__ kt, float* __restrict__ rc,
    int cap, int C, int* __restrict__ wide, int* __restrict__ err, int wide_err) {
  constexpr int CG = KD / 8;
  constexpr int RG = 128 / CG;
  constexpr int RPG = 128 / RG;
  __shared__ float tot[2][RG][KD];
  __shared__ float gfirst[KT ? 2 : 1][KT ? RG : 1][KD];  // g at each row group's first row
  __shared__ float wsum[2][4];
  __shared__ int s_span;  // largest |exponent| of the block's anchored factors (float bits)
  if (threadIdx.x == 0) s_span = 0;

  const int half = threadIdx.x >> 7, tid = threadIdx.x & 127;
  const int blk = blockIdx.x * 2 + half;  // 128-row block of this half
  const int bh = blockIdx.y;
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  const int cg = tid % CG, rg = tid / CG;
  const int t0 = blk * kBlockRows + rg * RPG;
  const int nrows = T - t0 >= RPG ? RPG : (T - t0 > 0 ? T - t0 : 0);
  const size_t qrow = static_cast<size_t>(HQ) * KD;  // elements between time steps (q, g)
  const size_t krow = static_cast<size_t>(H) * KD;   // (k)
  const size_t rbase = static_cast<size_t>(b) * T + (t0 < T ? t0 : 0);
  const Tin* gb = g + rbase * qrow + static_cast<size_t>(hq) * KD + cg * 8;
  const Tin* qb = q + rbase * qrow + static_cast<size_t>(hq) * KD + cg * 8;
  const Tin* kb = k + rbase * krow + static_cast<size_t>(kvh) * KD + cg * 8;

  // ---- pass 1: g summed over this thread's rows
  float2 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.f, 0.f);
  constexpr int U1 = 4;
  static_assert(RPG % U1 == 0, "row batch must divide the rows per thread");
  auto add_rows = [&](const Raw8<Tin>* gv, int n) {
#pragma unroll
    for (int u = 0; u < U1; ++u) {
      if (u < n) {
        float f[8];
        gv[u].get(f);
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[c] = __fadd2_rn(acc[c], make_float2(f[2 * c], f[2 * c + 1]));
      }
    }
  };
  if (nrows == RPG) {
#pragma unroll 1
    for (int m0 = 0; m0 < RPG; m0 += U1) {
      Raw8<Tin> gv[U1];
#pragma unroll
      for (int u = 0; u < U1; ++u) gv[u].load(gb + static_cast<size_t>(m0 + u) * qrow);
      if (KT && m0 == 0) {
        float f[8];
        gv[0].get(f);
#pragma unroll
        for (int c = 0; c < 8; ++c) gfirst[KT ? half : 0][KT ? rg : 0][cg * 8 + c] = f[c];
      }
      add_rows(gv, U1);
    }
  } else {
#pragma unroll 1
    for (int m0 = 0; m0 < nrows; m0 += U1) {
      Raw8<Tin> gv[U1];
#pragma unroll
      for (int u = 0; u < U1; ++u)
        if (m0 + u < nrows) gv[u].load(gb + static_cast<size_t>(m0 + u) * qrow);
      if (KT && m0 == 0) {
        float f[8];
        gv[0].get(f);
#pragma unroll
        for (int c = 0; c < 8; ++c) gfirst[KT ? half : 0][KT ? rg : 0][cg * 8 + c] = f[c];
      }
      add_rows(gv, nrows - m0);
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    tot[half][rg][cg * 8 + 2 * c] = acc[c].x;
    tot[half][rg][cg * 8 + 2 * c + 1] = acc[c].y;
  }
  __syncthreads();

  // Decode cache: this thread's rows lie in one chunk (C is a multiple of RPG
  // and divides 128); its anchor R = G at the chunk's first row, block-local.
  const int rgc = ((rg * RPG) / C) * C / RPG;  // row group that opens the chunk
  // qa: query exponent (G_t - AQ) log2 e, advanced per row; ka: (AK - AQ) log2 e;
  // za: (R_chunk - AQ) log2 e (cache rows only)
  float qa[8], ka[8], za[KT ? 8 : 1];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float pre = 0.f, all = 0.f, first = 0.f, cpre = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      const float x = tot[half][r][cg * 8 + c];
      all += x;
      if (r < rg) pre += x;
      if (r < rgc) cpre += x;
      if (half == 1) first += tot[0][r][cg * 8 + c];
    }
    // first = g summed over the first half of the query block (0 in half 0)
    qa[c] = (first + pre) * kLog2e;
    ka[c] = (first + all) * kLog2e;
    if (KT) {
      const float cst = cpre + gfirst[KT ? half : 0][KT ? rgc : 0][cg * 8 + c];
      za[KT ? c : 0] = (first + cst) * kLog2e;
      if (rg == rgc && t0 < T) {  // block-local anchor of the chunk; a later pass adds the
        const int ncap = (cap + C - 1) / C;  // block's offset
        rc[((static_cast<size_t>(b) * ncap + t0 / C) * HQ + hq) * KD + cg * 8 + c] = cst;
      }
    }
    if (rg == 0 && blk < NB) bsum[(static_cast<size_t>(bh) * NB + blk) * KD + cg * 8 + c] = all;
  }

  // ---- pass 2: qh = q 2^qa, kh = k 2^(ka - qa) (and cache rows k 2^(za - qa))
  Tin* qo = qh + (static_cast<size_t>(bh) * T + (t0 < T ? t0 : 0)) * KD + cg * 8;
  Tin* ko = kh + (static_cast<size_t>(bh) * T + (t0 < T ? t0 : 0)) * KD + cg * 8;
  Tin* zo = KT ? kt + ((static_cast<size_t>(b) * cap + (t0 < T ? t0 : 0)) * HQ + hq) * KD + cg * 8
               : nullptr;
  // |G_t - AQ| over this thread's rows and channels (log2 units): the exponent
  // of the query factor, and at each half's last row of the in-block key-tile
  // factor exp(AQ - AK).
  float span = 0.f;
  float kspan = 0.f;  // largest exponent of an emitted cache row (log2 units)
  auto do_row = [&](const Raw8<Tin>& gv, const Raw8<Tin>& rq, const Raw8<Tin>& rk, int m) {
    float f[8], x[8], y[8], z[8];
    gv.get(f);
    rq.get(x);
    rk.get(y);
    // exp(a) as 2^(a log2 e): one MUFU op each (relative error ~2^-22)
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const float2 a = __ffma2_rn(make_float2(f[c], f[c + 1]), make_float2(kLog2e, kLog2e),
                                  make_float2(qa[c], qa[c + 1]));
      qa[c] = a.x;
      qa[c + 1] = a.y;
      span = fmaxf(span, fmaxf(fabsf(a.x), fabsf(a.y)));
      const float2 kk = __fadd2_rn(make_float2(ka[c], ka[c + 1]), make_float2(-a.x, -a.y));
      if (KT) {
        const float2 zz = __fadd2_rn(make_float2(za[KT ? c : 0], za[KT ? c + 1 : 0]),
                                     make_float2(-a.x, -a.y));
        kspan = fmaxf(kspan, fmaxf(zz.x, zz.y));
        const float2 zr = __fmul2_rn(make_float2(y[c], y[c + 1]),
                                     make_float2(ex2_approx(zz.x), ex2_approx(zz.y)));
        z[c] = zr.x;
        z[c + 1] = zr.y;
      }
      const float2 xr = __fmul2_rn(make_float2(x[c], x[c + 1]),
                                   make_float2(ex2_approx(a.x), ex2_approx(a.y)));
      const float2 yr = __fmul2_rn(make_float2(y[c], y[c + 1]),
                                   make_float2(ex2_approx(kk.x), ex2_approx(kk.y)));
      x[c] = xr.x; x[c + 1] = xr.y;
      y[c] = yr.x; y[c + 1] = yr.y;
    }
    store8(qo + static_cast<size_t>(m) * KD, x);
    store8(ko + static_cast<size_t>(m) * KD, y);
    if (KT) store8(zo + static_cast<size_t>(m) * qrow, z);
  };
  constexpr int U2 = (sizeof(Tin) == 2 && !KT) ? 2 : 1;
  if (nrows == RPG) {
#pragma unroll 1
    for (int m0 = 0; m0 < RPG; m0 += U2) {
      Raw8<Tin> gv[U2], rq[U2], rk[U2];
#pragma unroll
      for (int u = 0; u < U2; ++u) {
        gv[u].load(gb + static_cast<size_t>(m0 + u) * qrow);
        rq[u].load(qb + static_cast<size_t>(m0 + u) * qrow);
        rk[u].load(kb + static_cast<size_t>(m0 + u) * krow);
      }
#pragma unroll
      for (int u = 0; u < U2; ++u) do_row(gv[u], rq[u], rk[u], m0 + u);
    }
  } else {
#pragma unroll 1
    for (int m = 0; m < nrows; ++m) {
      Raw8<Tin> gv, rq, rk;
      gv.load(gb + static_cast<size_t>(m) * qrow);
      rq.load(qb + static_cast<size_t>(m) * qrow);
      rk.load(kb + static_cast<size_t>(m) * krow);
      do_row(gv, rq, rk, m);
    }
  }

  if (KT && kspan > kCacheRangeLog2) atomicOr(err, kDevErrRange);
  // Non-negative floats order like their bit patterns; one shared atomic per warp.
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) span = fmaxf(span, __shfl_xor_sync(0xffffffffu, span, off));
  if ((threadIdx.x & 31) == 0 && span > 0.f) atomicMax(&s_span, __float_as_int(span));
  __syncthreads();
  if (threadIdx.x == 0) {
    const int w = __int_as_float(s_span) > kPrefillSpanNats * kLog2e ? 1 : 0;
    wide[static_cast<size_t>(bh) * gridDim.x + blockIdx.x] = w;
    if (w && wide_err) atomicOr(err, kDevErrRange);
  }

  // Scalar gate: negated 128-block-local inclusive prefix (log2 units), one row per thread.
  if (gs != nullptr) {
    const int t = blk * kBlockRows + tid;
    float x = (t < T) ? load1(gs + (static_cast<size_t>(b) * T + t) * HQ + hq) * kLog2e : 0.f;
    const int lane = tid & 31, wid = tid >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) wsum[half][wid] = x;
    __syncthreads();
    for (int w = 0; w < wid; ++w) x += wsum[half][w];
    if (blk < NB) {
      ssl[static_cast<size_t>(bh) * NB * kBlockRows + blk * kBlockRows + tid] = -x;  // negated
      if (tid == kBlockRows - 1) ssb[static_cast<size_t>(bh) * NB + blk] = x;
    }
    // Key-side gate term as two extra bf16 channels of the key operand (the
    // query operand carries ones there), so the QK contraction adds it: the
    // attention kernel scales S by scale * log2(e), so hi + lo = -x / (scale *
    // log2(e)) to ~16 significant bits.
    if (kx != nullptr && t < T) {
      const float val = -x * inv_scale;
      const __nv_bfloat16 hi = __float2bfloat16_rn(val);
      const __nv_bfloat16 lo = __float2bfloat16_rn(val - __bfloat162float(hi));
      uint4 u;
      u.x = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
            (static_cast<uint32_t>(__bfloat16_as_ushort(lo)) << 16);
      u.y = u.z = u.w = 0u;
      uint4* dst = reinterpret_cast<uint4*>(kx + (static_cast<size_t>(bh) * T + t) * 16);
      dst[0] = u;
      dst[1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // First admitted key of each row for packed documents (shared by all heads).
  if (cu != nullptr && bh == 0) {
    const int t = blk * kBlockRows + tid;
    if (t < T) {
      int lo = 0, hi = nseq;  // largest d with cu[d] <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid;
      }
      int s = cu[lo];
      s = s < 0 ? 0 : (s > t ? t : s);
      if (window > 0 && t - window + 1 > s) s = t - window + 1;
      rowlo[t] = s;
    }
  }
}

// TMA-staged prepass for bf16 inputs whose T is a multiple of 256 (no decode-
// cache output): the same arithmetic as prep_local_kernel, fed by bulk tensor
// copies.  One CTA per (256-row block, batch*query head): the block's g tile
// (256 rows x K) is copied into shared memory once and serves both passes; the
// q and k rows stream through a two-stage ring.  Consumer thread (cg, rg) owns 8
// channels of a run of RPG consecutive rows, so a ring stage that brings 2 rows
// of every thread's run (one 5-D copy per 64-channel box: rows, row groups, head,
// batch) gives every thread work.  A producer warp issues the copies; all loads
// are in flight without holding registers.  Two (K = 128) or three (K = 64) CTAs
// per SM.
template <int KD>
struct PrepTmaCfg {
  static constexpr int CG = KD / 8;       // channel groups of 8
  static constexpr int RG = 256 / CG;     // row groups of the 256-row block
  static constexpr int RPG = 256 / RG;    // rows per row group
  static constexpr int NBOX = KD / 64;    // 64-channel boxes
  static constexpr int RPS = 2;           // rows of each row group per ring stage
  static constexpr int NSTG = RPG / RPS;  // stages per block
  static constexpr int NS = 2;            // ring depth
  static constexpr int G_BOX = RG * RPG * 128;  // one box of the g tile
  static constexpr int A_BOX = RG * RPS * 128;  // one box of one array in a stage
  static constexpr int STAGE = 2 * NBOX * A_BOX;  // q then k
  static constexpr int OFF_G = 0;
  static constexpr int OFF_R = NBOX * G_BOX;
  static constexpr int OFF_TOT = OFF_R + NS * STAGE;  // float [RG][KD]
  static constexpr int OFF_BAR = OFF_TOT + RG * KD * 4;
  static constexpr int SMEM = OFF_BAR + (1 + 2 * NS) * 8 + 16;
};

template <int KD>
__global__ void __launch_bounds__(288, 1) prep_tma_kernel(
    const __grid_constant__ CUtensorMap tmGt, const __grid_constant__ CUtensorMap tmQr,
    const __grid_constant__ CUtensorMap tmKr, const __nv_bfloat16* __restrict__ gs,
    const int32_t* __restrict__ cu, int nseq, int window, int T, int HQ, int H, int NB,
    __nv_bfloat16* __restrict__ qh, __nv_bfloat16* __restrict__ kh, float* __restrict__ bsum,
    float* __restrict__ ssl, float* __restrict__ ssb, __nv_bfloat16* __restrict__ kx,
    float inv_scale, int* __restrict__ rowlo, int* __restrict__ wide, int* __restrict__ err,
    int wide_err, uint64_t wait_ns) {
  using PC = PrepTmaCfg<KD>;
  extern __shared__ __align__(128) uint8_t psm[];
  float* tot = reinterpret_cast<float*>(psm + PC::OFF_TOT);
  uint64_t* gfull = reinterpret_cast<uint64_t*>(psm + PC::OFF_BAR);
  uint64_t* full = gfull + 1;
  uint64_t* empty = full + PC::NS;
  int* abort_flag = reinterpret_cast<int*>(empty + PC::NS);
  int* s_span = abort_flag + 1;
  __shared__ float wsum[2][4];

  const int bp = blockIdx.x, bh = blockIdx.y;  // 256-row block, batch*query head
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  if (threadIdx.x == 0) {
    mbar_init(gfull, 1);
    for (int i = 0; i < PC::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 8);  // one arrival per consumer warp
    }
    *abort_flag = 0;
    *s_span = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, err, wait_ns};

  if (threadIdx.x >= 256) {
    // ------------------------------------------------------------- producer
    if (threadIdx.x == 256) {
      tma_prefetch_desc(&tmGt);
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmKr);
      const int grp0 = bp * PC::RG;  // the block's first row group
      mbar_arrive_expect_tx(gfull, PC::NBOX * PC::G_BOX);
      for (int x = 0; x < PC::NBOX; ++x)
        tma_load_5d(psm + PC::OFF_G + x * PC::G_BOX, &tmGt, gfull, x * 64, 0, grp0, hq, b);
      int issued = 0;
      for (int st = 0; st < PC::NSTG; ++st) {
        const int slot = st % PC::NS;
        if (st >= PC::NS && !mbar_wait(&empty[slot], ((st / PC::NS) - 1) & 1, wc)) break;
        uint8_t* dst = psm + PC::OFF_R + slot * PC::STAGE;
        mbar_arrive_expect_tx(&full[slot], PC::STAGE);
        for (int x = 0; x < PC::NBOX; ++x) {
          tma_load_5d(dst + x * PC::A_BOX, &tmQr, &full[slot], x * 64, st * PC::RPS, grp0, hq, b);
          tma_load_5d(dst + (PC::NBOX + x) * PC::A_BOX, &tmKr, &full[slot], x * 64, st * PC::RPS,
                      grp0, kvh, b);
        }
        issued = st + 1;
      }
      // every copy issued lands before the CTA may exit
      mbar_drain(gfull, 0, wait_ns);
      for (int st = issued > PC::NS ? issued - PC::NS : 0; st < issued; ++st)
        mbar_drain(&full[st % PC::NS], (st / PC::NS) & 1, wait_ns);
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int tid = threadIdx.x;
  const int cg = tid % PC::CG, rg = tid / PC::CG;
  const int box = cg >> 3, cw = cg & 7;  // 64-channel box, 16-byte chunk within its row
  const int half = (rg * PC::RPG) >> 7;  // the 128-row key block of this thread's rows
  const int t0 = bp * 256 + rg * PC::RPG;
  const uint8_t* gt = psm + PC::OFF_G + box * PC::G_BOX + (rg * PC::RPG) * 128 + cw * 16;

  // ---- pass 1: g summed over this thread's rows (from the resident g tile)
  bool ok = mbar_wait(gfull, 0, wc);
  float2 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float2(0.f, 0.f);
  if (ok) {
#pragma unroll 4
    for (int m = 0; m < PC::RPG; ++m) {
      float f[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(gt + m * 128), f);
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] = __fadd2_rn(acc[c], make_float2(f[2 * c], f[2 * c + 1]));
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    tot[rg * KD + cg * 8 + 2 * c] = acc[c].x;
    tot[rg * KD + cg * 8 + 2 * c + 1] = acc[c].y;
  }
  ok = !bar_red_or(1, 256, !ok);  // (a consumer-only barrier: the producer does not join)
  // qa: query exponent (G_t - AQ) log2 e, advanced per row; ka: (AK - AQ) log2 e
  constexpr int RGH = PC::RG / 2;  // row groups per 128-row half
  float qa[8], ka[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float pre = 0.f, all = 0.f, first = 0.f;
#pragma unroll
    for (int r = 0; r < RGH; ++r) {
      const float x = tot[(half * RGH + r) * KD + cg * 8 + c];
      all += x;
      if (half * RGH + r < rg) pre += x;
      if (half == 1) first += tot[r * KD + cg * 8 + c];
    }
    qa[c] = (first + pre) * kLog2e;
    ka[c] = (first + all) * kLog2e;
    if (rg == half * RGH && bp * 2 + half < NB)
      bsum[(static_cast<size_t>(bh) * NB + bp * 2 + half) * KD + cg * 8 + c] = all;
  }

  // ---- pass 2: qh = q 2^qa, kh = k 2^(ka - qa), q and k rows from the ring
  __nv_bfloat16* qo = qh + (static_cast<size_t>(bh) * T + t0) * KD + cg * 8;
  __nv_bfloat16* ko = kh + (static_cast<size_t>(bh) * T + t0) * KD + cg * 8;
  float span = 0.f;
  for (int st = 0; ok && st < PC::NSTG; ++st) {
    const int slot = st % PC::NS;
    const bool got = mbar_wait(&full[slot], (st / PC::NS) & 1, wc);
    if (!__all_sync(0xffffffffu, got)) {
      ok = false;
      break;
    }
    const uint8_t* sq = psm + PC::OFF_R + slot * PC::STAGE + box * PC::A_BOX +
                        (rg * PC::RPS) * 128 + cw * 16;
    const uint8_t* sk = sq + PC::NBOX * PC::A_BOX;
#pragma unroll
    for (int r = 0; r < PC::RPS; ++r) {
      const int m = st * PC::RPS + r;
      float f[8], x[8], y[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(gt + m * 128), f);
      load8(reinterpret_cast<const __nv_bfloat16*>(sq + r * 128), x);
      load8(reinterpret_cast<const __nv_bfloat16*>(sk + r * 128), y);
      // exp(a) as 2^(a log2 e): one MUFU op each (relative error ~2^-22)
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        const float2 a = __ffma2_rn(make_float2(f[c], f[c + 1]), make_float2(kLog2e, kLog2e),
                                    make_float2(qa[c], qa[c + 1]));
        qa[c] = a.x;
        qa[c + 1] = a.y;
        span = fmaxf(span, fmaxf(fabsf(a.x), fabsf(a.y)));
        const float2 kk = __fadd2_rn(make_float2(ka[c], ka[c + 1]), make_float2(-a.x, -a.y));
        const float2 xr = __fmul2_rn(make_float2(x[c], x[c + 1]),
                                     make_float2(ex2_approx(a.x), ex2_approx(a.y)));
        const float2 yr = __fmul2_rn(make_float2(y[c], y[c + 1]),
                                     make_float2(ex2_approx(kk.x), ex2_approx(kk.y)));
        x[c] = xr.x; x[c + 1] = xr.y;
        y[c] = yr.x; y[c + 1] = yr.y;
      }
      store8(qo + static_cast<size_t>(m) * KD, x);
      store8(ko + static_cast<size_t>(m) * KD, y);
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[slot]);  // this warp no longer reads the stage
  }

#pragma unroll
  for (int off = 16; off > 0; off >>= 1) span = fmaxf(span, __shfl_xor_sync(0xffffffffu, span, off));
  if ((tid & 31) == 0 && span > 0.f) atomicMax(s_span, __float_as_int(span));
  named_bar_sync(1, 256);
  if (tid == 0) {
    const int w = __int_as_float(*s_span) > kPrefillSpanNats * kLog2e ? 1 : 0;
    wide[static_cast<size_t>(bh) * gridDim.x + bp] = w;
    if (w && wide_err) atomicOr(err, kDevErrRange);
  }

  // Scalar gate: negated 128-block-local inclusive prefix (log2 units), one row per thread.
  const int blk = bp * 2 + (tid >> 7), tr = tid & 127, hf = tid >> 7;
  if (gs != nullptr) {
    const int t = blk * kBlockRows + tr;
    float x = (t < T) ? load1(gs + (static_cast<size_t>(b) * T + t) * HQ + hq) * kLog2e : 0.f;
    const int lane = tr & 31, wid = tr >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) wsum[hf][wid] = x;
    named_bar_sync(1, 256);
    for (int w = 0; w < wid; ++w) x += wsum[hf][w];
    if (blk < NB) {
      ssl[static_cast<size_t>(bh) * NB * kBlockRows + blk * kBlockRows + tr] = -x;  // negated
      if (tr == kBlockRows - 1) ssb[static_cast<size_t>(bh) * NB + blk] = x;
    }
    // key-side gate term as two extra bf16 channels of the key operand (hi + lo =
    // -x / (scale * log2(e)) to ~16 significant bits; the query side carries ones)
    if (kx != nullptr && t < T) {
      const float val = -x * inv_scale;
      const __nv_bfloat16 hi = __float2bfloat16_rn(val);
      const __nv_bfloat16 lo = __float2bfloat16_rn(val - __bfloat162float(hi));
      uint4 u;
      u.x = static_cast<uint32_t>(__bfloat16_as_ushort(hi)) |
            (static_cast<uint32_t>(__bfloat16_as_ushort(lo)) << 16);
      u.y = u.z = u.w = 0u;
      uint4* dst = reinterpret_cast<uint4*>(kx + (static_cast<size_t>(bh) * T + t) * 16);
      dst[0] = u;
      dst[1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // First admitted key of each row for packed documents (shared by all heads).
  if (cu != nullptr && bh == 0) {
    const int t = blk * kBlockRows + tr;
    if (t < T) {
      int lo = 0, hi = nseq;  // largest d with cu[d] <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid;
      }
      int s0 = cu[lo];
      s0 = s0 < 0 ? 0 : (s0 > t ? t : s0);
      if (window > 0 && t - window + 1 > s0) s0 = t - window + 1;
      rowlo[t] = s0;
    }
  }
}

// Exclusive scan of the block sums over the blocks of one (batch, head): one
// warp per channel, lane l owning blocks [l PB, (l + 1) PB); each lane sums its
// blocks, a shuffle scan gives every lane the sum before its first block, and
// the lanes write their blocks' AQ (before) and AK (after).  Warp 8 of the
// first channel group scans the gate's block sums the same way.  Grid (batch *
// heads, KD / 8), 288 threads.
__device__ __forceinline__ float warp_excl_scan(float v, int lane) {
  float x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  return x - v;
}

template <int KD>
__global__ void __launch_bounds__(288) prep_scan_kernel(
    const float* __restrict__ bsum, const float* __restrict__ ssb, int NB, float* __restrict__ AQ,
    float* __restrict__ AK, float* __restrict__ ssa, float* __restrict__ plast) {
  const int bh = blockIdx.x, cgrp = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int PB = (NB + 31) / 32;
  const int i0 = lane * PB, i1 = min(NB, i0 + PB);
  if (warp < 8) {
    const int n = cgrp * 8 + warp;
    const size_t base = static_cast<size_t>(bh) * NB * KD + n;
    float own = 0.f;
    for (int i = i0; i < i1; ++i) own += bsum[base + static_cast<size_t>(i) * KD];
    float acc = warp_excl_scan(own, lane);
    for (int i = i0; i < i1; ++i) {
      const size_t at = base + static_cast<size_t>(i) * KD;
      AQ[at] = acc;
      acc += bsum[at];
      AK[at] = acc;
    }
    if (plast != nullptr) {
      const float all = __shfl_sync(0xffffffffu, acc, 31);  // lane 31 ends at the last block
      if (lane == 0) plast[static_cast<size_t>(bh) * KD + n] = all * kLog2e;
    }
  } else if (cgrp == 0 && ssb != nullptr) {
    const size_t base = static_cast<size_t>(bh) * NB;
    float own = 0.f;
    for (int i = i0; i < i1; ++i) own += ssb[base + i];
    float acc = warp_excl_scan(own, lane);
    for (int i = i0; i < i1; ++i) {
      *reinterpret_cast<float4*>(ssa + (base + i) * 4) = make_float4(acc, 0.f, 0.f, 0.f);
      acc += ssb[base + i];
    }
  }
}

// Decode cache anchors (when the prefill emits the cache): the prepass left
// each chunk's block-local G in its slot; add the block's prefix, in log2 units.
// One CTA per (batch * query head, chunk), one thread per channel.
template <int KD>
__global__ void __launch_bounds__(KD) cache_anchor_kernel(const float* __restrict__ AQ, int NB,
                                                          int HQ, int cap, int C, int nchunk,
                                                          float* __restrict__ rc) {
  const int bh = static_cast<int>(blockIdx.x) / nchunk, c = static_cast<int>(blockIdx.x) % nchunk;
  const int b = bh / HQ, hq = bh % HQ, n = threadIdx.x;
  const int ncap = (cap + C - 1) / C;
  const int blk = c * C / kBlockRows;
  float* slot = rc + ((static_cast<size_t>(b) * ncap + c) * HQ + hq) * KD + n;
  *slot = (*slot + AQ[(static_cast<size_t>(bh) * NB + blk) * KD + n]) * kLog2e;
}

// The TMA-staged prepass: bf16, no cache output, T a multiple of 256.  Returns
// false (nothing launched) when its tensor maps cannot be encoded.
template <int KD>
bool prep_tma(const FwdArgs& a, const FwdWork& w, cudaStream_t st, cudaError_t* e) {
  using PC = PrepTmaCfg<KD>;
  const int BHQ = a.B * a.HQ;
  CUtensorMap tmGt, tmQr, tmKr;
  const cuuint64_t grp = static_cast<cuuint64_t>(a.T) / PC::RPG;
  {
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(PC::RPG), grp,
                                static_cast<cuuint64_t>(a.HQ), static_cast<cuuint64_t>(a.B)};
    const cuuint64_t row = static_cast<cuuint64_t>(a.HQ) * KD * 2;
    const cuuint64_t strides[4] = {row, row * PC::RPG, static_cast<cuuint64_t>(KD) * 2,
                                   row * static_cast<cuuint64_t>(a.T)};
    const cuuint32_t boxg[5] = {64, static_cast<cuuint32_t>(PC::RPG),
                                static_cast<cuuint32_t>(PC::RG), 1, 1};
    const cuuint32_t boxq[5] = {64, static_cast<cuuint32_t>(PC::RPS),
                                static_cast<cuuint32_t>(PC::RG), 1, 1};
    if (!encode_tiled(&tmGt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.g, dims, strides, boxg,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tiled(&tmQr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.q, dims, strides, boxq,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  {
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(PC::RPG), grp,
                                static_cast<cuuint64_t>(a.H), static_cast<cuuint64_t>(a.B)};
    const cuuint64_t row = static_cast<cuuint64_t>(a.H) * KD * 2;
    const cuuint64_t strides[4] = {row, row * PC::RPG, static_cast<cuuint64_t>(KD) * 2,
                                   row * static_cast<cuuint64_t>(a.T)};
    const cuuint32_t boxk[5] = {64, static_cast<cuuint32_t>(PC::RPS),
                                static_cast<cuuint32_t>(PC::RG), 1, 1};
    if (!encode_tiled(&tmKr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.k, dims, strides, boxk,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  auto kern = prep_tma_kernel<KD>;
  *e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::SMEM);
  if (*e != cudaSuccess) return true;
  kern<<<dim3(a.T / 256, BHQ), 288, PC::SMEM, st>>>(
      tmGt, tmQr, tmKr, static_cast<const __nv_bfloat16*>(a.g_scalar), a.cu_seqlens, a.num_seqs,
      a.window, a.T, a.HQ, a.H, a.NB, static_cast<__nv_bfloat16*>(w.qh),
      static_cast<__nv_bfloat16*>(w.kh), w.bsum, w.ssl, w.ssb, static_cast<__nv_bfloat16*>(w.kx),
      1.f / (a.scale * kLog2e), w.rowlo, w.wide, a.err, a.wide_is_error ? 1 : 0, a.wait_ns);
  *e = cudaGetLastError();
  return true;
}

template <typename Tin, int KD>
cudaError_t prep_impl(const FwdArgs& a, const FwdWork& w, cudaStream_t st) {
  const int BHQ = a.B * a.HQ;
  dim3 grid((a.NB + 1) / 2, BHQ);
  bool staged = false;
  cudaError_t e = cudaSuccess;
  if constexpr (sizeof(Tin) == 2) {
    if (a.kt_out == nullptr && a.T % 256 == 0) staged = prep_tma<KD>(a, w, st, &e);
  }
  if (staged) {
    if (e != cudaSuccess) return e;
  } else {
    auto kern = a.kt_out != nullptr ? prep_local_kernel<Tin, KD, true>
                                     : prep_local_kernel<Tin, KD, false>;
    kern<<<grid, 256, 0, st>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.g),
        static_cast<const Tin*>(a.g_scalar), a.cu_seqlens, a.num_seqs, a.window, a.T, a.HQ, a.H,
        a.NB, static_cast<Tin*>(w.qh), static_cast<Tin*>(w.kh), w.bsum, w.ssl, w.ssb,
        sizeof(Tin) == 2 ? static_cast<__nv_bfloat16*>(w.kx) : nullptr, 1.f / (a.scale * kLog2e),
        w.rowlo, static_cast<Tin*>(a.kt_out), a.r_out, a.cache_cap, a.cache_chunk, w.wide, a.err,
        a.wide_is_error ? 1 : 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  prep_scan_kernel<KD><<<dim3(BHQ, KD / 8), 288, 0, st>>>(w.bsum, a.g_scalar ? w.ssb : nullptr, a.NB, w.AQ,
                                                 w.AK, w.ssa, a.kt_out ? a.plast_out : nullptr);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.kt_out == nullptr) return e;
  const int nchunk = (a.T + a.cache_chunk - 1) / a.cache_chunk;  // chunks that start below T
  cache_anchor_kernel<KD><<<static_cast<unsigned>(BHQ) * nchunk, KD, 0, st>>>(
      w.AQ, a.NB, a.HQ, a.cache_cap, a.cache_chunk, nchunk, a.r_out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep(const FwdArgs& a, const FwdWork& w, bool bf16, cudaStream_t st) {
  if (bf16) {
    return a.K == 64 ? prep_impl<__nv_bfloat16, 64>(a, w, st) : prep_impl<__nv_bfloat16, 128>(a, w, st);
  }
  return a.K == 64 ? prep_impl<float, 64>(a, w, st) : prep_impl<float, 128>(a, w, st);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t fwd_workspace_layout(int B, int T, int HQ, int K, bool bf16, FwdWork* w, char* base) {
  const size_t BHQ = static_cast<size_t>(B) * HQ;
  const size_t NB = (static_cast<size_t>(T) + kBlockRows - 1) / kBlockRows;
  const size_t esz = bf16 ? 2 : 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return base ? static_cast<void*>(base + o) : nullptr;
  };
  FwdWork tmp;
  FwdWork* p = w ? w : &tmp;
  p->qh = take(BHQ * T * K * esz);
  p->kh = take(BHQ * T * K * esz);
  p->bsum = static_cast<float*>(take(BHQ * NB * K * 4));
  p->AQ = static_cast<float*>(take(BHQ * NB * K * 4));
  p->AK = static_cast<float*>(take(BHQ * NB * K * 4));
  p->ssl = static_cast<float*>(take(BHQ * NB * kBlockRows * 4));
  p->ssb = static_cast<float*>(take(BHQ * NB * 4));
  p->ssa = static_cast<float*>(take(BHQ * NB * 16));
  p->kx = take(BHQ * static_cast<size_t>(T) * 16 * 2);
  p->rowlo = static_cast<int*>(take(NB * kBlockRows * 4));  // padded: 128-row bulk copies
  p->wide = static_cast<int*>(take(BHQ * ((NB + 1) / 2) * 4));
  p->lse_ws = static_cast<float*>(take(BHQ * static_cast<size_t>(T) * 4));
  return off;
}

}  // namespace wall
