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

template <typename Tin, int KD>
cudaError_t prep_impl(const FwdArgs& a, const FwdWork& w, cudaStream_t st) {
  const int BHQ = a.B * a.HQ;
  dim3 grid((a.NB + 1) / 2, BHQ);
  auto kern = a.kt_out != nullptr ? prep_local_kernel<Tin, KD, true>
                                   : prep_local_kernel<Tin, KD, false>;
  kern<<<grid, 256, 0, st>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.g),
      static_cast<const Tin*>(a.g_scalar), a.cu_seqlens, a.num_seqs, a.window, a.T, a.HQ, a.H,
      a.NB, static_cast<Tin*>(w.qh), static_cast<Tin*>(w.kh), w.bsum, w.ssl, w.ssb,
      sizeof(Tin) == 2 ? static_cast<__nv_bfloat16*>(w.kx) : nullptr, 1.f / (a.scale * kLog2e),
      w.rowlo, static_cast<Tin*>(a.kt_out), a.r_out, a.cache_cap, a.cache_chunk, w.wide, a.err,
      a.wide_is_error ? 1 : 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
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
