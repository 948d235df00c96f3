// Exact in-block pairs of Wall attention for strongly decaying channels.
//
// The anchored tiles of the prefill (wall_prep.cu) split the per-channel
// factor exp(G[i] - G[j]) of the Wall Attention README's intro formula over
// 256-row block anchors.  Across blocks every factor is at most 1 for g <= 0;
// inside a block the query factor and the key-tile factor span up to 256 rows
// each in opposite directions, and once that span leaves the fp32/bf16
// exponent range (tens of nats: a channel with log-decay of a few units per
// token) the product is 0 * inf.  The prepass flags such "wide" blocks; the
// attention kernels skip their own key tiles, and this kernel evaluates the
// block's pairs (i, j both in the block, j <= i) with factors that never
// exceed 1, then merges them with the attention kernel's result for keys
// before the block through (o, lse).
//
// Factorisation inside a wide block, by 16-row sub-blocks I (queries) and
// J (keys), all exponents sums of the g values between the two rows:
//   J < I:  exp(G_i - G_j) = exp(G_i - A_I) * exp(A_I - A'_J) * exp(A'_J - G_j)
//           with A_I = G just before I and A'_J = G at J's last row: a prefix
//           inside I, the sum of the sub-blocks strictly between, and a suffix
//           inside J;
//   J = I:  exp(sum_{t=j+1..i} g_t) per pair, accumulated row by row.
// For g <= 0 each factor is at most 1, and each exponent is a sum of terms of
// one sign, so it is accurate to fp32 rounding at any decay strength.
//
// One CTA (128 threads) takes one wide block at a time; thread (a, cg) owns
// query row a of the current sub-block and channel group cg (K/8 channels of
// the dot products, V/8 of the output).  Row statistics are reduced over the 8
// lanes of a row with warp shuffles.  The softmax over the row's in-block keys
// is exact (two passes over at most 256 logits in shared memory).
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

constexpr int kSub = 16;          // rows per sub-block
constexpr int kBlk = 2 * kBlockRows;  // rows per query block (the prepass's anchor block)


template <typename T>
__device__ __forceinline__ void load_n(const T* p, float* f, int n) {
  for (int c = 0; c < n; c += 8) load8(p + c, f + c);
}

__device__ __forceinline__ float exp_nat(float x) { return ex2_approx(x * kLog2e); }

template <typename T>
__device__ __forceinline__ void store_n(T* p, const float* f, int n) {
  for (int c = 0; c < n; c += 8) store8(p + c, f + c);
}

// Sum over the 8 lanes (channel groups) of one query row.
__device__ __forceinline__ float row_sum8(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}
__device__ __forceinline__ float row_max8(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  return x;
}

template <typename Tin, int KD, int VD>
__global__ void __launch_bounds__(128) wall_fwd_diag_kernel(const DiagParams p) {
  constexpr int CPT = KD / 8;  // dot-product channels per thread: n = c * 8 + cg
  constexpr int VPT = VD / 8;  // output channels per thread: cg * VPT + c
  constexpr int XS = kBlk + 8; // logit row stride (rows of a warp land 8 banks apart)
  __shared__ float sG[kSub][KD];       // g of the query sub-block I
  __shared__ float sKI[kSub][KD];      // k of I (the diagonal sub-block's keys)
  __shared__ float sKJ[kSub][KD];      // key sub-block J: k * exp(suffix of g inside J)
  __shared__ float sC[KD];             // exp(g summed over the sub-blocks strictly between)
  __shared__ float sGsI[kSub];         // g_scalar of I
  __shared__ float sGsJ[kSub];         // g_scalar suffix inside J
  __shared__ float sGb;                // g_scalar summed strictly between J and I
  __shared__ float sX[kSub][XS];       // logits, then probabilities, of the block's keys
  __shared__ int list[128];
  __shared__ int nlist;

  const Tin* q = static_cast<const Tin*>(p.q);
  const Tin* k = static_cast<const Tin*>(p.k);
  const Tin* g = static_cast<const Tin*>(p.g);
  const Tin* gs = static_cast<const Tin*>(p.gs);
  const Tin* v = static_cast<const Tin*>(p.v);
  Tin* o = static_cast<Tin*>(p.o);
  const int tid = threadIdx.x, a = tid >> 3, cg = tid & 7;
  const int nblocks = p.B * p.HQ * p.NQB;
  const int G = gridDim.x;
  const size_t qrow = static_cast<size_t>(p.HQ) * KD, krow = static_cast<size_t>(p.H) * KD;
  const size_t vrow = static_cast<size_t>(p.H) * VD, orow = static_cast<size_t>(p.HQ) * VD;

  for (int base = 0; base < nblocks; base += 128 * G) {
    // Gather this CTA's wide blocks of the round (flags read in parallel).
    if (tid == 0) nlist = 0;
    __syncthreads();
    const int idx = base + tid * G + static_cast<int>(blockIdx.x);
    if (idx < nblocks && p.wide[idx] != 0) list[atomicAdd(&nlist, 1)] = idx;
    __syncthreads();
    const int cnt = nlist;
    for (int e = 0; e < cnt; ++e) {
      const int blk = list[e];
      const int bh = blk / p.NQB, qb = blk % p.NQB;
      const int b = bh / p.HQ, hq = bh % p.HQ, kvh = hq / (p.HQ / p.H);
      const int r0 = qb * kBlk, rend = min(r0 + kBlk, p.Tb);
      const Tin* qB = q + static_cast<size_t>(b) * p.Tb * qrow + static_cast<size_t>(hq) * KD;
      const Tin* kB = k + static_cast<size_t>(b) * p.Tb * krow + static_cast<size_t>(kvh) * KD;
      const Tin* gB = g + static_cast<size_t>(b) * p.Tb * qrow + static_cast<size_t>(hq) * KD;
      const Tin* gsB = gs ? gs + static_cast<size_t>(b) * p.Tb * p.HQ + hq : nullptr;
      const Tin* vB = v + (static_cast<size_t>(b) * p.vT + p.voff) * vrow +
                      static_cast<size_t>(kvh) * VD;
      Tin* oB = o + static_cast<size_t>(b) * p.Tb * orow + static_cast<size_t>(hq) * VD;
      float* lB = p.lse + static_cast<size_t>(b) * p.Tb * p.HQ + hq;
      const int nsub = (rend - r0 + kSub - 1) / kSub;

      for (int I = 0; I < nsub; ++I) {
        const int i0 = r0 + I * kSub;
        for (int x = tid; x < kSub * KD; x += 128) {
          const int r = x / KD, n = x % KD, t = i0 + r;
          const bool ok = t < rend;
          sG[r][n] = ok ? load1(gB + static_cast<size_t>(t) * qrow + n) : 0.f;
          sKI[r][n] = ok ? load1(kB + static_cast<size_t>(t) * krow + n) : 0.f;
        }
        if (tid < kSub) {
          const int t = i0 + tid;
          sGsI[tid] = (gsB != nullptr && t < rend) ? load1(gsB + static_cast<size_t>(t) * p.HQ) : 0.f;
        }
        __syncthreads();

        const int i = i0 + a;
        const bool row_ok = i < rend;
        int lo;  // first admitted key, local row index
        {
          int lo_abs = 0;
          if (p.rowlo != nullptr) lo_abs = p.rowlo[p.pos0 + (row_ok ? i : r0)];
          else if (p.window > 0) lo_abs = max(0, p.pos0 + i - p.window + 1);
          lo = lo_abs - p.pos0;
        }
        // Query row: raw (diagonal sub-block) and times exp(G_i - A_I) (earlier sub-blocks).
        float qraw[CPT], qI[CPT];
        {
          float gl[CPT];
#pragma unroll
          for (int c = 0; c < CPT; ++c) gl[c] = 0.f;
          for (int t = 0; t <= a; ++t) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) gl[c] += sG[t][c * 8 + cg];
          }
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            qraw[c] = row_ok ? load1(qB + static_cast<size_t>(i) * qrow + c * 8 + cg) : 0.f;
            qI[c] = qraw[c] * exp_nat(gl[c]);
          }
        }
        float gsl = 0.f;  // g_scalar prefix inside I up to row a
        for (int t = 0; t <= a; ++t) gsl += sGsI[t];

        // Diagonal sub-block: keys bb <= a of I, decay summed from row a down to bb + 1.
        {
          float d[CPT];
#pragma unroll
          for (int c = 0; c < CPT; ++c) d[c] = 0.f;
          float dgs = 0.f;
#pragma unroll 1
          for (int bb = kSub - 1; bb >= 0; --bb) {
            if (bb < a) {
#pragma unroll
              for (int c = 0; c < CPT; ++c) d[c] += sG[bb + 1][c * 8 + cg];
              dgs += sGsI[bb + 1];
            }
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c)
              part = fmaf(qraw[c] * sKI[bb][c * 8 + cg], exp_nat(d[c]), part);
            part = row_sum8(part);
            if (cg == 0 && bb <= a) {
              float xv = p.scale * part + dgs;
              if (i0 + bb < lo) xv = -INFINITY;
              sX[a][I * kSub + bb] = xv;
            }
          }
        }

        // Earlier key sub-blocks J = I-1 .. 0.  Thread n < K keeps channel n's
        // g summed over the sub-blocks strictly between J and I (cs).
        float cs = 0.f, gsb = 0.f;
        for (int J = I - 1; J >= 0; --J) {
          const int j0 = r0 + J * kSub;
          if (tid < KD) {
            const int n = tid;
            float kv[kSub], gv[kSub];
#pragma unroll
            for (int jj = 0; jj < kSub; ++jj) {
              const size_t t = static_cast<size_t>(j0 + jj);
              kv[jj] = load1(kB + t * krow + n);
              gv[jj] = load1(gB + t * qrow + n);
            }
            float suf = 0.f;  // g summed over J's rows after jj
#pragma unroll
            for (int jj = kSub - 1; jj >= 0; --jj) {
              sKJ[jj][n] = kv[jj] * exp_nat(suf);
              suf += gv[jj];
            }
            sC[n] = exp_nat(cs);
            cs += suf;
          }
          if (tid == 0 && gsB != nullptr) {
            float suf = 0.f;
            for (int jj = kSub - 1; jj >= 0; --jj) {
              sGsJ[jj] = suf;
              suf += load1(gsB + static_cast<size_t>(j0 + jj) * p.HQ);
            }
            sGb = gsb;
            gsb += suf;
          }
          __syncthreads();
          float qc[CPT];
#pragma unroll
          for (int c = 0; c < CPT; ++c) qc[c] = qI[c] * sC[c * 8 + cg];
          const float gq = gsB != nullptr ? gsl + sGb : 0.f;
#pragma unroll 4
          for (int jj = 0; jj < kSub; ++jj) {
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) part = fmaf(qc[c], sKJ[jj][c * 8 + cg], part);
            part = row_sum8(part);
            if (cg == 0) {
              float xv = p.scale * part + (gsB != nullptr ? gq + sGsJ[jj] : 0.f);
              if (j0 + jj < lo) xv = -INFINITY;
              sX[a][J * kSub + jj] = xv;
            }
          }
          __syncthreads();
        }

        // Exact softmax over the row's in-block keys 0 .. I*16 + a (local to the block).
        const int nk = I * kSub + a + 1;
        const int jmax = min((I + 1) * kSub, rend - r0);
        __syncwarp();
        float m = -INFINITY;
        for (int j = cg; j < nk; j += 8) m = fmaxf(m, sX[a][j]);
        m = row_max8(m);
        float l = 0.f;
        for (int j = cg; j < jmax; j += 8) {
          const float pj = (j < nk && m != -INFINITY) ? exp_nat(sX[a][j] - m) : 0.f;
          sX[a][j] = pj;
          l += pj;
        }
        l = row_sum8(l);
        __syncwarp();
        float acc[VPT];
#pragma unroll
        for (int c = 0; c < VPT; ++c) acc[c] = 0.f;
        for (int j = 0; j < jmax; ++j) {
          const float pj = sX[a][j];
          float vv[VPT];
          load_n(vB + static_cast<size_t>(r0 + j) * vrow + cg * VPT, vv, VPT);
#pragma unroll
          for (int c = 0; c < VPT; ++c) acc[c] = fmaf(pj, vv[c], acc[c]);
        }

        // Merge with the attention kernel's result for the keys before the block.
        if (row_ok) {
          float* lp = lB + static_cast<size_t>(i) * p.HQ;
          Tin* op = oB + static_cast<size_t>(i) * orow + cg * VPT;
          float lse_f;
          if (lo < r0) {
            const float L1 = *lp;
            const float L2 = m + logf(l);
            const float M = fmaxf(L1, L2);
            lse_f = M + logf(expf(L1 - M) + expf(L2 - M));
            const float wo = expf(L1 - lse_f), wd = expf(m - lse_f);
            float o1[VPT];
            load_n(op, o1, VPT);
#pragma unroll
            for (int c = 0; c < VPT; ++c) acc[c] = fmaf(o1[c], wo, acc[c] * wd);
          } else {
            float Z = l;
            if (p.sink != nullptr) Z += expf(p.sink[hq] - m);
            lse_f = m + logf(Z);
            const float inv = 1.f / Z;
#pragma unroll
            for (int c = 0; c < VPT; ++c) acc[c] *= inv;
          }
          __syncwarp(0xffu << (tid & 24));  // the row's 8 lanes have read lse before it changes
          store_n(op, acc, VPT);
          if (cg == 0) *lp = lse_f;
        }
        __syncthreads();
      }
    }
    __syncthreads();
  }
}

template <typename Tin, int KD, int VD>
cudaError_t diag_impl(const DiagParams& p, cudaStream_t st) {
  const int nblocks = p.B * p.HQ * p.NQB;
  if (nblocks <= 0) return cudaSuccess;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = nblocks < 4 * nsm ? nblocks : 4 * nsm;
  wall_fwd_diag_kernel<Tin, KD, VD><<<grid, 128, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t diag_dispatch(const DiagParams& p, int K, int V, cudaStream_t st) {
  if (K == 64 && V == 64) return diag_impl<Tin, 64, 64>(p, st);
  if (K == 64 && V == 128) return diag_impl<Tin, 64, 128>(p, st);
  if (K == 128 && V == 64) return diag_impl<Tin, 128, 64>(p, st);
  if (K == 128 && V == 128) return diag_impl<Tin, 128, 128>(p, st);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_diag(const DiagParams& p, bool bf16, int K, int V, cudaStream_t st) {
  return bf16 ? diag_dispatch<__nv_bfloat16>(p, K, V, st) : diag_dispatch<float>(p, K, V, st);
}

cudaError_t launch_fwd_diag(const FwdArgs& a, const FwdWork& w, bool bf16, cudaStream_t st) {
  DiagParams p;
  p.q = a.q; p.k = a.k; p.g = a.g; p.gs = a.g_scalar; p.v = a.v;
  p.sink = a.sink;
  p.rowlo = a.cu_seqlens ? w.rowlo : nullptr;
  p.wide = w.wide;
  p.window = a.window;
  p.B = a.B; p.Tb = a.T; p.HQ = a.HQ; p.H = a.H; p.NQB = (a.NB + 1) / 2;
  p.vT = a.T; p.voff = 0; p.pos0 = 0;
  p.scale = a.scale;
  p.o = a.o;
  p.lse = a.lse != nullptr ? a.lse : w.lse_ws;
  return launch_diag(p, bf16, a.K, a.V, st);
}

}  // namespace wall
