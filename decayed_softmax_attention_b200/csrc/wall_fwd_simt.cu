// Wall attention prefill forward for fp32 inputs: exact fp32 arithmetic on the
// CUDA cores (TF32 tensor-core products would round the operands to 10-bit
// mantissas, far outside the fp32 tolerance).
//
// Same factorisation as the bf16 tensor-core kernel (Wall Attention README
// intro formula): S = Qh * diag(exp(AQ - AK)) * Kh^T on the anchored operands
// of the prepass, then a streaming softmax over 64-key tiles.  One CTA per
// 64-row query block of one (batch, query head); 256 threads as a 16 x 16 grid,
// each owning a 4 x 4 patch of S and a 4 x (V/16) patch of O.  A row's
// statistics are reduced across the 16 threads that share it with warp
// shuffles.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

constexpr int SB = 64;  // rows per query block / keys per tile

template <int KD, int VD, bool HAS_GS>
__global__ void __launch_bounds__(256) wall_fwd_simt_kernel(
    const float* __restrict__ qh, const float* __restrict__ kh, const float* __restrict__ v,
    const float* __restrict__ AQ, const float* __restrict__ AK, const float* __restrict__ ssl,
    const float* __restrict__ ssa, const float* __restrict__ sink, const int* __restrict__ rowlo,
    const int* __restrict__ wide, int window, int B, int T, int HQ, int H, int NB, float sc, float* __restrict__ o,
    float* __restrict__ lse) {
  constexpr int VC = VD / 16;  // O columns per thread
  extern __shared__ float sm[];
  float* sQT = sm;                  // [KD][SB]   anchored q, transposed
  float* sKT = sQT + KD * SB;       // [KD][SB]   rescaled key tile, transposed
  float* sV = sKT + KD * SB;        // [SB][VD]
  float* sPT = sV + SB * VD;        // [SB][SB]   probabilities, transposed
  float* sCv = sPT + SB * SB;       // [KD]       per-pair channel factors
  float* sCol = sCv + KD;           // [SB]       key-side gate terms
  __shared__ int s_lo;

  const int nqb = (T + SB - 1) / SB;
  const int BHQ = B * HQ;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x / BHQ);
  const int bh = static_cast<int>(blockIdx.x % BHQ);
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  const int q0 = qb * SB;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int ablk = 2 * (q0 / (2 * kBlockRows));  // query anchor (256-row blocks)
  const int rblk = q0 / kBlockRows;                // 128-row block of these rows

  if (tid == 0) s_lo = 0x7fffffff;
  // anchored q block, transposed
  for (int e = tid; e < SB * KD; e += 256) {
    const int r = e / KD, n = e % KD;
    const int t = q0 + r;
    sQT[n * SB + r] = (t < T) ? qh[(static_cast<size_t>(bh) * T + t) * KD + n] : 0.f;
  }
  __syncthreads();
  int lo[4], hi[4];
  float rowA[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = q0 + ty * 4 + a;
    const bool ok = i < T;
    lo[a] = 0;
    if (ok) {
      if (rowlo != nullptr) lo[a] = rowlo[i];
      else if (window > 0) lo[a] = max(0, i - window + 1);
      if (tx == 0) atomicMin(&s_lo, lo[a]);
    }
    hi[a] = ok ? i : -1;
    rowA[a] = 0.f;
    if (HAS_GS) rowA[a] = ssa[(static_cast<size_t>(bh) * NB + rblk) * 4] -
                          ssl[static_cast<size_t>(bh) * NB * kBlockRows + min(i, NB * kBlockRows - 1)];
  }
  __syncthreads();
  // A wide 256-row block (strong decay inside it) leaves its own keys to the
  // diagonal kernel.
  const int a0 = q0 / (2 * kBlockRows);
  const bool is_wide = wide[static_cast<size_t>(bh) * ((NB + 1) / 2) + a0] != 0;
  const int kt_hi = is_wide ? a0 * (2 * kBlockRows / SB) - 1 : min(q0 + SB - 1, T - 1) / SB;
  const int kt_lo = s_lo == 0x7fffffff ? kt_hi : s_lo / SB;

  float m[4], l[4], acc[4][VC];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    m[a] = -INFINITY;
    l[a] = 0.f;
#pragma unroll
    for (int c = 0; c < VC; ++c) acc[a][c] = 0.f;
  }

  for (int kt = kt_hi; kt >= kt_lo; --kt) {
    const int j0 = kt * SB;
    const int kblk = j0 / kBlockRows;
    if (tid < KD)
      sCv[tid] = exp2f((AQ[(static_cast<size_t>(bh) * NB + ablk) * KD + tid] -
                        AK[(static_cast<size_t>(bh) * NB + kblk) * KD + tid]) * kLog2e);
    if (HAS_GS && tid < SB)
      sCol[tid] = ssa[(static_cast<size_t>(bh) * NB + kblk) * 4] -
                  ssl[static_cast<size_t>(bh) * NB * kBlockRows + j0 + tid];
    __syncthreads();
    for (int e = tid; e < SB * KD; e += 256) {
      const int r = e / KD, n = e % KD;
      const int t = j0 + r;
      sKT[n * SB + r] = (t < T) ? kh[(static_cast<size_t>(bh) * T + t) * KD + n] * sCv[n] : 0.f;
    }
    for (int e = tid; e < SB * VD; e += 256) {
      const int r = e / VD, c = e % VD;
      const int t = j0 + r;
      sV[r * VD + c] = (t < T) ? v[((static_cast<size_t>(b) * T + t) * H + kvh) * VD + c] : 0.f;
    }
    __syncthreads();

    float s[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[a][c] = 0.f;
#pragma unroll 8
    for (int n = 0; n < KD; ++n) {
      const float4 qv = *reinterpret_cast<const float4*>(sQT + n * SB + ty * 4);
      const float4 kv = *reinterpret_cast<const float4*>(sKT + n * SB + tx * 4);
      const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
      const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) s[a][c] = fmaf(qa[a], ka[c], s[a][c]);
    }
    // logits in log2 units, masked
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + tx * 4 + c;
        float x = s[a][c] * sc;
        if (HAS_GS) x += rowA[a] - sCol[tx * 4 + c];
        if (j < lo[a] || j > hi[a]) x = -INFINITY;
        s[a][c] = x;
        mt = fmaxf(mt, x);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float mn = fmaxf(m[a], mt);
      const float base = (mn == -INFINITY) ? 0.f : mn;
      const float alpha = exp2f(m[a] - base);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float pv = exp2f(s[a][c] - base);
        s[a][c] = pv;
        rs += pv;
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
      l[a] = l[a] * alpha + rs;
      m[a] = mn;
#pragma unroll
      for (int c = 0; c < VC; ++c) acc[a][c] *= alpha;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<float4*>(sPT + (tx * 4 + c) * SB + ty * 4) =
          make_float4(s[0][c], s[1][c], s[2][c], s[3][c]);
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < SB; ++j) {
      const float4 pv = *reinterpret_cast<const float4*>(sPT + j * SB + ty * 4);
      const float pa[4] = {pv.x, pv.y, pv.z, pv.w};
      float vv[VC];
#pragma unroll
      for (int c = 0; c < VC; c += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(sV + j * VD + tx * VC + c);
        vv[c] = t4.x; vv[c + 1] = t4.y; vv[c + 2] = t4.z; vv[c + 3] = t4.w;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < VC; ++c) acc[a][c] = fmaf(pa[a], vv[c], acc[a][c]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = q0 + ty * 4 + a;
    if (i >= T) continue;
    float Z = l[a];
    if (sink != nullptr) Z += exp2f(sink[hq] * kLog2e - m[a]);
    const float inv = 1.f / Z;
    float* orow = o + ((static_cast<size_t>(b) * T + i) * HQ + hq) * VD + tx * VC;
#pragma unroll
    for (int c = 0; c < VC; c += 4)
      *reinterpret_cast<float4*>(orow + c) =
          make_float4(acc[a][c] * inv, acc[a][c + 1] * inv, acc[a][c + 2] * inv, acc[a][c + 3] * inv);
    if (lse != nullptr && tx == 0)
      lse[(static_cast<size_t>(b) * T + i) * HQ + hq] = (m[a] + log2f(Z)) * kLn2;
  }
}

template <int KD, int VD, bool HAS_GS>
cudaError_t simt_impl(const FwdArgs& a, const FwdWork& w, cudaStream_t st) {
  auto kern = wall_fwd_simt_kernel<KD, VD, HAS_GS>;
  const int smem = (2 * KD * SB + SB * VD + SB * SB + KD + SB) * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nqb = (a.T + SB - 1) / SB;
  const unsigned grid = static_cast<unsigned>(nqb) * a.B * a.HQ;
  kern<<<grid, 256, smem, st>>>(static_cast<const float*>(w.qh), static_cast<const float*>(w.kh),
                                static_cast<const float*>(a.v), w.AQ, w.AK, w.ssl, w.ssa, a.sink,
                                a.cu_seqlens ? w.rowlo : nullptr, w.wide, a.window, a.B, a.T,
                                a.HQ, a.H, a.NB, a.scale * kLog2e, static_cast<float*>(a.o),
                                a.lse != nullptr ? a.lse : w.lse_ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, const FwdWork& w, cudaStream_t st) {
  const bool gs = a.g_scalar != nullptr;
#define WALL_SIMT(KD_, VD_)                                                              \
  if (a.K == KD_ && a.V == VD_)                                                          \
    return gs ? simt_impl<KD_, VD_, true>(a, w, st) : simt_impl<KD_, VD_, false>(a, w, st);
  WALL_SIMT(64, 64)
  WALL_SIMT(64, 128)
  WALL_SIMT(128, 64)
  WALL_SIMT(128, 128)
#undef WALL_SIMT
  return cudaErrorInvalidValue;
}

}  // namespace wall
