// Wall attention decode path (Wall Attention README, "Decode"):
//
//   cache build / append:  P = cumsum(g) / ln 2,  R_c = P[c * C] (chunk start),
//                          k_tilde[j] = k[j] * exp2(R_{j/C} - P[j])
//   single-step decode:    x_j = scale * sum_n q[n] k_tilde[j,n] exp2(p_curr[n] - R_{j/C}[n])
//
// The decode is a GEMV-like pass that streams k_tilde and v from HBM once.
// Grid = (split, KV head, batch); one CTA serves the HQ/H query heads that
// share a KV head, so each v row is read once for the whole group.  Inside a
// warp, lane l covers a contiguous slice of the group's concatenated k_tilde
// row (16-byte vector loads); per-head dot products are reduced with warp
// shuffles.  Each CTA writes (o, max, sum) partials per head; a combine pass
// merges the splits (warp-shuffle reductions) and adds the sink.
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// ----------------------------------------------------------------- vector loads
template <typename T, int N>
__device__ __forceinline__ void load_n(const T* p, float* f);

template <int N>
__device__ __forceinline__ void load_n_bf16(const __nv_bfloat16* p, float* f) {
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 8) load8(p + i, f + i);
  } else if constexpr (N == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  } else {
    static_assert(N == 2, "unsupported vector width");
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = bf16_lo(u); f[1] = bf16_hi(u);
  }
}
template <int N>
__device__ __forceinline__ void load_n_f32(const float* p, float* f) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 u = *reinterpret_cast<const float4*>(p + i);
      f[i] = u.x; f[i + 1] = u.y; f[i + 2] = u.z; f[i + 3] = u.w;
    }
  } else {
    static_assert(N == 2, "unsupported vector width");
    const float2 u = *reinterpret_cast<const float2*>(p);
    f[0] = u.x; f[1] = u.y;
  }
}
template <typename T, int N>
__device__ __forceinline__ void load_n(const T* p, float* f) {
  if constexpr (sizeof(T) == 2) load_n_bf16<N>(reinterpret_cast<const __nv_bfloat16*>(p), f);
  else load_n_f32<N>(reinterpret_cast<const float*>(p), f);
}

__device__ __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store1(float* p, float x) { *p = x; }

// ----------------------------------------------------------------- cache build / append
// One CTA per (batch, query head) walks the new rows chunk by chunk, carrying
// the running prefix P.  Thread layout per chunk: CG channel groups of 8 x RG
// row groups of RPG rows.
template <typename T, int KD, int RPG>
__global__ void __launch_bounds__(256) cache_build_kernel(
    const T* __restrict__ k_new, const T* __restrict__ g_new, const float* __restrict__ p_prev,
    int t_start, int T_new, int cap, int HQ, int H, T* __restrict__ k_tilde,
    float* __restrict__ r_cache, float* __restrict__ p_last) {
  constexpr int CG = KD / 8;
  constexpr int RG = 256 / CG;
  constexpr int C = RG * RPG;
  __shared__ float tot[2][RG][KD];
  __shared__ float rloc[2][KD];

  const int bh = blockIdx.x;
  const int b = bh / HQ, hq = bh % HQ, kvh = hq / (HQ / H);
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  const int ch = cg * 8;
  const int ncap = (cap + C - 1) / C;
  const int t_end = t_start + T_new;

  float carry[8];
#pragma unroll
  for (int c = 0; c < 8; ++c)
    carry[c] = p_prev ? p_prev[static_cast<size_t>(bh) * KD + ch + c] : 0.f;

  int buf = 0;
  for (int c0 = (t_start / C) * C; c0 < t_end; c0 += C, buf ^= 1) {
    const int chunk = c0 / C;
    const bool fresh = c0 >= t_start;  // this call writes the chunk's anchor
    float acc[8], loc[RPG][8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
    for (int m = 0; m < RPG; ++m) {
      const int t = c0 + rg * RPG + m;
      if (t >= t_start && t < t_end) {
        float f[8];
        load8(g_new + ((static_cast<size_t>(b) * T_new + (t - t_start)) * HQ + hq) * KD + ch, f);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += f[c] * kLog2e;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) loc[m][c] = acc[c];
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) tot[buf][rg][ch + c] = acc[c];
    if (fresh && rg == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) rloc[buf][ch + c] = loc[0][c];
    }
    __syncthreads();
    float pre[8], total[8], R[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float a = 0.f, all = 0.f;
      for (int r = 0; r < RG; ++r) {
        const float x = tot[buf][r][ch + c];
        all += x;
        if (r < rg) a += x;
      }
      pre[c] = a;
      total[c] = all;
    }
    float* rrow = r_cache + ((static_cast<size_t>(b) * ncap + chunk) * HQ + hq) * KD + ch;
    if (fresh) {
#pragma unroll
      for (int c = 0; c < 8; ++c) R[c] = rloc[buf][ch + c];  // local to this chunk's start
      if (rg == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) rrow[c] = carry[c] + R[c];
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) R[c] = rrow[c] - carry[c];  // anchor written by an earlier call
    }
#pragma unroll
    for (int m = 0; m < RPG; ++m) {
      const int t = c0 + rg * RPG + m;
      if (t >= t_start && t < t_end) {
        float kf[8];
        load8(k_new + ((static_cast<size_t>(b) * T_new + (t - t_start)) * H + kvh) * KD + ch, kf);
#pragma unroll
        for (int c = 0; c < 8; ++c) kf[c] *= exp2f(R[c] - (pre[c] + loc[m][c]));
        store8(k_tilde + ((static_cast<size_t>(b) * cap + t) * HQ + hq) * KD + ch, kf);
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) carry[c] += total[c];
  }
  if (rg == 0) {
#pragma unroll
    for (int c = 0; c < 8; ++c) p_last[static_cast<size_t>(bh) * KD + ch + c] = carry[c];
  }
}

// ----------------------------------------------------------------- split-KV decode
constexpr int kDecWarps = 4;
constexpr int kRowBatch = 8;

template <typename T, int KD, int VD, int G>
__global__ void __launch_bounds__(kDecWarps * 32) decode_split_kernel(
    const T* __restrict__ q, const float* __restrict__ p_curr, const T* __restrict__ v,
    const T* __restrict__ k_tilde, const float* __restrict__ r_cache, int T_kv, int cap, int HQ,
    int H, int C, int cps, int nsplit, float sc, float* __restrict__ part) {
  constexpr int LPH = 32 / G;    // lanes per query head
  constexpr int CPL = KD / LPH;  // k_tilde channels per lane
  constexpr int VPL = VD / 32;   // v channels per lane
  __shared__ float sm_m[kDecWarps][G], sm_l[kDecWarps][G];
  __shared__ __align__(16) float sm_o[kDecWarps][G][VD];

  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hl = lane / LPH;
  const int hq = h * G + hl;
  const int cofs = (lane % LPH) * CPL;
  const int nchunks = (T_kv + C - 1) / C;
  const int ncap = (cap + C - 1) / C;

  float qv[CPL], pc[CPL];
  load_n<T, CPL>(q + (static_cast<size_t>(b) * HQ + hq) * KD + cofs, qv);
  load_n<float, CPL>(p_curr + (static_cast<size_t>(b) * HQ + hq) * KD + cofs, pc);

  float m = -INFINITY, l = 0.f;
  float o[G][VPL];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int c = 0; c < VPL; ++c) o[hh][c] = 0.f;

  const size_t krow = static_cast<size_t>(HQ) * KD;
  const size_t vrow = static_cast<size_t>(H) * VD;
  const T* kbase = k_tilde + static_cast<size_t>(b) * cap * krow + static_cast<size_t>(h) * G * KD +
                   static_cast<size_t>(lane) * CPL;
  const T* vbase = v + static_cast<size_t>(b) * cap * vrow + static_cast<size_t>(h) * VD + lane * VPL;

  const int ck_end = min((s + 1) * cps, nchunks);
  for (int ck = s * cps + warp; ck < ck_end; ck += kDecWarps) {
    float qt[CPL], R[CPL];
    load_n<float, CPL>(r_cache + ((static_cast<size_t>(b) * ncap + ck) * HQ + hq) * KD + cofs, R);
#pragma unroll
    for (int e = 0; e < CPL; ++e) qt[e] = qv[e] * sc * exp2f(pc[e] - R[e]);
    const int r0 = ck * C, r1 = min(r0 + C, T_kv);
    for (int j = r0; j < r1; j += kRowBatch) {
      float sres[kRowBatch], vv[kRowBatch][VPL];
#pragma unroll
      for (int rr = 0; rr < kRowBatch; ++rr) {
        const int jj = j + rr;
        float part_dot = 0.f;
        if (jj < r1) {
          float kf[CPL];
          load_n<T, CPL>(kbase + static_cast<size_t>(jj) * krow, kf);
          load_n<T, VPL>(vbase + static_cast<size_t>(jj) * vrow, vv[rr]);
#pragma unroll
          for (int e = 0; e < CPL; ++e) part_dot = fmaf(qt[e], kf[e], part_dot);
        } else {
#pragma unroll
          for (int c = 0; c < VPL; ++c) vv[rr][c] = 0.f;
        }
        sres[rr] = part_dot;
      }
#pragma unroll
      for (int rr = 0; rr < kRowBatch; ++rr) {
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1)
          sres[rr] += __shfl_xor_sync(0xffffffffu, sres[rr], off);
        if (j + rr >= r1) sres[rr] = -INFINITY;
      }
      float mloc = sres[0];
#pragma unroll
      for (int rr = 1; rr < kRowBatch; ++rr) mloc = fmaxf(mloc, sres[rr]);
      const float mn = fmaxf(m, mloc);  // finite: row j is always admitted
      const float alpha = exp2f(m - mn);
      float pr[kRowBatch], rs = 0.f;
#pragma unroll
      for (int rr = 0; rr < kRowBatch; ++rr) {
        pr[rr] = exp2f(sres[rr] - mn);
        rs += pr[rr];
      }
      l = l * alpha + rs;
      m = mn;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float ah = __shfl_sync(0xffffffffu, alpha, hh * LPH);
#pragma unroll
        for (int c = 0; c < VPL; ++c) o[hh][c] *= ah;
#pragma unroll
        for (int rr = 0; rr < kRowBatch; ++rr) {
          const float ph = __shfl_sync(0xffffffffu, pr[rr], hh * LPH);
#pragma unroll
          for (int c = 0; c < VPL; ++c) o[hh][c] = fmaf(ph, vv[rr][c], o[hh][c]);
        }
      }
    }
  }

  // merge the warps of this CTA
  if (lane % LPH == 0) {
    sm_m[warp][hl] = m;
    sm_l[warp][hl] = l;
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int c = 0; c < VPL; ++c) sm_o[warp][hh][lane * VPL + c] = o[hh][c];
  __syncthreads();
  for (int e = threadIdx.x; e < G * (VD + 2); e += kDecWarps * 32) {
    const int hh = e / (VD + 2), c = e % (VD + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w][hh]);
    float val;
    if (M == -INFINITY) {
      val = (c == VD) ? -INFINITY : 0.f;
    } else if (c == VD) {
      val = M;
    } else {
      val = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = exp2f(sm_m[w][hh] - M);
        val += wt * (c == VD + 1 ? sm_l[w][hh] : sm_o[w][hh][c]);
      }
    }
    part[((static_cast<size_t>(b) * HQ + h * G + hh) * nsplit + s) * (VD + 2) + c] = val;
  }
}

// One warp per (batch, query head): merge the split partials, add the sink.
template <typename T, int VD>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part,
                                                             int nsplit, int nbh, int HQ,
                                                             const float* __restrict__ sink,
                                                             T* __restrict__ o,
                                                             float* __restrict__ lse) {
  constexpr int VPL = VD / 32;
  const int bhq = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bhq >= nbh) return;
  const float* pp = part + static_cast<size_t>(bhq) * nsplit * (VD + 2);
  float M = -INFINITY;
  for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, pp[s * (VD + 2) + VD]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float sink2 = sink ? sink[bhq % HQ] * kLog2e : -INFINITY;
  M = fmaxf(M, sink2);
  float Z = 0.f;
  for (int s = lane; s < nsplit; s += 32) {
    const float ms = pp[s * (VD + 2) + VD];
    if (ms != -INFINITY) Z += exp2f(ms - M) * pp[s * (VD + 2) + VD + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, off);
  if (sink) Z += exp2f(sink2 - M);
  float acc[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) acc[c] = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = pp[s * (VD + 2) + VD];
    if (ms == -INFINITY) continue;
    const float wt = exp2f(ms - M);
#pragma unroll
    for (int c = 0; c < VPL; ++c) acc[c] = fmaf(wt, pp[s * (VD + 2) + lane * VPL + c], acc[c]);
  }
  const float inv = 1.f / Z;
#pragma unroll
  for (int c = 0; c < VPL; ++c) store1(o + static_cast<size_t>(bhq) * VD + lane * VPL + c, acc[c] * inv);
  if (lse != nullptr && lane == 0) lse[bhq] = (M + log2f(Z)) * kLn2;
}

template <typename T, int KD, int RPG>
cudaError_t cache_impl(const CacheArgs& a, cudaStream_t st) {
  cache_build_kernel<T, KD, RPG><<<a.B * a.HQ, 256, 0, st>>>(
      static_cast<const T*>(a.k_new), static_cast<const T*>(a.g_new), a.p_prev, a.t_start,
      a.T_new, a.cap, a.HQ, a.H, static_cast<T*>(a.k_tilde), a.r_cache, a.p_last);
  return cudaGetLastError();
}

template <typename T, int KD>
cudaError_t cache_dispatch(const CacheArgs& a, cudaStream_t st) {
  constexpr int RG = 256 / (KD / 8);
  const int rpg = a.chunk / RG;
  switch (rpg) {
    case 1: return cache_impl<T, KD, 1>(a, st);
    case 2: return cache_impl<T, KD, 2>(a, st);
    case 4: return cache_impl<T, KD, 4>(a, st);
    case 8: return cache_impl<T, KD, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int KD, int VD, int G>
cudaError_t decode_impl(const DecodeArgs& a, cudaStream_t st) {
  const int nchunks = (a.T_kv + a.chunk - 1) / a.chunk;
  const int cps = (nchunks + a.nsplit - 1) / a.nsplit;
  dim3 grid(a.nsplit, a.H, a.B);
  decode_split_kernel<T, KD, VD, G><<<grid, kDecWarps * 32, 0, st>>>(
      static_cast<const T*>(a.q), a.p_curr, static_cast<const T*>(a.v),
      static_cast<const T*>(a.k_tilde), a.r_cache, a.T_kv, a.cap, a.HQ, a.H, a.chunk, cps,
      a.nsplit, a.scale * kLog2e, a.part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.mid_event != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(a.mid_event), st);
  const int nbh = a.B * a.HQ;
  decode_combine_kernel<T, VD><<<(nbh + 3) / 4, 128, 0, st>>>(a.part, a.nsplit, nbh, a.HQ, a.sink,
                                                             static_cast<T*>(a.o), a.lse);
  return cudaGetLastError();
}

template <typename T, int KD, int VD>
cudaError_t decode_by_group(const DecodeArgs& a, cudaStream_t st) {
  switch (a.HQ / a.H) {
    case 1: return decode_impl<T, KD, VD, 1>(a, st);
    case 2: return decode_impl<T, KD, VD, 2>(a, st);
    case 4: return decode_impl<T, KD, VD, 4>(a, st);
    case 8: return decode_impl<T, KD, VD, 8>(a, st);
    case 16: return decode_impl<T, KD, VD, 16>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t decode_by_dims(const DecodeArgs& a, cudaStream_t st) {
  if (a.K == 64 && a.V == 64) return decode_by_group<T, 64, 64>(a, st);
  if (a.K == 64 && a.V == 128) return decode_by_group<T, 64, 128>(a, st);
  if (a.K == 128 && a.V == 64) return decode_by_group<T, 128, 64>(a, st);
  if (a.K == 128 && a.V == 128) return decode_by_group<T, 128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_cache_build(const CacheArgs& a, bool bf16, cudaStream_t st) {
  if (bf16) return a.K == 64 ? cache_dispatch<__nv_bfloat16, 64>(a, st) : cache_dispatch<__nv_bfloat16, 128>(a, st);
  return a.K == 64 ? cache_dispatch<float, 64>(a, st) : cache_dispatch<float, 128>(a, st);
}

bool decode_supported(int K, int V, int group) {
  const bool kv = (K == 64 || K == 128) && (V == 64 || V == 128);
  const bool g = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
  return kv && g;
}

// Upper bound on the split count: enough CTAs to fill every SM several times
// over, never more splits than chunks.  Non-decreasing in T_kv.
int decode_max_splits(int B, int T_kv, int HQ, int H, int chunk) {
  (void)HQ;
  const long nchunks = (static_cast<long>(T_kv) + chunk - 1) / chunk;
  const long target = 148L * 8;
  const long groups = static_cast<long>(B) * H;
  long ns = (target + groups - 1) / groups;
  if (ns < 1) ns = 1;
  if (ns > nchunks) ns = nchunks;
  return static_cast<int>(ns);
}

// Splits actually launched: chunks are dealt out evenly, so trailing splits
// are never empty.  Never above decode_max_splits().
int decode_num_splits(int B, int T_kv, int HQ, int H, int chunk) {
  const int ns = decode_max_splits(B, T_kv, HQ, H, chunk);
  const int nchunks = (T_kv + chunk - 1) / chunk;
  const int cps = (nchunks + ns - 1) / ns;
  return (nchunks + cps - 1) / cps;
}

size_t decode_workspace_bytes(int B, int HQ, int V, int nsplit) {
  return static_cast<size_t>(B) * HQ * nsplit * (V + 2) * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? decode_by_dims<__nv_bfloat16>(a, st) : decode_by_dims<float>(a, st);
}

}  // namespace wall
