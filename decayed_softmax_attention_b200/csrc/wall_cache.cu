// Wall attention decode cache build / append (Wall Attention README, "Decode"):
//   P = cumsum(g) / ln 2,  R_c = P[c * C] (first row of chunk c),
//   k_tilde[j] = k[j] * exp2(R_{j/C} - P[j])
#include "wall_common.cuh"
#include "wall_internal.h"

namespace wall {
namespace {

// ----------------------------------------------------------------- cache build / append
// The prefix P runs along time, so each (batch, query head) sequence is walked
// in order by TPS = K/4 threads, each owning four channels for the whole walk:
// the prefix is a running sum in registers, with no exchange between threads.
// A warp covers one sequence (K = 128) or two (K = 64).  The rows come
// through a TMA ring in shared memory, so many stages of loads are in flight
// without holding registers.
//
// Precision: the running sum is kept as carry (P at the end of the previous
// chunk) + loc (sum inside the current chunk), so exp2(R_c - P[j]) is taken
// from chunk-local values only; anchors are stored as carry + loc.
template <typename T>
struct Vec4;  // four consecutive channels
template <>
struct Vec4<__nv_bfloat16> {
  uint2 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint2*>(p); }
  __device__ __forceinline__ void get(float* f) const {
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* f) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
  }
};
template <>
struct Vec4<float> {
  float4 u;
  __device__ __forceinline__ void load(const float* p) { u = *reinterpret_cast<const float4*>(p); }
  __device__ __forceinline__ void get(float* f) const { f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w; }
  __device__ __forceinline__ static void store(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

// Rows reach the CTA through a ring of NS shared-memory stages filled by TMA,
// D rows per stage: g of HPC consecutive query heads ([D][HPC][K]) and k of
// the NKV KV heads they use ([D][NKV][K]).  One producer thread issues the
// copies; consumer thread (head hl, channels ch..ch+3) walks the rows in order.
template <typename T, int KD>
struct CacheCfg {
  static constexpr int ESZ = static_cast<int>(sizeof(T));
  static constexpr int TPS = KD / 4;         // threads per sequence
  static constexpr int HMAX = 128 / TPS;     // query heads per CTA at most
  static constexpr int D = 32 / ESZ;         // rows per stage (16 bf16, 8 fp32)
  static constexpr int NS = 4;               // stages in the ring
  static constexpr int ROWB = KD * ESZ;      // bytes of one head row
};

template <typename T, int KD>
__global__ void __launch_bounds__(160) cache_build_kernel(
    const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmK,
    const float* __restrict__ p_prev, int t_start, int T_new, int cap, int HQ, int G, int HPC,
    int NKV, int C, T* __restrict__ k_tilde, float* __restrict__ r_cache,
    float* __restrict__ p_last, int* err, uint64_t wait_ns) {
  using CC = CacheCfg<T, KD>;
  constexpr int D = CC::D;
  extern __shared__ __align__(128) uint8_t csm[];
  const int gbytes = D * HPC * CC::ROWB;
  const int stage = gbytes + D * NKV * CC::ROWB;
  uint64_t* full = reinterpret_cast<uint64_t*>(csm + CC::NS * stage);
  uint64_t* empty = full + CC::NS;
  int* abort_flag = reinterpret_cast<int*>(empty + CC::NS);
  const int ncons = HPC * CC::TPS;
  const int nwc = (ncons + 31) / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hq0 = blockIdx.x * HPC, b = blockIdx.y;
  const int nst = (T_new + D - 1) / D;

  if (threadIdx.x == 0) {
    for (int i = 0; i < CC::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], nwc);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, err, wait_ns};

  if (warp == nwc) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmK);
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const int slot = i % CC::NS;
        if (i >= CC::NS && !mbar_wait(&empty[slot], ((i / CC::NS) - 1) & 1, wc)) break;
        uint8_t* st = csm + slot * stage;
        mbar_arrive_expect_tx(&full[slot], stage);
        tma_load_4d(st, &tmG, &full[slot], 0, hq0, i * D, b);
        tma_load_4d(st + gbytes, &tmK, &full[slot], 0, hq0 / G, i * D, b);
        issued = i + 1;
      }
      for (int i = issued > CC::NS ? issued - CC::NS : 0; i < issued; ++i)
        mbar_drain(&full[i % CC::NS], (i / CC::NS) & 1, wait_ns);
    }
    return;
  }
  // --------------------------------------------------------------- consumers
  const int ct = threadIdx.x;
  const bool active = ct < ncons;
  const int hl = active ? ct / CC::TPS : 0;
  const int kl = hl / G;  // local KV head (0 when the CTA's heads share one)
  const int ch = (ct % CC::TPS) * 4;
  const int hq = hq0 + hl;
  const size_t bh = static_cast<size_t>(b) * HQ + hq;
  const int ncap = (cap + C - 1) / C;
  const size_t hstep = static_cast<size_t>(HQ) * KD;
  T* op = k_tilde + ((static_cast<size_t>(b) * cap + t_start) * HQ + hq) * KD + ch;
  float* rp = r_cache + (static_cast<size_t>(b) * ncap * HQ + hq) * KD + ch;  // + chunk * hstep

  float carry[4], loc[4], r0[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    carry[c] = (active && p_prev) ? p_prev[bh * KD + ch + c] : 0.f;
    loc[c] = 0.f;
    r0[c] = 0.f;
  }
  if (active && t_start % C != 0) {
    // the chunk holding t_start was anchored by an earlier call
    const float* rr = rp + static_cast<size_t>(t_start / C) * hstep;
#pragma unroll
    for (int c = 0; c < 4; ++c) r0[c] = rr[c] - carry[c];
  }

  const int cmask = C - 1;  // C is a power of two
  const int cshift = __ffs(C) - 1;
  const int gstr = HPC * KD, kstr = NKV * KD;  // shared-memory row strides (elements)
  // One row: fold g into the prefix, anchor at a chunk head, rescale k.
  auto row = [&](const T* g_s, const T* k_s, T* o_g, bool head, int ta) {
    Vec4<T> gv, kv;
    gv.load(g_s);
    kv.load(k_s);
    float g[4], k[4];
    gv.get(g);
    kv.get(k);
    if (head) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        carry[c] += loc[c];
        loc[c] = 0.f;
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) loc[c] = fmaf(g[c], kLog2e, loc[c]);
    if (head) {
#pragma unroll
      for (int c = 0; c < 4; ++c) r0[c] = loc[c];
      *reinterpret_cast<float4*>(rp + static_cast<size_t>(ta >> cshift) * hstep) =
          make_float4(carry[0] + loc[0], carry[1] + loc[1], carry[2] + loc[2], carry[3] + loc[3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) k[c] *= ex2_approx(r0[c] - loc[c]);
    Vec4<T>::store(o_g, k);
  };

  bool ok = true;
  for (int i = 0; i < nst; ++i) {
    const int slot = i % CC::NS;
    const bool got = mbar_wait(&full[slot], (i / CC::NS) & 1, wc);
    if (!__all_sync(0xffffffffu, got)) {
      ok = false;
      break;
    }
    const uint8_t* st = csm + slot * stage;
    const T* sg = reinterpret_cast<const T*>(st) + hl * KD + ch;
    const T* sk = reinterpret_cast<const T*>(st + gbytes) + kl * KD + ch;
    if (active) {
      const int t0 = i * D;
      const int ta0 = t_start + t0;
      const int hr = (C - (ta0 & cmask)) & cmask;  // stage row that opens a chunk (>= D: none)
      T* ob = op + static_cast<size_t>(t0) * hstep;
      if (t0 + D <= T_new) {
#pragma unroll
        for (int r = 0; r < D; ++r) {
          row(sg, sk, ob, r == hr, ta0 + r);
          sg += gstr;
          sk += kstr;
          ob += hstep;
        }
      } else {
        for (int r = 0; r < T_new - t0; ++r) {
          row(sg, sk, ob, r == hr, ta0 + r);
          sg += gstr;
          sk += kstr;
          ob += hstep;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  if (ok && active)
    *reinterpret_cast<float4*>(p_last + bh * KD + ch) =
        make_float4(carry[0] + loc[0], carry[1] + loc[1], carry[2] + loc[2], carry[3] + loc[3]);
}

template <typename T, int KD>
cudaError_t cache_impl(const CacheArgs& a, cudaStream_t st) {
  using CC = CacheCfg<T, KD>;
  const int G = a.HQ / a.H;
  int hpc = 1;  // query heads per CTA: a power of two dividing HQ, nested with G
  for (int h = CC::HMAX; h > 1; h >>= 1) {
    if (a.HQ % h == 0 && (G % h == 0 || h % G == 0)) {
      hpc = h;
      break;
    }
  }
  const int nkv = hpc >= G ? hpc / G : 1;
  if (a.B > 65535) return cudaErrorInvalidValue;
  const CUtensorMapDataType tdt =
      sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const cuuint64_t esz = sizeof(T);
  CUtensorMap tmG, tmK;
  {  // g_new [B, T_new, HQ, K]
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.HQ),
                                static_cast<cuuint64_t>(a.T_new), static_cast<cuuint64_t>(a.B)};
    const cuuint64_t strides[3] = {KD * esz, static_cast<cuuint64_t>(a.HQ) * KD * esz,
                                   static_cast<cuuint64_t>(a.T_new) * a.HQ * KD * esz};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(KD), static_cast<cuuint32_t>(hpc),
                               static_cast<cuuint32_t>(CC::D), 1};
    if (!encode_tiled(&tmG, tdt, 4, a.g_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  {  // k_new [B, T_new, H, K]
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(a.H),
                                static_cast<cuuint64_t>(a.T_new), static_cast<cuuint64_t>(a.B)};
    const cuuint64_t strides[3] = {KD * esz, static_cast<cuuint64_t>(a.H) * KD * esz,
                                   static_cast<cuuint64_t>(a.T_new) * a.H * KD * esz};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(KD), static_cast<cuuint32_t>(nkv),
                               static_cast<cuuint32_t>(CC::D), 1};
    if (!encode_tiled(&tmK, tdt, 4, a.k_new, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  const int stage = CC::D * (hpc + nkv) * CC::ROWB;
  const int smem = CC::NS * stage + 2 * CC::NS * 8 + 16;
  auto kern = cache_build_kernel<T, KD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nwc = (hpc * CC::TPS + 31) / 32;
  dim3 grid(a.HQ / hpc, a.B);
  kern<<<grid, (nwc + 1) * 32, smem, st>>>(tmG, tmK, a.p_prev, a.t_start, a.T_new, a.cap, a.HQ, G,
                                           hpc, nkv, a.chunk, static_cast<T*>(a.k_tilde),
                                           a.r_cache, a.p_last, a.err, a.wait_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cache_build(const CacheArgs& a, bool bf16, cudaStream_t st) {
  if (bf16) return a.K == 64 ? cache_impl<__nv_bfloat16, 64>(a, st) : cache_impl<__nv_bfloat16, 128>(a, st);
  return a.K == 64 ? cache_impl<float, 64>(a, st) : cache_impl<float, 128>(a, st);
}

}  // namespace wall
