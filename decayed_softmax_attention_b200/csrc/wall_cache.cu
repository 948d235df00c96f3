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

template <typename T, int KD, bool PAGED>
__global__ void __launch_bounds__(160) cache_build_kernel(
    const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmK,
    const float* __restrict__ p_prev, int t_start, int T_new, PageMap pm, int HQ, int G, int HPC,
    int NKV, int C, int seg_first, int seg_rows, T* __restrict__ k_tilde,
    float* __restrict__ r_cache, float* __restrict__ p_last, int* err, uint64_t wait_ns,
    int fault) {
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
  // Rows [rb, re) of this call (relative to t_start): all of them, or one
  // chunk-aligned segment (blockIdx.z) whose starting prefix an earlier pass
  // left in the anchor slot of its first chunk.
  const bool segmented = seg_rows > 0;
  const int rb = segmented ? seg_first + static_cast<int>(blockIdx.z) * seg_rows : 0;
  const int re = segmented ? min(rb + seg_rows, T_new) : T_new;
  const int nst = (re - rb + D - 1) / D;

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
        if (!(fault == 3 && i == 0)) {  // testing hook: starve the consumers
          mbar_arrive_expect_tx(&full[slot], stage);
          tma_load_4d(st, &tmG, &full[slot], 0, hq0, rb + i * D, b);
          tma_load_4d(st + gbytes, &tmK, &full[slot], 0, hq0 / G, rb + i * D, b);
        }
        issued = i + 1;
      }
      for (int i = issued > CC::NS ? issued - CC::NS : 0; i < issued; ++i)
        if (!(fault == 3 && i == 0)) mbar_drain(&full[i % CC::NS], (i / CC::NS) & 1, wait_ns);
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
  // this thread's four channels of cache row ta / of the anchor of ta's chunk:
  // dense caches step through rows with one add, paged ones go through the table
  const size_t hstep = static_cast<size_t>(HQ) * KD;
  T* const op = k_tilde + (static_cast<size_t>(b) * pm.cap * HQ + hq) * KD + ch;
  float* const rp = r_cache + (static_cast<size_t>(b) * ((pm.cap + C - 1) / C) * HQ + hq) * KD + ch;
  const int cshift = __ffs(C) - 1;  // C is a power of two
  auto krow = [=](int ta) -> T* {
    if constexpr (PAGED) return k_tilde + (pm.row(b, ta) * HQ + hq) * KD + ch;
    else return op + static_cast<size_t>(ta) * hstep;
  };
  auto rslot = [=](int ta) -> float* {
    if constexpr (PAGED) return r_cache + (pm.chunk(b, ta, C) * HQ + hq) * KD + ch;
    else return rp + static_cast<size_t>(ta >> cshift) * hstep;
  };

  float carry[4], loc[4], r0[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    carry[c] = (active && p_prev && !segmented) ? p_prev[bh * KD + ch + c] : 0.f;
    loc[c] = 0.f;
    r0[c] = 0.f;
  }
  if (active && segmented) {
    // P just before the segment (read before this thread overwrites the slot
    // with the chunk's anchor at the segment's first row)
    const float4 c4 = *reinterpret_cast<const float4*>(rslot(t_start + rb));
    carry[0] = c4.x;
    carry[1] = c4.y;
    carry[2] = c4.z;
    carry[3] = c4.w;
  } else if (active && t_start % C != 0) {
    // the chunk holding t_start was anchored by an earlier call
    const float* rr = rslot(t_start);
#pragma unroll
    for (int c = 0; c < 4; ++c) r0[c] = rr[c] - carry[c];
  }

  const int cmask = C - 1;  // C is a power of two
  const int gstr = HPC * KD, kstr = NKV * KD;  // shared-memory row strides (elements)
  float kx = 0.f;  // largest exponent R_c - P_j of this thread's rows (cache range check)
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
      *reinterpret_cast<float4*>(rslot(ta)) =
          make_float4(carry[0] + loc[0], carry[1] + loc[1], carry[2] + loc[2], carry[3] + loc[3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      kx = fmaxf(kx, r0[c] - loc[c]);
      k[c] *= ex2_approx(r0[c] - loc[c]);
    }
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
      const int t0 = rb + i * D;
      const int ta0 = t_start + t0;
      const int hr = (C - (ta0 & cmask)) & cmask;  // stage row that opens a chunk (>= D: none)
      T* ob = PAGED ? nullptr : krow(ta0);
      if (t0 + D <= re) {
#pragma unroll
        for (int r = 0; r < D; ++r) {
          row(sg, sk, PAGED ? krow(ta0 + r) : ob, r == hr, ta0 + r);
          sg += gstr;
          sk += kstr;
          if (!PAGED) ob += hstep;
        }
      } else {
        for (int r = 0; r < re - t0; ++r) {
          row(sg, sk, PAGED ? krow(ta0 + r) : ob, r == hr, ta0 + r);
          sg += gstr;
          sk += kstr;
          if (!PAGED) ob += hstep;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  if (ok && active && !segmented)
    *reinterpret_cast<float4*>(p_last + bh * KD + ch) =
        make_float4(carry[0] + loc[0], carry[1] + loc[1], carry[2] + loc[2], carry[3] + loc[3]);
  if (kx > kCacheRangeLog2) atomicOr(err, kDevErrRange);
}

__device__ __forceinline__ void store_one(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_one(float* p, float x) { *p = x; }

// Segmented build, pass 1 (when B * HQ / HPC CTAs cannot fill the GPU): for
// every (batch, query head, chunk-aligned segment) the channel sums of g over
// the segment (log2 units, summed chunk by chunk like the walk's carry), kept
// in the anchor slot of the segment's first chunk until pass 3 overwrites it.
template <typename T, int KD>
__global__ void __launch_bounds__(128) cache_segsum_kernel(
    const T* __restrict__ g_new, int t_start, int T_new, PageMap pm, int HQ, int HPC, int C,
    int seg_first, int seg_rows, float* __restrict__ r_cache) {
  using CC = CacheCfg<T, KD>;
  constexpr int U = 8;  // rows whose loads are issued together
  const int ct = threadIdx.x;
  if (ct >= HPC * CC::TPS) return;
  const int hl = ct / CC::TPS, ch = (ct % CC::TPS) * 4;
  const int hq = static_cast<int>(blockIdx.x) * HPC + hl, b = blockIdx.y;
  const int rb = seg_first + static_cast<int>(blockIdx.z) * seg_rows;
  const int re = min(rb + seg_rows, T_new);
  const size_t gstep = static_cast<size_t>(HQ) * KD;
  const T* gp = g_new + (static_cast<size_t>(b) * T_new * HQ + hq) * KD + ch;
  float tot[4] = {0.f, 0.f, 0.f, 0.f}, loc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int t0 = rb; t0 < re; t0 += U) {
    Vec4<T> v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (t0 + u < re) v[u].load(gp + static_cast<size_t>(t0 + u) * gstep);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (t0 + u < re) {
        if (((t_start + t0 + u) & (C - 1)) == 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tot[c] += loc[c];
            loc[c] = 0.f;
          }
        }
        float g[4];
        v[u].get(g);
#pragma unroll
        for (int c = 0; c < 4; ++c) loc[c] = fmaf(g[c], kLog2e, loc[c]);
      }
    }
  }
  float* rr = r_cache + (pm.chunk(b, t_start + rb, C) * HQ + hq) * KD + ch;
  *reinterpret_cast<float4*>(rr) =
      make_float4(tot[0] + loc[0], tot[1] + loc[1], tot[2] + loc[2], tot[3] + loc[3]);
}

// Segmented build, pass 2: one thread per (batch, query head, channel).  The
// rows of a partial first chunk (t_start inside a chunk anchored by an earlier
// call) are rescaled here; then the segment sums become the prefix P just
// before each segment (in place, in order), and the final P goes to p_last.
template <typename T, int KD>
__global__ void __launch_bounds__(128) cache_segscan_kernel(
    const T* __restrict__ k_new, const T* __restrict__ g_new, const float* __restrict__ p_prev,
    int B, int t_start, int T_new, PageMap pm, int HQ, int H, int C, int seg_first, int seg_rows,
    int nseg, T* __restrict__ k_tilde, float* __restrict__ r_cache, float* __restrict__ p_last,
    int* err) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(B) * HQ * KD) return;
  const int n = static_cast<int>(idx % KD);
  const long bh = idx / KD;
  const int b = static_cast<int>(bh / HQ), hq = static_cast<int>(bh % HQ), kvh = hq / (HQ / H);
  auto rslot = [&](int ta) { return r_cache + (pm.chunk(b, ta, C) * HQ + hq) * KD + n; };
  float carry = p_prev ? p_prev[static_cast<size_t>(bh) * KD + n] : 0.f;
  if (seg_first > 0) {
    const float r0 = *rslot(t_start) - carry;
    float loc = 0.f;
    for (int t = 0; t < seg_first; ++t) {
      const size_t row = static_cast<size_t>(b) * T_new + t;
      loc = fmaf(load1(g_new + (row * HQ + hq) * KD + n), kLog2e, loc);
      const float kv = load1(k_new + (row * H + kvh) * KD + n);
      store_one(k_tilde + (pm.row(b, t_start + t) * HQ + hq) * KD + n, kv * ex2_approx(r0 - loc));
    }
    if (r0 - loc > kCacheRangeLog2) atomicOr(err, kDevErrRange);
    carry += loc;
  }
  for (int s = 0; s < nseg; ++s) {
    float* rr = rslot(t_start + seg_first + s * seg_rows);
    const float tot = *rr;
    *rr = carry;
    carry += tot;
  }
  p_last[static_cast<size_t>(bh) * KD + n] = carry;
}

// One-token append at a per-row position (batches whose sequences have
// different lengths).  Thread: (batch row, query head, four channels).
template <typename T, int KD>
__global__ void __launch_bounds__(128) cache_append_varlen_kernel(
    const T* __restrict__ k_new, const T* __restrict__ g_new, const float* __restrict__ p_prev,
    const int* __restrict__ t_pos, int B, PageMap pm, int HQ, int H, int C,
    T* __restrict__ k_tilde, float* __restrict__ r_cache, float* __restrict__ p_last, int* err) {
  constexpr int TPS = KD / 4;
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(B) * HQ * TPS) return;
  const int ch = static_cast<int>(idx % TPS) * 4;
  const long bh = idx / TPS;
  const int b = static_cast<int>(bh / HQ), hq = static_cast<int>(bh % HQ), kvh = hq / (HQ / H);
  const int t = min(max(t_pos[b], 0), pm.rows() - 1);  // clamped to the cache
  Vec4<T> gv, kv;
  gv.load(g_new + (static_cast<size_t>(b) * HQ + hq) * KD + ch);
  kv.load(k_new + (static_cast<size_t>(b) * H + kvh) * KD + ch);
  float g[4], k[4], P[4];
  gv.get(g);
  kv.get(k);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float prev = t > 0 ? p_prev[static_cast<size_t>(bh) * KD + ch + c] : 0.f;
    P[c] = fmaf(g[c], kLog2e, prev);
  }
  float* rr = r_cache + (pm.chunk(b, t, C) * HQ + hq) * KD + ch;
  if (t % C == 0) {
    *reinterpret_cast<float4*>(rr) = make_float4(P[0], P[1], P[2], P[3]);  // new chunk anchor
  } else {
    const float4 R = *reinterpret_cast<const float4*>(rr);
    if (fmaxf(fmaxf(R.x - P[0], R.y - P[1]), fmaxf(R.z - P[2], R.w - P[3])) > kCacheRangeLog2)
      atomicOr(err, kDevErrRange);
    k[0] *= ex2_approx(R.x - P[0]);
    k[1] *= ex2_approx(R.y - P[1]);
    k[2] *= ex2_approx(R.z - P[2]);
    k[3] *= ex2_approx(R.w - P[3]);
  }
  Vec4<T>::store(k_tilde + (pm.row(b, t) * HQ + hq) * KD + ch, k);
  *reinterpret_cast<float4*>(p_last + static_cast<size_t>(bh) * KD + ch) =
      make_float4(P[0], P[1], P[2], P[3]);
}

// ----------------------------------------------------------------- scalar-gate cache
// PS[t] = (PS before t_start) + sum_{u <= t} g_scalar[u] * log2(e): the scalar
// gate's prefix in the exp2 units of the decode cache, one fp32 per (row,
// query head).  Thread (segment of kGateSeg rows, head): head fastest, so a
// warp reads whole rows.  Three passes: segment sums (kept in the cache row
// that opens the segment), their prefix per head, then the rows.
constexpr int kGateSeg = 256;

template <typename T>
__global__ void __launch_bounds__(256) gate_segsum_kernel(const T* __restrict__ gs_new,
                                                          int t_start, int T_new, int HQ,
                                                          PageMap pm, float* __restrict__ gcache) {
  const int nseg = (T_new + kGateSeg - 1) / kGateSeg;
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(nseg) * HQ) return;
  const int hq = static_cast<int>(idx % HQ), seg = static_cast<int>(idx / HQ), b = blockIdx.y;
  const int r0 = seg * kGateSeg, r1 = min(r0 + kGateSeg, T_new);
  const T* src = gs_new + (static_cast<size_t>(b) * T_new) * HQ + hq;
  float acc = 0.f;
  for (int r = r0; r < r1; ++r) acc = fmaf(load1(src + static_cast<size_t>(r) * HQ), kLog2e, acc);
  gcache[pm.row(b, t_start + r0) * HQ + hq] = acc;
}

// One thread per (batch, head): the segment sums become the prefix before each
// segment, in place; the total goes to gs_last.
__global__ void __launch_bounds__(128) gate_scan_kernel(const float* __restrict__ gs_prev,
                                                        int B, int t_start, int T_new, int HQ,
                                                        PageMap pm, float* __restrict__ gcache,
                                                        float* __restrict__ gs_last) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(B) * HQ) return;
  const int b = static_cast<int>(idx / HQ), hq = static_cast<int>(idx % HQ);
  float carry = (t_start > 0 && gs_prev != nullptr) ? gs_prev[idx] : 0.f;
  const int nseg = (T_new + kGateSeg - 1) / kGateSeg;
  for (int sg = 0; sg < nseg; ++sg) {
    float* slot = gcache + pm.row(b, t_start + sg * kGateSeg) * HQ + hq;
    const float tot = *slot;
    *slot = carry;
    carry += tot;
  }
  gs_last[idx] = carry;
}

template <typename T>
__global__ void __launch_bounds__(256) gate_write_kernel(const T* __restrict__ gs_new, int t_start,
                                                         int T_new, int HQ, PageMap pm,
                                                         float* __restrict__ gcache) {
  const int nseg = (T_new + kGateSeg - 1) / kGateSeg;
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(nseg) * HQ) return;
  const int hq = static_cast<int>(idx % HQ), seg = static_cast<int>(idx / HQ), b = blockIdx.y;
  const int r0 = seg * kGateSeg, r1 = min(r0 + kGateSeg, T_new);
  const T* src = gs_new + (static_cast<size_t>(b) * T_new) * HQ + hq;
  float acc = gcache[pm.row(b, t_start + r0) * HQ + hq];  // prefix before the segment
  for (int r = r0; r < r1; ++r) {
    acc = fmaf(load1(src + static_cast<size_t>(r) * HQ), kLog2e, acc);
    gcache[pm.row(b, t_start + r) * HQ + hq] = acc;
  }
}

// One token per batch row at its own position t_pos[b]: thread per (batch, head).
template <typename T>
__global__ void __launch_bounds__(128) gate_append_kernel(const T* __restrict__ gs_new,
                                                          const float* __restrict__ gs_prev,
                                                          const int* __restrict__ t_pos, int B,
                                                          int HQ, PageMap pm,
                                                          float* __restrict__ gcache,
                                                          float* __restrict__ gs_last) {
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(B) * HQ) return;
  const int b = static_cast<int>(idx / HQ), hq = static_cast<int>(idx % HQ);
  const int t = min(max(t_pos[b], 0), pm.rows() - 1);
  const float prev = t > 0 ? gs_prev[idx] : 0.f;
  const float ps = fmaf(load1(gs_new + idx), kLog2e, prev);
  gcache[pm.row(b, t) * HQ + hq] = ps;
  gs_last[idx] = ps;
}

template <typename T>
cudaError_t gate_impl(const GateArgs& a, cudaStream_t st) {
  const T* gs = static_cast<const T*>(a.gs_new);
  if (a.t_pos != nullptr) {
    const long n = static_cast<long>(a.B) * a.HQ;
    gate_append_kernel<T><<<static_cast<unsigned>((n + 127) / 128), 128, 0, st>>>(
        gs, a.gs_prev, a.t_pos, a.B, a.HQ, a.pm, a.gcache, a.gs_last);
    return cudaGetLastError();
  }
  const int nseg = (a.T_new + kGateSeg - 1) / kGateSeg;
  const long nthr = static_cast<long>(nseg) * a.HQ;
  const dim3 grid(static_cast<unsigned>((nthr + 255) / 256), a.B);
  gate_segsum_kernel<T><<<grid, 256, 0, st>>>(gs, a.t_start, a.T_new, a.HQ, a.pm, a.gcache);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long nbh = static_cast<long>(a.B) * a.HQ;
  gate_scan_kernel<<<static_cast<unsigned>((nbh + 127) / 128), 128, 0, st>>>(
      a.gs_prev, a.B, a.t_start, a.T_new, a.HQ, a.pm, a.gcache, a.gs_last);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gate_write_kernel<T><<<grid, 256, 0, st>>>(gs, a.t_start, a.T_new, a.HQ, a.pm, a.gcache);
  return cudaGetLastError();
}

template <typename T, int KD>
cudaError_t append_varlen_impl(const CacheArgs& a, const int* t_pos, cudaStream_t st) {
  const long n = static_cast<long>(a.B) * a.HQ * (KD / 4);
  cache_append_varlen_kernel<T, KD><<<static_cast<unsigned>((n + 127) / 128), 128, 0, st>>>(
      static_cast<const T*>(a.k_new), static_cast<const T*>(a.g_new), a.p_prev, t_pos, a.B, a.pm,
      a.HQ, a.H, a.chunk, static_cast<T*>(a.k_tilde), a.r_cache, a.p_last, a.err);
  return cudaGetLastError();
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
  // Split each sequence into chunk-aligned segments when the (batch, head
  // group) CTAs alone would leave most SMs idle and there are enough rows.
  const int ctas = a.B * (a.HQ / hpc);
  int seg_first = 0, seg_rows = 0, nseg = 0;
  {
    const int c0 = (a.t_start + a.chunk - 1) / a.chunk * a.chunk;
    const int head = min(c0 - a.t_start, a.T_new);  // rows of a partial first chunk
    const int rest = a.T_new - head;
    if (ctas < 148 && rest >= 4 * a.chunk) {
      const int want = (296 + ctas - 1) / ctas;  // segments per sequence group: ~2 CTAs per SM
      int L = (rest + want - 1) / want;
      L = max(4 * a.chunk, (L + a.chunk - 1) / a.chunk * a.chunk);
      seg_first = head;
      seg_rows = L;
      nseg = (rest + L - 1) / L;
    }
  }
  const int stage = CC::D * (hpc + nkv) * CC::ROWB;
  const int smem = CC::NS * stage + 2 * CC::NS * 8 + 16;
  auto kern = a.pm.paged() ? cache_build_kernel<T, KD, true> : cache_build_kernel<T, KD, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (nseg > 0) {
    cache_segsum_kernel<T, KD><<<dim3(a.HQ / hpc, a.B, nseg), 128, 0, st>>>(
        static_cast<const T*>(a.g_new), a.t_start, a.T_new, a.pm, a.HQ, hpc, a.chunk, seg_first,
        seg_rows, a.r_cache);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long nthr = static_cast<long>(a.B) * a.HQ * KD;
    cache_segscan_kernel<T, KD><<<static_cast<unsigned>((nthr + 127) / 128), 128, 0, st>>>(
        static_cast<const T*>(a.k_new), static_cast<const T*>(a.g_new), a.p_prev, a.B, a.t_start,
        a.T_new, a.pm, a.HQ, a.H, a.chunk, seg_first, seg_rows, nseg,
        static_cast<T*>(a.k_tilde), a.r_cache, a.p_last, a.err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int nwc = (hpc * CC::TPS + 31) / 32;
  dim3 grid(a.HQ / hpc, a.B, nseg > 0 ? nseg : 1);
  kern<<<grid, (nwc + 1) * 32, smem, st>>>(tmG, tmK, a.p_prev, a.t_start, a.T_new, a.pm, a.HQ, G,
                                           hpc, nkv, a.chunk, seg_first, seg_rows,
                                           static_cast<T*>(a.k_tilde), a.r_cache, a.p_last,
                                           a.err, a.wait_ns, a.fault);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append_varlen(const CacheArgs& a, const int* t_pos, bool bf16, cudaStream_t st) {
  if (bf16) {
    return a.K == 64 ? append_varlen_impl<__nv_bfloat16, 64>(a, t_pos, st)
                     : append_varlen_impl<__nv_bfloat16, 128>(a, t_pos, st);
  }
  return a.K == 64 ? append_varlen_impl<float, 64>(a, t_pos, st)
                   : append_varlen_impl<float, 128>(a, t_pos, st);
}

cudaError_t launch_gate_cache(const GateArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? gate_impl<__nv_bfloat16>(a, st) : gate_impl<float>(a, st);
}

cudaError_t launch_cache_build(const CacheArgs& a, bool bf16, cudaStream_t st) {
  if (bf16) return a.K == 64 ? cache_impl<__nv_bfloat16, 64>(a, st) : cache_impl<__nv_bfloat16, 128>(a, st);
  return a.K == 64 ? cache_impl<float, 64>(a, st) : cache_impl<float, 128>(a, st);
}

}  // namespace wall
