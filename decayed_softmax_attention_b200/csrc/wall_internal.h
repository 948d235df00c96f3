// Host-side launchers shared by the translation units of the Wall attention
// library.  Not part of the public C ABI (include/wall_attn.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace wall {

constexpr int kBlockRows = 128;

// Device address of this device's error word (bit 0: a bounded wait gave up).
int* device_error_word();
// Current limit of every bounded device-side wait, in nanoseconds.
uint64_t wait_limit_ns();
// Current testing fault mode (wall_debug_set_fault); 0 in normal operation.
int fault_mode();
// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link): unit element strides, zero fill out of bounds.  strides in bytes.
bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                  const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                  CUtensorMapSwizzle swizzle);  // anchor block / tile height shared by the prefill kernels

// Workspace of the prefill forward.  NB = ceil(T / 128) anchor blocks.
//   qh, kh  [B*HQ][T][K]   anchored q and k (input dtype):
//           qh[t] = q[t] * exp(G[t] - AQ[2 * (t / 256)]),  kh[t] = k[t] * exp(AK[t / 128] - G[t])
//           (query anchors per 256-row block, key anchors per 128-row block)
//   bsum    [B*HQ][NB][K]  per-128-row-block sum of g (natural log)
//   AQ, AK  [B*HQ][NB][K]  G just before the block's first row / at its last row
//   ssl     [B*HQ][NB*128] minus the block-local inclusive prefix of g_scalar * log2(e)
//   ssb     [B*HQ][NB]     block sum of g_scalar * log2(e)
//   ssa     [B*HQ][NB][4]  prefix of g_scalar * log2(e) before the block ([0] used)
//   kx      [B*HQ][T][16]  bf16 key-side gate channels for the QK contraction:
//           (hi, lo, 0, ..., 0) with hi + lo = ssl[t] / (scale * log2(e)), bf16 head/tail
//   rowlo   [NB*128]       first admitted key per row (packed documents only; rows < T set)
//   wide    [B*HQ][NQB]    int32, NQB = ceil(T / 256): 1 when the anchored factors of the
//           256-row query block would span more than kPrefillSpanNats in some channel
//           (strong decay); the attention kernels then skip the block's own key tiles
//           and the diagonal kernel evaluates those pairs exactly
//   lse_ws  [B*T*HQ]       fp32 lse when the caller passes none (the diagonal kernel
//           merges through lse)
struct FwdWork {
  void* qh;
  void* kh;
  float* bsum;
  float* AQ;
  float* AK;
  float* ssl;
  float* ssb;
  float* ssa;
  void* kx;
  int* rowlo;
  int* wide;
  float* lse_ws;
};

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* g_scalar;
  const float* sink;
  const int32_t* cu_seqlens;
  int num_seqs;
  int window;
  int B, T, HQ, H, K, V, NB;
  float scale;
  void* o;
  float* lse;
  int* err;
  uint64_t wait_ns;
  int fault;
  // Decode cache emitted by the prepass (null k_tilde: none).
  void* kt_out = nullptr;     // [B, cap, HQ, K] input dtype
  float* r_out = nullptr;     // [B, ceil(cap/chunk), HQ, K] fp32
  float* plast_out = nullptr; // [B, HQ, K] fp32
  int cache_cap = 0, cache_chunk = 64;
  // Set by callers that cannot evaluate wide blocks exactly (the backward): the
  // prepass then records kDevErrRange in the error word for every wide block.
  bool wide_is_error = false;
};

size_t fwd_workspace_layout(int B, int T, int HQ, int K, bool bf16, FwdWork* w, char* base);

cudaError_t launch_prep(const FwdArgs& a, const FwdWork& w, bool bf16, cudaStream_t st);
cudaError_t launch_fwd_tc(const FwdArgs& a, const FwdWork& w, const CUtensorMap& tmQ,
                          const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKX,
                          cudaStream_t st);
cudaError_t launch_fwd_simt(const FwdArgs& a, const FwdWork& w, cudaStream_t st);
// Exact in-block pairs of the wide query blocks (both dtypes), merged with the
// attention kernel's (o, lse) of the same rows.  Runs after the attention kernel,
// which must have covered exactly the keys before each wide block.
struct DiagParams {
  const void* q;      // [B, Tb, HQ, K]
  const void* k;      // [B, Tb, H, K]
  const void* g;      // [B, Tb, HQ, K]
  const void* gs;     // [B, Tb, HQ] or null
  const void* v;      // local row t of batch row b: row (b * vT + voff + t) of [*, H, V]
  const float* sink;  // [HQ] or null
  const int* rowlo;   // first admitted key (absolute position) per row, or null
  const int* wide;    // [B*HQ][NQB] flags, NQB = ceil(Tb / 256)
  int window;
  int B, Tb, HQ, H, NQB;
  int vT, voff;
  int pos0;           // absolute position of local row 0 (window, rowlo)
  float scale;
  void* o;            // [B, Tb, HQ, V]: the attention kernel's rows on entry
  float* lse;         // [B, Tb, HQ]: likewise (natural log, sink included)
};
cudaError_t launch_diag(const DiagParams& p, bool bf16, int K, int V, cudaStream_t st);
cudaError_t launch_fwd_diag(const FwdArgs& a, const FwdWork& w, bool bf16, cudaStream_t st);

// Backward of the prefill.  Inputs as FwdArgs plus the forward's o and lse,
// dO (and optional dlse); outputs dq, dk, dv, dg, dg_scalar (input dtype) and
// dsink (fp32).
struct BwdArgs {
  FwdArgs f;            // forward inputs (f.o / f.lse: the forward's outputs)
  const void* dout;     // [B, T, HQ, V]
  const float* dlse;    // [B, T, HQ] or null
  void* dq;             // [B, T, HQ, K]
  void* dk;             // [B, T, H, K]
  void* dv;             // [B, T, H, V]
  void* dg;             // [B, T, HQ, K]
  void* dg_scalar;      // [B, T, HQ] (with g_scalar)
  float* dsink;         // [HQ] (with sink)
  // optional cudaEvent_t recorded before the key-block contraction, between it
  // and the query-block contraction, and after the latter (profiling hook)
  void* ev[3] = {nullptr, nullptr, nullptr};
};

// Backward workspace (after the forward prepass's own FwdWork):
//   rowt, colt, delta [B*HQ][NB*128] fp32 (padded rows: 16-byte aligned tiles);
//   psd, rsA, rsB [B*HQ][T] fp32; accQ, accK [B*HQ][T][K] fp32;
//   dvh [B*HQ][T][V] fp32; head, carry [B*HQ][NB][K+1]; sinkblk [B*HQ][NB].
struct BwdWork {
  float* rowt;   // Gs log2(e) - lse log2(e) per query row
  float* colt;   // Gs log2(e) per key row (g_scalar only)
  float* delta;  // dO.o - dlse
  float* psd;
  float* rsA;
  float* rsB;
  float* accQ;
  float* accK;
  float* dvh;
  float* head;
  float* carry;
  float* sinkblk;
};
size_t bwd_workspace_layout(int B, int T, int HQ, int K, int V, bool bf16, FwdWork* fw,
                            BwdWork* bw, char* base);
// Everything after the prepass: bwd_pre, the two contraction kernels, the post
// passes and the reductions.
cudaError_t launch_bwd(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw, bool bf16,
                       cudaStream_t st);
// The two bf16 tensor-core contraction kernels (key-block, query-block).
cudaError_t launch_bwd_tc(const BwdArgs& a, const FwdWork& fw, const BwdWork& bw,
                          cudaStream_t st);

// Where cache row t of batch row b lives.  Dense caches: row b * cap + t of a
// [B, cap, ...] array.  Paged caches (block tables, as in PagedAttention): a
// pool of nblk blocks of bs rows; row t of batch row b is row t % bs of block
// bt[b * maxblk + t / bs] (clamped into the pool, so a bad table entry never
// addresses memory outside it).  Anchor chunks of C rows never straddle a
// block (bs is a multiple of C).
struct PageMap {
  const int* bt = nullptr;
  int maxblk = 0, bs = 0, nblk = 0;
  int cap = 0;
  __host__ __device__ bool paged() const { return bt != nullptr; }
  // rows a batch row can hold
  __host__ __device__ int rows() const { return bt ? maxblk * bs : cap; }
#ifdef __CUDACC__
  __device__ __forceinline__ int block_of(int b, int t) const {
    const int pb = __ldg(bt + static_cast<size_t>(b) * maxblk + t / bs);
    return pb < 0 ? 0 : (pb >= nblk ? nblk - 1 : pb);
  }
  __device__ __forceinline__ size_t row(int b, int t) const {
    if (!bt) return static_cast<size_t>(b) * cap + t;
    return static_cast<size_t>(block_of(b, t)) * bs + t % bs;
  }
  // anchor slot of the chunk holding row t
  __device__ __forceinline__ size_t chunk(int b, int t, int C) const {
    if (!bt) return static_cast<size_t>(b) * ((cap + C - 1) / C) + t / C;
    return static_cast<size_t>(block_of(b, t)) * (bs / C) + (t % bs) / C;
  }
#endif
};

struct CacheArgs {
  const void* k_new;
  const void* g_new;
  const float* p_prev;
  int B, t_start, T_new, cap, HQ, H, K, chunk;
  void* k_tilde;
  float* r_cache;
  float* p_last;
  int* err;          // device error word (bounded waits)
  uint64_t wait_ns;  // limit of each bounded wait
  int fault;         // testing hook: 3 = producer skips its first stage
  PageMap pm;        // paged cache (pm.bt set) or dense (pm.cap = cap)
};
cudaError_t launch_cache_build(const CacheArgs& a, bool bf16, cudaStream_t st);
// Scalar-gate cache: PS = prefix of g_scalar * log2(e) per (row, query head),
// rows t_start .. t_start + T_new - 1 (t_pos null) or one row per batch row at
// t_pos[b].  gcache [B, cap, HQ] (dense) or [nblk, bs, HQ] (paged) fp32.
struct GateArgs {
  const void* gs_new;     // [B, T_new, HQ] input dtype
  const float* gs_prev;   // [B, HQ] PS before the first new row (null at row 0)
  const int* t_pos;       // [B] or null
  int B, t_start, T_new, HQ;
  float* gcache;
  float* gs_last;         // [B, HQ] PS at the last new row
  PageMap pm;
};
cudaError_t launch_gate_cache(const GateArgs& a, bool bf16, cudaStream_t st);

// One token per batch row at row b's own position t_pos[b] (device int32 [B]).
cudaError_t launch_append_varlen(const CacheArgs& a, const int* t_pos, bool bf16, cudaStream_t st);

// A chunk of M new tokens at positions t0 .. t0 + M - 1 (chunked prefill,
// multi-token decode): append its keys to the dense cache, then its queries
// attend cache rows 0 .. t0 + i.  bf16 only.
struct ChunkArgs {
  const void* q;       // [B, M, HQ, K]
  const void* k_new;   // [B, M, H, K]
  const void* g_new;   // [B, M, HQ, K]
  const float* p_prev; // [B, HQ, K] P at row t0 - 1 (null iff t0 == 0)
  const float* sink;
  int window;
  int B, t0, M, cap, HQ, H, K, V, chunk;
  bool bf16;           // element type of q, k_new, g_new, gs_new, k_tilde, v_cache, o
  float scale;
  void* k_tilde;       // [B, cap, HQ, K]
  float* r_cache;      // [B, ceil(cap/chunk), HQ, K]
  float* p_last;       // [B, HQ, K]
  const void* v_cache; // [B, cap, H, V] (rows t0 .. t0 + M - 1 written by the caller)
  void* o;             // [B, M, HQ, V]
  float* lse;          // [B, M, HQ] or null
  void* workspace;
  int* err;
  uint64_t wait_ns;
  void* ev_mid = nullptr;  // optional event recorded before the attention kernel
  int fault = 0;           // testing hook: 6 = chunk tile kernel, 7 = few-token split kernel
  // scalar gate (null gs_new: none): the chunk's g_scalar [B, M, HQ] (input dtype), PS
  // at row t0 - 1 [B, HQ] (null iff t0 == 0), the gate cache [B, cap, HQ] (rows t0 ..
  // written here) and PS at the chunk's last row [B, HQ] (may alias gs_prev)
  const void* gs_new = nullptr;
  const float* gs_prev = nullptr;
  float* gs_cache = nullptr;
  float* gs_last = nullptr;
};
size_t chunk_workspace_bytes(int B, int M, int cap, int HQ, int H, int K, int V, int chunk,
                             bool bf16);
cudaError_t launch_chunk(const ChunkArgs& a, cudaStream_t st);
// Few-token bf16 chunks (M <= 2 * 16 / group) and fp32 chunks of any length
// attend through a split-KV pass in the decode's style instead of 128-row
// tensor-core query tiles (power-of-two groups).
bool chunk_split_applies(int M, int HQ, int H, bool bf16);
size_t chunk_split_part_bytes(int B, int M, int cap, int HQ, int H, int V, int chunk);
// The few-token split pass on the tensor cores (bf16, groups of 1, 2, 4 or 8):
// writes the same per-split partials as the SIMT pass.
template <int KD, int VD, int G>
cudaError_t launch_chunk_mma(const ChunkArgs& a, const void* qh, const float* AQ, const int* wide,
                             float* part, int ck_lo, int cps, int nsplit, int ntg,
                             cudaStream_t st);
cudaError_t launch_chunk_split(const ChunkArgs& a, const void* qh, const float* AQ,
                               const int* wide, float* lse, float* part, cudaStream_t st);
// The decode's split combine (merge per-split partials, add the sink).
cudaError_t launch_decode_combine(const float* part, int nsplit, int nbh, int HQ,
                                  const float* sink, void* o, float* lse, int V, bool bf16,
                                  cudaStream_t st);

// Append fused into the decode step: the new token's k, g, v (one per batch
// row) join the cache inside the decode kernel.  In this mode DecodeArgs'
// p_curr holds P of the previous row (p_prev) and the kernel writes P_last.
struct DecodeFuse {
  const void* k_new = nullptr;  // [B, H, K]
  const void* g_new = nullptr;  // [B, HQ, K]
  const void* v_new = nullptr;  // [B, H, V]
  float* p_last = nullptr;      // [B, HQ, K], must not overlap p_prev
  void* k_tilde = nullptr;      // the cache, written at each batch row's new row
  float* r_cache = nullptr;
  void* v = nullptr;
  // scalar gate (with DecodeArgs::gs_cache): the new token's g_scalar [B, HQ] (input
  // dtype), PS at the previous row [B, HQ] and PS at the new row (out, another buffer)
  const void* gs_new = nullptr;
  const float* gs_prev = nullptr;
  float* gs_last = nullptr;
};

struct DecodeArgs {
  const void* q;
  const float* p_curr;
  const void* v;
  const void* k_tilde;
  const float* r_cache;
  const float* sink;
  int B, T_kv, cap, HQ, H, K, V, chunk;
  float scale;
  void* o;
  float* lse;
  float* part;  // workspace
  int nsplit;
  void* mid_event;  // optional cudaEvent_t recorded between the split and combine kernels
  int* err;         // device error word
  uint64_t wait_ns; // bounded-wait limit
  int fault;        // testing hook: 2 = producer skips its first stage
  const int* seqlens = nullptr;  // optional device int32 [B]: rows of each batch row's cache
  PageMap pm;                    // paged cache (pm.bt set; seqlens required) or dense
  DecodeFuse fuse;               // fuse.k_new set: append the new row inside the decode
  const float* gs_cache = nullptr;  // scalar-gate cache (null: no gate) [B, cap, HQ] / pool
  const float* gs_curr = nullptr;   // [B, HQ] PS of the current row
};
int decode_max_splits(int B, int T_kv, int HQ, int H, int chunk);
int decode_num_splits(int B, int T_kv, int HQ, int H, int chunk, int ctas_per_sm = 1);
// CTAs of the decode's split pass resident on an SM: the tensor-core pass
// (bf16, groups of 1-8) runs several small CTAs, the SIMT pass one.
int decode_ctas_per_sm(int K, int V, int group, bool bf16);
size_t decode_workspace_bytes(int B, int HQ, int V, int nsplit);
bool decode_supported(int K, int V, int group);
cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st);
// The decode's split pass on the tensor cores (bf16, groups of 1, 2, 4 or 8):
// writes the same per-split partials as the SIMT split kernel (the combine
// is the caller's).
template <int KD, int VD, int G>
cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t st);

}  // namespace wall
