// C ABI of the Wall attention library: argument validation, workspace
// layout, TMA descriptor encoding and kernel launches.  Every public entry
// point validates everything it can on the host before queuing any work and
// reports problems as wall_status_t; nothing here aborts or synchronises
// (unless WALL_DEBUG_SYNC=1).
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "wall_attn.h"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace {

__device__ int g_wall_err;  // per-device error word (bit 0: a bounded wait gave up)

std::atomic<int> g_fault_mode{0};
std::atomic<int> g_wait_ms{2000};
std::atomic<void*> g_stage_ev[3] = {};

// Records the caller's profiling event `i` (if any) on `st`.
void stage_event(int i, cudaStream_t st) {
  void* e = g_stage_ev[i].load();
  if (e != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(e), st);
}

bool debug_sync() {
  static const bool on = [] {
    const char* s = std::getenv("WALL_DEBUG_SYNC");
    return s != nullptr && s[0] == '1';
  }();
  return on;
}

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
int* g_err_addr[kMaxDevices] = {};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

wall_status_t finish(cudaError_t e, cudaStream_t st) {
  if (e != cudaSuccess) return WALL_ERR_CUDA;
  if (debug_sync()) return wall_device_error(reinterpret_cast<wall_stream_t>(st));
  return WALL_OK;
}

bool supported_dim(int x) { return x == 64 || x == 128; }

}  // namespace

namespace wall {

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (g_err_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wall_err) != cudaSuccess) return nullptr;
    g_err_addr[dev] = static_cast<int*>(p);
  }
  return g_err_addr[dev];
}

uint64_t wait_limit_ns() { return static_cast<uint64_t>(g_wait_ms.load()) * 1000000ull; }
int fault_mode() { return g_fault_mode.load(); }

bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                  const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                  CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace wall

extern "C" {

const char* wall_status_string(wall_status_t s) {
  switch (s) {
    case WALL_OK: return "WALL_OK";
    case WALL_ERR_INVALID_ARG: return "WALL_ERR_INVALID_ARG: bad pointer, shape, size or alignment";
    case WALL_ERR_UNSUPPORTED: return "WALL_ERR_UNSUPPORTED: head dimension, group size or chunk not supported";
    case WALL_ERR_CUDA: return "WALL_ERR_CUDA: a CUDA call failed";
    case WALL_ERR_DEVICE_TIMEOUT: return "WALL_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
    case WALL_ERR_WORKSPACE: return "WALL_ERR_WORKSPACE: workspace too small";
    case WALL_ERR_RANGE:
      return "WALL_ERR_RANGE: decay within one anchor span exceeds the representable range";
  }
  return "WALL_ERR_UNKNOWN";
}

size_t wall_attn_fwd_workspace_size(int B, int T, int HQ, int H, int K, int V, wall_dtype_t dt) {
  (void)H;
  (void)V;
  if (B <= 0 || T <= 0 || HQ <= 0 || K <= 0) return 0;
  return wall::fwd_workspace_layout(B, T, HQ, K, dt == WALL_DTYPE_BF16, nullptr, nullptr);
}

}  // extern "C"

namespace {

// Decode cache outputs of wall_attn_fwd_with_cache (validated by the caller).
struct CacheOut {
  void* k_tilde;
  float* r_cache;
  float* p_last;
  int cap, chunk;
};

wall_status_t fwd_impl(const void* q, const void* k, const void* v, const void* g,
                       const void* g_scalar, const float* sink_bias, int window,
                       const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ, int H,
                       int K, int V, wall_dtype_t dt, float scale, void* o, float* lse,
                       void* workspace, size_t workspace_bytes, wall_stream_t stream,
                       const CacheOut* co) {
  if (B < 0 || T < 0 || HQ <= 0 || H <= 0 || HQ % H != 0) return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (!supported_dim(K) || !supported_dim(V)) return WALL_ERR_UNSUPPORTED;
  if (cu_seqlens != nullptr && (B != 1 || num_seqs < 1)) return WALL_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return WALL_OK;
  const size_t esz = dt == WALL_DTYPE_BF16 ? 2 : 4;
  if (!q || !k || !v || !g || !o || !workspace) return WALL_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
      !aligned(o, 16) || !aligned(workspace, 256))
    return WALL_ERR_INVALID_ARG;
  if ((g_scalar && !aligned(g_scalar, esz)) || (sink_bias && !aligned(sink_bias, 4)) ||
      (lse && !aligned(lse, 4)) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return WALL_ERR_INVALID_ARG;
  const long long NB = (static_cast<long long>(T) + wall::kBlockRows - 1) / wall::kBlockRows;
  if (NB * B * HQ > 0x7fffffffLL) return WALL_ERR_UNSUPPORTED;
  const bool bf16 = dt == WALL_DTYPE_BF16;
  const size_t need = wall::fwd_workspace_layout(B, T, HQ, K, bf16, nullptr, nullptr);
  if (workspace_bytes < need) return WALL_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.f / std::sqrt(static_cast<float>(K));

  int* err = wall::device_error_word();
  if (err == nullptr) return WALL_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  wall::FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.g_scalar = g_scalar; a.sink = sink_bias;
  a.cu_seqlens = cu_seqlens; a.num_seqs = num_seqs; a.window = window > 0 ? window : 0;
  a.B = B; a.T = T; a.HQ = HQ; a.H = H; a.K = K; a.V = V; a.NB = static_cast<int>(NB);
  a.scale = scale; a.o = o; a.lse = lse; a.err = err;
  a.wait_ns = wall::wait_limit_ns();
  a.fault = g_fault_mode.load();
  if (co != nullptr) {
    a.kt_out = co->k_tilde;
    a.r_out = co->r_cache;
    a.plast_out = co->p_last;
    a.cache_cap = co->cap;
    a.cache_chunk = co->chunk;
  }
  wall::FwdWork w;
  wall::fwd_workspace_layout(B, T, HQ, K, bf16, &w, static_cast<char*>(workspace));

  stage_event(0, st);
  cudaError_t e = wall::launch_prep(a, w, bf16, st);
  if (e != cudaSuccess) return WALL_ERR_CUDA;
  stage_event(1, st);
  if (!bf16) {
    e = wall::launch_fwd_simt(a, w, st);
    stage_event(2, st);
    if (e == cudaSuccess) e = wall::launch_fwd_diag(a, w, bf16, st);
    return finish(e, st);
  }

  CUtensorMap tmQ, tmK, tmV;
  {  // anchored q / k: [B*HQ][T][K], 64-channel x 128-row boxes, 128-byte swizzle
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(T),
                                static_cast<cuuint64_t>(B) * HQ};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2,
                                   static_cast<cuuint64_t>(T) * K * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!wall::encode_tiled(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.qh, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_128B) ||
        !wall::encode_tiled(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.kh, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_128B))
      return WALL_ERR_CUDA;
  }
  {  // v: [B, T, H, V], 64-channel x 128-row boxes, 128-byte swizzle
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(V), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(V) * 2,
                                   static_cast<cuuint64_t>(H) * V * 2,
                                   static_cast<cuuint64_t>(T) * H * V * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    if (!wall::encode_tiled(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_128B))
      return WALL_ERR_CUDA;
  }
  CUtensorMap tmKX = tmK;
  if (g_scalar != nullptr) {  // key-side gate channels: [B*HQ][T][16] bf16, 32-byte swizzle
    const cuuint64_t dims[3] = {16, static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B) * HQ};
    const cuuint64_t strides[2] = {32, static_cast<cuuint64_t>(T) * 32};
    const cuuint32_t box[3] = {16, 128, 1};
    if (!wall::encode_tiled(&tmKX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.kx, dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_32B))
      return WALL_ERR_CUDA;
  }
  e = wall::launch_fwd_tc(a, w, tmQ, tmK, tmV, tmKX, st);
  stage_event(2, st);
  if (e == cudaSuccess) e = wall::launch_fwd_diag(a, w, bf16, st);
  return finish(e, st);
}

}  // namespace

extern "C" {

wall_status_t wall_attn_fwd(const void* q, const void* k, const void* v, const void* g,
                            const void* g_scalar, const float* sink_bias, int window,
                            const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ, int H,
                            int K, int V, wall_dtype_t dt, float scale, void* o, float* lse,
                            void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  return fwd_impl(q, k, v, g, g_scalar, sink_bias, window, cu_seqlens, num_seqs, B, T, HQ, H, K,
                  V, dt, scale, o, lse, workspace, workspace_bytes, stream, nullptr);
}

wall_status_t wall_attn_fwd_with_cache(const void* q, const void* k, const void* v, const void* g,
                                       const void* g_scalar, const float* sink_bias, int window,
                                       int B, int T, int HQ, int H, int K, int V, wall_dtype_t dt,
                                       float scale, void* o, float* lse, void* workspace,
                                       size_t workspace_bytes, int cap, int chunk, void* k_tilde,
                                       float* r_cache, float* p_last, wall_stream_t stream) {
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (cap < T || cap < 0) return WALL_ERR_INVALID_ARG;
  if (B > 0 && T > 0) {
    if (!k_tilde || !r_cache || !p_last) return WALL_ERR_INVALID_ARG;
    if (!aligned(k_tilde, 16) || !aligned(r_cache, 16) || !aligned(p_last, 16))
      return WALL_ERR_INVALID_ARG;
  }
  const CacheOut co{k_tilde, r_cache, p_last, cap, chunk};
  return fwd_impl(q, k, v, g, g_scalar, sink_bias, window, nullptr, 0, B, T, HQ, H, K, V, dt,
                  scale, o, lse, workspace, workspace_bytes, stream, &co);
}

size_t wall_attn_bwd_workspace_size(int B, int T, int HQ, int H, int K, int V, wall_dtype_t dt) {
  (void)H;
  if (B <= 0 || T <= 0 || HQ <= 0 || K <= 0 || V <= 0) return 0;
  return wall::bwd_workspace_layout(B, T, HQ, K, V, dt == WALL_DTYPE_BF16, nullptr, nullptr,
                                    nullptr);
}

wall_status_t wall_attn_bwd(const void* q, const void* k, const void* v, const void* g,
                            const void* g_scalar, const float* sink_bias, int window,
                            const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ, int H,
                            int K, int V, wall_dtype_t dt, float scale, const void* o,
                            const float* lse, const void* dout, const float* dlse, void* dq,
                            void* dk, void* dv, void* dg, void* dg_scalar, float* dsink,
                            void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  if (B < 0 || T < 0 || HQ <= 0 || H <= 0 || HQ % H != 0) return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (!supported_dim(K) || !supported_dim(V)) return WALL_ERR_UNSUPPORTED;
  if (cu_seqlens != nullptr && (B != 1 || num_seqs < 1)) return WALL_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return WALL_OK;
  const size_t esz = dt == WALL_DTYPE_BF16 ? 2 : 4;
  if (!q || !k || !v || !g || !o || !lse || !dout || !dq || !dk || !dv || !dg || !workspace)
    return WALL_ERR_INVALID_ARG;
  if ((g_scalar == nullptr) != (dg_scalar == nullptr)) return WALL_ERR_INVALID_ARG;
  if ((sink_bias == nullptr) != (dsink == nullptr)) return WALL_ERR_INVALID_ARG;
  const void* a16[] = {q, k, v, g, o, dout, dq, dk, dv, dg};
  for (const void* p : a16)
    if (!aligned(p, 16)) return WALL_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(lse, 4) || (dlse && !aligned(dlse, 4)) ||
      (g_scalar && !aligned(g_scalar, esz)) || (dg_scalar && !aligned(dg_scalar, esz)) ||
      (sink_bias && !aligned(sink_bias, 4)) || (dsink && !aligned(dsink, 4)) ||
      (cu_seqlens && !aligned(cu_seqlens, 4)))
    return WALL_ERR_INVALID_ARG;
  const long long NB = (static_cast<long long>(T) + wall::kBlockRows - 1) / wall::kBlockRows;
  if (NB * B * HQ > 0x7fffffffLL || static_cast<long long>(B) * T * HQ > 0x3fffffffLL)
    return WALL_ERR_UNSUPPORTED;
  const bool bf16 = dt == WALL_DTYPE_BF16;
  const size_t need = wall::bwd_workspace_layout(B, T, HQ, K, V, bf16, nullptr, nullptr, nullptr);
  if (workspace_bytes < need) return WALL_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.f / std::sqrt(static_cast<float>(K));

  int* err = wall::device_error_word();
  if (err == nullptr) return WALL_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  wall::BwdArgs a;
  wall::FwdArgs& f = a.f;
  f.q = q; f.k = k; f.v = v; f.g = g; f.g_scalar = g_scalar; f.sink = sink_bias;
  f.cu_seqlens = cu_seqlens; f.num_seqs = num_seqs; f.window = window > 0 ? window : 0;
  f.B = B; f.T = T; f.HQ = HQ; f.H = H; f.K = K; f.V = V; f.NB = static_cast<int>(NB);
  f.scale = scale; f.o = const_cast<void*>(o); f.lse = const_cast<float*>(lse); f.err = err;
  f.wait_ns = wall::wait_limit_ns();
  f.fault = g_fault_mode.load();
  f.wide_is_error = true;  // the backward's tiles have no exact path for wide blocks yet
  a.dout = dout; a.dlse = dlse;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dg_scalar = dg_scalar; a.dsink = dsink;
  for (int i = 0; i < 3; ++i) a.ev[i] = g_stage_ev[i].load();
  wall::FwdWork fw;
  wall::BwdWork bw;
  wall::bwd_workspace_layout(B, T, HQ, K, V, bf16, &fw, &bw, static_cast<char*>(workspace));

  cudaError_t e = wall::launch_prep(f, fw, bf16, st);
  if (e != cudaSuccess) return WALL_ERR_CUDA;
  return finish(wall::launch_bwd(a, fw, bw, bf16, st), st);
}

static wall_status_t build_entry(const void* k_new, const void* g_new, const float* p_prev,
                                 int B, int t_start, int T_new, int cap, int HQ, int H, int K,
                                 int chunk, wall_dtype_t dt, void* k_tilde, float* r_cache,
                                 float* p_last, wall_stream_t stream, const wall::PageMap* pm) {
  if (B < 0 || t_start < 0 || T_new < 0 || cap < 0 || HQ <= 0 || H <= 0 || HQ % H != 0)
    return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (static_cast<long long>(t_start) + T_new > cap) return WALL_ERR_INVALID_ARG;
  if (!supported_dim(K)) return WALL_ERR_UNSUPPORTED;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (B == 0 || T_new == 0) return WALL_OK;
  if ((t_start > 0) != (p_prev != nullptr)) return WALL_ERR_INVALID_ARG;
  if (!k_new || !g_new || !k_tilde || !r_cache || !p_last) return WALL_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(g_new, 16) || !aligned(k_tilde, 16) ||
      !aligned(r_cache, 16) || !aligned(p_last, 16) || (p_prev && !aligned(p_prev, 16)))
    return WALL_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * HQ > 0x7fffffffLL) return WALL_ERR_UNSUPPORTED;
  wall::CacheArgs a;
  a.k_new = k_new; a.g_new = g_new; a.p_prev = p_prev;
  a.B = B; a.t_start = t_start; a.T_new = T_new; a.cap = cap; a.HQ = HQ; a.H = H; a.K = K;
  a.chunk = chunk; a.k_tilde = k_tilde; a.r_cache = r_cache; a.p_last = p_last;
  a.err = wall::device_error_word();
  if (a.err == nullptr) return WALL_ERR_CUDA;
  a.wait_ns = wall::wait_limit_ns();
  a.fault = wall::fault_mode();
  if (pm != nullptr) a.pm = *pm;
  a.pm.cap = cap;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(wall::launch_cache_build(a, dt == WALL_DTYPE_BF16, st), st);
}

wall_status_t wall_build_kv_cache(const void* k_new, const void* g_new, const float* p_prev,
                                  int B, int t_start, int T_new, int cap, int HQ, int H, int K,
                                  int chunk, wall_dtype_t dt, void* k_tilde, float* r_cache,
                                  float* p_last, wall_stream_t stream) {
  return build_entry(k_new, g_new, p_prev, B, t_start, T_new, cap, HQ, H, K, chunk, dt, k_tilde,
                     r_cache, p_last, stream, nullptr);
}

// Checks shared by the paged calls; fills *pm.  Returns WALL_OK or an error.
static wall_status_t page_map(const int32_t* block_table, int max_blocks, int num_blocks,
                              int block_size, int chunk, int B, wall::PageMap* pm) {
  if (max_blocks < 1 || num_blocks < 1 || block_size < 1) return WALL_ERR_INVALID_ARG;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (block_size % chunk != 0 || block_size > (1 << 20)) return WALL_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * block_size > 0x7fffffffLL ||
      static_cast<long long>(num_blocks) * block_size > 0x7fffffffLL ||
      static_cast<long long>(B) * max_blocks > 0x7fffffffLL)
    return WALL_ERR_UNSUPPORTED;
  if (B > 0 && (block_table == nullptr || !aligned(block_table, 4))) return WALL_ERR_INVALID_ARG;
  pm->bt = block_table;
  pm->maxblk = max_blocks;
  pm->bs = block_size;
  pm->nblk = num_blocks;
  return WALL_OK;
}

wall_status_t wall_build_kv_cache_paged(const void* k_new, const void* g_new,
                                        const float* p_prev, const int32_t* block_table,
                                        int max_blocks, int B, int t_start, int T_new,
                                        int num_blocks, int block_size, int HQ, int H, int K,
                                        int chunk, wall_dtype_t dt, void* k_tilde_pool,
                                        float* r_pool, float* p_last, wall_stream_t stream) {
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  return build_entry(k_new, g_new, p_prev, B, t_start, T_new, max_blocks * block_size, HQ, H, K,
                     chunk, dt, k_tilde_pool, r_pool, p_last, stream, &pm);
}

static wall_status_t append_entry(const void* k_new, const void* g_new, const float* p_prev,
                                  const int32_t* t_pos, int B, int cap, int HQ, int H, int K,
                                  int chunk, wall_dtype_t dt, void* k_tilde, float* r_cache,
                                  float* p_last, wall_stream_t stream, const wall::PageMap* pm) {
  if (B < 0 || cap < 1 || HQ <= 0 || H <= 0 || HQ % H != 0) return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (!supported_dim(K)) return WALL_ERR_UNSUPPORTED;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  if (!k_new || !g_new || !p_prev || !t_pos || !k_tilde || !r_cache || !p_last)
    return WALL_ERR_INVALID_ARG;
  const size_t esz = dt == WALL_DTYPE_BF16 ? 2 : 4;
  if (!aligned(k_new, 4 * esz) || !aligned(g_new, 4 * esz) || !aligned(k_tilde, 4 * esz) ||
      !aligned(r_cache, 16) || !aligned(p_last, 16) || !aligned(p_prev, 16) || !aligned(t_pos, 4))
    return WALL_ERR_INVALID_ARG;
  wall::CacheArgs a;
  a.k_new = k_new; a.g_new = g_new; a.p_prev = p_prev;
  a.B = B; a.t_start = 0; a.T_new = 1; a.cap = cap; a.HQ = HQ; a.H = H; a.K = K;
  a.chunk = chunk; a.k_tilde = k_tilde; a.r_cache = r_cache; a.p_last = p_last;
  a.err = wall::device_error_word(); a.wait_ns = 0; a.fault = 0;
  if (a.err == nullptr) return WALL_ERR_CUDA;
  if (pm != nullptr) a.pm = *pm;
  a.pm.cap = cap;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(wall::launch_append_varlen(a, t_pos, dt == WALL_DTYPE_BF16, st), st);
}

wall_status_t wall_append_kv_cache_varlen(const void* k_new, const void* g_new,
                                          const float* p_prev, const int32_t* t_pos, int B,
                                          int cap, int HQ, int H, int K, int chunk,
                                          wall_dtype_t dt, void* k_tilde, float* r_cache,
                                          float* p_last, wall_stream_t stream) {
  return append_entry(k_new, g_new, p_prev, t_pos, B, cap, HQ, H, K, chunk, dt, k_tilde, r_cache,
                      p_last, stream, nullptr);
}

wall_status_t wall_append_kv_cache_paged(const void* k_new, const void* g_new,
                                         const float* p_prev, const int32_t* t_pos,
                                         const int32_t* block_table, int max_blocks, int B,
                                         int num_blocks, int block_size, int HQ, int H, int K,
                                         int chunk, wall_dtype_t dt, void* k_tilde_pool,
                                         float* r_pool, float* p_last, wall_stream_t stream) {
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  return append_entry(k_new, g_new, p_prev, t_pos, B, max_blocks * block_size, HQ, H, K, chunk,
                      dt, k_tilde_pool, r_pool, p_last, stream, &pm);
}

size_t wall_attn_decode_workspace_size(int B, int T_kv, int HQ, int H, int V, int chunk) {
  if (B <= 0 || T_kv <= 0 || HQ <= 0 || H <= 0 || V <= 0 || chunk <= 0) return 0;
  const int ns = wall::decode_max_splits(B, T_kv, HQ, H, chunk);
  return wall::decode_workspace_bytes(B, HQ, V, ns);
}

static wall_status_t decode_entry(const void* q, const float* p_curr, const void* v,
                                  const void* k_tilde, const float* r_cache,
                                  const float* sink_bias, const int32_t* seqlens, int B, int T_kv,
                                  int cap, int HQ, int H, int K, int V, int chunk,
                                  wall_dtype_t dt, float scale, void* o, float* lse,
                                  void* workspace, size_t workspace_bytes, wall_stream_t stream,
                                  const wall::PageMap* pm = nullptr,
                                  const float* gs_cache = nullptr,
                                  const float* gs_curr = nullptr,
                                  const wall::DecodeFuse* fu = nullptr) {
  if (B < 0 || T_kv < 1 || cap < T_kv || HQ <= 0 || H <= 0 || HQ % H != 0)
    return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (!wall::decode_supported(K, V, HQ / H)) return WALL_ERR_UNSUPPORTED;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  if (!q || !p_curr || !v || !k_tilde || !r_cache || !o || !workspace) return WALL_ERR_INVALID_ARG;
  if (seqlens && !aligned(seqlens, 4)) return WALL_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(p_curr, 16) || !aligned(v, 16) || !aligned(k_tilde, 16) ||
      !aligned(r_cache, 16) || !aligned(o, 16) || !aligned(workspace, 16) ||
      (sink_bias && !aligned(sink_bias, 4)) || (lse && !aligned(lse, 4)))
    return WALL_ERR_INVALID_ARG;
  if (fu != nullptr) {
    if (!fu->k_new || !fu->g_new || !fu->v_new || !fu->p_last || !aligned(fu->k_new, 16) ||
        !aligned(fu->g_new, 16) || !aligned(fu->v_new, 16) || !aligned(fu->p_last, 16))
      return WALL_ERR_INVALID_ARG;
    // other CTAs read p_prev while the one holding a row's new token writes P_last
    const size_t pb = static_cast<size_t>(B) * HQ * K * sizeof(float);
    const char* a0 = reinterpret_cast<const char*>(p_curr);
    const char* a1 = reinterpret_cast<const char*>(fu->p_last);
    if (a0 < a1 + pb && a1 < a0 + pb) return WALL_ERR_INVALID_ARG;
    if (gs_cache != nullptr) {  // gated step: the new token's g_scalar, PS in and out
      if (!fu->gs_new || !fu->gs_last || (T_kv > 1 && !fu->gs_prev) || !aligned(fu->gs_last, 4) ||
          (fu->gs_prev && !aligned(fu->gs_prev, 4)))
        return WALL_ERR_INVALID_ARG;
      const size_t gb = static_cast<size_t>(B) * HQ * sizeof(float);
      const char* g0 = reinterpret_cast<const char*>(fu->gs_prev);
      const char* g1 = reinterpret_cast<const char*>(fu->gs_last);
      if (g0 != nullptr && g0 < g1 + gb && g1 < g0 + gb) return WALL_ERR_INVALID_ARG;
    }
  }
  const int ns = wall::decode_num_splits(
      B, T_kv, HQ, H, chunk, wall::decode_ctas_per_sm(K, V, HQ / H, dt == WALL_DTYPE_BF16));
  if (workspace_bytes < wall::decode_workspace_bytes(B, HQ, V, ns)) return WALL_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.f / std::sqrt(static_cast<float>(K));
  wall::DecodeArgs a;
  a.q = q; a.p_curr = p_curr; a.v = v; a.k_tilde = k_tilde; a.r_cache = r_cache;
  a.sink = sink_bias; a.B = B; a.T_kv = T_kv; a.cap = cap; a.HQ = HQ; a.H = H; a.K = K;
  a.V = V; a.chunk = chunk; a.scale = scale; a.o = o; a.lse = lse;
  a.part = static_cast<float*>(workspace); a.nsplit = ns;
  a.mid_event = g_stage_ev[1].load();
  a.err = wall::device_error_word();
  if (a.err == nullptr) return WALL_ERR_CUDA;
  a.wait_ns = wall::wait_limit_ns();
  a.fault = wall::fault_mode();
  a.seqlens = seqlens;
  if (pm != nullptr) a.pm = *pm;
  a.pm.cap = cap;
  a.gs_cache = gs_cache;
  a.gs_curr = gs_curr;
  if (fu != nullptr) a.fuse = *fu;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  stage_event(0, st);
  const cudaError_t e = wall::launch_decode(a, dt == WALL_DTYPE_BF16, st);
  stage_event(2, st);
  return finish(e, st);
}

wall_status_t wall_attn_decode(const void* q, const float* p_curr, const void* v,
                               const void* k_tilde, const float* r_cache, const float* sink_bias,
                               int B, int T_kv, int cap, int HQ, int H, int K, int V, int chunk,
                               wall_dtype_t dt, float scale, void* o, float* lse, void* workspace,
                               size_t workspace_bytes, wall_stream_t stream) {
  return decode_entry(q, p_curr, v, k_tilde, r_cache, sink_bias, nullptr, B, T_kv, cap, HQ, H, K,
                      V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream);
}

wall_status_t wall_attn_decode_varlen(const void* q, const float* p_curr, const void* v,
                                      const void* k_tilde, const float* r_cache,
                                      const float* sink_bias, const int32_t* seqlens_kv, int B,
                                      int max_T_kv, int cap, int HQ, int H, int K, int V,
                                      int chunk, wall_dtype_t dt, float scale, void* o,
                                      float* lse, void* workspace, size_t workspace_bytes,
                                      wall_stream_t stream) {
  if (B > 0 && seqlens_kv == nullptr) return WALL_ERR_INVALID_ARG;
  return decode_entry(q, p_curr, v, k_tilde, r_cache, sink_bias, seqlens_kv, B, max_T_kv, cap, HQ,
                      H, K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream);
}

wall_status_t wall_attn_decode_paged(const void* q, const float* p_curr, const void* v_pool,
                                     const void* k_tilde_pool, const float* r_pool,
                                     const float* sink_bias, const int32_t* seqlens_kv,
                                     const int32_t* block_table, int max_blocks, int B,
                                     int num_blocks, int block_size, int HQ, int H, int K, int V,
                                     int chunk, wall_dtype_t dt, float scale, void* o, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     wall_stream_t stream) {
  if (B > 0 && seqlens_kv == nullptr) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  const int rows = max_blocks * block_size;
  return decode_entry(q, p_curr, v_pool, k_tilde_pool, r_pool, sink_bias, seqlens_kv, B, rows,
                      rows, HQ, H, K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes,
                      stream, &pm);
}

wall_status_t wall_attn_decode_step(const void* q, const void* k_new, const void* g_new,
                                    const void* v_new, const float* p_prev, float* p_last,
                                    const float* sink_bias, const int32_t* seqlens_kv,
                                    const int32_t* block_table, int max_blocks, int num_blocks,
                                    int block_size, int B, int T_kv, int cap, int HQ, int H,
                                    int K, int V, int chunk, wall_dtype_t dt, float scale,
                                    void* k_tilde, float* r_cache, void* v_cache, void* o,
                                    float* lse, void* workspace, size_t workspace_bytes,
                                    wall_stream_t stream) {
  wall::DecodeFuse fu;
  fu.k_new = k_new; fu.g_new = g_new; fu.v_new = v_new; fu.p_last = p_last;
  fu.k_tilde = k_tilde; fu.r_cache = r_cache; fu.v = v_cache;
  if (block_table == nullptr)
    return decode_entry(q, p_prev, v_cache, k_tilde, r_cache, sink_bias, seqlens_kv, B, T_kv, cap,
                        HQ, H, K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream,
                        nullptr, nullptr, nullptr, &fu);
  if (B > 0 && seqlens_kv == nullptr) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  const int rows = max_blocks * block_size;
  (void)cap;
  return decode_entry(q, p_prev, v_cache, k_tilde, r_cache, sink_bias, seqlens_kv, B,
                      T_kv < rows ? T_kv : rows, rows, HQ, H, K, V, chunk, dt, scale, o, lse,
                      workspace, workspace_bytes, stream, &pm, nullptr, nullptr, &fu);
}

wall_status_t wall_attn_decode_step_gated(
    const void* q, const void* k_new, const void* g_new, const void* v_new, const void* gs_new,
    const float* p_prev, float* p_last, const float* gs_prev, float* gs_last, float* gs_cache,
    const float* sink_bias, const int32_t* seqlens_kv, const int32_t* block_table, int max_blocks,
    int num_blocks, int block_size, int B, int T_kv, int cap, int HQ, int H, int K, int V,
    int chunk, wall_dtype_t dt, float scale, void* k_tilde, float* r_cache, void* v_cache,
    void* o, float* lse, void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  if (B > 0 && (gs_cache == nullptr || gs_new == nullptr || !aligned(gs_cache, 4)))
    return WALL_ERR_INVALID_ARG;
  wall::DecodeFuse fu;
  fu.k_new = k_new; fu.g_new = g_new; fu.v_new = v_new; fu.p_last = p_last;
  fu.k_tilde = k_tilde; fu.r_cache = r_cache; fu.v = v_cache;
  fu.gs_new = gs_new; fu.gs_prev = gs_prev; fu.gs_last = gs_last;
  if (block_table == nullptr)
    return decode_entry(q, p_prev, v_cache, k_tilde, r_cache, sink_bias, seqlens_kv, B, T_kv, cap,
                        HQ, H, K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream,
                        nullptr, gs_cache, nullptr, &fu);
  if (B > 0 && seqlens_kv == nullptr) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  const int rows = max_blocks * block_size;
  (void)cap;
  return decode_entry(q, p_prev, v_cache, k_tilde, r_cache, sink_bias, seqlens_kv, B,
                      T_kv < rows ? T_kv : rows, rows, HQ, H, K, V, chunk, dt, scale, o, lse,
                      workspace, workspace_bytes, stream, &pm, gs_cache, nullptr, &fu);
}

// Gate cache entries: dense when block_table is NULL (gs_cache [B, cap, HQ]),
// paged otherwise (gs_cache [num_blocks, block_size, HQ]).
static wall_status_t gate_map(const int32_t* block_table, int max_blocks, int num_blocks,
                              int block_size, int B, int cap, wall::PageMap* pm) {
  if (block_table == nullptr) {
    if (cap < 1) return WALL_ERR_INVALID_ARG;
    pm->cap = cap;
    return WALL_OK;
  }
  // any block size works for the gate cache (one value per row and head)
  if (max_blocks < 1 || num_blocks < 1 || block_size < 1) return WALL_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks) * block_size > 0x7fffffffLL ||
      static_cast<long long>(num_blocks) * block_size > 0x7fffffffLL)
    return WALL_ERR_UNSUPPORTED;
  if (!aligned(block_table, 4)) return WALL_ERR_INVALID_ARG;
  pm->bt = block_table;
  pm->maxblk = max_blocks;
  pm->bs = block_size;
  pm->nblk = num_blocks;
  pm->cap = max_blocks * block_size;
  (void)B;
  return WALL_OK;
}

wall_status_t wall_build_gate_cache(const void* gs_new, const float* gs_prev,
                                    const int32_t* block_table, int max_blocks, int num_blocks,
                                    int block_size, int B, int t_start, int T_new, int cap, int HQ,
                                    wall_dtype_t dt, float* gs_cache, float* gs_last,
                                    wall_stream_t stream) {
  if (B < 0 || t_start < 0 || T_new < 0 || HQ <= 0) return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = gate_map(block_table, max_blocks, num_blocks, block_size, B, cap, &pm);
  if (ps != WALL_OK) return ps;
  if (static_cast<long long>(t_start) + T_new > pm.rows()) return WALL_ERR_INVALID_ARG;
  if (B == 0 || T_new == 0) return WALL_OK;
  if ((t_start > 0) != (gs_prev != nullptr)) return WALL_ERR_INVALID_ARG;
  if (!gs_new || !gs_cache || !gs_last) return WALL_ERR_INVALID_ARG;
  if (!aligned(gs_cache, 4) || !aligned(gs_last, 4) || (gs_prev && !aligned(gs_prev, 4)) ||
      !aligned(gs_new, dt == WALL_DTYPE_BF16 ? 2 : 4))
    return WALL_ERR_INVALID_ARG;
  if (B > 65535) return WALL_ERR_UNSUPPORTED;
  wall::GateArgs a;
  a.gs_new = gs_new; a.gs_prev = gs_prev; a.t_pos = nullptr;
  a.B = B; a.t_start = t_start; a.T_new = T_new; a.HQ = HQ;
  a.gcache = gs_cache; a.gs_last = gs_last; a.pm = pm;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(wall::launch_gate_cache(a, dt == WALL_DTYPE_BF16, st), st);
}

wall_status_t wall_append_gate_cache(const void* gs_new, const float* gs_prev,
                                     const int32_t* t_pos, const int32_t* block_table,
                                     int max_blocks, int num_blocks, int block_size, int B,
                                     int cap, int HQ, wall_dtype_t dt, float* gs_cache,
                                     float* gs_last, wall_stream_t stream) {
  if (B < 0 || HQ <= 0) return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = gate_map(block_table, max_blocks, num_blocks, block_size, B, cap, &pm);
  if (ps != WALL_OK) return ps;
  if (B == 0) return WALL_OK;
  if (!gs_new || !gs_prev || !t_pos || !gs_cache || !gs_last) return WALL_ERR_INVALID_ARG;
  if (!aligned(gs_cache, 4) || !aligned(gs_last, 4) || !aligned(gs_prev, 4) ||
      !aligned(t_pos, 4) || !aligned(gs_new, dt == WALL_DTYPE_BF16 ? 2 : 4))
    return WALL_ERR_INVALID_ARG;
  wall::GateArgs a;
  a.gs_new = gs_new; a.gs_prev = gs_prev; a.t_pos = t_pos;
  a.B = B; a.t_start = 0; a.T_new = 1; a.HQ = HQ;
  a.gcache = gs_cache; a.gs_last = gs_last; a.pm = pm;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(wall::launch_gate_cache(a, dt == WALL_DTYPE_BF16, st), st);
}

wall_status_t wall_attn_decode_gated(const void* q, const float* p_curr, const float* gs_curr,
                                     const void* v, const void* k_tilde, const float* r_cache,
                                     const float* gs_cache, const float* sink_bias,
                                     const int32_t* seqlens_kv, const int32_t* block_table,
                                     int max_blocks, int num_blocks, int block_size, int B,
                                     int T_kv, int cap, int HQ, int H, int K, int V, int chunk,
                                     wall_dtype_t dt, float scale, void* o, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     wall_stream_t stream) {
  if (B > 0 && (gs_curr == nullptr || gs_cache == nullptr)) return WALL_ERR_INVALID_ARG;
  if (B > 0 && (!aligned(gs_curr, 4) || !aligned(gs_cache, 4))) return WALL_ERR_INVALID_ARG;
  if (block_table == nullptr) {
    return decode_entry(q, p_curr, v, k_tilde, r_cache, sink_bias, seqlens_kv, B, T_kv, cap, HQ,
                        H, K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream,
                        nullptr, gs_cache, gs_curr);
  }
  if (B > 0 && seqlens_kv == nullptr) return WALL_ERR_INVALID_ARG;
  wall::PageMap pm;
  const wall_status_t ps = page_map(block_table, max_blocks, num_blocks, block_size, chunk, B, &pm);
  if (ps != WALL_OK) return ps;
  const int rows = max_blocks * block_size;
  return decode_entry(q, p_curr, v, k_tilde, r_cache, sink_bias, seqlens_kv, B, rows, rows, HQ, H,
                      K, V, chunk, dt, scale, o, lse, workspace, workspace_bytes, stream, &pm,
                      gs_cache, gs_curr);
}

size_t wall_attn_chunk_workspace_size(int B, int M, int cap, int HQ, int H, int K, int V,
                                      int chunk, wall_dtype_t dt) {
  if (B <= 0 || M <= 0 || cap <= 0 || HQ <= 0 || H <= 0 || HQ % H != 0 || K <= 0 || V <= 0 ||
      chunk <= 0)
    return 0;
  return wall::chunk_workspace_bytes(B, M, cap, HQ, H, K, V, chunk, dt != WALL_DTYPE_F32);
}

static wall_status_t chunk_impl(const void* q, const void* k_new, const void* g_new,
                              const float* p_prev, const float* sink_bias, int window, int B,
                              int t_start, int M, int cap, int HQ, int H, int K, int V, int chunk,
                              wall_dtype_t dt, float scale, void* k_tilde, float* r_cache,
                              float* p_last, const void* v_cache, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, wall_stream_t stream,
                              const void* gs_new, const float* gs_prev, float* gs_cache,
                              float* gs_last) {
  if (B < 0 || t_start < 0 || M < 0 || cap < 0 || HQ <= 0 || H <= 0 || HQ % H != 0)
    return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  const bool bf16 = dt == WALL_DTYPE_BF16;
  if (!supported_dim(K) || !supported_dim(V)) return WALL_ERR_UNSUPPORTED;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (static_cast<long long>(t_start) + M > cap) return WALL_ERR_INVALID_ARG;
  if (B == 0 || M == 0) return WALL_OK;
  // fp32 chunks take the split-KV pass: power-of-two groups, B * M * HQ rows in an int
  if (!bf16 && (!wall::chunk_split_applies(M, HQ, H, false) ||
                static_cast<long long>(B) * M * HQ > 0x7fffffffLL))
    return WALL_ERR_UNSUPPORTED;
  if ((t_start > 0) != (p_prev != nullptr)) return WALL_ERR_INVALID_ARG;
  if (gs_new != nullptr) {  // scalar gate: g_scalar of the chunk, PS in and out, gate cache
    if (!gs_cache || !gs_last || (t_start > 0) != (gs_prev != nullptr) ||
        !aligned(gs_new, bf16 ? 2 : 4) || !aligned(gs_cache, 4) || !aligned(gs_last, 4) ||
        (gs_prev && !aligned(gs_prev, 4)))
      return WALL_ERR_INVALID_ARG;
  }
  const void* a16[] = {q, k_new, g_new, k_tilde, r_cache, p_last, v_cache, o, workspace};
  for (const void* ptr : a16)
    if (ptr == nullptr || !aligned(ptr, 16)) return WALL_ERR_INVALID_ARG;
  if ((p_prev && !aligned(p_prev, 16)) || (sink_bias && !aligned(sink_bias, 4)) ||
      (lse && !aligned(lse, 4)) || !aligned(workspace, 256))
    return WALL_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * HQ * ((M + 255) / 256) > 0x7fffffffLL || B > 65535)
    return WALL_ERR_UNSUPPORTED;
  if (workspace_bytes < wall::chunk_workspace_bytes(B, M, cap, HQ, H, K, V, chunk, bf16))
    return WALL_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.f / std::sqrt(static_cast<float>(K));
  wall::ChunkArgs a;
  a.q = q; a.k_new = k_new; a.g_new = g_new; a.p_prev = p_prev; a.sink = sink_bias;
  a.window = window > 0 ? window : 0;
  a.B = B; a.t0 = t_start; a.M = M; a.cap = cap; a.HQ = HQ; a.H = H; a.K = K; a.V = V;
  a.chunk = chunk; a.bf16 = bf16; a.scale = scale; a.k_tilde = k_tilde; a.r_cache = r_cache; a.p_last = p_last;
  a.v_cache = v_cache; a.o = o; a.lse = lse; a.workspace = workspace;
  a.fault = wall::fault_mode();
  a.gs_new = gs_new; a.gs_prev = gs_prev; a.gs_cache = gs_cache; a.gs_last = gs_last;
  a.err = wall::device_error_word();
  if (a.err == nullptr) return WALL_ERR_CUDA;
  a.wait_ns = wall::wait_limit_ns();
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  stage_event(0, st);
  a.ev_mid = g_stage_ev[1].load();
  const cudaError_t e = wall::launch_chunk(a, st);
  stage_event(2, st);
  return finish(e, st);
}

wall_status_t wall_attn_chunk(const void* q, const void* k_new, const void* g_new,
                              const float* p_prev, const float* sink_bias, int window, int B,
                              int t_start, int M, int cap, int HQ, int H, int K, int V, int chunk,
                              wall_dtype_t dt, float scale, void* k_tilde, float* r_cache,
                              float* p_last, const void* v_cache, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, wall_stream_t stream) {
  return chunk_impl(q, k_new, g_new, p_prev, sink_bias, window, B, t_start, M, cap, HQ, H, K, V,
                    chunk, dt, scale, k_tilde, r_cache, p_last, v_cache, o, lse, workspace,
                    workspace_bytes, stream, nullptr, nullptr, nullptr, nullptr);
}

wall_status_t wall_attn_chunk_gated(const void* q, const void* k_new, const void* g_new,
                                    const void* gs_new, const float* p_prev, const float* gs_prev,
                                    const float* sink_bias, int window, int B, int t_start, int M,
                                    int cap, int HQ, int H, int K, int V, int chunk,
                                    wall_dtype_t dt, float scale, void* k_tilde, float* r_cache,
                                    float* p_last, float* gs_cache, float* gs_last,
                                    const void* v_cache, void* o, float* lse, void* workspace,
                                    size_t workspace_bytes, wall_stream_t stream) {
  if (B > 0 && M > 0 && gs_new == nullptr) return WALL_ERR_INVALID_ARG;
  return chunk_impl(q, k_new, g_new, p_prev, sink_bias, window, B, t_start, M, cap, HQ, H, K, V,
                    chunk, dt, scale, k_tilde, r_cache, p_last, v_cache, o, lse, workspace,
                    workspace_bytes, stream, gs_new, gs_prev, gs_cache, gs_last);
}

wall_status_t wall_device_error(wall_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return WALL_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_wall_err, sizeof(int)) != cudaSuccess) return WALL_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_wall_err, &zero, sizeof(int)) != cudaSuccess) return WALL_ERR_CUDA;
    return (h & wall::kDevErrTimeout) ? WALL_ERR_DEVICE_TIMEOUT : WALL_ERR_RANGE;
  }
  return WALL_OK;
}

void wall_debug_set_stage_events(void* before, void* between, void* after) {
  g_stage_ev[0].store(before);
  g_stage_ev[1].store(between);
  g_stage_ev[2].store(after);
}

void wall_debug_set_fault(int mode, int wait_ms) {
  g_fault_mode.store(mode);
  g_wait_ms.store(wait_ms > 0 ? wait_ms : 2000);
}

}  // extern "C"
