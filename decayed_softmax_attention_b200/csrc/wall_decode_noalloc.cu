// wall_attn_decode_noalloc: the split-KV decode of wall_attn_decode, for
// callers that cannot hand the library any scratch memory.
//
// The split pass writes one (o, max, sum) partial per (batch, query head,
// split) and the combine pass reads them back.  Here those partials live in a
// fixed, file-scope device array (kScratchBytes per device, reserved when the
// library is loaded and held until the process exits) instead of a
// caller-provided workspace, so the call allocates nothing.  Host code only
// knows the array by its symbol: its device address is looked up once per
// device with cudaGetSymbolAddress and passed to the kernels as a pointer.
#include <mutex>

#include "wall_attn.h"
#include "wall_common.cuh"
#include "wall_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB of split partials per device
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);

static __device__ __align__(256) float g_decode_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
wall_status_t scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WALL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return WALL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return WALL_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return WALL_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" wall_status_t wall_attn_decode_noalloc(
    const void* q, const float* p_curr, const void* v, const void* k_tilde, const float* r_cache,
    const float* sink_bias, int B, int T_kv, int cap, int HQ, int H, int K, int V, int chunk,
    wall_dtype_t dt, float scale, void* o, float* lse, wall_stream_t stream) {
  if (B < 0 || T_kv < 1 || cap < T_kv || HQ <= 0 || H <= 0 || HQ % H != 0)
    return WALL_ERR_INVALID_ARG;
  if (dt != WALL_DTYPE_F32 && dt != WALL_DTYPE_BF16) return WALL_ERR_INVALID_ARG;
  if (!wall::decode_supported(K, V, HQ / H)) return WALL_ERR_UNSUPPORTED;
  if (chunk != 32 && chunk != 64 && chunk != 128) return WALL_ERR_UNSUPPORTED;
  if (B == 0) return WALL_OK;
  if (!q || !p_curr || !v || !k_tilde || !r_cache || !o) return WALL_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(p_curr, 16) || !aligned(v, 16) || !aligned(k_tilde, 16) ||
      !aligned(r_cache, 16) || !aligned(o, 16) || (sink_bias && !aligned(sink_bias, 4)) ||
      (lse && !aligned(lse, 4)))
    return WALL_ERR_INVALID_ARG;

  // Split count: as wall_attn_decode chooses it, but never more splits than the
  // fixed scratch holds.  Beyond one split per (batch, query head) it cannot run.
  const size_t per_split = static_cast<size_t>(B) * HQ * (V + 2);
  const size_t fit = kScratchFloats / per_split;
  if (fit < 1) return WALL_ERR_WORKSPACE;
  const int nchunks = (T_kv + chunk - 1) / chunk;
  int ns = wall::decode_num_splits(B, T_kv, HQ, H, chunk,
                                   wall::decode_ctas_per_sm(K, V, HQ / H, dt == WALL_DTYPE_BF16));
  if (static_cast<size_t>(ns) > fit) {
    const int capped = static_cast<int>(fit);
    const int cps = (nchunks + capped - 1) / capped;
    ns = (nchunks + cps - 1) / cps;
  }

  float* scratch = nullptr;
  const wall_status_t s = scratch_address(&scratch);
  if (s != WALL_OK) return s;
  if (!(scale > 0.f) || !(scale < INFINITY)) scale = 1.f / sqrtf(static_cast<float>(K));

  wall::DecodeArgs a;
  a.q = q; a.p_curr = p_curr; a.v = v; a.k_tilde = k_tilde; a.r_cache = r_cache;
  a.sink = sink_bias; a.B = B; a.T_kv = T_kv; a.cap = cap; a.HQ = HQ; a.H = H; a.K = K;
  a.pm.cap = cap;
  a.V = V; a.chunk = chunk; a.scale = scale; a.o = o; a.lse = lse;
  a.part = scratch; a.nsplit = ns; a.mid_event = nullptr;
  a.err = wall::device_error_word();
  if (a.err == nullptr) return WALL_ERR_CUDA;
  a.wait_ns = wall::wait_limit_ns();
  a.fault = wall::fault_mode();
  const cudaError_t e = wall::launch_decode(a, dt == WALL_DTYPE_BF16,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WALL_OK : WALL_ERR_CUDA;
}
