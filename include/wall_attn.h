/*
 * wall_attn.h -- C ABI of the B200 (sm_100a) Wall attention library.
 *
 * Wall attention ("decayed softmax attention") scores a query/key pair (i, j)
 * by the q.k dot product in which every channel n carries the learned decay
 * accumulated between the two positions (Wall Attention README, intro):
 *
 *   x(i,j) = scale * sum_n q[i,n] k[j,n] exp(G[i,n] - G[j,n]) + Gs[i] - Gs[j]
 *
 * with G the inclusive cumulative sum of the per-channel log-decay g over
 * time and Gs that of the optional scalar gate g_scalar.  Softmax runs over
 * the admitted keys j <= i (plus an optional sink logit); g = 0 gives vanilla
 * causal softmax attention.
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, last dimension contiguous, in DEVICE
 *     memory, and owned by the caller.  The library never allocates, frees or
 *     synchronises (except when the environment variable WALL_DEBUG_SYNC=1 is
 *     set, which makes every call synchronise and report device errors).
 *   - Every call is asynchronous on `stream` (NULL = the legacy default stream)
 *     and is reentrant; the only global mutable state is the per-device
 *     error word read by wall_device_error().
 *   - Element types: `wall_dtype_t` selects bf16 or fp32 for q, k, v, g,
 *     g_scalar, o and k_tilde; sink_bias, lse, p_prev/p_last/p_curr and
 *     r_cache are always fp32.
 *   - Supported head dims: K, V in {64, 128}; HQ % H == 0 (GQA: query head hq
 *     reads KV head hq / (HQ / H)).  Anything else: WALL_ERR_UNSUPPORTED.
 *   - Pointers must be 16-byte aligned; a misaligned or NULL required pointer,
 *     a negative size or an inconsistent shape returns WALL_ERR_INVALID_ARG
 *     before any work is queued.  Errors never abort the process; there is no
 *     CPU fallback.
 */
#ifndef WALL_ATTN_H_
#define WALL_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the driver's opaque stream struct). */
struct CUstream_st;
typedef struct CUstream_st* wall_stream_t;

typedef enum {
  WALL_OK = 0,
  WALL_ERR_INVALID_ARG = 1,    /* bad pointer, shape, size or alignment */
  WALL_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. K = 96) */
  WALL_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed */
  WALL_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait gave up */
  WALL_ERR_WORKSPACE = 5,      /* workspace too small */
  WALL_ERR_RANGE = 6           /* decay too strong for a decode cache chunk, or (backward)
                                  for the anchored tiles: see wall_device_error */
} wall_status_t;

typedef enum { WALL_DTYPE_F32 = 0, WALL_DTYPE_BF16 = 1 } wall_dtype_t;

/* Human-readable name of a status code (static string). */
const char* wall_status_string(wall_status_t status);

/*
 * Prefill forward (Wall Attention README, "Usage / Training-Prefill"):
 *   o = wall_attn(q, k, v, g, scale, g_scalar, sink_bias, window_size, cu_seqlens)
 *
 *   q         [B, T, HQ, K]  dtype dt
 *   k         [B, T, H,  K]  dtype dt
 *   v         [B, T, H,  V]  dtype dt
 *   g         [B, T, HQ, K]  dtype dt  per-channel log-decay (natural log)
 *   g_scalar  [B, T, HQ]     dtype dt  nullable; additive FoX-style gate: the
 *                                      logit gains Gs[i] - Gs[j]
 *   sink_bias [HQ]           fp32      nullable; one extra logit per head with
 *                                      a zero value (adds to the normaliser)
 *   window    keep keys with 0 <= i - j < window; window <= 0: no window
 *   cu_seqlens int32 [num_seqs + 1] device, nullable; variable-length packing
 *             (requires B == 1): cu[0] = 0, cu[num_seqs] = T, strictly
 *             increasing; attention never crosses a document boundary and the
 *             cumulative sums restart at each document.  The values are read
 *             on the device only; out-of-range values are clamped, never
 *             dereferenced out of bounds, but give unspecified results.
 *   scale     softmax scale on the decayed q.k sum; <= 0 means K^-0.5
 *   o         [B, T, HQ, V]  dtype dt  output
 *   lse       [B, T, HQ]     fp32      nullable; natural-log normaliser,
 *                                      sink included
 *   workspace caller-owned device scratch of at least
 *             wall_attn_fwd_workspace_size(...) bytes, 256-byte aligned; its
 *             contents need no initialisation and are clobbered.
 * T == 0 (or B == 0) is a no-op returning WALL_OK.
 */
size_t wall_attn_fwd_workspace_size(int B, int T, int HQ, int H, int K, int V,
                                    wall_dtype_t dt);

wall_status_t wall_attn_fwd(const void* q, const void* k, const void* v, const void* g,
                            const void* g_scalar, const float* sink_bias, int window,
                            const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ,
                            int H, int K, int V, wall_dtype_t dt, float scale, void* o,
                            float* lse, void* workspace, size_t workspace_bytes,
                            wall_stream_t stream);

/*
 * Prefill forward that also emits the decode cache of its rows (Wall Attention
 * README, "Decode": the cache the decode path attends over, built here as a
 * side output of the prefill prepass instead of a separate
 * wall_build_kv_cache pass).  Same arguments and results as wall_attn_fwd,
 * without packed documents (one sequence per batch row), plus:
 *   cap      rows of the cache (>= T); chunk in {32, 64, 128}
 *   k_tilde  [B, cap, HQ, K] dtype dt   out: rows 0 .. T-1 (others untouched)
 *   r_cache  [B, ceil(cap/chunk), HQ, K] fp32  out: anchors of chunks starting below T
 *   p_last   [B, HQ, K] fp32            out: P at row T-1
 * The result equals wall_build_kv_cache(k, g, NULL, B, 0, T, cap, ...) up to
 * fp32 rounding; further tokens are appended with wall_build_kv_cache
 * (t_start = T, p_prev = p_last).  All three pointers 16-byte aligned.
 */
wall_status_t wall_attn_fwd_with_cache(const void* q, const void* k, const void* v, const void* g,
                                       const void* g_scalar, const float* sink_bias, int window,
                                       int B, int T, int HQ, int H, int K, int V, wall_dtype_t dt,
                                       float scale, void* o, float* lse, void* workspace,
                                       size_t workspace_bytes, int cap, int chunk, void* k_tilde,
                                       float* r_cache, float* p_last, wall_stream_t stream);

/*
 * Prefill backward (Wall Attention README, intro formula and "Usage /
 * Training-Prefill"; its "code structure" section names the backward pass):
 * the gradients of a loss L through o (and, optionally, lse) of
 * wall_attn_fwd with respect to every input.  Same inputs and shapes as
 * wall_attn_fwd, plus
 *   o         [B, T, HQ, V]  dtype dt  the forward's output for these inputs
 *   lse       [B, T, HQ]     fp32      the forward's lse (required)
 *   dout      [B, T, HQ, V]  dtype dt  dL/do
 *   dlse      [B, T, HQ]     fp32      nullable; dL/dlse (0 when NULL)
 * and the outputs (all written in full, caller-owned):
 *   dq        [B, T, HQ, K]  dtype dt
 *   dk        [B, T, H,  K]  dtype dt  summed over the query heads of each KV group
 *   dv        [B, T, H,  V]  dtype dt  likewise
 *   dg        [B, T, HQ, K]  dtype dt
 *   dg_scalar [B, T, HQ]     dtype dt  required iff g_scalar != NULL
 *   dsink     [HQ]           fp32      required iff sink_bias != NULL; summed over B
 *   workspace at least wall_attn_bwd_workspace_size(...) bytes, 256-byte
 *             aligned, clobbered.
 * The softmax statistics come from lse: o and lse must be those of the same
 * inputs (the forward's own outputs).  Deterministic: no atomics, fixed
 * reduction orders.  T == 0 (or B == 0) is a no-op returning WALL_OK.
 */
size_t wall_attn_bwd_workspace_size(int B, int T, int HQ, int H, int K, int V,
                                    wall_dtype_t dt);

wall_status_t wall_attn_bwd(const void* q, const void* k, const void* v, const void* g,
                            const void* g_scalar, const float* sink_bias, int window,
                            const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ,
                            int H, int K, int V, wall_dtype_t dt, float scale, const void* o,
                            const float* lse, const void* dout, const float* dlse, void* dq,
                            void* dk, void* dv, void* dg, void* dg_scalar, float* dsink,
                            void* workspace, size_t workspace_bytes, wall_stream_t stream);

/*
 * Decode cache build / append (Wall Attention README, "Decode"):
 *   P = cumsum(g) * (1/ln 2);  k_tilde[j] = k[j] * exp2(R_c - P[j])
 * with one anchor vector R_c = P[c * chunk] per chunk of `chunk` tokens (the
 * chunk's first token, so appending never rewrites earlier rows).
 * Writes cache rows t_start .. t_start + T_new - 1.
 *
 *   k_new   [B, T_new, H,  K]  dtype dt   keys of the new tokens
 *   g_new   [B, T_new, HQ, K]  dtype dt   log-decay of the new tokens
 *   p_prev  [B, HQ, K] fp32    P at row t_start - 1; NULL iff t_start == 0
 *   k_tilde [B, cap, HQ, K]    dtype dt   cache (rows below t_start untouched)
 *   r_cache [B, ceil(cap/chunk), HQ, K] fp32  anchors; a chunk whose first row
 *           is below t_start must already hold its anchor (it is read)
 *   p_last  [B, HQ, K] fp32    out: P at row t_start + T_new - 1 (pass it as
 *           p_curr to wall_attn_decode and as p_prev to the next append)
 * Requires 0 <= t_start, t_start + T_new <= cap, chunk in {32, 64, 128}
 * (WALL_ERR_UNSUPPORTED otherwise).  p_last may alias p_prev.  T_new == 0 is
 * a no-op.
 */
wall_status_t wall_build_kv_cache(const void* k_new, const void* g_new, const float* p_prev,
                                  int B, int t_start, int T_new, int cap, int HQ, int H, int K,
                                  int chunk, wall_dtype_t dt, void* k_tilde, float* r_cache,
                                  float* p_last, wall_stream_t stream);

/*
 * One-token append per batch row at that row's own position (batches whose
 * sequences have different lengths; Wall Attention README, "Decode" append): for each
 * b, row t = t_pos[b] of the cache gets k_tilde from k_new[b] and g_new[b];
 * a chunk starting at t gets its anchor; p_last[b] = P at row t.
 *   k_new [B, 1, H, K], g_new [B, 1, HQ, K]  dtype dt
 *   p_prev [B, HQ, K] fp32  P at row t_pos[b] - 1 (ignored where t_pos[b] == 0)
 *   t_pos  device int32 [B], values in [0, cap) (clamped on the device); a row
 *          appended inside a chunk needs that chunk's anchor already written
 *   k_tilde, r_cache, chunk as for wall_build_kv_cache; p_last may alias p_prev
 * Use with wall_attn_decode_varlen (seqlens_kv[b] = t_pos[b] + 1).
 */
wall_status_t wall_append_kv_cache_varlen(const void* k_new, const void* g_new,
                                          const float* p_prev, const int32_t* t_pos, int B,
                                          int cap, int HQ, int H, int K, int chunk,
                                          wall_dtype_t dt, void* k_tilde, float* r_cache,
                                          float* p_last, wall_stream_t stream);

/*
 * Single-step decode over the pre-rescaled cache (Wall Attention README,
 * "Decode"): the current query attends cache rows 0 .. T_kv - 1 (the current
 * token included: append first, then attend):
 *   x_j = scale * sum_n q[n] k_tilde[j,n] exp2(p_curr[n] - R_{j/chunk}[n])
 *
 *   q        [B, 1, HQ, K]  dtype dt
 *   p_curr   [B, 1, HQ, K]  fp32  P at the current token (p_last of the append)
 *   v        [B, cap, H, V] dtype dt  value cache (rows < T_kv valid)
 *   k_tilde  [B, cap, HQ, K] dtype dt, r_cache [B, ceil(cap/chunk), HQ, K] fp32
 *   sink_bias [HQ] fp32, nullable
 *   o        [B, 1, HQ, V]  dtype dt;  lse [B, 1, HQ] fp32, nullable
 *   workspace >= wall_attn_decode_workspace_size(B, T_kv, HQ, H, V, chunk)
 *            bytes, 16-byte aligned, no initialisation needed.
 * Split-KV: partial (o, max, sum) per split, merged by a combine pass.  The
 * split count grows with T_kv, so a workspace sized for T_kv = cap serves
 * every step of a streaming loop.
 * Requires 1 <= T_kv <= cap, chunk in {32, 64, 128}, HQ / H in
 * {1, 2, 4, 8, 16}.  No g_scalar term here (the README's decode call takes
 * none); wall_attn_decode_gated adds it.
 */
size_t wall_attn_decode_workspace_size(int B, int T_kv, int HQ, int H, int V, int chunk);

wall_status_t wall_attn_decode(const void* q, const float* p_curr, const void* v,
                               const void* k_tilde, const float* r_cache, const float* sink_bias,
                               int B, int T_kv, int cap, int HQ, int H, int K, int V, int chunk,
                               wall_dtype_t dt, float scale, void* o, float* lse, void* workspace,
                               size_t workspace_bytes, wall_stream_t stream);

/*
 * Decode over a batch whose cached sequences have different lengths (the
 * README's decode takes one length for the whole batch).  Same as
 * wall_attn_decode except:
 *   seqlens_kv  device int32 [B]: batch row b attends its cache rows
 *               0 .. seqlens_kv[b] - 1; values must lie in [1, max_T_kv]
 *               (they are clamped to it on the device)
 *   max_T_kv    the largest length (<= cap); size the workspace with
 *               wall_attn_decode_workspace_size(B, max_T_kv, HQ, H, V, chunk)
 * p_curr[b] must be P at row seqlens_kv[b] - 1 of that row.
 */
wall_status_t wall_attn_decode_varlen(const void* q, const float* p_curr, const void* v,
                                      const void* k_tilde, const float* r_cache,
                                      const float* sink_bias, const int32_t* seqlens_kv, int B,
                                      int max_T_kv, int cap, int HQ, int H, int K, int V,
                                      int chunk, wall_dtype_t dt, float scale, void* o,
                                      float* lse, void* workspace, size_t workspace_bytes,
                                      wall_stream_t stream);

/*
 * Paged decode caches (block tables, after the PagedAttention scheme the pages
 * describe: a pool of fixed-size physical blocks; each sequence lists the
 * blocks that hold its logical rows).  Row t of batch row b lives in row
 * t % block_size of pool block block_table[b * max_blocks + t / block_size].
 *   block_table  device int32 [B, max_blocks]; entries must lie in
 *                [0, num_blocks) (they are clamped into the pool on the device,
 *                so a bad entry never addresses memory outside it)
 *   k_tilde_pool [num_blocks, block_size, HQ, K]  dtype dt
 *   r_pool       [num_blocks, block_size / chunk, HQ, K] fp32 (anchors of the
 *                block's chunks)
 *   v_pool       [num_blocks, block_size, H, V]   dtype dt (caller-written, as
 *                the dense v cache)
 * block_size must be a multiple of chunk (so a chunk never straddles a block).
 * Each call is the dense call of the same name with the cache rows addressed
 * through the table; a batch row's capacity is max_blocks * block_size rows.
 * wall_attn_decode_paged requires seqlens_kv (as wall_attn_decode_varlen);
 * size its workspace with wall_attn_decode_workspace_size(B, max_blocks *
 * block_size, HQ, H, V, chunk).
 */
wall_status_t wall_build_kv_cache_paged(const void* k_new, const void* g_new,
                                        const float* p_prev, const int32_t* block_table,
                                        int max_blocks, int B, int t_start, int T_new,
                                        int num_blocks, int block_size, int HQ, int H, int K,
                                        int chunk, wall_dtype_t dt, void* k_tilde_pool,
                                        float* r_pool, float* p_last, wall_stream_t stream);

wall_status_t wall_append_kv_cache_paged(const void* k_new, const void* g_new,
                                         const float* p_prev, const int32_t* t_pos,
                                         const int32_t* block_table, int max_blocks, int B,
                                         int num_blocks, int block_size, int HQ, int H, int K,
                                         int chunk, wall_dtype_t dt, void* k_tilde_pool,
                                         float* r_pool, float* p_last, wall_stream_t stream);

wall_status_t wall_attn_decode_paged(const void* q, const float* p_curr, const void* v_pool,
                                     const void* k_tilde_pool, const float* r_pool,
                                     const float* sink_bias, const int32_t* seqlens_kv,
                                     const int32_t* block_table, int max_blocks, int B,
                                     int num_blocks, int block_size, int HQ, int H, int K, int V,
                                     int chunk, wall_dtype_t dt, float scale, void* o, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     wall_stream_t stream);

/*
 * One decode step with the append fused in (Wall Attention README, "Decode":
 * the streaming loop appends each new token to the cache, then attends it).
 * One new token per batch row, at row t_b = T_b - 1 where T_b is the row's
 * length after this step: T_kv (seqlens_kv NULL) or seqlens_kv[b].  The call
 * writes that row exactly as wall_append_kv_cache_varlen(t_pos = t_b) does
 * (k_tilde row, the chunk's anchor when t_b % chunk == 0, P_last = p_prev +
 * g_new * log2(e)), stores v_new in the value cache's row t_b, and returns
 * o / lse of the token's query over rows 0 .. t_b, all in the decode's kernel
 * launches (no separate append).
 *   q      [B, 1, HQ, K]   k_new [B, 1, H, K]   g_new [B, 1, HQ, K]
 *   v_new  [B, 1, H, V]    (dtype dt)
 *   p_prev [B, HQ, K] fp32 = P at row t_b - 1 (read only where t_b > 0)
 *   p_last [B, HQ, K] fp32, written; must not overlap p_prev (several CTAs
 *          read p_prev while one writes P_last): WALL_ERR_INVALID_ARG
 *   dense  (block_table NULL): k_tilde [B, cap, HQ, K], r_cache
 *          [B, ceil(cap / chunk), HQ, K] fp32, v_cache [B, cap, H, V];
 *          T_kv <= cap; max_blocks, num_blocks, block_size ignored
 *   paged  (block_table set): the pools of wall_attn_decode_paged;
 *          seqlens_kv required; cap ignored
 *   T_kv   the largest T_b (values of seqlens_kv above it are clamped to it)
 * Workspace: wall_attn_decode_workspace_size(B, T_kv, HQ, H, V, chunk) (paged:
 * with T_kv = max_blocks * block_size).  With the scalar gate use
 * wall_attn_decode_step_gated below.
 */
wall_status_t wall_attn_decode_step(const void* q, const void* k_new, const void* g_new,
                                    const void* v_new, const float* p_prev, float* p_last,
                                    const float* sink_bias, const int32_t* seqlens_kv,
                                    const int32_t* block_table, int max_blocks, int num_blocks,
                                    int block_size, int B, int T_kv, int cap, int HQ, int H,
                                    int K, int V, int chunk, wall_dtype_t dt, float scale,
                                    void* k_tilde, float* r_cache, void* v_cache, void* o,
                                    float* lse, void* workspace, size_t workspace_bytes,
                                    wall_stream_t stream);

/*
 * wall_attn_decode_step with the scalar gate (the forward's additive term
 * Gs[t] - Gs[j], Wall Attention README "Usage" optional arguments, through the
 * gate cache described below): the same arguments plus
 *   gs_new   [B, 1, HQ] dtype dt   the new token's g_scalar
 *   gs_prev  [B, HQ] fp32          PS at row t_b - 1 (read only where t_b > 0)
 *   gs_last  [B, HQ] fp32          out: PS at row t_b; must not overlap gs_prev
 *   gs_cache the gate cache (dense [B, cap, HQ] or the pool [num_blocks,
 *            block_size, HQ] of the same block table), row t_b written
 * Row j's logit gains (PS[t_b] - PS[j]) ln 2; the new row's own term is 0.
 */
wall_status_t wall_attn_decode_step_gated(
    const void* q, const void* k_new, const void* g_new, const void* v_new, const void* gs_new,
    const float* p_prev, float* p_last, const float* gs_prev, float* gs_last, float* gs_cache,
    const float* sink_bias, const int32_t* seqlens_kv, const int32_t* block_table, int max_blocks,
    int num_blocks, int block_size, int B, int T_kv, int cap, int HQ, int H, int K, int V,
    int chunk, wall_dtype_t dt, float scale, void* k_tilde, float* r_cache, void* v_cache,
    void* o, float* lse, void* workspace, size_t workspace_bytes, wall_stream_t stream);

/*
 * Scalar gate in decode (the forward's g_scalar term Gs[t] - Gs[j] through the
 * cache; the README's decode call has no gate, so these calls are separate).
 * The gate cache holds PS[t] = sum_{u <= t} g_scalar[u] * log2(e) per (row,
 * query head), fp32, in the exp2 units of P:
 *   dense  gs_cache [B, cap, HQ]                       (block_table NULL)
 *   paged  gs_cache [num_blocks, block_size, HQ]       (same table as k_tilde)
 * wall_build_gate_cache writes rows t_start .. t_start + T_new - 1 from
 * gs_new [B, T_new, HQ] (dtype dt); gs_prev [B, HQ] = PS at row t_start - 1
 * (NULL iff t_start == 0); gs_last [B, HQ] = PS at the last new row.
 * wall_append_gate_cache writes one row per batch row at t_pos[b] (device
 * int32 [B]) from gs_new [B, 1, HQ], with gs_prev = PS at row t_pos[b] - 1.
 * wall_attn_decode_gated is wall_attn_decode (block_table NULL, seqlens_kv
 * optional) or wall_attn_decode_paged (block_table set, seqlens_kv required)
 * plus gs_curr [B, HQ] = PS at the current row and the gate cache; the logit
 * of row j gains (gs_curr - gs_cache[j]) ln 2.  Workspace as for those calls.
 */
wall_status_t wall_build_gate_cache(const void* gs_new, const float* gs_prev,
                                    const int32_t* block_table, int max_blocks, int num_blocks,
                                    int block_size, int B, int t_start, int T_new, int cap, int HQ,
                                    wall_dtype_t dt, float* gs_cache, float* gs_last,
                                    wall_stream_t stream);

wall_status_t wall_append_gate_cache(const void* gs_new, const float* gs_prev,
                                     const int32_t* t_pos, const int32_t* block_table,
                                     int max_blocks, int num_blocks, int block_size, int B,
                                     int cap, int HQ, wall_dtype_t dt, float* gs_cache,
                                     float* gs_last, wall_stream_t stream);

wall_status_t wall_attn_decode_gated(const void* q, const float* p_curr, const float* gs_curr,
                                     const void* v, const void* k_tilde, const float* r_cache,
                                     const float* gs_cache, const float* sink_bias,
                                     const int32_t* seqlens_kv, const int32_t* block_table,
                                     int max_blocks, int num_blocks, int block_size, int B,
                                     int T_kv, int cap, int HQ, int H, int K, int V, int chunk,
                                     wall_dtype_t dt, float scale, void* o, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     wall_stream_t stream);

/*
 * A chunk of new tokens against the cache (chunked prefill; multi-token
 * decode): M tokens at positions t_start .. t_start + M - 1 of each batch row.
 * The call first appends their keys to the dense decode cache exactly as
 * wall_build_kv_cache(k_new, g_new, p_prev, B, t_start, M, cap, ...) does
 * (k_tilde rows, chunk anchors, p_last), then every new query i attends cache
 * rows 0 .. t_start + i (causal; window > 0 keeps t_start + i - j < window;
 * optional sink), with the cache's per-chunk anchors folded into tile rescales
 * (Wall Attention README "Decode" cache, the forward's score).  The result
 * equals rows t_start .. t_start + M - 1 of the prefill of the whole sequence.
 *   q        [B, M, HQ, K]   k_new [B, M, H, K]   g_new [B, M, HQ, K]   (dt)
 *   v_cache  [B, cap, H, V]  rows t_start .. t_start + M - 1 already hold the
 *            chunk's values (caller-written, as for the decode)
 *   o        [B, M, HQ, V] dt;  lse [B, M, HQ] fp32 (nullable)
 *   workspace >= wall_attn_chunk_workspace_size(B, M, cap, HQ, H, K, V, chunk, dt)
 *            bytes, 256-aligned
 * The scalar gate goes through wall_attn_chunk_gated below.
 * bf16: a chunk of at most 2 * 16 / (HQ / H) tokens (multi-token decode)
 * attends through a split-KV pass that streams the cache once per KV head;
 * longer chunks through 128-row tensor-core query tiles.  Both give the same
 * result within the usual tolerance.
 * fp32 (the exact path, no tensor cores): every chunk takes the split-KV pass,
 * each group of 16 / (HQ / H) tokens streaming the cache rows it can see;
 * HQ / H must be 1, 2, 4, 8 or 16 and B * M * HQ < 2^31, else
 * WALL_ERR_UNSUPPORTED.
 */
size_t wall_attn_chunk_workspace_size(int B, int M, int cap, int HQ, int H, int K, int V,
                                      int chunk, wall_dtype_t dt);

wall_status_t wall_attn_chunk(const void* q, const void* k_new, const void* g_new,
                              const float* p_prev, const float* sink_bias, int window, int B,
                              int t_start, int M, int cap, int HQ, int H, int K, int V, int chunk,
                              wall_dtype_t dt, float scale, void* k_tilde, float* r_cache,
                              float* p_last, const void* v_cache, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, wall_stream_t stream);

/*
 * wall_attn_chunk with the scalar gate (the forward's additive term Gs[i] - Gs[j],
 * Wall Attention README "Usage" optional arguments): the chunk's gate prefixes
 * join the gate cache first, exactly as wall_build_gate_cache(gs_new, gs_prev,
 * t_start, ...) writes them, then query i's logit of cache row j gains
 * (PS[t_start + i] - PS[j]) ln 2.
 *   gs_new    [B, M, HQ] dt            the chunk's g_scalar
 *   gs_prev   [B, HQ] fp32             PS at row t_start - 1 (NULL iff t_start == 0)
 *   gs_cache  [B, cap, HQ] fp32        the dense gate cache (rows t_start .. written)
 *   gs_last   [B, HQ] fp32             out: PS at the chunk's last row (may alias gs_prev)
 * Other arguments and the workspace as wall_attn_chunk.
 */
wall_status_t wall_attn_chunk_gated(const void* q, const void* k_new, const void* g_new,
                                    const void* gs_new, const float* p_prev, const float* gs_prev,
                                    const float* sink_bias, int window, int B, int t_start, int M,
                                    int cap, int HQ, int H, int K, int V, int chunk,
                                    wall_dtype_t dt, float scale, void* k_tilde, float* r_cache,
                                    float* p_last, float* gs_cache, float* gs_last,
                                    const void* v_cache, void* o, float* lse, void* workspace,
                                    size_t workspace_bytes, wall_stream_t stream);

/*
 * Decode without scratch allocation (no counterpart in the paper: this entry
 * point exists for callers of this library, not for the method).
 *
 * Same arguments and result as wall_attn_decode, minus the workspace.  Some
 * callers cannot allocate device memory at decode time: an inference server or
 * host application that owns every byte of device memory through its own
 * planner or pool and forbids outside allocations, a token loop that must not
 * stall on an allocator (cudaMalloc can synchronise the device), or plain C
 * code that is handed tensor pointers and no allocator at all.  This call
 * keeps the split partials in a fixed 4 MiB array in the library's own device
 * memory (one per GPU that loads the library, held until the process exits)
 * and calls no cudaMalloc, cudaFree or allocating library routine.
 *
 *   - Limit: one (V + 2)-float partial per (batch row, query head, split) must
 *     fit in 4 MiB.  The split count is lowered as needed (results stay within
 *     the usual tolerance); if even one split per (batch row, query head) does
 *     not fit (B * HQ * (V + 2) * 4 bytes > 4 MiB, e.g. B * HQ > 8065 at
 *     V = 128) the call returns WALL_ERR_WORKSPACE before queuing any work.
 *   - The array is shared by every call on the device and keeps the last
 *     call's contents; nothing in it needs to start at zero (the split pass
 *     writes every partial the combine pass reads).  Calls whose kernels
 *     overlap on the GPU (different streams without ordering between them)
 *     race on the array and give wrong results: order them on one stream.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture begins.
 */
wall_status_t wall_attn_decode_noalloc(const void* q, const float* p_curr, const void* v,
                                       const void* k_tilde, const float* r_cache,
                                       const float* sink_bias, int B, int T_kv, int cap, int HQ,
                                       int H, int K, int V, int chunk, wall_dtype_t dt,
                                       float scale, void* o, float* lse, wall_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word.
 * Returns WALL_ERR_DEVICE_TIMEOUT if any kernel since the last read gave up a
 * bounded wait (its outputs are then unspecified); else WALL_ERR_RANGE if a
 * kernel met decay it cannot represent (outputs unspecified where it did):
 *   - a decode-cache row whose factor exp2(R_c - P_j) exceeds 2^100, i.e. a
 *     channel decayed by more than ~69 nats since its chunk's first row
 *     (the Wall Attention README's cache keeps one anchor per chunk; a
 *     smaller chunk raises the bound), written by any cache build, append,
 *     fused decode step or prefill that emits the cache;
 *   - wall_attn_bwd on inputs with a 256-row block whose decay exceeds 64 nats
 *     in some channel.
 * The prefill and chunk outputs themselves are exact for any g <= 0.
 * WALL_ERR_CUDA if the synchronisation failed, WALL_OK otherwise.
 */
wall_status_t wall_device_error(wall_stream_t stream);

/*
 * Testing hook (not for production use): while mode is set, the producer of
 * one kernel skips its first load, so that kernel's consumers' bounded waits
 * run out and report WALL_ERR_DEVICE_TIMEOUT through the error word (no GPU
 * fault, no hang: every wait gives up after about wait_ms milliseconds):
 *   mode 1: prefill attention (first K/V tile), mode 2: decode split (first
 *   k_tilde/v stage), mode 3: cache build (first g/k stage), mode 4: backward
 *   key-block kernel (first query tile), mode 5: backward query-block kernel
 *   (first key tile; bf16 only), mode 6: wall_attn_chunk's tensor-core tile
 *   kernel (first cache key tile), mode 7: wall_attn_chunk's few-token split
 *   kernel (first k_tilde/v stage).
 * Outputs of the starved call are unspecified.  mode 0 restores normal
 * operation.  wait_ms <= 0 keeps the default limit (2000 ms).
 */
void wall_debug_set_fault(int mode, int wait_ms);

/*
 * Profiling hook (not for production use): while set, every wall_attn_fwd
 * records the caller's CUDA events (cudaEvent_t, NULL = skip) on its stream
 * before the prepass (`before`), between the prepass and the main attention
 * kernel (`between`) and after the main kernel (`after`); every
 * wall_attn_decode records them before the split kernel, between the split and
 * the combine kernel, and after the combine.  Lets a caller time each kernel
 * with events on the launching stream.  Process-global; not thread-safe.
 */
void wall_debug_set_stage_events(void* before, void* between, void* after);

#ifdef __cplusplus
}
#endif

#endif /* WALL_ATTN_H_ */
