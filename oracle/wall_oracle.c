/*
 * Wall attention CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, double-precision evaluation of what the Wall attention hot path
 * computes.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this file's library.  It shares no code, header or constant
 * with the CUDA path (decayed_softmax_attention_b200/csrc).
 *
 * Sources (the Wall Attention GitHub README, as mirrored on news.ainew.jp):
 *   - intro: a pair (i, j) is scored by sum_n q[i,n] k[j,n] weighted, per
 *     channel n, by the learned decay accumulated between the two positions;
 *     g = 0 gives vanilla softmax attention.  The accumulated decay between
 *     j <= i is exp(G[i,n] - G[j,n]) with G the inclusive cumulative sum of
 *     the per-channel log-decay g over time.
 *   - "Usage / Training-Prefill": shapes q [B,T,HQ,K], k [B,T,H,K],
 *     v [B,T,H,V], g [B,T,HQ,K]; optional g_scalar [B,T,HQ] (a FoX-style
 *     additive gate), sink_bias [HQ] (attention sink), window_size (sliding
 *     window), cu_seqlens (variable-length packing, B == 1).
 *   - "Decode (cache build)": P = cumsum(g) * (1/ln 2) (exp2 domain),
 *     k_tilde[j] = k[j] * exp2(R_c - P[j]) with one anchor vector R_c per
 *     chunk of C tokens; the decode reads k_tilde and r_cache.
 * Readings of points the page leaves open:
 *   - scale multiplies only the decayed q.k sum (not g_scalar, not the sink);
 *   - g_scalar adds Gs[i] - Gs[j] to the logit, Gs its inclusive cumsum;
 *   - sink_bias is one extra logit per head with a zero value vector;
 *   - window W keeps keys with 0 <= i - j < W (W counts the query itself),
 *     following the sliding-window mask_mod statement on the FlexAttention
 *     review page ("technical mechanism" section); W <= 0 means no window;
 *   - cumulative sums restart at every cu_seqlens document start;
 *   - query head hq reads KV head hq / (HQ / H);
 *   - lse is the natural-log normaliser, sink included;
 *   - the cache anchor is R_c = P[c*C], the chunk's first token;
 *   - the backward differentiates o (and, when given, lse) with respect to
 *     every input; the sink gradient sums over the batch, k and v gradients
 *     over the query heads of a KV group.
 *
 * Inputs are float32 arrays holding already-rounded values (bf16 or fp32);
 * every value is widened to double on use.  No blocking, fusion or reordering
 * beyond the definitions above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2

/* Document [s, e) that contains token t (whole row [0, T) without packing). */
static void doc_of(const int32_t* cu, int nseq, int T, int t, int* s, int* e) {
  if (!cu) {
    *s = 0;
    *e = T;
    return;
  }
  for (int d = 0; d < nseq; ++d) {
    if (t >= cu[d] && t < cu[d + 1]) {
      *s = cu[d];
      *e = cu[d + 1];
      return;
    }
  }
  *s = t;
  *e = t + 1;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

/*
 * Prefill forward, by the definition.
 *
 * For every requested row r = b*T + t and every query head hq:
 *   kv = hq / (HQ/H);  [s, e) = document of t;
 *   G[u,n]  = sum_{w=s..u} g[b,w,hq,n]        (inclusive, restarts at s)
 *   Gs[u]   = sum_{w=s..u} g_scalar[b,w,hq]   (0 without g_scalar)
 *   keys j in [s, t] with (window <= 0 or t - j < window);
 *   x_j = scale * sum_n q[t,n] k[j,n] exp(G[t,n] - G[j,n]) + Gs[t] - Gs[j];
 *   M = max(x_j, sink);  Z = sum_j exp(x_j - M) + exp(sink - M);
 *   o = sum_j exp(x_j - M) v[j] / Z;  lse = M + log Z.
 * rows == NULL means every row (nrows must be B*T).  o: [nrows, HQ, V],
 * lse: [nrows, HQ], both double.
 */
int wall_oracle_fwd(const float* q, const float* k, const float* v, const float* g,
                    const float* g_scalar, const float* sink, int window,
                    const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ, int H,
                    int K, int V, double scale, const int64_t* rows, int64_t nrows,
                    double* o, double* lse, int nthreads) {
  if (B <= 0 || T <= 0 || HQ <= 0 || H <= 0 || K <= 0 || V <= 0 || HQ % H) return ORACLE_BAD_ARG;
  if (cu_seqlens && (B != 1 || num_seqs <= 0 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T))
    return ORACLE_BAD_ARG;
  if (!rows && nrows != (int64_t)B * T) return ORACLE_BAD_ARG;
  const int group = HQ / H;
  set_threads(nthreads);
  int status = ORACLE_OK;

#pragma omp parallel
  {
    double* G = (double*)malloc(sizeof(double) * (size_t)T * K);
    double* Gs = (double*)malloc(sizeof(double) * (size_t)T);
    double* x = (double*)malloc(sizeof(double) * (size_t)T);
    if (!G || !Gs || !x) {
#pragma omp atomic write
      status = ORACLE_NO_MEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t bh = 0; bh < (int64_t)B * HQ; ++bh) {
        const int b = (int)(bh / HQ), hq = (int)(bh % HQ), kv = hq / group;
        /* inclusive prefix sums, restarting at each document start */
        for (int u = 0; u < T; ++u) {
          int s, e;
          doc_of(cu_seqlens, num_seqs, T, u, &s, &e);
          const float* gu = g + (((size_t)b * T + u) * HQ + hq) * K;
          for (int n = 0; n < K; ++n)
            G[(size_t)u * K + n] = (u == s ? 0.0 : G[(size_t)(u - 1) * K + n]) + (double)gu[n];
          const double gsu = g_scalar ? (double)g_scalar[((size_t)b * T + u) * HQ + hq] : 0.0;
          Gs[u] = (u == s ? 0.0 : Gs[u - 1]) + gsu;
        }
        for (int64_t r = 0; r < nrows; ++r) {
          const int64_t row = rows ? rows[r] : r;
          if (row / T != b) continue;
          const int t = (int)(row % T);
          int s, e;
          doc_of(cu_seqlens, num_seqs, T, t, &s, &e);
          int j0 = s;
          if (window > 0 && t - window + 1 > j0) j0 = t - window + 1;
          const float* qt = q + (((size_t)b * T + t) * HQ + hq) * K;
          const double* Gt = G + (size_t)t * K;
          double M = -INFINITY;
          for (int j = j0; j <= t; ++j) {
            const float* kj = k + (((size_t)b * T + j) * H + kv) * K;
            const double* Gj = G + (size_t)j * K;
            double dot = 0.0;
            for (int n = 0; n < K; ++n) dot += (double)qt[n] * (double)kj[n] * exp(Gt[n] - Gj[n]);
            x[j] = scale * dot + (Gs[t] - Gs[j]);
            if (x[j] > M) M = x[j];
          }
          const double sb = sink ? (double)sink[hq] : -INFINITY;
          if (sb > M) M = sb;
          double Z = sink ? exp(sb - M) : 0.0;
          double* orow = o + ((size_t)r * HQ + hq) * V;
          for (int c = 0; c < V; ++c) orow[c] = 0.0;
          for (int j = j0; j <= t; ++j) {
            const double w = exp(x[j] - M);
            Z += w;
            const float* vj = v + (((size_t)b * T + j) * H + kv) * V;
            for (int c = 0; c < V; ++c) orow[c] += w * (double)vj[c];
          }
          for (int c = 0; c < V; ++c) orow[c] /= Z;
          lse[(size_t)r * HQ + hq] = M + log(Z);
        }
      }
    }
    free(G);
    free(Gs);
    free(x);
  }
  return status;
}

/*
 * Decode cache build, following the README's "Decode" section.
 *   P[t,n]  = (1/ln 2) * sum_{u=0..t} g[b,u,hq,n]        (exp2-domain prefix)
 *   R[c,n]  = P[c*C, n]           (chunk-start anchor; or anchors[] if given)
 *   k_tilde[t,hq,n] = k[t, kv(hq), n] * 2^(R[t/C, n] - P[t, n])
 * Outputs (double): k_tilde [B,T,HQ,K], r_cache [B,ceil(T/C),HQ,K], P [B,T,HQ,K].
 * `anchors` (nullable, [B,ceil(T/C),HQ,K]) replaces R to test that the choice of
 * anchor leaves every decode score unchanged.
 */
int wall_oracle_kv_cache(const float* k, const float* g, int B, int T, int HQ, int H, int K,
                         int C, const double* anchors, double* k_tilde, double* r_cache,
                         double* P, int nthreads) {
  if (B <= 0 || T <= 0 || HQ <= 0 || H <= 0 || K <= 0 || C <= 0 || HQ % H) return ORACLE_BAD_ARG;
  const int group = HQ / H;
  const int nc = (T + C - 1) / C;
  const double rcp_ln2 = 1.0 / log(2.0);
  set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * HQ; ++bh) {
    const int b = (int)(bh / HQ), hq = (int)(bh % HQ), kv = hq / group;
    for (int n = 0; n < K; ++n) {
      double acc = 0.0;
      for (int t = 0; t < T; ++t) {
        acc += (double)g[(((size_t)b * T + t) * HQ + hq) * K + n];
        P[(((size_t)b * T + t) * HQ + hq) * K + n] = acc * rcp_ln2;
      }
      for (int c = 0; c < nc; ++c) {
        const size_t ridx = (((size_t)b * nc + c) * HQ + hq) * K + n;
        r_cache[ridx] = anchors ? anchors[ridx] : P[(((size_t)b * T + (size_t)c * C) * HQ + hq) * K + n];
      }
      for (int t = 0; t < T; ++t) {
        const size_t pidx = (((size_t)b * T + t) * HQ + hq) * K + n;
        const double R = r_cache[(((size_t)b * nc + t / C) * HQ + hq) * K + n];
        k_tilde[pidx] = (double)k[(((size_t)b * T + t) * H + kv) * K + n] * exp2(R - P[pidx]);
      }
    }
  }
  return ORACLE_OK;
}

/*
 * Single-step decode over the pre-rescaled cache, following the README's
 * "Decode" section: for the current query q (its prefix P = p_curr) and cached
 * keys j in [0, T_kv):
 *   x_j = scale * sum_n q[n] * k_tilde[j,n] * 2^(p_curr[n] - R[j/C, n])
 *   softmax over j (plus the optional sink logit), o = sum_j w_j v[j].
 * q [B,HQ,K] float; p_curr [B,HQ,K], k_tilde [B,cap,HQ,K], r_cache
 * [B,ceil(cap/C),HQ,K] double; v [B,cap,H,V] float.  o [B,HQ,V], lse [B,HQ].
 * With the scalar gate (gs_curr [B,HQ] and gs_cache [B,cap,HQ], both double,
 * nullable together): PS = cumsum(g_scalar) * (1/ln 2) in the same exp2 units
 * as P, and the logit gains (gs_curr - gs_cache[j]) * ln 2 = Gs[t] - Gs[j].
 */
int wall_oracle_decode_cache(const float* q, const double* p_curr, const float* v,
                             const double* k_tilde, const double* r_cache, const float* sink,
                             const double* gs_curr, const double* gs_cache,
                             int B, int T_kv, int cap, int HQ, int H, int K, int V, int C,
                             double scale, double* o, double* lse, int nthreads) {
  if (B <= 0 || T_kv <= 0 || cap < T_kv || HQ <= 0 || H <= 0 || K <= 0 || V <= 0 || C <= 0 ||
      HQ % H)
    return ORACLE_BAD_ARG;
  const int group = HQ / H;
  const int nc = (cap + C - 1) / C;
  set_threads(nthreads);
  int status = ORACLE_OK;
#pragma omp parallel
  {
    double* x = (double*)malloc(sizeof(double) * (size_t)T_kv);
    if (!x) {
#pragma omp atomic write
      status = ORACLE_NO_MEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t bh = 0; bh < (int64_t)B * HQ; ++bh) {
        const int b = (int)(bh / HQ), hq = (int)(bh % HQ), kv = hq / group;
        const float* qv = q + ((size_t)b * HQ + hq) * K;
        const double* pc = p_curr + ((size_t)b * HQ + hq) * K;
        double M = -INFINITY;
        for (int j = 0; j < T_kv; ++j) {
          const double* kt = k_tilde + (((size_t)b * cap + j) * HQ + hq) * K;
          const double* R = r_cache + (((size_t)b * nc + j / C) * HQ + hq) * K;
          double dot = 0.0;
          for (int n = 0; n < K; ++n) dot += (double)qv[n] * kt[n] * exp2(pc[n] - R[n]);
          x[j] = scale * dot;
          if (gs_cache)
            x[j] += (gs_curr[(size_t)b * HQ + hq] - gs_cache[((size_t)b * cap + j) * HQ + hq]) *
                    log(2.0);
          if (x[j] > M) M = x[j];
        }
        const double sb = sink ? (double)sink[hq] : -INFINITY;
        if (sb > M) M = sb;
        double Z = sink ? exp(sb - M) : 0.0;
        double* orow = o + ((size_t)b * HQ + hq) * V;
        for (int c = 0; c < V; ++c) orow[c] = 0.0;
        for (int j = 0; j < T_kv; ++j) {
          const double w = exp(x[j] - M);
          Z += w;
          const float* vj = v + (((size_t)b * cap + j) * H + kv) * V;
          for (int c = 0; c < V; ++c) orow[c] += w * (double)vj[c];
        }
        for (int c = 0; c < V; ++c) orow[c] /= Z;
        lse[(size_t)b * HQ + hq] = M + log(Z);
      }
    }
    free(x);
  }
  return status;
}

/*
 * Prefill backward, by differentiating the forward definition above (the
 * README's intro and "Usage / Training-Prefill" sections define what is
 * differentiated; its "code structure" section names the backward pass).
 * With dO = dL/do and dl = dL/dlse (0 when dlse is NULL), per row t and head hq:
 *   p_j = exp(x_j - lse), p_s = exp(sink - lse),  D = sum_c dO[t,c] o[t,c]
 *   dx_j = p_j * (dO[t].v[j] - D + dl)                 (softmax Jacobian)
 *   dq[t,n]   += scale dx_j k[j,n] exp(G[t,n] - G[j,n])
 *   dk_h[j,n] += scale dx_j q[t,n] exp(G[t,n] - G[j,n])  (per query head)
 *   dv_h[j,c] += p_j dO[t,c]
 *   dG[t,n] += scale dx_j q[t,n] k[j,n] exp(...),  dG[j,n] -= the same term
 *   dGs[t]  += dx_j,  dGs[j] -= dx_j
 *   dsink_bh += p_s * (dl - D)                         (the sink's value is 0)
 * and, G and Gs being inclusive prefix sums restarting at each document start,
 *   dg[u] = sum_{w=u..e-1} dG[w],  dg_scalar[u] = sum_{w=u..e-1} dGs[w].
 * Outputs (double): dq, dk_h, dg [B,T,HQ,K]; dv_h [B,T,HQ,V]; dg_scalar [B,T,HQ]
 * (nullable); dsink_bh [B,HQ] (nullable).  dk_h and dv_h are per query head:
 * the caller sums the heads of a KV group (and dsink_bh over b).
 * o_in [B,T,HQ,V] and lse_in [B,T,HQ] (nullable) replace the recomputed forward
 * output and normaliser in D and p: the backward evaluated from given forward
 * results, as a backward kernel that receives them does.  NULL: exact values.
 * s2 (nullable, 11 arrays): for every output element, the sum of the SQUARES of
 * the terms it sums (a scale for rounding-error tolerances, not a result):
 * s2[0] dq, s2[1] dk_h, s2[3] dg (reverse prefix sums of the squared dG terms),
 * [B,T,HQ,K]; s2[2] dv_h [B,T,HQ,V]; s2[4] dg_scalar [B,T,HQ]; s2[5] dsink [B,HQ];
 * s2[6..10]: the same for dq, dk_h, dg, dg_scalar, dsink with each term's
 * dO.v[j] - D + dl replaced by |dO.v[j]| + |D - dl| (its size before that
 * difference cancels).
 */
int wall_oracle_bwd(const float* q, const float* k, const float* v, const float* g,
                    const float* g_scalar, const float* sink, int window,
                    const int32_t* cu_seqlens, int num_seqs, int B, int T, int HQ, int H,
                    int K, int V, double scale, const float* dout, const float* dlse,
                    const float* o_in, const float* lse_in, double* dq, double* dk_h,
                    double* dv_h, double* dg, double* dg_scalar, double* dsink_bh,
                    double* const* s2, int nthreads) {
  if (B <= 0 || T <= 0 || HQ <= 0 || H <= 0 || K <= 0 || V <= 0 || HQ % H) return ORACLE_BAD_ARG;
  if (cu_seqlens && (B != 1 || num_seqs <= 0 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T))
    return ORACLE_BAD_ARG;
  const int group = HQ / H;
  set_threads(nthreads);
  int status = ORACLE_OK;

#pragma omp parallel
  {
    double* G = (double*)malloc(sizeof(double) * (size_t)T * K);
    double* Gs = (double*)malloc(sizeof(double) * (size_t)T);
    double* dG = (double*)malloc(sizeof(double) * (size_t)T * K);
    double* dGs = (double*)malloc(sizeof(double) * (size_t)T);
    double* qG = (double*)malloc(sizeof(double) * (size_t)T * K);  /* squared dG terms */
    double* qGs = (double*)malloc(sizeof(double) * (size_t)T);
    double* aG = (double*)malloc(sizeof(double) * (size_t)T * K);  /* same, absolute */
    double* aGs = (double*)malloc(sizeof(double) * (size_t)T);
    double* x = (double*)malloc(sizeof(double) * (size_t)T);
    double* orow = (double*)malloc(sizeof(double) * (size_t)V);
    if (!G || !Gs || !dG || !dGs || !x || !orow || !qG || !qGs || !aG || !aGs) {
#pragma omp atomic write
      status = ORACLE_NO_MEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t bh = 0; bh < (int64_t)B * HQ; ++bh) {
        const int b = (int)(bh / HQ), hq = (int)(bh % HQ), kv = hq / group;
#define IDX_K(t) ((((size_t)b * T + (t)) * HQ + hq) * K)
#define IDX_V(t) ((((size_t)b * T + (t)) * HQ + hq) * V)
        for (int u = 0; u < T; ++u) {
          int s, e;
          doc_of(cu_seqlens, num_seqs, T, u, &s, &e);
          const float* gu = g + IDX_K(u);
          for (int n = 0; n < K; ++n) {
            G[(size_t)u * K + n] = (u == s ? 0.0 : G[(size_t)(u - 1) * K + n]) + (double)gu[n];
            dG[(size_t)u * K + n] = 0.0;
            qG[(size_t)u * K + n] = aG[(size_t)u * K + n] = 0.0;
            dq[IDX_K(u) + n] = 0.0;
            dk_h[IDX_K(u) + n] = 0.0;
            if (s2) s2[0][IDX_K(u) + n] = s2[1][IDX_K(u) + n] = 0.0;
            if (s2) s2[6][IDX_K(u) + n] = s2[7][IDX_K(u) + n] = 0.0;
          }
          for (int c = 0; c < V; ++c) {
            dv_h[IDX_V(u) + c] = 0.0;
            if (s2) s2[2][IDX_V(u) + c] = 0.0;
          }
          qGs[u] = aGs[u] = 0.0;
          const double gsu = g_scalar ? (double)g_scalar[((size_t)b * T + u) * HQ + hq] : 0.0;
          Gs[u] = (u == s ? 0.0 : Gs[u - 1]) + gsu;
          dGs[u] = 0.0;
        }
        double dsink = 0.0, qsink = 0.0, asink = 0.0;
        for (int t = 0; t < T; ++t) {
          int s, e;
          doc_of(cu_seqlens, num_seqs, T, t, &s, &e);
          int j0 = s;
          if (window > 0 && t - window + 1 > j0) j0 = t - window + 1;
          const float* qt = q + IDX_K(t);
          const float* dot_ = dout + IDX_V(t);
          const double* Gt = G + (size_t)t * K;
          /* forward again: logits, max, normaliser, output row */
          double M = -INFINITY;
          for (int j = j0; j <= t; ++j) {
            const float* kj = k + (((size_t)b * T + j) * H + kv) * K;
            const double* Gj = G + (size_t)j * K;
            double dot = 0.0;
            for (int n = 0; n < K; ++n) dot += (double)qt[n] * (double)kj[n] * exp(Gt[n] - Gj[n]);
            x[j] = scale * dot + (Gs[t] - Gs[j]);
            if (x[j] > M) M = x[j];
          }
          const double sb = sink ? (double)sink[hq] : -INFINITY;
          if (sb > M) M = sb;
          double Z = sink ? exp(sb - M) : 0.0;
          for (int j = j0; j <= t; ++j) Z += exp(x[j] - M);
          const double lse = lse_in ? (double)lse_in[((size_t)b * T + t) * HQ + hq] : M + log(Z);
          for (int c = 0; c < V; ++c) orow[c] = 0.0;
          if (o_in) {
            for (int c = 0; c < V; ++c) orow[c] = (double)o_in[IDX_V(t) + c];
          } else {
            for (int j = j0; j <= t; ++j) {
              const double p = exp(x[j] - lse);
              const float* vj = v + (((size_t)b * T + j) * H + kv) * V;
              for (int c = 0; c < V; ++c) orow[c] += p * (double)vj[c];
            }
          }
          double D = 0.0;
          for (int c = 0; c < V; ++c) D += (double)dot_[c] * orow[c];
          const double dl = dlse ? (double)dlse[((size_t)b * T + t) * HQ + hq] : 0.0;
          /* backward through the softmax and the decayed scores */
          for (int j = j0; j <= t; ++j) {
            const double p = exp(x[j] - lse);
            const float* kj = k + (((size_t)b * T + j) * H + kv) * K;
            const float* vj = v + (((size_t)b * T + j) * H + kv) * V;
            const double* Gj = G + (size_t)j * K;
            double dP = 0.0;
            for (int c = 0; c < V; ++c) dP += (double)dot_[c] * (double)vj[c];
            const double dx = p * (dP - D + dl);
            const double dxa = p * (fabs(dP) + fabs(D - dl));
            for (int c = 0; c < V; ++c) {
              dv_h[IDX_V(j) + c] += p * (double)dot_[c];
              if (s2) s2[2][IDX_V(j) + c] += (p * (double)dot_[c]) * (p * (double)dot_[c]);
            }
            for (int n = 0; n < K; ++n) {
              const double w = scale * dx * exp(Gt[n] - Gj[n]);
              dq[IDX_K(t) + n] += w * (double)kj[n];
              dk_h[IDX_K(j) + n] += w * (double)qt[n];
              const double term = w * (double)qt[n] * (double)kj[n];
              dG[(size_t)t * K + n] += term;
              dG[(size_t)j * K + n] -= term;
              if (s2) {
                const double wa = scale * dxa * exp(Gt[n] - Gj[n]);
                const double ta = wa * (double)qt[n] * (double)kj[n];
                s2[0][IDX_K(t) + n] += (w * (double)kj[n]) * (w * (double)kj[n]);
                s2[1][IDX_K(j) + n] += (w * (double)qt[n]) * (w * (double)qt[n]);
                s2[6][IDX_K(t) + n] += (wa * (double)kj[n]) * (wa * (double)kj[n]);
                s2[7][IDX_K(j) + n] += (wa * (double)qt[n]) * (wa * (double)qt[n]);
                qG[(size_t)t * K + n] += term * term;
                qG[(size_t)j * K + n] += term * term;
                aG[(size_t)t * K + n] += ta * ta;
                aG[(size_t)j * K + n] += ta * ta;
              }
            }
            dGs[t] += dx;
            dGs[j] -= dx;
            qGs[t] += dx * dx;
            qGs[j] += dx * dx;
            aGs[t] += dxa * dxa;
            aGs[j] += dxa * dxa;
          }
          if (sink) {
            const double ps = exp(sb - lse);
            dsink += ps * (dl - D);
            qsink += (ps * (dl - D)) * (ps * (dl - D));
            asink += (ps * (fabs(dl) + fabs(D))) * (ps * (fabs(dl) + fabs(D)));
          }
        }
        /* reverse prefix sums inside each document */
        for (int n = 0; n < K; ++n) {
          double acc = 0.0, acc2 = 0.0, acc3 = 0.0;
          for (int u = T - 1; u >= 0; --u) {
            int s, e;
            doc_of(cu_seqlens, num_seqs, T, u, &s, &e);
            if (u == e - 1) acc = acc2 = acc3 = 0.0;
            acc += dG[(size_t)u * K + n];
            acc2 += qG[(size_t)u * K + n];
            acc3 += aG[(size_t)u * K + n];
            dg[IDX_K(u) + n] = acc;
            if (s2) {
              s2[3][IDX_K(u) + n] = acc2;
              s2[8][IDX_K(u) + n] = acc3;
            }
          }
        }
        if (dg_scalar) {
          double acc = 0.0, acc2 = 0.0, acc3 = 0.0;
          for (int u = T - 1; u >= 0; --u) {
            int s, e;
            doc_of(cu_seqlens, num_seqs, T, u, &s, &e);
            if (u == e - 1) acc = acc2 = acc3 = 0.0;
            acc += dGs[u];
            acc2 += qGs[u];
            acc3 += aGs[u];
            dg_scalar[((size_t)b * T + u) * HQ + hq] = acc;
            if (s2) {
              s2[4][((size_t)b * T + u) * HQ + hq] = acc2;
              s2[9][((size_t)b * T + u) * HQ + hq] = acc3;
            }
          }
        }
        if (dsink_bh) dsink_bh[bh] = dsink;
        if (s2) {
          s2[5][bh] = qsink;
          s2[10][bh] = asink;
        }
#undef IDX_K
#undef IDX_V
      }
    }
    free(G);
    free(Gs);
    free(dG);
    free(dGs);
    free(x);
    free(orow);
    free(qG);
    free(qGs);
    free(aG);
    free(aGs);
  }
  return status;
}

int wall_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
