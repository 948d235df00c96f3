"""Wall attention CPU oracle (double precision) -- TEST INFRASTRUCTURE ONLY.

Python wrapper over ``wall_oracle.c``.  Only ``tests/``, ``__graft_entry__.smoke``
and the benchmark's CPU-baseline leg may import this package; the product path
(``decayed_softmax_attention_b200``) never does.  The oracle shares no code with
the CUDA path: inputs are numpy float32 arrays holding already-rounded values,
outputs are float64.

Functions (each follows the Wall Attention README; see the C file's header for
the exact formulas and the readings taken where the page is silent):
  wall_fwd           -- prefill forward by the pairwise definition
  kv_cache           -- P, r_cache and k_tilde of the "Decode" section
  decode_from_cache  -- one decode step over (k_tilde, r_cache), optionally with the gate
  gate_cache         -- the scalar gate's prefix PS in exp2 units (decode with g_scalar)
  wall_bwd           -- gradients of the prefill forward (analytic, by the definition)
  wall_bwd_rows      -- the same gradients at selected query / key rows (numpy, for long T)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wall_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE double, OpenMP). Returns the .so path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-std=c11", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i, d, i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
    lib.wall_oracle_fwd.argtypes = [P, P, P, P, P, P, i, P, i, i, i, i, i, i, i, d, P, i64, P, P, i]
    lib.wall_oracle_kv_cache.argtypes = [P, P, i, i, i, i, i, i, P, P, P, P, i]
    lib.wall_oracle_decode_cache.argtypes = [P, P, P, P, P, P, P, P, i, i, i, i, i, i, i, i, d, P,
                                             P, i]
    lib.wall_oracle_bwd.argtypes = [P, P, P, P, P, P, i, P, i, i, i, i, i, i, i, d, P, P,
                                    P, P, P, P, P, P, P, P, P, i]
    for f in (lib.wall_oracle_fwd, lib.wall_oracle_kv_cache, lib.wall_oracle_decode_cache,
              lib.wall_oracle_bwd):
        f.restype = ctypes.c_int
    lib.wall_oracle_max_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def max_threads() -> int:
    return int(_load().wall_oracle_max_threads())


def _f32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().float().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def wall_fwd(q, k, v, g, g_scalar=None, sink_bias=None, window=0, cu_seqlens=None,
             scale=None, rows=None, threads=0):
    """Prefill forward by the definition.

    q [B,T,HQ,K], k [B,T,H,K], v [B,T,H,V], g [B,T,HQ,K]; g_scalar [B,T,HQ] or None;
    sink_bias [HQ] or None; cu_seqlens int [N+1] or None (B == 1).
    rows: None (all rows) or an int array of flattened b*T + t indices.
    Returns (o, lse): o [B,T,HQ,V] / [nrows,HQ,V], lse [B,T,HQ] / [nrows,HQ], float64.
    """
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(g)
    gs, sink = _f32(g_scalar), _f32(sink_bias)
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    cu = None
    nseq = 0
    if cu_seqlens is not None:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
        nseq = cu.shape[0] - 1
    if scale is None or scale <= 0:
        scale = K ** -0.5
    if rows is None:
        nrows, rows_arr = B * T, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = rows_arr.shape[0]
    o = np.empty((nrows, HQ, V), dtype=np.float64)
    lse = np.empty((nrows, HQ), dtype=np.float64)
    rc = _load().wall_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gs), _ptr(sink),
                                 int(window or 0), _ptr(cu), nseq, B, T, HQ, H, K, V, float(scale),
                                 _ptr(rows_arr), nrows, _ptr(o), _ptr(lse), int(threads))
    _check(rc, "wall_fwd")
    if rows is None:
        return o.reshape(B, T, HQ, V), lse.reshape(B, T, HQ)
    return o, lse


def kv_cache(k, g, HQ=None, chunk=64, anchors=None, threads=0):
    """P, r_cache and k_tilde of the decode cache (double).

    k [B,T,H,K], g [B,T,HQ,K]. anchors: optional [B,ceil(T/C),HQ,K] replacing R_c.
    Returns (k_tilde [B,T,HQ,K], r_cache [B,ceil(T/C),HQ,K], P [B,T,HQ,K]).
    """
    k, g = _f32(k), _f32(g)
    B, T, H, K = k.shape
    HQ = g.shape[2]
    nc = (T + chunk - 1) // chunk
    kt = np.empty((B, T, HQ, K), dtype=np.float64)
    rc_ = np.empty((B, nc, HQ, K), dtype=np.float64)
    P = np.empty((B, T, HQ, K), dtype=np.float64)
    anc = _f64(anchors)
    rc = _load().wall_oracle_kv_cache(_ptr(k), _ptr(g), B, T, HQ, H, K, int(chunk), _ptr(anc),
                                      _ptr(kt), _ptr(rc_), _ptr(P), int(threads))
    _check(rc, "kv_cache")
    return kt, rc_, P


def gate_cache(g_scalar):
    """PS = cumsum(g_scalar over time) * (1/ln 2) [B,T,HQ] (double): the scalar gate's prefix in
    the exp2 units of the decode cache."""
    gs = np.asarray(_f32(g_scalar), dtype=np.float64)
    return np.cumsum(gs, axis=1) / np.log(2.0)


def decode_from_cache(q, p_curr, v, k_tilde, r_cache, T_kv, sink_bias=None, chunk=64,
                      scale=None, gs_curr=None, gs_cache=None, threads=0):
    """One decode step over the pre-rescaled cache (double).

    q [B,HQ,K] (or [B,1,HQ,K]); p_curr [B,HQ,K]; v [B,cap,H,V]; k_tilde [B,cap,HQ,K];
    r_cache [B,ceil(cap/C),HQ,K]; the first T_kv cache rows are attended.
    gs_curr [B,HQ] / gs_cache [B,cap,HQ] (optional, together): the scalar gate's prefix PS
    (see gate_cache) at the current row and at every cache row.
    Returns (o [B,HQ,V], lse [B,HQ]).
    """
    q = _f32(q)
    q = q.reshape(q.shape[0], q.shape[-2], q.shape[-1])
    p = _f64(np.asarray(p_curr).reshape(q.shape))
    v, kt, r = _f32(v), _f64(k_tilde), _f64(r_cache)
    sink = _f32(sink_bias)
    B, HQ, K = q.shape
    cap, H, V = v.shape[1], v.shape[2], v.shape[3]
    if scale is None or scale <= 0:
        scale = K ** -0.5
    o = np.empty((B, HQ, V), dtype=np.float64)
    lse = np.empty((B, HQ), dtype=np.float64)
    gcur = None if gs_curr is None else _f64(np.asarray(gs_curr).reshape(B, HQ))
    gcache = None if gs_cache is None else _f64(gs_cache)
    if (gcur is None) != (gcache is None):
        raise ValueError("gs_curr and gs_cache go together")
    rc = _load().wall_oracle_decode_cache(_ptr(q), _ptr(p), _ptr(v), _ptr(kt), _ptr(r), _ptr(sink),
                                          _ptr(gcur), _ptr(gcache),
                                          B, int(T_kv), cap, HQ, H, K, V, int(chunk), float(scale),
                                          _ptr(o), _ptr(lse), int(threads))
    _check(rc, "decode_from_cache")
    return o, lse



def wall_bwd(q, k, v, g, do, g_scalar=None, sink_bias=None, window=0, cu_seqlens=None,
             scale=None, dlse=None, o=None, lse=None, scales=False, threads=0):
    """Gradients of the prefill forward (double), by differentiating the definition.

    Same inputs as ``wall_fwd`` plus do [B,T,HQ,V] (dL/do) and optional dlse [B,T,HQ].
    o [B,T,HQ,V] / lse [B,T,HQ] (optional): given forward results used in place of the
    exact ones (in D = dO.o and p = exp(x - lse)); None: recomputed exactly.
    Returns a dict: dq [B,T,HQ,K], dk [B,T,H,K], dv [B,T,H,V], dg [B,T,HQ,K],
    dg_scalar [B,T,HQ] (None without g_scalar), dsink [HQ] (None without sink_bias).
    dk and dv sum the query heads of each KV group; dsink sums the batch.
    scales=True adds "sigma": per output, the root of the sum of squares of the terms
    each element sums (a scale for rounding-error tolerances, not a result), and
    "sigma_abs": the same with each softmax-Jacobian factor dO.v - D + dlse taken as
    |dO.v| + |D - dlse| (its size before that difference cancels; dv has no such factor).
    """
    q, k, v, g, do = _f32(q), _f32(k), _f32(v), _f32(g), _f32(do)
    gs, sink, dl = _f32(g_scalar), _f32(sink_bias), _f32(dlse)
    o_in, lse_in = _f32(o), _f32(lse)
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    cu = None
    nseq = 0
    if cu_seqlens is not None:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
        nseq = cu.shape[0] - 1
    if scale is None or scale <= 0:
        scale = K ** -0.5
    dq = np.empty((B, T, HQ, K))
    dkh = np.empty((B, T, HQ, K))
    dvh = np.empty((B, T, HQ, V))
    dg = np.empty((B, T, HQ, K))
    dgs = np.empty((B, T, HQ)) if gs is not None else None
    dsb = np.empty((B, HQ)) if sink is not None else None
    s2 = s2ptr = None
    if scales:
        s2 = [np.zeros((B, T, HQ, K)), np.zeros((B, T, HQ, K)), np.zeros((B, T, HQ, V)),
              np.zeros((B, T, HQ, K)), np.zeros((B, T, HQ)), np.zeros((B, HQ)),
              np.zeros((B, T, HQ, K)), np.zeros((B, T, HQ, K)), np.zeros((B, T, HQ, K)),
              np.zeros((B, T, HQ)), np.zeros((B, HQ))]
        s2ptr = (ctypes.c_void_p * 11)(*[a.ctypes.data for a in s2])
    rc = _load().wall_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gs), _ptr(sink),
                                 int(window or 0), _ptr(cu), nseq, B, T, HQ, H, K, V,
                                 float(scale), _ptr(do), _ptr(dl), _ptr(o_in), _ptr(lse_in),
                                 _ptr(dq), _ptr(dkh),
                                 _ptr(dvh), _ptr(dg), _ptr(dgs), _ptr(dsb),
                                 None if s2ptr is None else ctypes.cast(s2ptr, ctypes.c_void_p),
                                 int(threads))
    _check(rc, "wall_bwd")
    grp = HQ // H
    dk = dkh.reshape(B, T, H, grp, K).sum(axis=3)
    dv = dvh.reshape(B, T, H, grp, V).sum(axis=3)
    out = dict(dq=dq, dk=dk, dv=dv, dg=dg, dg_scalar=dgs,
               dsink=None if dsb is None else dsb.sum(axis=0))
    if scales:
        out["sigma"] = dict(
            dq=np.sqrt(s2[0]), dk=np.sqrt(s2[1].reshape(B, T, H, grp, K).sum(axis=3)),
            dv=np.sqrt(s2[2].reshape(B, T, H, grp, V).sum(axis=3)), dg=np.sqrt(s2[3]),
            dg_scalar=np.sqrt(s2[4]) if gs is not None else None,
            dsink=np.sqrt(s2[5].sum(axis=0)) if sink is not None else None)
        out["sigma_abs"] = dict(
            dq=np.sqrt(s2[6]), dk=np.sqrt(s2[7].reshape(B, T, H, grp, K).sum(axis=3)),
            dv=out["sigma"]["dv"], dg=np.sqrt(s2[8]),
            dg_scalar=np.sqrt(s2[9]) if gs is not None else None,
            dsink=np.sqrt(s2[10].sum(axis=0)) if sink is not None else None)
    return out


def wall_bwd_rows(q, k, v, g, do, o, lse, q_rows=(), k_rows=(), g_scalar=None, window=0,
                  cu_seqlens=None, scale=None, dlse=None, batch=0, tail=0, tail_heads=None):
    """Selected rows of the prefill backward of one batch row, in double precision, straight
    from the definition (numpy; for long sequences where the full oracle is too slow).

    The same gradients as ``wall_bwd`` with given o / lse (the sink enters through lse
    only): dq at query rows ``q_rows`` [n, HQ, K]; dk [n, H, K] and dv [n, H, V] at key rows
    ``k_rows``, summed over the query heads of each KV group.  With p = exp(x - lse) and
    dS = p (dO.v - dO.o + dlse):
        dq_i = scale sum_j dS_ij k_j exp(G_i - G_j)
        dk_j = scale sum_i dS_ij q_i exp(G_i - G_j),   dv_j = sum_i p_ij dO_i
    over the admitted pairs (causal, same document, window).  Also returns "sigma" and
    "sigma_abs" for each, defined as in ``wall_bwd``.

    tail > 0 adds dg [tail, HQ, K] (and dg_scalar [tail, HQ] with g_scalar) at the last
    ``tail`` rows, which must lie in the last document.  G is an inclusive prefix sum, so
    dg_u is the sum over rows t >= u of the document of
        dG_t = q_t * dq_t - k_t * dk_t^(hq)    (dk of query head hq alone)
    and dg_scalar_u that of dGs_t = sum_j dS_tj - sum_i dS_it; the last rows need only
    the last rows' terms.  sigma: the root of the sum of squares of every pair term the
    element sums, as ``wall_bwd`` defines it.  tail_heads: the query heads to compute
    (default all); the tail arrays then hold those heads in that order.
    """
    cv = lambda x: None if x is None else _f64(_f32(x))[batch]
    q, k, v, g, do, o, lse = (cv(x) for x in (q, k, v, g, do, o, lse))
    gs, dl = cv(g_scalar), cv(dlse)
    T, HQ, K = q.shape
    H, V = k.shape[1], v.shape[2]
    grp = HQ // H
    if scale is None or scale <= 0:
        scale = K ** -0.5
    G = np.cumsum(g, axis=0)                                   # [T, HQ, K], natural log
    Gs = np.cumsum(gs, axis=0) if gs is not None else np.zeros((T, HQ))
    doc = np.zeros(T, dtype=np.int64)
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens.detach().cpu().numpy() if hasattr(cu_seqlens, "detach")
                        else cu_seqlens, dtype=np.int64)
        for d_ in range(len(cu) - 1):
            doc[cu[d_]:cu[d_ + 1]] = d_
    delta = np.einsum("thv,thv->th", do, o) - (dl if dl is not None else 0.0)
    pos = np.arange(T)

    def pairs(i, j):  # admitted (query i, key j) for arrays i, j of equal shape
        ok = (j <= i) & (doc[i] == doc[j])
        if window and window > 0:
            ok &= (i - j) < window
        return ok

    q_rows, k_rows = list(q_rows), list(k_rows)
    out = {n: np.zeros(s) for n, s in (("dq", (len(q_rows), HQ, K)), ("dk", (len(k_rows), H, K)),
                                         ("dv", (len(k_rows), H, V)))}
    s2 = {n: np.zeros_like(a) for n, a in out.items()}
    sa = {n: np.zeros_like(a) for n, a in out.items()}
    for r, i in enumerate(q_rows):
        js = pos[pairs(np.full(T, i), pos)]
        for hq in range(HQ):
            kv = hq // grp
            dec = np.exp(G[i, hq][None, :] - G[js, hq])               # [nj, K]
            x = scale * (q[i, hq][None, :] * k[js, kv] * dec).sum(axis=1) + Gs[i, hq] - Gs[js, hq]
            p = np.exp(x - lse[i, hq])
            dP = v[js, kv] @ do[i, hq]
            t = scale * (p * (dP - delta[i, hq]))[:, None] * k[js, kv] * dec
            ta = scale * (p * (np.abs(dP) + np.abs(delta[i, hq])))[:, None] * k[js, kv] * dec
            out["dq"][r, hq] = t.sum(axis=0)
            s2["dq"][r, hq] = (t * t).sum(axis=0)
            sa["dq"][r, hq] = (ta * ta).sum(axis=0)
    for r, j in enumerate(k_rows):
        is_ = pos[pairs(pos, np.full(T, j))]
        for hq in range(HQ):
            kv = hq // grp
            dec = np.exp(G[is_, hq] - G[j, hq][None, :])              # [ni, K]
            x = scale * (q[is_, hq] * k[j, kv][None, :] * dec).sum(axis=1) + Gs[is_, hq] - Gs[j, hq]
            p = np.exp(x - lse[is_, hq])
            dP = do[is_, hq] @ v[j, kv]
            t = scale * (p * (dP - delta[is_, hq]))[:, None] * q[is_, hq] * dec
            ta = scale * (p * (np.abs(dP) + np.abs(delta[is_, hq])))[:, None] * q[is_, hq] * dec
            tv = p[:, None] * do[is_, hq]
            out["dk"][r, kv] += t.sum(axis=0)
            s2["dk"][r, kv] += (t * t).sum(axis=0)
            sa["dk"][r, kv] += (ta * ta).sum(axis=0)
            out["dv"][r, kv] += tv.sum(axis=0)
            s2["dv"][r, kv] += (tv * tv).sum(axis=0)
            sa["dv"][r, kv] += (tv * tv).sum(axis=0)
    if tail > 0:
        t0 = T - tail
        assert doc[t0] == doc[T - 1], "the tail rows must lie in one (the last) document"
        heads = list(range(HQ)) if tail_heads is None else list(tail_heads)
        nh = len(heads)
        dG = np.zeros((tail, nh, K))
        dGs = np.zeros((tail, nh))
        gq2, gqa = np.zeros((tail, nh, K)), np.zeros((tail, nh, K))
        gs2, gsa = np.zeros((tail, nh)), np.zeros((tail, nh))
        for r, t in enumerate(range(t0, T)):
            js = pos[pairs(np.full(T, t), pos)]       # row t as the query
            is_ = pos[pairs(pos, np.full(T, t))]      # row t as the key
            for hi, hq in enumerate(heads):
                kv = hq // grp
                dec = np.exp(G[t, hq][None, :] - G[js, hq])
                x = scale * (q[t, hq][None, :] * k[js, kv] * dec).sum(axis=1) + Gs[t, hq] - Gs[js, hq]
                p = np.exp(x - lse[t, hq])
                dP = v[js, kv] @ do[t, hq]
                ds = p * (dP - delta[t, hq])
                tq = q[t, hq][None, :] * scale * ds[:, None] * k[js, kv] * dec
                tqa = np.abs(q[t, hq])[None, :] * scale * (p * (np.abs(dP) + np.abs(delta[t, hq])))[:, None] * k[js, kv] * dec
                dec = np.exp(G[is_, hq] - G[t, hq][None, :])
                x = scale * (q[is_, hq] * k[t, kv][None, :] * dec).sum(axis=1) + Gs[is_, hq] - Gs[t, hq]
                p2 = np.exp(x - lse[is_, hq])
                dP2 = do[is_, hq] @ v[t, kv]
                ds2 = p2 * (dP2 - delta[is_, hq])
                tk = k[t, kv][None, :] * scale * ds2[:, None] * q[is_, hq] * dec
                tka = np.abs(k[t, kv])[None, :] * scale * (p2 * (np.abs(dP2) + np.abs(delta[is_, hq])))[:, None] * q[is_, hq] * dec
                dG[r, hi] = tq.sum(axis=0) - tk.sum(axis=0)
                dGs[r, hi] = ds.sum() - ds2.sum()
                gq2[r, hi] = (tq * tq).sum(axis=0) + (tk * tk).sum(axis=0)
                gqa[r, hi] = (tqa * tqa).sum(axis=0) + (tka * tka).sum(axis=0)
                gs2[r, hi] = (ds * ds).sum() + (ds2 * ds2).sum()
                da = p * (np.abs(dP) + np.abs(delta[t, hq]))
                da2 = p2 * (np.abs(dP2) + np.abs(delta[is_, hq]))
                gsa[r, hi] = (da * da).sum() + (da2 * da2).sum()
        rev = lambda a: np.cumsum(a[::-1], axis=0)[::-1]
        out["dg"] = rev(dG)
        s2["dg"], sa["dg"] = rev(gq2), rev(gqa)
        if gs is not None:
            out["dg_scalar"] = rev(dGs)
            s2["dg_scalar"], sa["dg_scalar"] = rev(gs2), rev(gsa)
    out["sigma"] = {n: np.sqrt(a) for n, a in s2.items()}
    out["sigma_abs"] = {n: np.sqrt(a) for n, a in sa.items()}
    return out
