"""Pins for the CPU oracle, independent of the oracle's own formulation.

Every check here compares the oracle with something the Wall Attention README
(intro, "Usage", "Decode", "Tests" sections) or plain mathematics fixes:
  - g = 0 reduces to vanilla causal softmax attention (README intro), checked
    against a textbook dense softmax written with numpy matrix ops;
  - brute force on T <= 12 in pure Python, with the accumulated decay formed as
    a product of per-step factors exp(g_u) (no cumulative sum at all);
  - a two-token example worked by hand (fixes the inclusive-sum convention and
    the direction of the decay);
  - invariants: row weights plus sink mass sum to one, shifting g at a document
    start changes nothing, packing equals separate documents, GQA equals MHA
    with repeated K/V, window and sink limits, the pure-FoX special case;
  - the decode cache of the README's "Decode" section: any anchor choice leaves
    the decode unchanged and decode equals the prefill row, token by token.
"""
import math

import numpy as np
import pytest

import oracle

RTOL = 1e-11
ATOL = 1e-11


def _rand(rng, *shape):
    return rng.standard_normal(shape).astype(np.float32)


def _inputs(seed, B=1, T=20, HQ=4, H=2, K=8, V=6, gscale=0.3, gs=False, sink=False):
    rng = np.random.default_rng(seed)
    d = dict(q=_rand(rng, B, T, HQ, K), k=_rand(rng, B, T, H, K), v=_rand(rng, B, T, H, V),
             g=(gscale * _rand(rng, B, T, HQ, K)).astype(np.float32))
    d["g_scalar"] = (-np.abs(_rand(rng, B, T, HQ)) * 0.5).astype(np.float32) if gs else None
    d["sink_bias"] = _rand(rng, HQ) if sink else None
    return d


# ---------------------------------------------------------------- textbook g = 0
def _dense_softmax_attention(q, k, v, scale, window=0, cu=None):
    """Vanilla causal softmax attention, dense masked matrices (float64)."""
    B, T, HQ, K = q.shape
    H = k.shape[2]
    grp = HQ // H
    doc = np.zeros(T, dtype=np.int64)
    if cu is not None:
        for d in range(len(cu) - 1):
            doc[cu[d]:cu[d + 1]] = d
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    allowed = (j <= i) & (doc[:, None] == doc[None, :])
    if window > 0:
        allowed &= (i - j) < window
    o = np.zeros((B, T, HQ, v.shape[3]))
    lse = np.zeros((B, T, HQ))
    for b in range(B):
        for h in range(HQ):
            qq = q[b, :, h, :].astype(np.float64)
            kk = k[b, :, h // grp, :].astype(np.float64)
            vv = v[b, :, h // grp, :].astype(np.float64)
            logits = np.where(allowed, scale * qq @ kk.T, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            z = e.sum(axis=1, keepdims=True)
            o[b, :, h, :] = (e / z) @ vv
            lse[b, :, h] = (m + np.log(z))[:, 0]
    return o, lse


@pytest.mark.parametrize("case", [
    dict(B=2, T=37, HQ=4, H=2, window=0, cu=None),
    dict(B=1, T=50, HQ=3, H=1, window=7, cu=None),
    dict(B=1, T=45, HQ=2, H=2, window=0, cu=[0, 1, 13, 30, 45]),
    dict(B=1, T=45, HQ=4, H=4, window=5, cu=[0, 20, 45]),
])
def test_g_zero_is_vanilla_softmax_attention(case):
    d = _inputs(1, B=case["B"], T=case["T"], HQ=case["HQ"], H=case["H"])
    g0 = np.zeros_like(d["g"])
    scale = 0.37
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], g0, window=case["window"],
                             cu_seqlens=case["cu"], scale=scale)
    o_ref, lse_ref = _dense_softmax_attention(d["q"], d["k"], d["v"], scale, case["window"],
                                              case["cu"])
    np.testing.assert_allclose(o, o_ref, rtol=RTOL, atol=ATOL)
    np.testing.assert_allclose(lse, lse_ref, rtol=RTOL, atol=ATOL)


# ---------------------------------------------------------------- brute force
def _brute(q, k, v, g, gs, sink, window, cu, scale):
    """Pure-Python loops; decay as a product of per-step factors exp(g_u)."""
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    grp = HQ // H
    starts = [0] * T
    if cu is not None:
        for d in range(len(cu) - 1):
            for t in range(cu[d], cu[d + 1]):
                starts[t] = cu[d]
    o = np.zeros((B, T, HQ, V))
    lse = np.zeros((B, T, HQ))
    for b in range(B):
        for h in range(HQ):
            kv = h // grp
            for i in range(T):
                keys = [j for j in range(starts[i], i + 1) if window <= 0 or i - j < window]
                logits = []
                for j in keys:
                    terms = []
                    for n in reversed(range(K)):
                        decay = math.prod(math.exp(float(g[b, u, h, n])) for u in range(j + 1, i + 1))
                        terms.append(float(q[b, i, h, n]) * float(k[b, j, kv, n]) * decay)
                    x = scale * math.fsum(terms)
                    if gs is not None:
                        x += math.fsum(float(gs[b, u, h]) for u in range(j + 1, i + 1))
                    logits.append(x)
                extra = [float(sink[h])] if sink is not None else []
                m = max(logits + extra)
                w = [math.exp(x - m) for x in logits]
                z = math.fsum(w + [math.exp(s - m) for s in extra])
                for c in range(V):
                    o[b, i, h, c] = math.fsum(wj * float(v[b, j, kv, c]) for wj, j in zip(w, keys)) / z
                lse[b, i, h] = m + math.log(z)
    return o, lse


@pytest.mark.parametrize("case", [
    dict(seed=2, B=1, T=12, HQ=2, H=1, K=3, V=2, gs=True, sink=True, window=0, cu=None),
    dict(seed=3, B=2, T=9, HQ=2, H=2, K=4, V=3, gs=False, sink=False, window=4, cu=None),
    dict(seed=4, B=1, T=11, HQ=4, H=2, K=2, V=2, gs=True, sink=False, window=3, cu=[0, 5, 6, 11]),
    dict(seed=5, B=1, T=10, HQ=1, H=1, K=5, V=1, gs=False, sink=True, window=0, cu=[0, 4, 10]),
])
def test_brute_force_small(case):
    d = _inputs(case["seed"], B=case["B"], T=case["T"], HQ=case["HQ"], H=case["H"], K=case["K"],
                V=case["V"], gscale=0.8, gs=case["gs"], sink=case["sink"])
    scale = 0.6
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             window=case["window"], cu_seqlens=case["cu"], scale=scale)
    o_ref, lse_ref = _brute(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                            case["window"], case["cu"], scale)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- worked by hand
def test_two_token_worked_example():
    """T=2, K=V=1, scale=1.  Row 1 sees key 0 through the decay exp(g[1]) only.

    q1 = 1, k0 = 2, k1 = 0, g1 = ln(1/2)  =>  x10 = 1*2*0.5 = 1, x11 = 0,
    o1 = (e*v0 + v1) / (e + 1), lse1 = ln(e + 1).  g0 (= 5) must not matter: the
    decay between j and i sums g over (j, i] only.
    """
    q = np.array([0.0, 1.0], np.float32).reshape(1, 2, 1, 1)
    k = np.array([2.0, 0.0], np.float32).reshape(1, 2, 1, 1)
    v = np.array([3.0, -1.0], np.float32).reshape(1, 2, 1, 1)
    g = np.array([5.0, math.log(0.5)], np.float32).reshape(1, 2, 1, 1)
    o, lse = oracle.wall_fwd(q, k, v, g, scale=1.0)
    e = math.e
    g1 = float(np.float32(math.log(0.5)))
    x10 = 2.0 * math.exp(g1)
    assert abs(x10 - 1.0) < 1e-7
    assert o[0, 0, 0, 0] == pytest.approx(3.0, abs=1e-15)          # row 0 sees only itself
    assert o[0, 1, 0, 0] == pytest.approx((math.exp(x10) * 3.0 - 1.0) / (math.exp(x10) + 1.0), rel=1e-14)
    assert lse[0, 1, 0] == pytest.approx(math.log(math.exp(x10) + 1.0), rel=1e-14)
    assert abs(o[0, 1, 0, 0] - (e * 3 - 1) / (e + 1)) < 1e-6


def test_constant_decay_closed_form():
    """K=1, g = gamma everywhere: the decay between j <= i is exp(gamma*(i-j))."""
    T, gamma, scale = 9, -0.45, 0.8
    rng = np.random.default_rng(7)
    q = _rand(rng, 1, T, 1, 1)
    k = _rand(rng, 1, T, 1, 1)
    v = _rand(rng, 1, T, 1, 1)
    g = np.full((1, T, 1, 1), gamma, np.float32)
    gam = float(np.float32(gamma))
    o, _ = oracle.wall_fwd(q, k, v, g, scale=scale)
    for i in range(T):
        x = np.array([scale * float(q[0, i, 0, 0]) * float(k[0, j, 0, 0]) * math.exp(gam * (i - j))
                      for j in range(i + 1)])
        w = np.exp(x - x.max())
        ref = float((w * v[0, :i + 1, 0, 0].astype(np.float64)).sum() / w.sum())
        assert o[0, i, 0, 0] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    # the opposite decay direction gives a different answer (the pin is sensitive to sign)
    o_flip, _ = oracle.wall_fwd(q, k, v, -g, scale=scale)
    assert np.max(np.abs(o_flip - o)) > 1e-3


# ---------------------------------------------------------------- invariants
def test_weights_sum_to_one_with_sink():
    """One-hot values make o the weight row; weights plus sink mass sum to 1."""
    T, HQ = 30, 2
    rng = np.random.default_rng(11)
    q = _rand(rng, 1, T, HQ, 4)
    k = _rand(rng, 1, T, 1, 4)
    g = (0.5 * _rand(rng, 1, T, HQ, 4)).astype(np.float32)
    gs = (-np.abs(_rand(rng, 1, T, HQ))).astype(np.float32)
    sink = np.array([0.7, -1.3], np.float32)
    v = np.eye(T, dtype=np.float32).reshape(1, T, 1, T)
    o, lse = oracle.wall_fwd(q, k, v, g, gs, sink, window=11)
    w = o[0]                                          # [T, HQ, T]
    sink_mass = np.exp(sink[None, :].astype(np.float64) - lse[0])
    np.testing.assert_allclose(w.sum(axis=2) + sink_mass, 1.0, rtol=0, atol=1e-13)
    i = np.arange(T)[:, None, None]
    j = np.arange(T)[None, None, :]
    assert np.all(w[np.broadcast_to((j > i) | (i - j >= 11), w.shape)] == 0.0)
    assert np.all(w >= 0.0)


def test_shift_of_g_at_document_start_is_invisible():
    d = _inputs(12, T=40, gs=True, sink=True)
    cu = [0, 17, 40]
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             cu_seqlens=cu)
    g2 = d["g"].copy()
    gs2 = d["g_scalar"].copy()
    for s in cu[:-1]:
        g2[:, s] += 3.0
        gs2[:, s] -= 2.0
    o2, lse2 = oracle.wall_fwd(d["q"], d["k"], d["v"], g2, gs2, d["sink_bias"], cu_seqlens=cu)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-12)


def test_packing_equals_separate_documents():
    d = _inputs(13, T=50, gs=True, sink=True)
    cu = [0, 1, 19, 33, 50]
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             window=9, cu_seqlens=cu)
    for s, e in zip(cu[:-1], cu[1:]):
        sl = slice(s, e)
        od, ld = oracle.wall_fwd(d["q"][:, sl], d["k"][:, sl], d["v"][:, sl], d["g"][:, sl],
                                 d["g_scalar"][:, sl], d["sink_bias"], window=9)
        np.testing.assert_allclose(o[:, sl], od, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[:, sl], ld, rtol=1e-12, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    d = _inputs(14, B=2, T=33, HQ=6, H=2, gs=True, sink=True)
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"])
    k_rep = np.repeat(d["k"], 3, axis=2)
    v_rep = np.repeat(d["v"], 3, axis=2)
    o2, lse2 = oracle.wall_fwd(d["q"], k_rep, v_rep, d["g"], d["g_scalar"], d["sink_bias"])
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13, atol=1e-13)


def test_window_limits():
    d = _inputs(15, T=25, gs=True)
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"])
    o_w, lse_w = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], window=25)
    np.testing.assert_array_equal(o_w, o)
    np.testing.assert_array_equal(lse_w, lse)
    o1, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], window=1)
    v_q = np.repeat(d["v"], 2, axis=2).astype(np.float64)    # HQ=4, H=2
    np.testing.assert_allclose(o1, v_q, rtol=1e-15, atol=0)


def test_sink_limit_equals_no_sink():
    d = _inputs(16, T=21, gs=True)
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"])
    sink = np.full(4, -1e30, np.float32)
    o2, lse2 = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], sink)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(lse2, lse)


def test_zero_query_gives_pure_fox_weights():
    """q = 0 removes the dot product: logits are Gs[i] - Gs[j] (FoX forgetting gate)."""
    T = 16
    rng = np.random.default_rng(17)
    q = np.zeros((1, T, 1, 4), np.float32)
    k = _rand(rng, 1, T, 1, 4)
    g = _rand(rng, 1, T, 1, 4)
    gs = (-np.abs(_rand(rng, 1, T, 1))).astype(np.float32)
    v = np.eye(T, dtype=np.float32).reshape(1, T, 1, T)
    o, _ = oracle.wall_fwd(q, k, v, g, gs)
    cum = np.cumsum(gs[0, :, 0].astype(np.float64))
    for i in range(T):
        w = np.exp(-(cum[:i + 1] - cum[i]))          # forget gate product over (j, i]
        np.testing.assert_allclose(o[0, i, 0, :i + 1], w / w.sum(), rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- decode cache
def test_cache_prefix_and_anchor_rows():
    rng = np.random.default_rng(18)
    B, T, HQ, H, K, C = 2, 70, 4, 2, 8, 16
    k = _rand(rng, B, T, H, K)
    g = (-np.abs(0.3 * _rand(rng, B, T, HQ, K))).astype(np.float32)
    kt, r, P = oracle.kv_cache(k, g, chunk=C)
    np.testing.assert_allclose(P, np.cumsum(g.astype(np.float64), axis=1) / np.log(2.0),
                               rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(r, P[:, ::C])               # chunk-start anchors
    k_q = np.repeat(k, HQ // H, axis=2).astype(np.float64)
    np.testing.assert_array_equal(kt[:, ::C], k_q[:, ::C])    # anchor row keeps its key
    # g <= 0: the chunk-start anchor lies above every later prefix, so keys only grow
    assert np.all(np.abs(kt) >= np.abs(k_q) * (1 - 1e-15))


@pytest.mark.parametrize("random_anchors", [False, True])
def test_decode_cache_equals_prefill_rows(random_anchors):
    """Decode at step t over cache rows [0, t] equals prefill row t (README "Tests")."""
    rng = np.random.default_rng(19 + int(random_anchors))
    B, T, HQ, H, K, V, C = 2, 75, 4, 2, 8, 5, 16
    q = _rand(rng, B, T, HQ, K)
    k = _rand(rng, B, T, H, K)
    v = _rand(rng, B, T, H, V)
    g = (-np.abs(0.4 * _rand(rng, B, T, HQ, K))).astype(np.float32)
    sink = _rand(rng, HQ)
    nc = (T + C - 1) // C
    anchors = 20.0 * rng.standard_normal((B, nc, HQ, K)) if random_anchors else None
    kt, r, P = oracle.kv_cache(k, g, chunk=C, anchors=anchors)
    o_pre, lse_pre = oracle.wall_fwd(q, k, v, g, sink_bias=sink)
    for t in range(T - 20, T):
        o, lse = oracle.decode_from_cache(q[:, t], P[:, t], v, kt, r, T_kv=t + 1, sink_bias=sink,
                                          chunk=C)
        np.testing.assert_allclose(o, o_pre[:, t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse, lse_pre[:, t], rtol=1e-10, atol=1e-12)


def test_plausible_mistakes_are_caught():
    """Planted mistakes in a copy of the inputs must move the oracle away from its pins."""
    d = _inputs(21, T=10, HQ=2, H=1, K=3, V=2, gscale=0.8)
    o, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], scale=0.6)
    # exclusive instead of inclusive prefix == shifting g by one step
    g_shift = np.concatenate([np.zeros_like(d["g"][:, :1]), d["g"][:, :-1]], axis=1)
    o_shift, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], g_shift, scale=0.6)
    assert np.max(np.abs(o_shift - o)) > 1e-3
    # transposed GQA map (kv = hq % H) differs once H > 1
    d2 = _inputs(22, T=10, HQ=4, H=2, K=3, V=2, gscale=0.8)
    o2, _ = oracle.wall_fwd(d2["q"], d2["k"], d2["v"], d2["g"])
    k_alt = d2["k"][:, :, [0, 1, 0, 1]]
    v_alt = d2["v"][:, :, [0, 1, 0, 1]]
    o_alt, _ = oracle.wall_fwd(d2["q"], k_alt, v_alt, d2["g"])
    k_rep = d2["k"][:, :, [0, 0, 1, 1]]
    v_rep = d2["v"][:, :, [0, 0, 1, 1]]
    o_rep, _ = oracle.wall_fwd(d2["q"], k_rep, v_rep, d2["g"])
    np.testing.assert_allclose(o_rep, o2, rtol=1e-13, atol=1e-13)
    assert np.max(np.abs(o_alt - o2)) > 1e-3


def test_decode_with_gate_equals_prefill_rows_with_g_scalar():
    """The scalar gate in decode: PS = cumsum(g_scalar)/ln2 per row, the logit gains
    (PS_t - PS_j) ln 2; decode at step t equals the prefill row t with g_scalar (README
    "Tests": decode == prefill), with and without a sink."""
    rng = np.random.default_rng(23)
    B, T, HQ, H, K, V, C = 2, 70, 4, 2, 8, 5, 16
    q, k, v = _rand(rng, B, T, HQ, K), _rand(rng, B, T, H, K), _rand(rng, B, T, H, V)
    g = (-np.abs(0.4 * _rand(rng, B, T, HQ, K))).astype(np.float32)
    gs = (-np.abs(0.7 * _rand(rng, B, T, HQ))).astype(np.float32)
    kt, r, P = oracle.kv_cache(k, g, chunk=C)
    PS = oracle.gate_cache(gs)
    np.testing.assert_allclose(PS[:, -1] * np.log(2.0), gs.astype(np.float64).sum(axis=1),
                               rtol=1e-12)
    for sink in (None, _rand(rng, HQ)):
        o_pre, lse_pre = oracle.wall_fwd(q, k, v, g, gs, sink_bias=sink)
        for t in (0, 17, 33, T - 1):
            o, lse = oracle.decode_from_cache(q[:, t], P[:, t], v, kt, r, T_kv=t + 1,
                                              sink_bias=sink, chunk=C, gs_curr=PS[:, t],
                                              gs_cache=PS)
            np.testing.assert_allclose(o, o_pre[:, t], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(lse, lse_pre[:, t], rtol=1e-10, atol=1e-12)
        # without the gate terms the decode no longer matches (the gate matters here)
        o, _ = oracle.decode_from_cache(q[:, T - 1], P[:, T - 1], v, kt, r, T_kv=T,
                                        sink_bias=sink, chunk=C)
        assert np.abs(o - o_pre[:, T - 1]).max() > 1e-3
