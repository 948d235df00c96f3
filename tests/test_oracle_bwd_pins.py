"""Pins for the oracle's backward pass, independent of its own formulation.

The backward differentiates what the Wall Attention README defines (intro and
"Usage / Training-Prefill" sections); its "code structure" and "Tests"
sections name the backward kernel and check it with finite differences.  Here:
  - central finite differences of the pure-Python brute-force forward (decay
    as a product of per-step factors exp(g_u), no prefix sums anywhere), with
    a loss L = sum(o * dO) + sum(lse * dlse), for every input including g,
    g_scalar and the sink;
  - g = 0 reduces to vanilla causal softmax attention: dq, dk, dv equal torch
    autograd through a textbook dense attention in float64;
  - invariants: shifting g (or g_scalar) at a document's first token changes
    nothing, so its gradient there is zero; sum_j dv_j = sum_t (1 - p_sink) dO_t;
  - a planted mistake in the analytic formula (on the CPU) is caught by the
    finite-difference pin.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_pins import _brute, _inputs

FD_H = 1e-5


def _loss(d, do, dlse, window, cu, scale, **over):
    a = {key: d[key] for key in ("q", "k", "v", "g", "g_scalar", "sink_bias")}
    a.update(over)
    o, lse = _brute(a["q"], a["k"], a["v"], a["g"], a["g_scalar"], a["sink_bias"], window, cu,
                    scale)
    val = float(np.sum(o * do))
    if dlse is not None:
        val += float(np.sum(lse * dlse))
    return val


def _fd_grad(d, name, do, dlse, window, cu, scale):
    base = np.asarray(d[name], dtype=np.float64)
    grad = np.zeros_like(base)
    it = np.nditer(base, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        hi = base.copy()
        lo = base.copy()
        hi[idx] += FD_H
        lo[idx] -= FD_H
        grad[idx] = (_loss(d, do, dlse, window, cu, scale, **{name: hi}) -
                     _loss(d, do, dlse, window, cu, scale, **{name: lo})) / (2 * FD_H)
    return grad


FD_CASES = [
    dict(seed=11, B=1, T=7, HQ=2, H=1, K=3, V=2, gs=True, sink=True, dlse=True, window=0, cu=None),
    dict(seed=12, B=2, T=6, HQ=2, H=2, K=2, V=3, gs=False, sink=False, dlse=False, window=3,
         cu=None),
    dict(seed=13, B=1, T=8, HQ=4, H=2, K=2, V=2, gs=True, sink=True, dlse=False, window=0,
         cu=[0, 3, 8]),
    dict(seed=14, B=1, T=8, HQ=2, H=1, K=3, V=2, gs=True, sink=False, dlse=True, window=4,
         cu=[0, 5, 6, 8]),
    # three query heads per KV head: dk, dv summed over a group of 3
    dict(seed=15, B=1, T=6, HQ=3, H=1, K=2, V=2, gs=True, sink=True, dlse=False, window=0,
         cu=[0, 2, 6]),
]


def _fd_setup(case):
    d = _inputs(case["seed"], B=case["B"], T=case["T"], HQ=case["HQ"], H=case["H"], K=case["K"],
                V=case["V"], gscale=0.5, gs=case["gs"], sink=case["sink"])
    # fp32-rounded values widened to double: the same point the oracle sees
    d = {key: (None if val is None else val.astype(np.float64)) for key, val in d.items()}
    rng = np.random.default_rng(case["seed"] + 100)
    do = rng.standard_normal((case["B"], case["T"], case["HQ"], case["V"])).astype(np.float32)
    dlse = (rng.standard_normal((case["B"], case["T"], case["HQ"])).astype(np.float32)
            if case["dlse"] else None)
    return d, do, dlse


def _analytic(d, do, dlse, case, scale, fn=None):
    fn = fn or oracle.wall_bwd
    return fn(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
              window=case["window"], cu_seqlens=case["cu"], scale=scale, dlse=dlse)


@pytest.mark.parametrize("case", FD_CASES)
def test_gradients_match_finite_differences_of_brute_force(case):
    d, do, dlse = _fd_setup(case)
    scale = 0.7
    got = _analytic(d, do, dlse, case, scale)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg")]
    if case["gs"]:
        names.append(("g_scalar", "dg_scalar"))
    if case["sink"]:
        names.append(("sink_bias", "dsink"))
    for inp, out in names:
        fd = _fd_grad(d, inp, do.astype(np.float64),
                      None if dlse is None else dlse.astype(np.float64), case["window"],
                      case["cu"], scale)
        np.testing.assert_allclose(got[out], fd, rtol=1e-6, atol=1e-7, err_msg=out)


def _textbook_grads(q, k, v, do, scale, window, cu):
    """torch autograd through dense masked softmax attention (float64), g = 0."""
    B, T, HQ, K = q.shape
    H = k.shape[2]
    grp = HQ // H
    doc = torch.zeros(T, dtype=torch.long)
    if cu is not None:
        for i in range(len(cu) - 1):
            doc[cu[i]:cu[i + 1]] = i
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (j <= i) & (doc[:, None] == doc[None, :])
    if window > 0:
        allowed &= (i - j) < window
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    qh = tq.permute(0, 2, 1, 3)
    kh = tk.permute(0, 2, 1, 3).repeat_interleave(grp, dim=1)
    vh = tv.permute(0, 2, 1, 3).repeat_interleave(grp, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=allowed,
                                                         scale=scale)
    o.backward(torch.tensor(do, dtype=torch.float64).permute(0, 2, 1, 3))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("case", [
    dict(B=2, T=33, HQ=4, H=2, window=0, cu=None),
    dict(B=1, T=40, HQ=3, H=1, window=6, cu=None),
    dict(B=1, T=41, HQ=2, H=2, window=0, cu=[0, 1, 17, 30, 41]),
])
def test_g_zero_gradients_equal_textbook_attention(case):
    d = _inputs(21, B=case["B"], T=case["T"], HQ=case["HQ"], H=case["H"], K=5, V=4)
    rng = np.random.default_rng(22)
    do = rng.standard_normal((case["B"], case["T"], case["HQ"], 4)).astype(np.float32)
    g0 = np.zeros_like(d["g"])
    got = oracle.wall_bwd(d["q"], d["k"], d["v"], g0, do, window=case["window"],
                          cu_seqlens=case["cu"], scale=0.45)
    dq, dk, dv = _textbook_grads(d["q"], d["k"], d["v"], do, 0.45, case["window"], case["cu"])
    np.testing.assert_allclose(got["dq"], dq, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(got["dk"], dk, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(got["dv"], dv, rtol=1e-10, atol=1e-11)


def test_document_start_gradients_vanish_and_value_gradients_sum():
    cu = [0, 9, 10, 31, 48]
    d = _inputs(31, B=1, T=48, HQ=4, H=2, K=6, V=5, gscale=0.4, gs=True, sink=True)
    rng = np.random.default_rng(32)
    do = rng.standard_normal((1, 48, 4, 5)).astype(np.float32)
    got = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                          cu_seqlens=cu, scale=0.5)
    big = np.abs(got["dg"]).max()
    for s in cu[:-1]:
        # g and g_scalar at a document's first token only shift every prefix of that document
        assert np.abs(got["dg"][0, s]).max() < 1e-12 * max(1.0, big)
        assert np.abs(got["dg_scalar"][0, s]).max() < 1e-12 * max(1.0, np.abs(got["dg_scalar"]).max())
    # each row's weights sum to 1 - p_sink, so sum_j dv_j = sum_t (1 - p_sink_t) dO_t per KV head
    _, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             cu_seqlens=cu, scale=0.5)
    keep = 1.0 - np.exp(d["sink_bias"][None, None, :] - lse)          # [B,T,HQ]
    want = (keep[..., None] * do).reshape(1, 48, 2, 2, 5).sum(axis=(1, 3))
    np.testing.assert_allclose(got["dv"].sum(axis=1), want, rtol=1e-11, atol=1e-11)


def test_planted_mistake_is_caught_by_finite_differences():
    """Drop the key-side decay term from the analytic dg (a plausible slip)."""
    case = FD_CASES[0]
    d, do, dlse = _fd_setup(case)
    scale = 0.7
    good = _analytic(d, do, dlse, case, scale)
    fd = _fd_grad(d, "g", do.astype(np.float64), dlse.astype(np.float64), case["window"],
                  case["cu"], scale)
    np.testing.assert_allclose(good["dg"], fd, rtol=1e-6, atol=1e-7)
    # the mistaken gradient keeps only the query-side term q * dq, prefix-summed backwards
    wrong_dG = np.asarray(d["q"]) * good["dq"]
    wrong = np.flip(np.cumsum(np.flip(wrong_dG, axis=1), axis=1), axis=1)
    assert np.abs(wrong - fd).max() > 1e-3


def test_given_forward_results_equal_recomputed_ones():
    """Passing the oracle's own o and lse changes nothing; a shifted lse scales p."""
    case = FD_CASES[2]
    d, do, dlse = _fd_setup(case)
    a = dict(window=case["window"], cu_seqlens=case["cu"], scale=0.7)
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"], **a)
    base = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"], **a)
    given = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                            o=o.astype(np.float32), lse=lse.astype(np.float32), **a)
    for name in ("dq", "dk", "dv", "dg", "dg_scalar", "dsink"):
        np.testing.assert_allclose(given[name], base[name], rtol=1e-5, atol=1e-6, err_msg=name)
    # every weight p = exp(x - lse) doubles when lse drops by ln 2: dv doubles exactly
    half = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                           o=o.astype(np.float32), lse=(lse - np.log(2.0)).astype(np.float32), **a)
    # (up to the fp32 rounding of the two lse arrays)
    np.testing.assert_allclose(half["dv"], 2.0 * given["dv"], rtol=2e-5, atol=1e-9)


@pytest.mark.parametrize("case", [
    dict(seed=41, B=2, T=37, HQ=4, H=2, K=6, V=5, gs=True, sink=True, window=0, cu=None,
         dlse=True, batch=1),
    dict(seed=42, B=1, T=45, HQ=4, H=1, K=4, V=3, gs=False, sink=False, window=9,
         cu=[0, 13, 14, 45], dlse=False, batch=0),
])
def test_row_backward_equals_full_oracle(case):
    """The numpy row backward (used at full size on the GPU machine) equals the C oracle's
    gradients and sigma scales at the sampled rows, given the same o and lse."""
    d = _inputs(case["seed"], B=case["B"], T=case["T"], HQ=case["HQ"], H=case["H"], K=case["K"],
                V=case["V"], gscale=0.3, gs=case["gs"], sink=case["sink"])
    rng = np.random.default_rng(case["seed"] + 1)
    do = rng.standard_normal((case["B"], case["T"], case["HQ"], case["V"])).astype(np.float32)
    dlse = (rng.standard_normal((case["B"], case["T"], case["HQ"])).astype(np.float32)
            if case["dlse"] else None)
    a = dict(window=case["window"], cu_seqlens=case["cu"], scale=0.6)
    o, lse = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"], **a)
    o, lse = o.astype(np.float32), lse.astype(np.float32)
    full = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                           dlse=dlse, o=o, lse=lse, scales=True, **a)
    qr, kr = [0, 1, 13, case["T"] - 2, case["T"] - 1], [0, 5, 13, 14, case["T"] - 1]
    rows = oracle.wall_bwd_rows(d["q"], d["k"], d["v"], d["g"], do, o, lse, q_rows=qr, k_rows=kr,
                                g_scalar=d["g_scalar"], dlse=dlse, batch=case["batch"], **a)
    b = case["batch"]
    # dg / dg_scalar at the last rows (the tail lies in the last document)
    tail = 9
    tr = list(range(case["T"] - tail, case["T"]))
    rt = oracle.wall_bwd_rows(d["q"], d["k"], d["v"], d["g"], do, o, lse, tail=tail,
                              g_scalar=d["g_scalar"], dlse=dlse, batch=case["batch"], **a)
    names = ["dg"] + (["dg_scalar"] if d["g_scalar"] is not None else [])
    for name in names:
        np.testing.assert_allclose(rt[name], full[name][b, tr], rtol=1e-9, atol=1e-12,
                                   err_msg=name)
        np.testing.assert_allclose(rt["sigma"][name], full["sigma"][name][b, tr], rtol=1e-9,
                                   atol=1e-12, err_msg="sigma " + name)
        np.testing.assert_allclose(rt["sigma_abs"][name], full["sigma_abs"][name][b, tr],
                                   rtol=1e-9, atol=1e-12, err_msg="sigma_abs " + name)
    for name, idx in (("dq", qr), ("dk", kr), ("dv", kr)):
        np.testing.assert_allclose(rows[name], full[name][b, idx], rtol=1e-9, atol=1e-12,
                                   err_msg=name)
        np.testing.assert_allclose(rows["sigma"][name], full["sigma"][name][b, idx], rtol=1e-9,
                                   atol=1e-12, err_msg="sigma " + name)
        np.testing.assert_allclose(rows["sigma_abs"][name], full["sigma_abs"][name][b, idx],
                                   rtol=1e-9, atol=1e-12, err_msg="sigma_abs " + name)
