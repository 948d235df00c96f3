"""GPU parity of the prefill backward (C ABI wall_attn_bwd) against the oracle.

The oracle differentiates the Wall Attention README's forward definition in
double precision (pinned by finite differences in test_oracle_bwd_pins.py).
The backward receives the forward's o and lse as inputs, so the oracle is
evaluated from the same given o and lse (its `o=`, `lse=` inputs) and every
gradient is compared element by element on the same seeded inputs.

Tolerance.  Each gradient element is a sum of many terms (dq[i] sums dS(i,j)
k[j] decay over keys, dg[u] sums the dG terms of rows u.. of the document, ...)
and the terms cancel heavily (dS sums to ~0 over a row), so an element can be
far smaller than what it sums.  The oracle returns, per element, sigma = the
root of the sum of the squared terms; rounding errors scale with sigma:
  bf16: |d| <= 10 u sigma + 2e-2 |ref|, u = 2^-8 (bf16 unit roundoff).
        Every term carries independent relative errors from its bf16 operands
        (p, dS, the rescaled q or k, the score's anchored operands): standard
        deviation <= 2u per term, so <= 2u sigma for the sum; 10 u is five
        standard deviations.  2e-2 |ref| is the forward's relative bound (it
        covers the bf16 rounding of the stored gradient).
  fp32: |d| <= 1e-4 sigma + 1e-4 |ref| (the forward's fp32 bound, sigma-scaled).
Both add 2^-18 sigma_abs: each term's factor dO.v[j] - delta is a difference of
two fp32 dot products of length V; sigma_abs takes the terms at their size
before that difference cancels (|dO.v| + |delta|), and 2^-18 covers the fp32
rounding of both products (about sqrt(V) 2^-24 each) with margin.
End to end (against the exact gradient, the forward's own rounding of o and
lse included): relative L2 error <= 2e-2 of sigma's L2 norm.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import ORACLE_THREADS

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8
BOUND = {torch.bfloat16: (10 * U_BF16, 2e-2), torch.float32: (1e-4, 1e-4)}
NAMES = ("dq", "dk", "dv", "dg", "dg_scalar", "dsink")


FP32_FLOOR = 2.0 ** -18


def assert_grad_close(got, ref, sigma, sigma_abs, dtype, what):
    a, rtol = BOUND[dtype]
    g = got.detach().double().cpu().numpy()
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    err = np.abs(g - r)
    bound = a * sigma + FP32_FLOOR * sigma_abs + rtol * np.abs(r)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside {a:.3g} sigma + {rtol}|ref|; "
            f"max err/sigma {float(np.nanmax(err / np.maximum(sigma, 1e-300))):.3e}; "
            f"first bad {idx.tolist()} got {[float(g[tuple(i)]) for i in idx]} "
            f"ref {[float(r[tuple(i)]) for i in idx]} sigma {[float(sigma[tuple(i)]) for i in idx]}")


def _run(spec, with_dlse=False, g_zero=False):
    import decayed_softmax_attention_b200 as wall
    d = W.gen_prefill(spec, device="cuda")
    if g_zero:
        d["g"] = torch.zeros_like(d["g"])
    dt = spec.torch_dtype
    gen = torch.Generator(device="cuda").manual_seed(spec.seed + 7)
    do = torch.randn(d["q"].shape[:3] + (spec.V,), generator=gen, device="cuda").to(dt)
    dlse = (torch.randn(d["q"].shape[:3], generator=gen, device="cuda")
            if with_dlse else None)
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                d["window"], d["cu_seqlens"], d["scale"], return_lse=True)
    got = wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, do, d["g_scalar"],
                             d["sink_bias"], d["window"], d["cu_seqlens"], d["scale"], dlse=dlse)
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    args = dict(window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"], dlse=dlse,
                threads=ORACLE_THREADS)
    ref = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                          o=o, lse=lse, scales=True, **args)
    exact = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], d["sink_bias"],
                            scales=True, **args)
    return got, ref, exact


def _check_all(got, ref, exact, dt, tag):
    for name in NAMES:
        if ref[name] is None:
            assert got.get(name) is None, name
            continue
        assert_grad_close(got[name], ref[name], ref["sigma"][name], ref["sigma_abs"][name], dt,
                          f"{tag}:{name}")
        # end to end, against the exact gradient
        g = got[name].detach().double().cpu().numpy()
        e = np.linalg.norm(g - exact[name]) / max(np.linalg.norm(exact["sigma"][name]), 1e-300)
        lim = 2e-2 if dt == torch.bfloat16 else 1e-4
        assert e <= lim, f"{tag}:{name} end-to-end relative L2 error {e:.3e} > {lim}"


CASES = [
    # the tiny fp32 workload (and its g = 0 vanilla special case below)
    W.PrefillSpec("bwd_tiny", B=1, T=256, HQ=2, H=2, K=64, V=64, dtype="f32", seed=11),
    # GQA, two batch rows, ragged tail
    W.PrefillSpec("bwd_gqa", B=2, T=300, HQ=8, H=4, K=64, V=64, dtype="bf16", seed=12),
    # long-prefill value distributions: decaying g and the scalar gate
    W.PrefillSpec("bwd_long", B=1, T=520, HQ=4, H=1, K=128, V=128, dtype="bf16",
                  g_kind="negsoftplus", g_scalar=True, seed=13),
    # packed documents (one of length 1) + window + sink
    W.PrefillSpec("bwd_varlen", B=1, T=518, HQ=4, H=2, K=128, V=128, dtype="bf16",
                  docs=(100, 37, 250, 1, 130), window=96, sink=True, seed=14),
    # fp32 with every option
    W.PrefillSpec("bwd_f32_all", B=1, T=333, HQ=2, H=1, K=128, V=64, dtype="f32",
                  g_kind="negsoftplus", g_scalar=True, sink=True, window=150,
                  docs=(200, 133), seed=15),
    W.PrefillSpec("bwd_k64v128", B=2, T=190, HQ=4, H=2, K=64, V=128, dtype="bf16",
                  g_scalar=True, sink=True, seed=16),
    # 3 query heads per KV head (the post pass's general group path), documents + gate
    W.PrefillSpec("bwd_group3", B=1, T=300, HQ=6, H=2, K=64, V=64, dtype="bf16",
                  g_scalar=True, docs=(90, 210), seed=17),
    # 8 query heads per KV head, ragged tail
    W.PrefillSpec("bwd_group8", B=1, T=270, HQ=8, H=1, K=128, V=128, dtype="bf16",
                  g_kind="negsoftplus", seed=18),
]


@pytest.mark.parametrize("spec", CASES, ids=lambda s: s.name)
def test_bwd_matches_oracle(spec):
    got, ref, exact = _run(spec)
    _check_all(got, ref, exact, spec.torch_dtype, spec.name)


@pytest.mark.parametrize("spec", [CASES[1], CASES[4]], ids=lambda s: s.name)
def test_bwd_with_dlse(spec):
    got, ref, exact = _run(spec, with_dlse=True)
    _check_all(got, ref, exact, spec.torch_dtype, spec.name + "+dlse")


def test_bwd_g_zero_is_vanilla():
    got, ref, exact = _run(CASES[0], g_zero=True)
    _check_all(got, ref, exact, torch.float32, "g0")


def test_bwd_document_starts_and_determinism():
    """dg vanishes at document starts (up to rounding); two runs are bit-identical."""
    import decayed_softmax_attention_b200 as wall
    spec = CASES[3]
    d = W.gen_prefill(spec, device="cuda")
    do = torch.randn(d["q"].shape[:3] + (spec.V,), device="cuda",
                     generator=torch.Generator(device="cuda").manual_seed(5)).to(torch.bfloat16)
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], None, d["sink_bias"],
                                d["window"], d["cu_seqlens"], d["scale"], return_lse=True)
    a = wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, do, None, d["sink_bias"],
                           d["window"], d["cu_seqlens"], d["scale"])
    b = wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, do, None, d["sink_bias"],
                           d["window"], d["cu_seqlens"], d["scale"])
    for name in ("dq", "dk", "dv", "dg", "dsink"):
        assert torch.equal(a[name], b[name]), name
    # exactly zero in exact arithmetic: what is left is rounding, within the parity bound
    ref = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, None, d["sink_bias"],
                          window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                          o=o, lse=lse, scales=True, threads=ORACLE_THREADS)
    dg = a["dg"].double().cpu().numpy()
    sig = ref["sigma"]["dg"]
    for s in d["cu_seqlens"][:-1].tolist():
        assert np.abs(ref["dg"][0, s]).max() <= 1e-9 * sig[0, s].max()
        assert (np.abs(dg[0, s]) <= BOUND[torch.bfloat16][0] * sig[0, s] +
                FP32_FLOOR * ref["sigma_abs"]["dg"][0, s]).all()
