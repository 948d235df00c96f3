"""Prefill backward at the long-prefill workload's full size (B=1, T=8192, HQ=32,
H=8, K=V=128, bf16, decaying g and the scalar gate), in the launch configuration the
benchmark times.

The full oracle is far too slow at this size, so the check is twofold:
  - where the oracle can compute one row at a time (``oracle.wall_bwd_rows``, numpy
    double, pinned to the full oracle in test_oracle_bwd_pins.py): dq at sampled query
    rows, dk and dv at sampled key rows (block edges, the first and last rows, middle
    rows), from the same o and lse, within the per-element sigma bound of test_gpu_bwd;
  - a property that holds at any size: every row's weights sum to 1 (no sink in this
    workload), so sum_j dv_j equals the sum of dO over all rows and the group's query
    heads, per KV head and channel;
  - dg and dg_scalar, the reverse prefix sums that cross all 64 row blocks: at the last
    160 rows (across the last block boundary) against the row oracle for four query
    heads, and at row 0, where they are exactly zero (the scores depend on G and Gs only
    through differences), so what remains there is the rounding of the whole chain.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.test_gpu_bwd import assert_grad_close

pytestmark = pytest.mark.gpu


def test_long_prefill_backward_sampled_rows():
    import decayed_softmax_attention_b200 as wall
    spec = W.PREFILL["long"]
    d = W.gen_prefill(spec, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(spec.seed + 7)
    do = torch.randn(d["q"].shape[:3] + (spec.V,), generator=gen, device="cuda").to(torch.bfloat16)
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                d["window"], d["cu_seqlens"], d["scale"], return_lse=True)
    got = wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, do, d["g_scalar"],
                             d["sink_bias"], d["window"], d["cu_seqlens"], d["scale"])
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    T = spec.T
    q_rows = [0, 1, 127, 128, 255, 4095, 5000, T - 1]
    k_rows = [0, 127, 128, 2049, 4096, T - 129, T - 2, T - 1]
    ref = oracle.wall_bwd_rows(d["q"], d["k"], d["v"], d["g"], do, o, lse, q_rows=q_rows,
                               k_rows=k_rows, g_scalar=d["g_scalar"], window=d["window"],
                               scale=d["scale"])
    for name, rows in (("dq", q_rows), ("dk", k_rows), ("dv", k_rows)):
        assert_grad_close(got[name][0, rows], ref[name], ref["sigma"][name],
                          ref["sigma_abs"][name], torch.bfloat16, f"full size {name}")
    # sum over all key rows of dv = sum over rows and the group's query heads of dO
    assert d["sink_bias"] is None  # no sink in this workload: every row's weights sum to 1
    dv = got["dv"][0].double()                                         # [T, H, V]
    want = do[0].double().reshape(T, spec.H, spec.HQ // spec.H, spec.V).sum(dim=(0, 2))
    have = dv.sum(dim=0)
    scale = dv.pow(2).sum(dim=0).sqrt()                                # per-element rounding scale
    err = (have - want).abs()
    bound = 10 * 2.0 ** -8 * scale + 1e-3 * want.abs()
    assert bool((err <= bound).all()), (
        f"sum_j dv_j vs sum dO: max err {float(err.max()):.3e}, "
        f"max bound {float(bound.max()):.3e}")

    # dg, dg_scalar at the last rows (they sum dG over the rows after them only)
    tail, heads = 160, [0, 9, 18, 31]
    rt = oracle.wall_bwd_rows(d["q"], d["k"], d["v"], d["g"], do, o, lse, tail=tail,
                              tail_heads=heads, g_scalar=d["g_scalar"], window=d["window"],
                              scale=d["scale"])
    for name, sl in (("dg", (0, slice(T - tail, T), heads)),
                     ("dg_scalar", (0, slice(T - tail, T), heads))):
        assert_grad_close(got[name][sl], rt[name], rt["sigma"][name], rt["sigma_abs"][name],
                          torch.bfloat16, f"full size {name} (last {tail} rows)")
    # row 0: zero in exact arithmetic; the sum of every row's dG, through all block carries
    dg0 = got["dg"][0, 0].double()                                     # [HQ, K]
    qdq = (d["q"][0].double() * got["dq"][0].double())                 # [T, HQ, K]
    s_dg = qdq.pow(2).sum(dim=0).sqrt()                                # rounding scale
    assert bool((dg0.abs() <= 0.05 * s_dg + 1e-6).all()), (
        f"dg at row 0: max |dg| {float(dg0.abs().max()):.3e} vs scale {float(s_dg.max()):.3e}")
    dgs = got["dg_scalar"][0].double()                                 # [T, HQ]
    steps = torch.cat([dgs[:-1] - dgs[1:], dgs[-1:]], dim=0)           # per-row dGs (rounded)
    s_gs = steps.pow(2).sum(dim=0).sqrt()
    assert bool((dgs[0].abs() <= 0.05 * s_gs + 1e-6).all()), (
        f"dg_scalar at row 0: max {float(dgs[0].abs().max()):.3e} vs scale {float(s_gs.max()):.3e}")
