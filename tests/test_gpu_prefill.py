"""GPU parity of wall_attn_fwd against the double-precision CPU oracle.

Every case draws seeded inputs (workloads.py), runs the CUDA path through the
C ABI, and compares o and lse element by element with the oracle on the same
values: all rows for sizes the oracle finishes in seconds, sampled rows for
the full-size workloads.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import ORACLE_THREADS, assert_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wall():
    import decayed_softmax_attention_b200 as w
    w.load_library()
    return w


def _run(wall, spec, rows=None):
    d = W.gen_prefill(spec, device="cuda")
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                                return_lse=True)
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                             rows=rows, threads=ORACLE_THREADS)
    if rows is None:
        return o, lse, ro, rl, spec
    B, T = spec.B, spec.T
    bi = torch.as_tensor(rows // T, device="cuda")
    ti = torch.as_tensor(rows % T, device="cuda")
    return o[bi, ti], lse[bi, ti], ro, rl, spec


def _check(res, name):
    o, lse, ro, rl, spec = res
    assert_close(o, ro, spec.torch_dtype, f"{name}: o")
    # lse is fp32 output; it carries the bf16 input rounding through the logits
    assert_close(lse, rl, spec.torch_dtype, f"{name}: lse")


@pytest.mark.parametrize("name", ["tiny", "tiny_g0", "gqa"])
def test_small_configs_all_rows(wall, name):
    _check(_run(wall, W.PREFILL[name]), name)


def test_tiny_g0_equals_vanilla_attention(wall):
    """g = 0 must reproduce vanilla causal softmax attention (README intro)."""
    spec = W.PREFILL["tiny_g0"]
    d = W.gen_prefill(spec, device="cuda")
    o = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"])
    q, k, v = (d[x].double().permute(0, 2, 1, 3) for x in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                           scale=d["scale"])
    assert_close(o, ref.permute(0, 2, 1, 3).cpu().numpy(), torch.float32, "g=0 vs SDPA")


def test_long_config_sampled_rows(wall):
    spec = W.PREFILL["long"]
    rows = sample_rows(spec.B, spec.T, extra=(255, 256, 4095, 4096, 8000), n_random=12)
    _check(_run(wall, spec, rows), "long T=8192")


def test_varlen_window_config_sampled_rows(wall):
    spec = W.PREFILL["varlen_window"]
    cu = np.cumsum((0,) + spec.docs)
    extra = []
    for s in cu[:-1]:
        extra += [int(s), int(s) + 1, int(s) + 2047, int(s) + 2048, int(s) + 2049]
    rows = sample_rows(spec.B, spec.T, extra=extra, n_random=16)
    _check(_run(wall, spec, rows), "varlen+window")


EDGE = [
    dict(T=1), dict(T=2), dict(T=127), dict(T=128), dict(T=129), dict(T=383),
    dict(T=300, window=1), dict(T=300, window=37), dict(T=300, window=128), dict(T=300, window=129),
    dict(T=300, window=5000),
    dict(T=260, docs=(1, 127, 1, 3, 128)), dict(T=515, docs=(200, 1, 314), window=64),
    dict(T=256, g_scalar=True, sink=True), dict(T=333, g_kind="negsoftplus", g_scalar=True),
    dict(T=257, K=64, V=128), dict(T=257, K=128, V=64), dict(T=200, HQ=4, H=1),
    dict(T=200, HQ=6, H=3, sink=True, window=50),
    dict(T=300, HQ=16, H=1), dict(T=200, HQ=8, H=1, window=100, g_scalar=True),
    # T a multiple of 256 (bf16 takes the TMA-staged prepass): documents, window, gate;
    # K = 64 with GQA
    dict(T=512, docs=(1, 255, 200, 56), window=100, g_scalar=True),
    dict(T=768, K=64, V=128, HQ=8, H=2, sink=True),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", EDGE, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_edge_cases(wall, dtype, case):
    base = W.PrefillSpec("edge", B=1, T=64, HQ=2, H=2, K=128, V=128, dtype=dtype, seed=77)
    c = dict(case)
    if "docs" in c:
        c["B"] = 1
    spec = replace(base, **c)
    if spec.docs is None and spec.B == 1 and "T" in c:
        spec = replace(spec, B=2)
    _check(_run(wall, spec), f"edge {case} {dtype}")


@pytest.mark.parametrize("seed", range(12))
def test_random_shapes(wall, seed):
    spec = W.random_prefill_spec(seed, dtype="bf16" if seed % 3 else "f32")
    _check(_run(wall, spec), spec.name)


def test_long_ragged_negative_decay_all_rows(wall):
    """Strong negative decay over several hundred blocks' worth of anchors (T=2000)."""
    spec = W.PrefillSpec("ragged", B=1, T=2000, HQ=4, H=2, K=128, V=128, dtype="bf16",
                         g_kind="negsoftplus", g_scalar=True, sink=True, seed=91)
    _check(_run(wall, spec), "ragged negsoftplus")


def test_repeat_calls_are_deterministic(wall):
    spec = W.PREFILL["gqa"]
    d = W.gen_prefill(spec, device="cuda")
    a = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"])
    b = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)
