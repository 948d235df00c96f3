"""Chunked prefill / multi-token decode against the cache (wall_attn_chunk).

A sequence fed in chunks (each chunk's keys appended to the decode cache, its
queries attending cache rows 0 .. t0 + i) must reproduce the prefill of the
whole sequence row for row (the oracle's rows), whatever the chunk sizes: a
single token (multi-token decode with M = 1), sizes that are not multiples
of the 128-row tiles, and chunks that start inside an anchor chunk.  The cache
buffers start as NaN, so a read of a row past the rows in use would show.

A few tokens per sequence (at most 2 * 16 / group: multi-token decode, e.g.
speculative verification) take the split-KV pass instead of the tensor-core
query tiles; FEW_CASES run every group size on both sides of that bound, with
one and two token groups per CTA, a partly filled second group, windows that
skip whole anchor chunks and enough prefix chunks for several splits.

fp32 caches take the split-KV pass for chunks of every length (F32_CASES):
chunks spanning several 256-row query blocks, every group size, windows, the
scalar gate and wide blocks (strong decay) inside a long chunk.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import ORACLE_THREADS, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wall():
    import decayed_softmax_attention_b200 as w
    w.load_library()
    return w


CASES = [
    dict(B=2, sizes=(300, 129, 1, 270), HQ=8, H=2, K=128, V=128, C=64, window=0, sink=True),
    dict(B=1, sizes=(1, 511, 2, 64), HQ=4, H=1, K=64, V=128, C=32, window=0, sink=False),
    dict(B=2, sizes=(200, 333, 17), HQ=4, H=2, K=128, V=64, C=128, window=150, sink=True),
    dict(B=1, sizes=(640,), HQ=16, H=2, K=128, V=128, C=64, window=0, sink=True),
]


# (group HQ / H: tokens per split-KV CTA 16 / group; chunks up to twice that take the split pass)
FEW_CASES = [
    dict(B=2, sizes=(700, 4, 8, 1, 7, 9, 3), HQ=8, H=2, K=128, V=128, C=64, window=0, sink=True),
    dict(B=1, sizes=(517, 16, 32, 5, 33), HQ=2, H=2, K=64, V=64, C=32, window=0, sink=False),
    dict(B=2, sizes=(300, 8, 16, 3), HQ=4, H=2, K=128, V=64, C=128, window=200, sink=True),
    dict(B=1, sizes=(450, 3, 4, 2, 5), HQ=8, H=1, K=64, V=128, C=64, window=0, sink=True),
    dict(B=3, sizes=(333, 1, 2, 1, 3), HQ=16, H=1, K=128, V=128, C=64, window=100, sink=False),
]


def _ids(c):
    return "-".join(map(str, c["sizes"])) + f"C{c['C']}G{c['HQ'] // c['H']}"


@pytest.mark.parametrize("case", CASES + FEW_CASES, ids=_ids)
def test_chunks_reproduce_the_prefill(wall, case):
    B, HQ, H, K, V, C = case["B"], case["HQ"], case["H"], case["K"], case["V"], case["C"]
    T = sum(case["sizes"])
    spec = W.PrefillSpec("chunk", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="negsoftplus", sink=case["sink"], window=case["window"], seed=101)
    d = W.gen_prefill(spec, device="cuda")
    cap = T + 37
    nan = float("nan")
    kt = torch.full((B, cap, HQ, K), nan, dtype=torch.bfloat16, device="cuda")
    rc = torch.full((B, (cap + C - 1) // C, HQ, K), nan, dtype=torch.float32, device="cuda")
    p = torch.full((B, HQ, K), nan, dtype=torch.float32, device="cuda")
    vc = torch.full((B, cap, H, V), nan, dtype=torch.bfloat16, device="cuda")
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                             window=d["window"], scale=d["scale"], threads=ORACLE_THREADS)
    t0 = 0
    for M in case["sizes"]:
        sl = slice(t0, t0 + M)
        vc[:, sl].copy_(d["v"][:, sl])
        lse = torch.empty((B, M, HQ), dtype=torch.float32, device="cuda")
        o = wall.wall_attn_chunk(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                                 d["g"][:, sl].contiguous(), kt, rc, p, vc, t0,
                                 sink_bias=d["sink_bias"], window=d["window"], scale=d["scale"],
                                 chunk=C, lse=lse)
        torch.cuda.synchronize()
        assert wall.wall_device_error() == 0
        assert_close(o, ro[:, sl], torch.bfloat16, f"chunk at {t0} (M={M})")
        assert_close(lse, rl[:, sl], torch.bfloat16, f"chunk lse at {t0} (M={M})")
        t0 += M
    # the cache the chunks built equals the oracle's
    ktr, _, P = oracle.kv_cache(d["k"], d["g"], chunk=C, threads=ORACLE_THREADS)
    assert_close(kt[:, :T], ktr, torch.bfloat16, "cache built by the chunks")
    np.testing.assert_allclose(p.double().cpu().numpy(), P[:, -1], rtol=1e-4, atol=1e-3)


def test_chunk_then_decode(wall):
    """A chunked prefill followed by single-token decode steps on the same cache."""
    B, HQ, H, K, V, C = 2, 8, 2, 128, 128, 64
    T0, S = 450, 6
    T = T0 + S
    spec = W.PrefillSpec("chunk_dec", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="negsoftplus", sink=True, seed=102)
    d = W.gen_prefill(spec, device="cuda")
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=torch.bfloat16, chunk=C)
    cache.v[:, :T0].copy_(d["v"][:, :T0])
    wall.wall_attn_chunk(d["q"][:, :T0].contiguous(), d["k"][:, :T0].contiguous(),
                         d["g"][:, :T0].contiguous(), cache.k_tilde, cache.r_cache, cache.p,
                         cache.v, 0, sink_bias=d["sink_bias"], scale=d["scale"], chunk=C)
    cache.length = T0
    rows = np.array([b * T + t for b in range(B) for t in range(T0, T)], dtype=np.int64)
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                            scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    ro = ro.reshape(B, S, HQ, V)
    for s_ in range(S):
        t = T0 + s_
        cache.append(d["k"][:, t:t + 1].contiguous(), d["g"][:, t:t + 1].contiguous(),
                     d["v"][:, t:t + 1].contiguous())
        o = cache.decode(d["q"][:, t:t + 1].contiguous(), sink_bias=d["sink_bias"],
                         scale=d["scale"])
        assert_close(o[:, 0], ro[:, s_], torch.bfloat16, f"decode after chunk, step {s_}")


GATED_CASES = [
    dict(B=2, sizes=(300, 129, 1, 270), HQ=8, H=2, K=128, V=128, C=64, window=0, sink=True,
         g_kind="negsoftplus"),
    dict(B=2, sizes=(517, 4, 8, 1, 3), HQ=8, H=2, K=128, V=64, C=32, window=150, sink=False,
         g_kind="negsoftplus"),
    dict(B=1, sizes=(600, 260), HQ=4, H=1, K=64, V=128, C=32, window=0, sink=True,
         g_kind="strong_cache"),  # wide blocks: the exact in-block pass carries the gate too
]


@pytest.mark.parametrize("case", GATED_CASES, ids=_ids)
def test_gated_chunks_reproduce_the_prefill(wall, case):
    """wall_attn_chunk_gated: chunks of a sequence with the scalar gate equal the oracle's
    prefill rows with g_scalar, through the tile kernel, the few-token split pass and the
    wide-block pass; the gate cache the chunks build equals the oracle's PS."""
    B, HQ, H, K, V, C = case["B"], case["HQ"], case["H"], case["K"], case["V"], case["C"]
    T = sum(case["sizes"])
    spec = W.PrefillSpec("chunk_gate", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind=case["g_kind"], g_scalar=True, sink=case["sink"],
                         window=case["window"], seed=103)
    d = W.gen_prefill(spec, device="cuda")
    cap = T + 9
    nan = float("nan")
    kt = torch.full((B, cap, HQ, K), nan, dtype=torch.bfloat16, device="cuda")
    rc = torch.full((B, (cap + C - 1) // C, HQ, K), nan, dtype=torch.float32, device="cuda")
    p = torch.full((B, HQ, K), nan, dtype=torch.float32, device="cuda")
    vc = torch.full((B, cap, H, V), nan, dtype=torch.bfloat16, device="cuda")
    gsc = torch.full((B, cap, HQ), nan, dtype=torch.float32, device="cuda")
    gsl = torch.full((B, HQ), nan, dtype=torch.float32, device="cuda")
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             window=d["window"], scale=d["scale"], threads=ORACLE_THREADS)
    t0 = 0
    for M in case["sizes"]:
        sl = slice(t0, t0 + M)
        vc[:, sl].copy_(d["v"][:, sl])
        lse = torch.empty((B, M, HQ), dtype=torch.float32, device="cuda")
        o = wall.wall_attn_chunk(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                                 d["g"][:, sl].contiguous(), kt, rc, p, vc, t0,
                                 sink_bias=d["sink_bias"], window=d["window"], scale=d["scale"],
                                 chunk=C, lse=lse, gs_new=d["g_scalar"][:, sl].contiguous(),
                                 gs_cache=gsc, gs_last=gsl)
        torch.cuda.synchronize()
        assert wall.wall_device_error() == 0
        assert_close(o, ro[:, sl], torch.bfloat16, f"gated chunk at {t0} (M={M})")
        assert_close(lse, rl[:, sl], torch.bfloat16, f"gated chunk lse at {t0} (M={M})")
        t0 += M
    PS = oracle.gate_cache(d["g_scalar"])
    np.testing.assert_allclose(gsc[:, :T].double().cpu().numpy(), PS, rtol=2e-6, atol=2e-5)
    np.testing.assert_allclose(gsl.double().cpu().numpy(), PS[:, -1], rtol=2e-6, atol=2e-5)


F32_CASES = [
    dict(B=2, sizes=(600, 300, 1, 5), HQ=8, H=2, K=128, V=128, C=64, window=0, sink=True,
         g_kind="negsoftplus", gate=False),
    dict(B=1, sizes=(513, 2, 270), HQ=2, H=2, K=64, V=64, C=32, window=0, sink=False,
         g_kind="negsoftplus", gate=True),
    dict(B=2, sizes=(333, 444), HQ=4, H=2, K=128, V=64, C=128, window=200, sink=True,
         g_kind="negsoftplus", gate=False),
    dict(B=1, sizes=(260, 31, 600), HQ=16, H=1, K=64, V=128, C=64, window=0, sink=True,
         g_kind="negsoftplus", gate=True),
    dict(B=1, sizes=(700, 300), HQ=8, H=1, K=128, V=128, C=32, window=0, sink=False,
         g_kind="strong_cache", gate=True),  # wide blocks inside long fp32 chunks
]


@pytest.mark.parametrize("case", F32_CASES, ids=_ids)
def test_fp32_chunks_reproduce_the_prefill(wall, case):
    """wall_attn_chunk(_gated) with fp32 inputs and cache: every chunk length through the
    split-KV pass, equal to the oracle's prefill rows at the fp32 tolerance."""
    B, HQ, H, K, V, C = case["B"], case["HQ"], case["H"], case["K"], case["V"], case["C"]
    T = sum(case["sizes"])
    spec = W.PrefillSpec("chunk_f32", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="f32",
                         g_kind=case["g_kind"], g_scalar=case["gate"], sink=case["sink"],
                         window=case["window"], seed=104)
    d = W.gen_prefill(spec, device="cuda")
    cap = T + 21
    nan = float("nan")
    f32 = torch.float32
    kt = torch.full((B, cap, HQ, K), nan, dtype=f32, device="cuda")
    rc = torch.full((B, (cap + C - 1) // C, HQ, K), nan, dtype=f32, device="cuda")
    p = torch.full((B, HQ, K), nan, dtype=f32, device="cuda")
    vc = torch.full((B, cap, H, V), nan, dtype=f32, device="cuda")
    gsc = torch.full((B, cap, HQ), nan, dtype=f32, device="cuda")
    gsl = torch.full((B, HQ), nan, dtype=f32, device="cuda")
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d.get("g_scalar"), d["sink_bias"],
                             window=d["window"], scale=d["scale"], threads=ORACLE_THREADS)
    t0 = 0
    for M in case["sizes"]:
        sl = slice(t0, t0 + M)
        vc[:, sl].copy_(d["v"][:, sl])
        lse = torch.empty((B, M, HQ), dtype=f32, device="cuda")
        gate = {}
        if case["gate"]:
            gate = dict(gs_new=d["g_scalar"][:, sl].contiguous(), gs_cache=gsc, gs_last=gsl)
        o = wall.wall_attn_chunk(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                                 d["g"][:, sl].contiguous(), kt, rc, p, vc, t0,
                                 sink_bias=d["sink_bias"], window=d["window"], scale=d["scale"],
                                 chunk=C, lse=lse, **gate)
        torch.cuda.synchronize()
        assert wall.wall_device_error() == 0
        assert o.dtype == f32
        assert_close(o, ro[:, sl], f32, f"fp32 chunk at {t0} (M={M})")
        assert_close(lse, rl[:, sl], f32, f"fp32 chunk lse at {t0} (M={M})")
        t0 += M
    ktr, _, P = oracle.kv_cache(d["k"], d["g"], chunk=C, threads=ORACLE_THREADS)
    # k_tilde = k 2^(R_c - P_j) from fp32 prefixes: a rounding of P (log2 units, ulp about
    # 2^-23 |P|) moves the factor by ln 2 times it, so under strong decay (|P| in the
    # thousands) the relative bound grows with max |P|; 16 roundings of headroom
    rtol_k = 1e-4 + 16 * 2.0 ** -23 * np.log(2.0) * float(np.abs(P).max())
    got = kt[:, :T].double().cpu().numpy()
    bad = ~(np.abs(got - ktr) <= 1e-4 + rtol_k * np.abs(ktr))
    assert not bad.any(), (f"fp32 cache built by the chunks: {int(bad.sum())} outside "
                           f"rtol {rtol_k:.2e}, first {np.argwhere(bad)[:3].tolist()}")
    np.testing.assert_allclose(p.double().cpu().numpy(), P[:, -1], rtol=1e-5, atol=1e-4)


def test_four_token_chunk_full_decode_workload(wall):
    """The benchmark's multi-token decode at full size (B=32, T_kv=32768 prefix, HQ=32, H=8,
    K=V=128, C=64, 4 new tokens per sequence through the tensor-core split pass): batch rows
    0 and 31 against the oracle's prefill rows of the 4 tokens."""
    spec = W.DECODE["decode"]
    Mt = 4
    d = W.gen_decode(spec, device="cuda")
    B, T0, HQ, H, K, V = spec.B, spec.T0, spec.HQ, spec.H, spec.K, spec.V
    cache = wall.KVCache(B, spec.cap, HQ, H, K, V, dtype=torch.bfloat16, chunk=spec.C)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    sl = slice(T0, T0 + Mt)
    cache.v[:, sl].copy_(d["v"][:, sl])
    q4 = d["q"][:, :Mt].contiguous()
    lse = torch.empty((B, Mt, HQ), dtype=torch.float32, device="cuda")
    o = wall.wall_attn_chunk(q4, d["k"][:, sl].contiguous(), d["g"][:, sl].contiguous(),
                             cache.k_tilde, cache.r_cache, cache.p, cache.v, T0,
                             scale=d["scale"], chunk=spec.C, lse=lse)
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    T = T0 + Mt
    for b in (0, 31):
        qf = torch.zeros((1, T, HQ, K), dtype=torch.bfloat16)
        qf[0, sl] = q4[b].cpu()
        rows = np.arange(T0, T, dtype=np.int64)
        ro, rl = oracle.wall_fwd(qf, d["k"][b:b + 1, :T].cpu(), d["v"][b:b + 1, :T].cpu(),
                                 d["g"][b:b + 1, :T].cpu(), scale=d["scale"], rows=rows,
                                 threads=ORACLE_THREADS)
        assert_close(o[b], ro.reshape(Mt, HQ, V), torch.bfloat16, f"4-token chunk b={b}")
        assert_close(lse[b], rl.reshape(Mt, HQ), torch.bfloat16, f"4-token chunk lse b={b}")
