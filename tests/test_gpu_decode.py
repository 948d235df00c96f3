"""GPU parity of the decode path (wall_build_kv_cache + wall_attn_decode).

Checks (Wall Attention README, "Decode" and "Tests"): the cache contents equal
the oracle's k_tilde / r_cache / P; every step of a streaming loop (append one
token, then attend) equals the oracle's prefill row for that token and the
GPU prefill row; appends of ragged sizes across chunk boundaries give the same
cache as one build; the full-size decode workload matches on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import ORACLE_THREADS, TOL, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wall():
    import decayed_softmax_attention_b200 as w
    w.load_library()
    return w


def _inputs(B, T, HQ, H, K, V, dtype, seed, sink=False):
    spec = W.PrefillSpec("dec", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype=dtype,
                         g_kind="negsoftplus", sink=sink, seed=seed)
    return spec, W.gen_prefill(spec, device="cuda")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("chunk", [32, 64, 128])
def test_cache_build_matches_oracle(wall, dtype, chunk):
    spec, d = _inputs(2, 300, 8, 2, 128, 128, dtype, seed=31)
    cache = wall.KVCache(2, 320, 8, 2, 128, 128, dtype=spec.torch_dtype, chunk=chunk)
    cache.append(d["k"], d["g"], d["v"])
    torch.cuda.synchronize()
    kt, r, P = oracle.kv_cache(d["k"], d["g"], chunk=chunk, threads=ORACLE_THREADS)
    assert_close(cache.k_tilde[:, :300], kt, spec.torch_dtype, "k_tilde")
    nc = (300 + chunk - 1) // chunk
    np.testing.assert_allclose(cache.r_cache[:, :nc].double().cpu().numpy(), r, rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(cache.p.double().cpu().numpy(), P[:, -1], rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("pieces", [(1,) * 70, (5, 59, 1, 64, 3, 100, 68), (64, 64, 64, 64, 44)])
def test_ragged_appends_equal_one_build(wall, pieces):
    T = sum(pieces)
    spec, d = _inputs(2, T, 4, 2, 64, 64, "bf16", seed=32)
    one = wall.KVCache(2, T, 4, 2, 64, 64, dtype=torch.bfloat16, chunk=64)
    one.append(d["k"], d["g"])
    many = wall.KVCache(2, T, 4, 2, 64, 64, dtype=torch.bfloat16, chunk=64)
    t = 0
    for n in pieces:
        many.append(d["k"][:, t:t + n].contiguous(), d["g"][:, t:t + n].contiguous())
        t += n
    torch.cuda.synchronize()
    kt, r, P = oracle.kv_cache(d["k"], d["g"], chunk=64)
    for c, name in ((one, "one build"), (many, "appends")):
        assert_close(c.k_tilde, kt, torch.bfloat16, f"k_tilde {name}")
        np.testing.assert_allclose(c.p.double().cpu().numpy(), P[:, -1], rtol=1e-5, atol=1e-4)
        np.testing.assert_allclose(c.r_cache.double().cpu().numpy(), r, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("dtype,B,HQ,H,K,pieces", [
    ("bf16", 1, 8, 2, 128, (37, 4000)),     # second append: partial chunk + 16 segments
    ("f32", 1, 4, 4, 64, (100, 3000, 5)),   # K = 64, fp32, a short tail append
    ("bf16", 3, 4, 1, 128, (0, 2500)),      # several batch rows, chunk-aligned start
])
def test_segmented_build_matches_oracle(wall, dtype, B, HQ, H, K, pieces):
    """Small batches split every sequence into chunk-aligned segments (segment sums,
    their prefix, then a parallel walk); the cache must equal the oracle's."""
    T = sum(pieces)
    spec, d = _inputs(B, T, HQ, H, K, K, dtype, seed=35)
    cache = wall.KVCache(B, T + 3, HQ, H, K, K, dtype=spec.torch_dtype, chunk=64)
    t = 0
    for n in pieces:
        if n:
            cache.append(d["k"][:, t:t + n].contiguous(), d["g"][:, t:t + n].contiguous())
        t += n
    torch.cuda.synchronize()
    kt, r, P = oracle.kv_cache(d["k"], d["g"], chunk=64, threads=ORACLE_THREADS)
    assert_close(cache.k_tilde[:, :T], kt, spec.torch_dtype, "k_tilde")
    nc = (T + 63) // 64
    np.testing.assert_allclose(cache.r_cache[:, :nc].double().cpu().numpy(), r, rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(cache.p.double().cpu().numpy(), P[:, -1], rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("dtype,B,T,HQ,H,K,V,chunk,gs", [
    ("bf16", 2, 1000, 8, 2, 128, 128, 64, True),
    ("f32", 1, 300, 4, 4, 64, 64, 32, False),
    ("bf16", 1, 517, 16, 4, 64, 128, 128, False),
])
def test_prefill_emits_decode_cache(wall, dtype, B, T, HQ, H, K, V, chunk, gs):
    """wall_attn_fwd(cache=...) writes the decode cache of its T rows: equal to the oracle's
    cache, the prefill output unchanged, and a decode step appended after it equal to the
    prefill row of the next token."""
    spec = W.PrefillSpec("emit", B=B, T=T + 1, HQ=HQ, H=H, K=K, V=V, dtype=dtype,
                         g_kind="negsoftplus", g_scalar=gs, seed=41)
    d = W.gen_prefill(spec, device="cuda")
    pre = {n: d[n][:, :T].contiguous() for n in ("q", "k", "v", "g")}
    gsc = d["g_scalar"][:, :T].contiguous() if gs else None
    cache = wall.KVCache(B, T + 8, HQ, H, K, V, dtype=spec.torch_dtype, chunk=chunk)
    o = wall.wall_attn_fwd(pre["q"], pre["k"], pre["v"], pre["g"], gsc, scale=d["scale"],
                           cache=cache)
    o_plain = wall.wall_attn_fwd(pre["q"], pre["k"], pre["v"], pre["g"], gsc, scale=d["scale"])
    torch.cuda.synchronize()
    assert cache.length == T
    assert torch.equal(o, o_plain)
    kt, r, P = oracle.kv_cache(pre["k"], pre["g"], chunk=chunk, threads=ORACLE_THREADS)
    assert_close(cache.k_tilde[:, :T], kt, spec.torch_dtype, "emitted k_tilde")
    nc = (T + chunk - 1) // chunk
    np.testing.assert_allclose(cache.r_cache[:, :nc].double().cpu().numpy(), r, rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(cache.p.double().cpu().numpy(), P[:, -1], rtol=1e-5, atol=1e-4)
    if not gs:  # decode has no gate term (README decode call takes none)
        cache.v[:, :T + 1].copy_(d["v"])
        cache.append(d["k"][:, T:T + 1].contiguous(), d["g"][:, T:T + 1].contiguous())
        od = cache.decode(d["q"][:, T:T + 1].contiguous(), scale=d["scale"])
        rows = [b * (T + 1) + T for b in range(B)]
        ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"], rows=rows,
                                threads=ORACLE_THREADS)
        assert_close(od[:, 0], ro, spec.torch_dtype, "decode after emitted cache")


@pytest.mark.parametrize("dtype,lens,HQ,H,K,V", [
    ("bf16", (100, 37, 200, 1, 129), 8, 2, 128, 128),
    ("f32", (64, 65, 3), 4, 4, 64, 64),
    ("bf16", (300, 5), 16, 1, 64, 128),
])
def test_decode_varlen_matches_prefill_rows(wall, dtype, lens, HQ, H, K, V):
    """Per-sequence cache lengths: batch row b attends rows [0, lens[b]) of one shared cache
    and must equal the prefill row lens[b] - 1 of its sequence."""
    B, T = len(lens), max(lens)
    spec, d = _inputs(B, T, HQ, H, K, V, dtype, seed=51, sink=True)
    cache = wall.KVCache(B, T + 4, HQ, H, K, V, dtype=spec.torch_dtype, chunk=64)
    cache.append(d["k"], d["g"], d["v"])
    _, _, P = oracle.kv_cache(d["k"], d["g"], chunk=64, threads=ORACLE_THREADS)
    p_curr = torch.tensor(np.stack([P[b, L - 1] for b, L in enumerate(lens)]),
                          dtype=torch.float32, device="cuda")[:, None].contiguous()
    q = torch.stack([d["q"][b, L - 1] for b, L in enumerate(lens)])[:, None].contiguous()
    seqlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lse = torch.empty((B, 1, HQ), dtype=torch.float32, device="cuda")
    o = wall.wall_attn_decode(q, p_curr, cache.v, cache.k_tilde, cache.r_cache, T,
                              sink_bias=d["sink_bias"], scale=d["scale"], lse=lse, seqlens=seqlens)
    rows = [b * T + L - 1 for b, L in enumerate(lens)]
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                             scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    assert_close(o[:, 0], ro, spec.torch_dtype, "varlen decode")
    np.testing.assert_allclose(lse[:, 0].double().cpu().numpy(), rl, rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("dtype,start,HQ,H,K,V,steps", [
    ("bf16", (60, 130, 1, 64), 8, 2, 128, 128, 12),
    ("f32", (31, 2), 4, 4, 64, 64, 6),
])
def test_varlen_streaming_append_and_decode(wall, dtype, start, HQ, H, K, V, steps):
    """A batch whose sequences have different lengths: per-row appends at each row's own
    position, then a per-row-length decode; every step must equal the prefill row of the
    token just appended, for every sequence."""
    B, T = len(start), max(start) + steps
    spec, d = _inputs(B, T, HQ, H, K, V, dtype, seed=61, sink=True)
    C = 64
    cap = T + 2
    dt = spec.torch_dtype
    kt = torch.zeros((B, cap, HQ, K), dtype=dt, device="cuda")
    rc = torch.zeros((B, (cap + C - 1) // C, HQ, K), dtype=torch.float32, device="cuda")
    p = torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda")
    vc = torch.zeros((B, cap, H, V), dtype=dt, device="cuda")
    for b, L in enumerate(start):  # each row's own prefix, built through a one-row view
        wall.wall_build_kv_cache(d["k"][b:b + 1, :L].contiguous(), d["g"][b:b + 1, :L].contiguous(),
                                 kt[b:b + 1], rc[b:b + 1], p[b:b + 1], chunk=C)
        vc[b, :T].copy_(d["v"][b])
    lens = list(start)
    for s_ in range(steps):
        t_pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
        k_new = torch.stack([d["k"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        g_new = torch.stack([d["g"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        wall.wall_append_kv_cache_varlen(k_new, g_new, kt, rc, p, t_pos, chunk=C)
        q = torch.stack([d["q"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        o = wall.wall_attn_decode(q, p[:, None].contiguous(), vc, kt, rc, max(lens) + 1,
                                  sink_bias=d["sink_bias"], scale=d["scale"], chunk=C,
                                  seqlens=t_pos + 1)
        rows = [b * T + L for b, L in enumerate(lens)]
        ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                                scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
        assert_close(o[:, 0], ro, dt, f"varlen step {s_}")
        lens = [L + 1 for L in lens]


STREAM = [
    dict(B=2, T0=200, steps=24, HQ=8, H=2, K=128, V=128, dtype="bf16", sink=True),
    dict(B=3, T0=130, steps=10, HQ=4, H=4, K=64, V=64, dtype="bf16", sink=False),
    dict(B=1, T0=64, steps=12, HQ=16, H=2, K=128, V=64, dtype="bf16", sink=True),
    dict(B=2, T0=100, steps=8, HQ=2, H=1, K=64, V=128, dtype="f32", sink=True),
    dict(B=2, T0=150, steps=6, HQ=16, H=1, K=64, V=128, dtype="bf16", sink=True),
    dict(B=1, T0=1, steps=5, HQ=4, H=1, K=128, V=128, dtype="bf16", sink=False),
]


@pytest.mark.parametrize("case", STREAM, ids=lambda c: f"B{c['B']}T{c['T0']}G{c['HQ']//c['H']}K{c['K']}V{c['V']}{c['dtype']}")
def test_streaming_decode_matches_prefill(wall, case):
    """Append then attend, token by token; compare with the oracle and with GPU prefill."""
    B, T0, S = case["B"], case["T0"], case["steps"]
    HQ, H, K, V = case["HQ"], case["H"], case["K"], case["V"]
    T = T0 + S
    spec, d = _inputs(B, T, HQ, H, K, V, case["dtype"], seed=33, sink=case["sink"])
    dt = spec.torch_dtype
    sink = d["sink_bias"]
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=dt, chunk=64)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    rows = np.array([b * T + t for b in range(B) for t in range(T0 - 1, T)], dtype=np.int64)
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=sink, scale=d["scale"],
                             rows=rows, threads=ORACLE_THREADS)
    ro = ro.reshape(B, S + 1, HQ, V)
    rl = rl.reshape(B, S + 1, HQ)
    o_pre, lse_pre = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=sink,
                                        scale=d["scale"], return_lse=True)
    lse = torch.empty((B, 1, HQ), dtype=torch.float32, device="cuda")
    # step 0 attends the prefix as built; then append + attend per new token
    for s in range(S + 1):
        t = T0 - 1 + s
        if s > 0:
            cache.append(d["k"][:, t:t + 1].contiguous(), d["g"][:, t:t + 1].contiguous(),
                         d["v"][:, t:t + 1].contiguous())
        q = d["q"][:, t:t + 1].contiguous()
        o = cache.decode(q, sink_bias=sink, scale=d["scale"], lse=lse)
        torch.cuda.synchronize()
        assert_close(o[:, 0], ro[:, s], dt, f"decode step {s} vs oracle")
        assert_close(lse[:, 0], rl[:, s], dt, f"decode lse step {s} vs oracle")
        # decode == prefill row (README "Tests"), both on the GPU: twice the tolerance
        atol, rtol = TOL[dt]
        diff = (o[:, 0].double() - o_pre[:, t].double()).abs()
        assert bool((diff <= 2 * atol + 2 * rtol * o_pre[:, t].double().abs()).all()), \
            f"decode step {s} vs GPU prefill: max {float(diff.max()):.3e}"
    assert wall.wall_device_error() == 0


def test_full_decode_workload_sampled(wall):
    """The decode workload (B=32, T_kv=32768 prefix, HQ=32, H=8, K=V=128, C=64):
    build the prefix, stream 3 steps, check batch rows 0 and 31 against the oracle."""
    spec = W.DECODE["decode"]
    steps = 3
    d = W.gen_decode(spec, device="cuda")
    B, T0, HQ, H, K, V = spec.B, spec.T0, spec.HQ, spec.H, spec.K, spec.V
    cache = wall.KVCache(B, spec.cap, HQ, H, K, V, dtype=torch.bfloat16, chunk=spec.C)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    outs = []
    for s in range(steps):
        t = T0 + s
        cache.append(d["k"][:, t:t + 1].contiguous(), d["g"][:, t:t + 1].contiguous(),
                     d["v"][:, t:t + 1].contiguous())
        outs.append(cache.decode(d["q"][:, s:s + 1].contiguous(), scale=d["scale"]).clone())
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    for b in (0, 31):
        T = T0 + steps
        qf = torch.zeros((1, T, HQ, K), dtype=torch.bfloat16)
        for s in range(steps):
            qf[0, T0 + s] = d["q"][b, s].cpu()
        rows = np.array([T0 + s for s in range(steps)], dtype=np.int64)
        ro, _ = oracle.wall_fwd(qf, d["k"][b:b + 1, :T].cpu(), d["v"][b:b + 1, :T].cpu(),
                                d["g"][b:b + 1, :T].cpu(), scale=d["scale"], rows=rows,
                                threads=ORACLE_THREADS)
        for s in range(steps):
            assert_close(outs[s][b, 0], ro[s], torch.bfloat16, f"full decode b={b} step {s}")
