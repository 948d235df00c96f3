"""The scalar gate (g_scalar) in decode, on the GPU.

The forward's gate term Gs[t] - Gs[j] reaches the decode through a gate cache
PS[j] = sum_{u <= j} g_scalar[u] log2(e) (exp2 units of the key cache): every
decode step must equal the oracle's prefill row of the token just appended with
g_scalar (Wall Attention README "Tests": decode == prefill), for dense caches,
per-sequence lengths and paged caches.
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


def _inputs(B, T, HQ, H, K, V, dtype, seed, sink=True):
    spec = W.PrefillSpec("gate", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype=dtype,
                         g_kind="negsoftplus", g_scalar=True, sink=sink, seed=seed)
    return spec, W.gen_prefill(spec, device="cuda")


@pytest.mark.parametrize("dtype,HQ,H,K,V", [("bf16", 8, 2, 128, 128), ("f32", 4, 4, 64, 128),
                                            ("bf16", 16, 1, 64, 64)])
def test_gated_streaming_decode_matches_prefill(wall, dtype, HQ, H, K, V):
    B, T0, S = 2, 300, 20
    T = T0 + S
    spec, d = _inputs(B, T, HQ, H, K, V, dtype, seed=91)
    dt = spec.torch_dtype
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=dt, chunk=64, gate=True)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous(), d["g_scalar"][:, :T0].contiguous())
    torch.cuda.synchronize()
    PS = oracle.gate_cache(d["g_scalar"])
    np.testing.assert_allclose(cache.gs_cache[:, :T0].double().cpu().numpy(), PS[:, :T0],
                               rtol=2e-6, atol=2e-5)
    rows = np.array([b * T + t for b in range(B) for t in range(T0 - 1, T)], dtype=np.int64)
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                            scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    ro = ro.reshape(B, S + 1, HQ, V)
    for s_ in range(S + 1):
        t = T0 - 1 + s_
        if s_ > 0:
            cache.append(d["k"][:, t:t + 1].contiguous(), d["g"][:, t:t + 1].contiguous(),
                         d["v"][:, t:t + 1].contiguous(), d["g_scalar"][:, t:t + 1].contiguous())
        o = cache.decode(d["q"][:, t:t + 1].contiguous(), sink_bias=d["sink_bias"],
                         scale=d["scale"])
        assert_close(o[:, 0], ro[:, s_], dt, f"gated decode step {s_}")
    assert wall.wall_device_error() == 0


def test_gated_varlen_append_and_decode(wall):
    """Per-sequence lengths: gate rows appended at each row's own position."""
    start, steps = (200, 65, 1), 12
    B, HQ, H, K, V, C = len(start), 8, 2, 128, 128, 64
    T = max(start) + steps
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=92)
    cap = T + 1
    kt = torch.zeros((B, cap, HQ, K), dtype=torch.bfloat16, device="cuda")
    rc = torch.zeros((B, (cap + C - 1) // C, HQ, K), dtype=torch.float32, device="cuda")
    p = torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda")
    vc = torch.zeros((B, cap, H, V), dtype=torch.bfloat16, device="cuda")
    gsc = torch.zeros((B, cap, HQ), dtype=torch.float32, device="cuda")
    gsl = torch.zeros((B, HQ), dtype=torch.float32, device="cuda")
    for b, L in enumerate(start):
        wall.wall_build_kv_cache(d["k"][b:b + 1, :L].contiguous(), d["g"][b:b + 1, :L].contiguous(),
                                 kt[b:b + 1], rc[b:b + 1], p[b:b + 1], chunk=C)
        wall.wall_build_gate_cache(d["g_scalar"][b:b + 1, :L].contiguous(), gsc[b:b + 1],
                                   gsl[b:b + 1])
        vc[b, :T].copy_(d["v"][b])
    lens = list(start)
    for s_ in range(steps):
        t_pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
        pick = lambda x: torch.stack([x[b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        wall.wall_append_kv_cache_varlen(pick(d["k"]), pick(d["g"]), kt, rc, p, t_pos, chunk=C)
        wall.wall_append_gate_cache(pick(d["g_scalar"]), gsc, gsl, t_pos)
        o = wall.wall_attn_decode_gated(pick(d["q"]), p[:, None].contiguous(), gsl, vc, kt, rc,
                                        gsc, T_kv=max(lens) + 1, seqlens=t_pos + 1,
                                        sink_bias=d["sink_bias"], scale=d["scale"], chunk=C)
        rows = [b * T + L for b, L in enumerate(lens)]
        ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
        assert_close(o[:, 0], ro, torch.bfloat16, f"gated varlen step {s_}")
        lens = [L + 1 for L in lens]


def test_gated_paged_streaming(wall):
    start, steps, bs = (130, 64), 40, 64
    B, HQ, H, K, V = len(start), 4, 1, 128, 64
    T = max(start) + steps
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=93)
    maxblk = (T + bs - 1) // bs
    cache = wall.PagedKVCache(B, num_blocks=B * maxblk + 1, block_size=bs, max_blocks=maxblk,
                              HQ=HQ, H=H, K=K, V=V, chunk=64, gate=True)
    for b, L in enumerate(start):
        cache.reserve(b, L)
    for b, L in enumerate(start):
        tb = cache.block_table[b:b + 1].contiguous()
        wall.wall_build_kv_cache_paged(d["k"][b:b + 1, :L].contiguous(),
                                       d["g"][b:b + 1, :L].contiguous(), tb, cache.k_tilde,
                                       cache.r_cache, cache.p[b:b + 1], chunk=64)
        wall.wall_build_gate_cache(d["g_scalar"][b:b + 1, :L].contiguous(), cache.gs_cache,
                                   cache.gs[b:b + 1], block_table=tb)
        rows = torch.tensor(cache.rows_of(b, 0, L), device="cuda")
        cache.v.view(-1, H, V)[rows] = d["v"][b, :L]
        cache.lengths[b] = L
    lens = list(start)
    for s_ in range(steps):
        pick = lambda x: torch.stack([x[b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        cache.append(pick(d["k"]), pick(d["g"]), pick(d["v"]), lens, gs_new=pick(d["g_scalar"]))
        o = cache.decode(pick(d["q"]), sink_bias=d["sink_bias"], scale=d["scale"])
        if s_ % 6 == 0 or s_ == steps - 1:
            rows = [b * T + L for b, L in enumerate(lens)]
            ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                    scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(o[:, 0], ro, torch.bfloat16, f"gated paged step {s_}")
        lens = [L + 1 for L in lens]
    assert wall.wall_device_error() == 0


@pytest.mark.parametrize("dtype,HQ,H,K,V,T0", [
    ("bf16", 8, 2, 128, 128, 190),   # staged gate rows (HQ % 4 == 0)
    ("f32", 4, 1, 64, 128, 0),       # from an empty cache: the first step has no PS before it
    ("bf16", 2, 2, 64, 64, 70),      # HQ = 2: gate rows loaded per lane
    ("bf16", 16, 1, 128, 64, 33),    # a group of 16 query heads
], ids=lambda x: str(x))
def test_gated_fused_step_matches_prefill(wall, dtype, HQ, H, K, V, T0):
    """The fused append + decode step with the scalar gate: every step equals the oracle's
    prefill row with g_scalar, and afterwards the gate cache equals the oracle's PS."""
    B, S = 2, 40
    T = T0 + S
    spec, d = _inputs(B, T, HQ, H, K, V, dtype, seed=94)
    dt = spec.torch_dtype
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=dt, chunk=64, gate=True)
    for t_ in (cache.k_tilde, cache.v, cache.r_cache, cache.gs_cache):
        t_.fill_(float("nan"))
    if T0 > 0:
        cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                     d["v"][:, :T0].contiguous(), d["g_scalar"][:, :T0].contiguous())
    rows = np.array([b * T + t for b in range(B) for t in range(T0, T)], dtype=np.int64)
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                            scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    ro = ro.reshape(B, S, HQ, V)
    for s_ in range(S):
        t = T0 + s_
        sl = slice(t, t + 1)
        o = cache.step(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(),
                       d["g"][:, sl].contiguous(), d["v"][:, sl].contiguous(),
                       sink_bias=d["sink_bias"], scale=d["scale"],
                       gs_new=d["g_scalar"][:, sl].contiguous())
        assert_close(o[:, 0], ro[:, s_], dt, f"gated fused step {s_}")
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    PS = oracle.gate_cache(d["g_scalar"])
    np.testing.assert_allclose(cache.gs_cache[:, :T].double().cpu().numpy(), PS[:, :T],
                               rtol=2e-6, atol=2e-5)
    np.testing.assert_allclose(cache.gs.double().cpu().numpy(), PS[:, T - 1], rtol=2e-6, atol=2e-5)


def test_gated_fused_step_paged(wall):
    """Paged caches with per-row lengths: gated fused steps through growing block tables."""
    start, steps, bs = (130, 64), 30, 64
    B, HQ, H, K, V = len(start), 4, 1, 128, 64
    T = max(start) + steps
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=95)
    maxblk = (T + bs - 1) // bs
    cache = wall.PagedKVCache(B, num_blocks=B * maxblk + 1, block_size=bs, max_blocks=maxblk,
                              HQ=HQ, H=H, K=K, V=V, chunk=64, gate=True)
    for b, L in enumerate(start):
        cache.reserve(b, L)
    for b, L in enumerate(start):
        tb = cache.block_table[b:b + 1].contiguous()
        wall.wall_build_kv_cache_paged(d["k"][b:b + 1, :L].contiguous(),
                                       d["g"][b:b + 1, :L].contiguous(), tb, cache.k_tilde,
                                       cache.r_cache, cache.p[b:b + 1], chunk=64)
        wall.wall_build_gate_cache(d["g_scalar"][b:b + 1, :L].contiguous(), cache.gs_cache,
                                   cache.gs[b:b + 1], block_table=tb)
        rows = torch.tensor(cache.rows_of(b, 0, L), device="cuda")
        cache.v.view(-1, H, V)[rows] = d["v"][b, :L]
        cache.lengths[b] = L
    lens = list(start)
    for s_ in range(steps):
        pick = lambda x: torch.stack([x[b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        o = cache.step(pick(d["q"]), pick(d["k"]), pick(d["g"]), pick(d["v"]), lens,
                       sink_bias=d["sink_bias"], scale=d["scale"], gs_new=pick(d["g_scalar"]))
        if s_ % 5 == 0 or s_ == steps - 1:
            rows = [b * T + L for b, L in enumerate(lens)]
            ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                    scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(o[:, 0], ro, torch.bfloat16, f"gated paged fused step {s_}")
        lens = [L + 1 for L in lens]
    assert wall.wall_device_error() == 0
