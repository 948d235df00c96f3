"""The decode step with the append fused in (C ABI wall_attn_decode_step).

Wall Attention README, "Decode": the streaming loop appends each new token to
the cache and then attends it.  The fused step does both in the decode's own
launches.  Checks, per step:
  - the output equals the separate append + decode within the decode's
    tolerance (the new row is scored after the streamed rows instead of in
    its stage, so the accumulation order differs) and the oracle's prefill row
    of the same token ("Tests": decode == prefill);
  - afterwards the cache holds, bit for bit, what the one-token appends
    (wall_append_kv_cache_varlen, whose arithmetic the step reproduces) wrote:
    k_tilde rows, chunk anchors, values, P_last;
over dense caches with one length (from an empty cache, across anchor-chunk
boundaries), dense caches with per-row lengths, and paged caches.
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
    spec = W.PrefillSpec("step", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype=dtype,
                         g_kind="negsoftplus", sink=sink, seed=seed)
    return spec, W.gen_prefill(spec, device="cuda")


def _row(d, name, b_rows, ts):
    """[B, 1, ...] slice of input `name` at position ts[b] of each batch row."""
    return torch.stack([d[name][b, t] for b, t in zip(b_rows, ts)])[:, None].contiguous()


CASES = [
    # bf16, prefix of 190 rows, 70 steps crossing the anchor chunks at 192 and 256
    dict(B=2, T0=190, steps=70, HQ=8, H=2, K=128, V=128, C=64, dtype="bf16"),
    # fp32 from an empty cache: the first step has no previous P; chunks of 32
    dict(B=2, T0=0, steps=40, HQ=4, H=1, K=64, V=128, C=32, dtype="f32"),
    # a group of 16 query heads (two lanes per head)
    dict(B=1, T0=60, steps=9, HQ=16, H=1, K=128, V=64, C=64, dtype="bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}G{c['HQ'] // c['H']}T0{c['T0']}")
def test_fused_step_equals_append_then_decode(wall, case):
    B, HQ, H, K, V, C = case["B"], case["HQ"], case["H"], case["K"], case["V"], case["C"]
    T0, S = case["T0"], case["steps"]
    T = T0 + S
    spec, d = _inputs(B, T, HQ, H, K, V, case["dtype"], seed=131)
    dt = spec.torch_dtype
    fused = wall.KVCache(B, T, HQ, H, K, V, dtype=dt, chunk=C)
    sep = wall.KVCache(B, T, HQ, H, K, V, dtype=dt, chunk=C)
    for c in (fused, sep):  # rows past the ones in use start as NaN
        c.k_tilde.fill_(float("nan"))
        c.v.fill_(float("nan"))
        c.r_cache.fill_(float("nan"))
        if T0 > 0:
            c.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                     d["v"][:, :T0].contiguous())
    rows = [b * T + t for b in range(B) for t in range(T0, T)]
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                            scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    ro = ro.reshape(B, S, HQ, V)
    for s_ in range(S):
        t = T0 + s_
        sl = slice(t, t + 1)
        q, k, g, v = (d[n][:, sl].contiguous() for n in ("q", "k", "g", "v"))
        oa = fused.step(q, k, g, v, sink_bias=d["sink_bias"], scale=d["scale"])
        tp = torch.full((B,), t, dtype=torch.int32, device="cuda")
        wall.wall_append_kv_cache_varlen(k, g, sep.k_tilde, sep.r_cache, sep.p, tp, chunk=C)
        sep.v[:, t].copy_(v[:, 0])
        sep.length += 1
        ob = sep.decode(q, sink_bias=d["sink_bias"], scale=d["scale"])
        torch.cuda.synchronize()
        assert torch.isfinite(oa.float()).all()
        assert_close(oa, ob.float().cpu().numpy(), dt, f"fused vs separate, step {s_}")
        assert_close(oa[:, 0], ro[:, s_], dt, f"fused step {s_} vs oracle")
    assert wall.wall_device_error() == 0
    assert fused.length == sep.length == T
    assert torch.equal(fused.k_tilde[:, :T], sep.k_tilde[:, :T])
    assert torch.equal(fused.v[:, :T], sep.v[:, :T])
    nc = (T + C - 1) // C
    assert torch.equal(fused.r_cache[:, :nc], sep.r_cache[:, :nc])
    assert torch.equal(fused.p, sep.p)


def test_fused_step_per_row_lengths_dense(wall):
    """Each batch row at its own position (dense caches, seqlens)."""
    B, HQ, H, K, V, C = 3, 8, 2, 128, 128, 64
    start, S = (130, 63, 1), 12
    T = max(start) + S
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=141)
    dt = torch.bfloat16
    kt = [torch.full((B, T, HQ, K), float("nan"), dtype=dt, device="cuda") for _ in range(2)]
    rc = [torch.full((B, (T + C - 1) // C, HQ, K), float("nan"), dtype=torch.float32,
                     device="cuda") for _ in range(2)]
    vc = [torch.full((B, T, H, V), float("nan"), dtype=dt, device="cuda") for _ in range(2)]
    p = [torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda") for _ in range(3)]
    for i in range(2):  # prefixes of different lengths, one batch row at a time
        for b, L in enumerate(start):
            wall.wall_build_kv_cache(d["k"][b:b + 1, :L].contiguous(), d["g"][b:b + 1, :L].contiguous(),
                                     kt[i][b:b + 1], rc[i][b:b + 1], p[i][b:b + 1], chunk=C)
            vc[i][b, :L].copy_(d["v"][b, :L])
    p[2].copy_(p[0])
    lens = list(start)
    pf, pf_next = p[0], p[2]
    for s_ in range(S):
        bs_ = list(range(B))
        q, k, g, v = (_row(d, n, bs_, lens) for n in ("q", "k", "g", "v"))
        seqlens = torch.tensor([L + 1 for L in lens], dtype=torch.int32, device="cuda")
        oa = wall.wall_attn_decode_step(q, k, g, v, kt[0], rc[0], vc[0], pf, pf_next,
                                        T_kv=max(lens) + 1, seqlens=seqlens,
                                        sink_bias=d["sink_bias"], scale=d["scale"], chunk=C)
        pf, pf_next = pf_next, pf
        tp = torch.tensor(lens, dtype=torch.int32, device="cuda")
        wall.wall_append_kv_cache_varlen(k, g, kt[1], rc[1], p[1], tp, chunk=C)
        for b, L in enumerate(lens):
            vc[1][b, L].copy_(v[b, 0])
        ob = wall.wall_attn_decode(q, p[1][:, None].contiguous(), vc[1], kt[1], rc[1],
                                   max(lens) + 1, sink_bias=d["sink_bias"], scale=d["scale"],
                                   chunk=C, seqlens=seqlens)
        torch.cuda.synchronize()
        assert_close(oa, ob.float().cpu().numpy(), dt, f"per-row fused vs separate, step {s_}")
        if s_ % 5 == 0 or s_ == S - 1:
            rows = [b * T + L for b, L in enumerate(lens)]
            ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                                    scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(oa[:, 0], ro, dt, f"per-row fused step {s_} vs oracle")
        lens = [L + 1 for L in lens]
    assert wall.wall_device_error() == 0
    for b, L in enumerate(lens):
        assert torch.equal(kt[0][b, :L], kt[1][b, :L])
        assert torch.equal(vc[0][b, :L], vc[1][b, :L])
        nc = (L + C - 1) // C
        assert torch.equal(rc[0][b, :nc], rc[1][b, :nc])
    assert torch.equal(pf, p[1])


@pytest.mark.parametrize("bs", [64, 128])
def test_fused_step_paged(wall, bs):
    """Paged caches: blocks handed out as the sequences grow; the fused step equals
    append + decode through the same tables, and the oracle's prefill rows."""
    start, S = (150, 63, 1), 40
    B, HQ, H, K, V, C = len(start), 8, 2, 128, 128, 64
    T = max(start) + S
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=151)
    maxblk = (T + bs - 1) // bs
    caches = [wall.PagedKVCache(B, num_blocks=B * maxblk + 2, block_size=bs, max_blocks=maxblk,
                                HQ=HQ, H=H, K=K, V=V, chunk=C) for _ in range(2)]
    for c in caches:
        c.k_tilde.fill_(float("nan"))
        c.v.fill_(float("nan"))
        for b, L in enumerate(start):
            c.reserve(b, L)
        for b, L in enumerate(start):
            wall.wall_build_kv_cache_paged(d["k"][b:b + 1, :L].contiguous(),
                                           d["g"][b:b + 1, :L].contiguous(),
                                           c.block_table[b:b + 1].contiguous(), c.k_tilde,
                                           c.r_cache, c.p[b:b + 1], chunk=C)
            rows = torch.tensor(c.rows_of(b, 0, L), device="cuda")
            c.v.view(-1, H, V)[rows] = d["v"][b, :L]
            c.lengths[b] = L
    fused, sep = caches
    lens = list(start)
    for s_ in range(S):
        q, k, g, v = (_row(d, n, range(B), lens) for n in ("q", "k", "g", "v"))
        oa = fused.step(q, k, g, v, lens, sink_bias=d["sink_bias"], scale=d["scale"])
        sep.append(k, g, v, lens)
        ob = sep.decode(q, sink_bias=d["sink_bias"], scale=d["scale"])
        torch.cuda.synchronize()
        assert_close(oa, ob.float().cpu().numpy(), torch.bfloat16, f"paged fused vs separate {s_}")
        if s_ % 9 == 0 or s_ == S - 1:
            rows = [b * T + L for b, L in enumerate(lens)]
            ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                                    scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(oa[:, 0], ro, torch.bfloat16, f"paged fused step {s_} vs oracle")
        lens = [L + 1 for L in lens]
    assert wall.wall_device_error() == 0
    assert fused.host_table == sep.host_table
    for b, L in enumerate(lens):
        rows = torch.tensor(fused.rows_of(b, 0, L), device="cuda")
        assert torch.equal(fused.k_tilde.view(-1, HQ, K)[rows], sep.k_tilde.view(-1, HQ, K)[rows])
        assert torch.equal(fused.v.view(-1, H, V)[rows], sep.v.view(-1, H, V)[rows])
    assert torch.equal(fused.p, sep.p)


def test_fused_step_full_decode_workload(wall):
    """The benchmark's decode loop at its full size (B=32, T_kv=32768 prefix, HQ=32, H=8,
    K=V=128, C=64): build the prefix, run 3 fused steps, and check batch rows 0 and 31
    against the oracle's prefill rows of the appended tokens."""
    spec = W.DECODE["decode"]
    steps = 3
    d = W.gen_decode(spec, device="cuda")
    B, T0, HQ, H, K, V = spec.B, spec.T0, spec.HQ, spec.H, spec.K, spec.V
    cache = wall.KVCache(B, spec.cap, HQ, H, K, V, dtype=torch.bfloat16, chunk=spec.C)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    outs = []
    for s_ in range(steps):
        t = T0 + s_
        k1, g1, v1 = (d[n][:, t:t + 1].contiguous() for n in ("k", "g", "v"))
        outs.append(cache.step(d["q"][:, s_:s_ + 1].contiguous(), k1, g1, v1,
                               scale=d["scale"]).clone())
    torch.cuda.synchronize()
    assert wall.wall_device_error() == 0
    T = T0 + steps
    for b in (0, 31):
        qf = torch.zeros((1, T, HQ, K), dtype=torch.bfloat16)
        for s_ in range(steps):
            qf[0, T0 + s_] = d["q"][b, s_].cpu()
        rows = np.array([T0 + s_ for s_ in range(steps)], dtype=np.int64)
        ro, _ = oracle.wall_fwd(qf, d["k"][b:b + 1, :T].cpu(), d["v"][b:b + 1, :T].cpu(),
                                d["g"][b:b + 1, :T].cpu(), scale=d["scale"], rows=rows,
                                threads=ORACLE_THREADS)
        for s_ in range(steps):
            assert_close(outs[s_][b, 0], ro[s_], torch.bfloat16, f"fused full decode b={b} step {s_}")
