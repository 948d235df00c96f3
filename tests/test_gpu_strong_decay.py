"""Parity under strong per-channel decay.

The method's log-decay g = -softplus(.) is unbounded below, and a channel that
forgets within a few tokens is inside its domain (Wall Attention README,
"Features": per-chunk anchors keep the exp2 factors bounded).  These cases put
such channels next to slowly decaying ones: constant g in {-0.5, -2, -8},
-softplus(N(0,1)+2), a single decay of 100 nats at a few rows, or every channel
strong.  The prefill must match the oracle wherever the anchored tensor-core
tiles would overflow (its wide 256-row blocks take the exact in-block pass);
the decode cache, whose format has one anchor per chunk, must either match
(decay within one chunk inside the representable range) or report
WALL_ERR_RANGE, never a silent NaN.
"""
from dataclasses import replace

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
    w.wall_device_error()  # start from a clear error word
    return w


def _prefill(wall, spec):
    d = W.gen_prefill(spec, device="cuda")
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                                window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                                return_lse=True)
    assert wall.wall_device_error() == 0
    ro, rl = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], d["sink_bias"],
                             window=d["window"], cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                             threads=ORACLE_THREADS)
    assert torch.isfinite(o.float()).all(), "non-finite output"
    assert_close(o, ro, spec.torch_dtype, f"{spec.name}: o")
    assert_close(lse, rl, spec.torch_dtype, f"{spec.name}: lse")
    return d, o, lse


PREFILL_CASES = [
    dict(T=300, g_kind="strong"),
    dict(T=2000, g_kind="strong", g_scalar=True, sink=True),
    dict(T=2000, g_kind="strong_all"),
    dict(T=1024, g_kind="strong", g_scalar=True),  # (bf16: the TMA-staged prepass)
    dict(T=1000, g_kind="spike", HQ=4, H=1),
    dict(T=777, g_kind="strong", window=300, sink=True),
    dict(T=700, g_kind="strong", docs=(1, 255, 300, 144), g_scalar=True),
    dict(T=513, g_kind="strong", K=64, V=128, HQ=6, H=3),
    dict(T=257, g_kind="strong_cache", K=128, V=64, window=1),
]


def _pid(c):
    return "-".join(f"{k}{v}" for k, v in c.items())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", PREFILL_CASES, ids=_pid)
def test_prefill_strong_decay_all_rows(wall, dtype, case):
    base = W.PrefillSpec("strong", B=2, T=64, HQ=4, H=2, K=128, V=128, dtype=dtype, seed=313)
    c = dict(case)
    if "docs" in c:
        c["B"] = 1
    _prefill(wall, replace(base, **c, name=f"strong {_pid(case)} {dtype}"))


def test_spike_blocks_only_change_their_own_rows(wall):
    """A 100-nat decay at one row only makes its own 256-row block wide: rows of the other
    blocks are computed by the tensor-core tiles alone, and every row still matches."""
    spec = W.PrefillSpec("spike", B=1, T=1536, HQ=2, H=2, K=128, V=128, dtype="bf16",
                         g_kind="spike", sink=True, seed=314)
    d, o, _ = _prefill(wall, spec)
    # the same inputs with the spikes removed differ only from the spike rows on
    g2 = d["g"].clone()
    for t in (spec.T // 3, (2 * spec.T) // 3):
        g2[:, t, :, 5] = d["g"][:, t - 1, :, 5]
    o2 = wall.wall_attn_fwd(d["q"], d["k"], d["v"], g2, None, d["sink_bias"], scale=d["scale"])
    torch.cuda.synchronize()
    t1 = spec.T // 3
    assert torch.equal(o[:, :t1], o2[:, :t1])


def _stream_decode(wall, spec, T0, steps, chunk, fused):
    """Build the cache of rows 0..T0-1, then append/attend `steps` tokens one by one;
    each step must equal the oracle's prefill row of that token."""
    d = W.gen_prefill(spec, device="cuda")
    B, HQ, H, K, V = spec.B, spec.HQ, spec.H, spec.K, spec.V
    cache = wall.KVCache(B, T0 + steps, HQ, H, K, V, dtype=spec.torch_dtype, chunk=chunk)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(), d["v"][:, :T0])
    rows = [b * spec.T + t for t in range(T0, T0 + steps) for b in range(B)]
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                            scale=d["scale"], rows=np.array(rows), threads=ORACLE_THREADS)
    ro = ro.reshape(steps, B, HQ, V)
    for s in range(steps):
        t = T0 + s
        q1 = d["q"][:, t:t + 1].contiguous()
        k1, g1, v1 = (d[n][:, t:t + 1].contiguous() for n in ("k", "g", "v"))
        if fused:
            o = cache.step(q1, k1, g1, v1, sink_bias=d["sink_bias"], scale=d["scale"])
        else:
            cache.append(k1, g1, v1)
            o = cache.decode(q1, sink_bias=d["sink_bias"], scale=d["scale"])
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all()
        assert_close(o[:, 0], ro[s], spec.torch_dtype, f"decode step {t}")
    return wall.wall_device_error()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("fused", [False, True])
def test_decode_strong_decay_within_cache_range(wall, dtype, fused):
    """Decay of up to ~62 nats within one 32-row anchor chunk is representable: the
    streaming decode equals the prefill rows (across several chunk boundaries)."""
    spec = W.PrefillSpec("dec-strong", B=2, T=400, HQ=8, H=2, K=128, V=128, dtype=dtype,
                         g_kind="strong_cache", sink=True, seed=315)
    assert _stream_decode(wall, spec, T0=330, steps=70, chunk=32, fused=fused) == 0


def test_cache_out_of_range_is_reported(wall):
    """A channel decaying by 8 nats per token spans ~500 nats within a 64-row chunk: the
    cache cannot hold those keys, so every path that writes such rows reports
    WALL_ERR_RANGE (build, one-token append, fused step, prefill emitting the cache)."""
    spec = W.PrefillSpec("range", B=1, T=200, HQ=4, H=2, K=128, V=128, dtype="bf16",
                         g_kind="strong", seed=316)
    d = W.gen_prefill(spec, device="cuda")
    cache = wall.KVCache(1, 256, 4, 2, 128, 128, dtype=torch.bfloat16, chunk=64)
    cache.append(d["k"][:, :100].contiguous(), d["g"][:, :100].contiguous(), d["v"][:, :100])
    assert wall.wall_device_error() == wall.WALL_ERR_RANGE
    cache.append(d["k"][:, 100:101].contiguous(), d["g"][:, 100:101].contiguous())
    assert wall.wall_device_error() == wall.WALL_ERR_RANGE
    cache.step(*(d[n][:, 101:102].contiguous() for n in ("q", "k", "g", "v")), scale=d["scale"])
    assert wall.wall_device_error() == wall.WALL_ERR_RANGE
    emit = wall.KVCache(1, 256, 4, 2, 128, 128, dtype=torch.bfloat16, chunk=64)
    o = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"], cache=emit)
    assert wall.wall_device_error() == wall.WALL_ERR_RANGE
    # the prefill output itself is exact all the same
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"],
                            threads=ORACLE_THREADS)
    assert_close(o, ro, torch.bfloat16, "prefill with an out-of-range cache")
    # mild decay afterwards: the error word is clear again
    mild = wall.KVCache(1, 256, 4, 2, 128, 128, dtype=torch.bfloat16, chunk=64)
    mild.append(d["k"], torch.full_like(d["g"], -0.01))
    assert wall.wall_device_error() == 0


CHUNK_CASES = [
    dict(B=2, sizes=(300, 129, 1, 270), HQ=8, H=2, K=128, V=128, window=0, sink=True),
    dict(B=1, sizes=(600, 3, 4, 1, 8), HQ=8, H=2, K=128, V=128, window=0, sink=False),
    dict(B=2, sizes=(200, 333, 17), HQ=4, H=2, K=128, V=64, window=150, sink=True),
    dict(B=1, sizes=(2, 511, 64), HQ=4, H=1, K=64, V=128, window=0, sink=True),
]


@pytest.mark.parametrize("case", CHUNK_CASES, ids=lambda c: "-".join(map(str, c["sizes"])))
def test_chunks_strong_decay(wall, case):
    """Chunked prefill / multi-token decode with strong decay (32-row anchor chunks): every
    chunk's rows equal the oracle's prefill rows, through the tensor-core tiles and the
    split pass alike."""
    B, HQ, H, K, V = case["B"], case["HQ"], case["H"], case["K"], case["V"]
    C = 32
    T = sum(case["sizes"])
    spec = W.PrefillSpec("chunk-strong", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="strong_cache", sink=case["sink"], window=case["window"],
                         seed=317)
    d = W.gen_prefill(spec, device="cuda")
    cap = T + 5
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
        assert wall.wall_device_error() == 0
        assert_close(o, ro[:, sl], torch.bfloat16, f"chunk at {t0} (+{M}) o")
        assert_close(lse, rl[:, sl], torch.bfloat16, f"chunk at {t0} (+{M}) lse")
        t0 += M


def test_backward_wide_blocks_report_range(wall):
    """The backward's tiles have no exact in-block pass yet: inputs with a wide block make
    wall_attn_bwd report WALL_ERR_RANGE (never silent NaN gradients); mild inputs do not."""
    spec = W.PrefillSpec("bwd-range", B=1, T=300, HQ=4, H=2, K=128, V=128, dtype="bf16",
                         g_kind="strong", seed=318)
    for kind, want in (("strong", wall.WALL_ERR_RANGE), ("negsoftplus", 0)):
        d = W.gen_prefill(replace(spec, g_kind=kind), device="cuda")
        o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"],
                                    return_lse=True)
        assert wall.wall_device_error() == 0
        wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, torch.ones_like(o),
                           scale=d["scale"])
        assert wall.wall_device_error() == want, kind
