"""wall_attn_decode_noalloc: decode for callers that cannot allocate scratch.

Collected last (file name) so that a run stopping at the first failure has
already run every other test.  Builds a small decode cache, then on two
consecutive streaming steps calls the no-allocation entry point through the C
ABI (ctypes, raw device pointers) and the regular workspace entry point, and
requires the two outputs to agree within the bf16 parity tolerance.  The
second call reuses the library's fixed scratch array left over from the first.
A second case runs the decode workload's head shape, where the split count must
be lowered to fit the scratch, against the oracle; a third checks that shapes
beyond the scratch are refused before any work is queued.
"""
import ctypes

import pytest
import torch

import workloads as W
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

BF16 = 1


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def test_noalloc_decode_matches_workspace_decode_twice():
    import decayed_softmax_attention_b200 as wall
    lib = wall.load_library()
    B, T0, HQ, H, K, V, C = 4, 300, 8, 2, 128, 128, 64
    spec = W.PrefillSpec("noalloc", B=B, T=T0 + 2, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="negsoftplus", sink=True, seed=41)
    d = W.gen_prefill(spec, device="cuda")
    cache = wall.KVCache(B, T0 + 2, HQ, H, K, V, dtype=torch.bfloat16, chunk=C)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    sink = d["sink_bias"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for step in range(2):
        t = T0 + step
        cache.append(d["k"][:, t:t + 1].contiguous(), d["g"][:, t:t + 1].contiguous(),
                     d["v"][:, t:t + 1].contiguous())
        q = d["q"][:, t:t + 1].contiguous()
        ref_lse = torch.empty((B, 1, HQ), dtype=torch.float32, device="cuda")
        ref = cache.decode(q, sink_bias=sink, scale=d["scale"], lse=ref_lse)
        out = torch.full((B, 1, HQ, V), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 1, HQ), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.wall_attn_decode_noalloc(
            _ptr(q), _ptr(cache.p), _ptr(cache.v), _ptr(cache.k_tilde), _ptr(cache.r_cache),
            _ptr(sink), B, cache.length, cache.cap, HQ, H, K, V, C, BF16, float(d["scale"]),
            _ptr(out), _ptr(lse), stream)
        assert st == 0, lib.wall_status_string(st).decode()
        torch.cuda.synchronize()
        assert wall.wall_device_error() == 0
        assert_close(out, ref.double().cpu().numpy(), torch.bfloat16, f"no-alloc step {step}")
        assert_close(lse, ref_lse.double().cpu().numpy(), torch.bfloat16, f"no-alloc lse {step}")


def test_noalloc_decode_split_cap_matches_oracle():
    """At the decode workload's head shape (B=32, HQ=32, H=8, K=V=128) a 4096-row cache
    wants more splits than the 4 MiB scratch holds, so the split count is lowered to fit
    (7 here).  Two calls in a row; batch rows 0 and 31 against the oracle's prefill row,
    every row against the workspace decode."""
    import numpy as np
    import oracle
    from tests.gpu_util import ORACLE_THREADS
    import decayed_softmax_attention_b200 as wall
    lib = wall.load_library()
    B, T, HQ, H, K, V, C = 32, 4096, 32, 8, 128, 128, 64
    assert 4 * 2 ** 20 // (B * HQ * (V + 2) * 4) == 7  # splits that fit the scratch
    spec = W.PrefillSpec("noalloc-cap", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="negsoftplus", seed=43)
    d = W.gen_prefill(spec, device="cuda")
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=torch.bfloat16, chunk=C)
    cache.append(d["k"], d["g"], d["v"])
    q = d["q"][:, T - 1:T].contiguous()
    ref = cache.decode(q, scale=d["scale"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rows = np.array([T - 1], dtype=np.int64)
    for call in range(2):
        out = torch.full((B, 1, HQ, V), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 1, HQ), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.wall_attn_decode_noalloc(
            _ptr(q), _ptr(cache.p), _ptr(cache.v), _ptr(cache.k_tilde), _ptr(cache.r_cache),
            None, B, T, cache.cap, HQ, H, K, V, C, BF16, float(d["scale"]), _ptr(out),
            _ptr(lse), stream)
        assert st == 0, lib.wall_status_string(st).decode()
        torch.cuda.synchronize()
        assert wall.wall_device_error() == 0
        assert_close(out, ref.double().cpu().numpy(), torch.bfloat16, f"capped call {call}")
        for b in (0, B - 1):
            ro, rl = oracle.wall_fwd(d["q"][b:b + 1].cpu(), d["k"][b:b + 1].cpu(),
                                     d["v"][b:b + 1].cpu(), d["g"][b:b + 1].cpu(),
                                     scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(out[b, 0], ro[0], torch.bfloat16, f"capped call {call} b={b} o")
            assert_close(lse[b, 0], rl[0], torch.bfloat16, f"capped call {call} b={b} lse")


def test_noalloc_decode_rejects_shapes_beyond_the_scratch():
    """B * HQ * (V + 2) floats above 4 MiB (B * HQ > 8065 at V = 128): WALL_ERR_WORKSPACE
    before any work is queued (the output keeps its NaN fill).  Buffers are sized for the
    call's shapes all the same."""
    import decayed_softmax_attention_b200 as wall
    lib = wall.load_library()
    B, HQ, H, K, V, C, cap = 256, 32, 8, 128, 128, 64, 1
    bf = dict(dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((B, 1, HQ, K), **bf)
    p = torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda")
    v = torch.zeros((B, cap, H, V), **bf)
    kt = torch.zeros((B, cap, HQ, K), **bf)
    rc = torch.zeros((B, 1, HQ, K), dtype=torch.float32, device="cuda")
    out = torch.full((B, 1, HQ, V), float("nan"), **bf)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.wall_attn_decode_noalloc(_ptr(q), _ptr(p), _ptr(v), _ptr(kt), _ptr(rc), None, B, 1,
                                      cap, HQ, H, K, V, C, BF16, 0.0, _ptr(out), None, stream)
    assert st == 5, lib.wall_status_string(st).decode()  # WALL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all()
