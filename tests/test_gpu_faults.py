"""Failure detection without a GPU fault: the kernels' bounded waits.

`wall_debug_set_fault(mode, ms)` makes one kernel's producer skip its first
load (1: prefill attention, 2: decode split, 3: cache build, 4 / 5: the
backward's key-block / query-block kernels, 6 / 7: the chunk path's tile and
few-token split kernels), so the
consumers' waits run out after `ms` milliseconds.  The kernel must then
wind down on its own (drain its copies, free tensor memory), report
WALL_ERR_DEVICE_TIMEOUT through the device error word, and leave the context
usable: the next normal call must succeed and match the oracle.  Nothing here
traps, faults or hangs the GPU.
"""
import pytest
import torch

import oracle
import workloads as W
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu

WALL_ERR_DEVICE_TIMEOUT = 4


def test_starved_consumers_time_out_and_recover():
    import decayed_softmax_attention_b200 as wall
    spec = W.PrefillSpec("fault", B=1, T=256, HQ=2, H=1, K=128, V=128, dtype="bf16",
                         g_scalar=True, seed=3)
    d = W.gen_prefill(spec, device="cuda")
    assert wall.wall_device_error() == 0
    wall.wall_debug_set_fault(1, 100)
    try:
        wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    # the error word is cleared by the read and the context still works
    o = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
    assert wall.wall_device_error() == 0
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"])
    assert_close(o, ro, torch.bfloat16, "after recovery")


def _decode_inputs(wall, B=2, T=300, HQ=8, H=2, K=128, seed=5):
    spec = W.PrefillSpec("fault_dec", B=B, T=T, HQ=HQ, H=H, K=K, V=K, dtype="bf16",
                         g_kind="negsoftplus", seed=seed)
    d = W.gen_prefill(spec, device="cuda")
    return spec, d


def test_decode_starved_consumers_time_out_and_recover():
    """Mode 2: the decode split kernel's producer skips its first stage."""
    import decayed_softmax_attention_b200 as wall
    spec, d = _decode_inputs(wall)
    cache = wall.KVCache(spec.B, spec.T, spec.HQ, spec.H, spec.K, spec.V, dtype=torch.bfloat16)
    cache.append(d["k"], d["g"], d["v"])
    q = d["q"][:, -1:].contiguous()
    assert wall.wall_device_error() == 0
    wall.wall_debug_set_fault(2, 100)
    try:
        cache.decode(q, scale=d["scale"])
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    o = cache.decode(q, scale=d["scale"])
    assert wall.wall_device_error() == 0
    # the decode of the last token equals the last prefill row of each sequence
    rows = [b * spec.T + spec.T - 1 for b in range(spec.B)]
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"], rows=rows)
    assert_close(o[:, 0], ro, torch.bfloat16, "decode after recovery")


def test_cache_build_starved_consumers_time_out_and_recover():
    """Mode 3: the cache build kernel's producer skips its first stage."""
    import decayed_softmax_attention_b200 as wall
    spec, d = _decode_inputs(wall, B=2, T=300, HQ=8, H=2, K=128, seed=6)
    assert wall.wall_device_error() == 0
    bad = wall.KVCache(spec.B, spec.T, spec.HQ, spec.H, spec.K, spec.V, dtype=torch.bfloat16)
    wall.wall_debug_set_fault(3, 100)
    try:
        bad.append(d["k"], d["g"])
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    good = wall.KVCache(spec.B, spec.T, spec.HQ, spec.H, spec.K, spec.V, dtype=torch.bfloat16)
    good.append(d["k"], d["g"])
    assert wall.wall_device_error() == 0
    kt, _, _ = oracle.kv_cache(d["k"], d["g"], chunk=64)
    assert_close(good.k_tilde, kt, torch.bfloat16, "cache after recovery")


def _bwd_case(wall):
    spec = W.PrefillSpec("fault_bwd", B=1, T=300, HQ=4, H=2, K=128, V=128, dtype="bf16",
                         g_kind="negsoftplus", g_scalar=True, seed=9)
    d = W.gen_prefill(spec, device="cuda")
    o, lse = wall.wall_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["g_scalar"], scale=d["scale"],
                                return_lse=True)
    do = torch.randn(o.shape, device="cuda",
                     generator=torch.Generator(device="cuda").manual_seed(4)).to(torch.bfloat16)
    return d, o, lse, do


@pytest.mark.parametrize("mode", [4, 5], ids=["key_block", "query_block"])
def test_backward_starved_consumers_time_out_and_recover(mode):
    """Modes 4 / 5: a backward contraction kernel's producer skips its first tile."""
    import decayed_softmax_attention_b200 as wall
    from tests.test_gpu_bwd import assert_grad_close
    d, o, lse, do = _bwd_case(wall)
    assert wall.wall_device_error() == 0

    def bwd():
        return wall.wall_attn_bwd(d["q"], d["k"], d["v"], d["g"], o, lse, do, d["g_scalar"],
                                  scale=d["scale"])

    wall.wall_debug_set_fault(mode, 100)
    try:
        bwd()
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    got = bwd()
    assert wall.wall_device_error() == 0
    ref = oracle.wall_bwd(d["q"], d["k"], d["v"], d["g"], do, d["g_scalar"], scale=d["scale"],
                          o=o, lse=lse, scales=True)
    for name in ("dq", "dk", "dv", "dg", "dg_scalar"):
        assert_grad_close(got[name], ref[name], ref["sigma"][name], ref["sigma_abs"][name],
                          torch.bfloat16, f"{name} after recovery")


@pytest.mark.parametrize("mode,M", [(6, 300), (7, 4)], ids=["chunk_tile", "chunk_split"])
def test_chunk_starved_consumers_time_out_and_recover(mode, M):
    """Modes 6 / 7: the chunk path's tensor-core tile kernel (a 300-token chunk) or its
    few-token split kernel (4 tokens) loses its first load; the call reports
    WALL_ERR_DEVICE_TIMEOUT and the same chunk, called again, matches the oracle."""
    import decayed_softmax_attention_b200 as wall
    B, T0, HQ, H, K, V, C = 2, 200, 8, 2, 128, 128, 64
    T = T0 + M
    spec = W.PrefillSpec("fault_chunk", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype="bf16",
                         g_kind="negsoftplus", seed=9)
    d = W.gen_prefill(spec, device="cuda")
    cache = wall.KVCache(B, T, HQ, H, K, V, dtype=torch.bfloat16, chunk=C)
    cache.append(d["k"][:, :T0].contiguous(), d["g"][:, :T0].contiguous(),
                 d["v"][:, :T0].contiguous())
    cache.v[:, T0:T].copy_(d["v"][:, T0:T])
    p_prev = cache.p.clone()
    sl = slice(T0, T)
    args = [d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(), d["g"][:, sl].contiguous(),
            cache.k_tilde, cache.r_cache, cache.p, cache.v, T0]
    assert wall.wall_device_error() == 0
    wall.wall_debug_set_fault(mode, 100)
    try:
        wall.wall_attn_chunk(*args, p_prev=p_prev, scale=d["scale"], chunk=C)
        status = wall.wall_device_error()
    finally:
        wall.wall_debug_set_fault(0, 0)
    assert status == WALL_ERR_DEVICE_TIMEOUT
    o = wall.wall_attn_chunk(*args, p_prev=p_prev, scale=d["scale"], chunk=C)
    assert wall.wall_device_error() == 0
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], scale=d["scale"])
    assert_close(o, ro[:, sl], torch.bfloat16, f"chunk after recovery (mode {mode})")
