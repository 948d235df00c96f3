"""wall_attn_decode_noalloc: decode for callers that cannot allocate scratch.

Collected last (file name) so that a run stopping at the first failure has
already run every other test.  Builds a small decode cache, then on two
consecutive streaming steps calls the no-allocation entry point through the C
ABI (ctypes, raw device pointers) and the regular workspace entry point, and
requires the two outputs to agree within the bf16 parity tolerance.  The
second call reuses the library's fixed scratch array left over from the first.
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
