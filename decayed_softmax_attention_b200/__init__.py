"""Wall attention (decayed softmax attention) for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/wall_attn.h``: argument
marshalling only (dtype/shape checks, device pointers, the current CUDA
stream, caller-side workspace allocation through torch).  Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback: any
entry point raises ImportError when the built library is missing, and
ValueError when a tensor does not live in CUDA device memory.

Public calls (same names as the C ABI):
  wall_attn_fwd(q, k, v, g, g_scalar=None, sink_bias=None, window=0,
                cu_seqlens=None, scale=None, return_lse=False)
  wall_build_kv_cache(k_new, g_new, k_tilde, r_cache, p_last, t_start=0,
                      p_prev=None, chunk=64)
  wall_attn_decode(q, p_curr, v, k_tilde, r_cache, T_kv, sink_bias=None,
                   scale=None, chunk=64, out=None, lse=None, workspace=None)
plus KVCache, a small helper that owns the cache tensors of a streaming loop.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "WallError", "lib_path", "load_library", "wall_attn_fwd", "wall_attn_fwd_workspace_size",
    "wall_build_kv_cache", "wall_attn_decode", "wall_attn_decode_workspace_size",
    "wall_attn_decode_noalloc", "wall_append_kv_cache_varlen", "wall_attn_bwd",
    "wall_attn_bwd_workspace_size", "wall_build_kv_cache_paged", "wall_append_kv_cache_paged",
    "wall_attn_decode_paged", "PagedKVCache", "wall_build_gate_cache", "wall_append_gate_cache",
    "wall_attn_decode_gated", "wall_attn_chunk", "wall_attn_chunk_workspace_size",
    "wall_attn_decode_step",
    "wall_device_error", "wall_debug_set_fault", "wall_debug_set_stage_events", "KVCache",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_lib", "libwall_attn.so")

WALL_OK = 0
WALL_ERR_DEVICE_TIMEOUT = 4
WALL_ERR_RANGE = 6
WALL_DTYPE_F32 = 0
WALL_DTYPE_BF16 = 1
_STATUS = {
    0: "WALL_OK", 1: "WALL_ERR_INVALID_ARG", 2: "WALL_ERR_UNSUPPORTED", 3: "WALL_ERR_CUDA",
    4: "WALL_ERR_DEVICE_TIMEOUT", 5: "WALL_ERR_WORKSPACE", 6: "WALL_ERR_RANGE",
}

EXPORTED_SYMBOLS = (
    "wall_status_string", "wall_attn_fwd_workspace_size", "wall_attn_fwd",
    "wall_build_kv_cache", "wall_attn_decode_workspace_size", "wall_attn_decode",
    "wall_device_error", "wall_debug_set_fault", "wall_debug_set_stage_events",
    "wall_attn_decode_noalloc", "wall_attn_fwd_with_cache", "wall_attn_decode_varlen",
    "wall_append_kv_cache_varlen", "wall_attn_bwd_workspace_size", "wall_attn_bwd",
    "wall_build_kv_cache_paged", "wall_append_kv_cache_paged", "wall_attn_decode_paged",
    "wall_build_gate_cache", "wall_append_gate_cache", "wall_attn_decode_gated",
    "wall_attn_chunk_workspace_size", "wall_attn_chunk", "wall_attn_decode_step",
    "wall_attn_decode_step_gated", "wall_attn_chunk_gated",
)


class WallError(RuntimeError):
    """A C-ABI call returned a status other than WALL_OK."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)} ({_lib_status_string(status)})")


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the in-tree CUDA library (build it with ``python -m decayed_softmax_attention_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"Wall attention CUDA library not built: {_LIB_PATH} is missing "
            "(run `python -m decayed_softmax_attention_b200.build`)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.wall_status_string.argtypes = [I]
    lib.wall_status_string.restype = ctypes.c_char_p
    lib.wall_attn_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.wall_attn_fwd_workspace_size.restype = S
    lib.wall_attn_fwd.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I, I, I, I, F, P, P, P, S, P]
    lib.wall_attn_fwd.restype = I
    lib.wall_attn_fwd_with_cache.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P,
                                             P, S, I, I, P, P, P, P]
    lib.wall_attn_fwd_with_cache.restype = I
    lib.wall_attn_bwd_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.wall_attn_bwd_workspace_size.restype = S
    lib.wall_attn_bwd.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I, I, I, I, F, P, P, P, P,
                                  P, P, P, P, P, P, P, S, P]
    lib.wall_attn_bwd.restype = I
    lib.wall_build_kv_cache_paged.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, P, P,
                                              P, P]
    lib.wall_build_kv_cache_paged.restype = I
    lib.wall_append_kv_cache_paged.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, P,
                                               P]
    lib.wall_append_kv_cache_paged.restype = I
    lib.wall_attn_decode_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I,
                                           F, P, P, P, S, P]
    lib.wall_attn_decode_paged.restype = I
    lib.wall_attn_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I,
                                          I, I, F, P, P, P, P, P, P, S, P]
    lib.wall_attn_decode_step.restype = I
    lib.wall_attn_decode_step_gated.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I,
                                                I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, S, P]
    lib.wall_attn_decode_step_gated.restype = I
    lib.wall_build_gate_cache.argtypes = [P, P, P, I, I, I, I, I, I, I, I, I, P, P, P]
    lib.wall_build_gate_cache.restype = I
    lib.wall_append_gate_cache.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P]
    lib.wall_append_gate_cache.restype = I
    lib.wall_attn_decode_gated.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I,
                                           I, I, I, F, P, P, P, S, P]
    lib.wall_attn_decode_gated.restype = I
    lib.wall_attn_chunk_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I]
    lib.wall_attn_chunk_workspace_size.restype = S
    lib.wall_attn_chunk.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, F, P, P, P, P,
                                    P, P, P, S, P]
    lib.wall_attn_chunk.restype = I
    lib.wall_attn_chunk_gated.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I,
                                          F, P, P, P, P, P, P, P, P, P, S, P]
    lib.wall_attn_chunk_gated.restype = I
    lib.wall_build_kv_cache.argtypes = [P, P, P, I, I, I, I, I, I, I, I, I, P, P, P, P]
    lib.wall_build_kv_cache.restype = I
    lib.wall_append_kv_cache_varlen.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P, P]
    lib.wall_append_kv_cache_varlen.restype = I
    lib.wall_attn_decode_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.wall_attn_decode_workspace_size.restype = S
    lib.wall_attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P, P, P, S, P]
    lib.wall_attn_decode.restype = I
    lib.wall_attn_decode_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P,
                                            P, P, S, P]
    lib.wall_attn_decode_varlen.restype = I
    lib.wall_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P, P, P]
    lib.wall_attn_decode_noalloc.restype = I
    lib.wall_device_error.argtypes = [P]
    lib.wall_device_error.restype = I
    lib.wall_debug_set_fault.argtypes = [I, I]
    lib.wall_debug_set_fault.restype = None
    lib.wall_debug_set_stage_events.argtypes = [P, P, P]
    lib.wall_debug_set_stage_events.restype = None
    _lib = lib
    return lib


def _lib_status_string(status: int) -> str:
    try:
        return load_library().wall_status_string(int(status)).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(status: int, what: str):
    if status != WALL_OK:
        raise WallError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return WALL_DTYPE_BF16
    if t.dtype == torch.float32:
        return WALL_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(t, name, dtype=None, shape=None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live in CUDA device memory")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


# ----------------------------------------------------------------- prefill
def wall_attn_fwd_workspace_size(B, T, HQ, H, K, V, dtype) -> int:
    code = WALL_DTYPE_BF16 if dtype == torch.bfloat16 else WALL_DTYPE_F32
    return int(load_library().wall_attn_fwd_workspace_size(B, T, HQ, H, K, V, code))


def wall_attn_fwd(q, k, v, g, g_scalar=None, sink_bias=None, window=0, cu_seqlens=None,
                  scale=None, return_lse=False, out=None, lse=None, workspace=None, cache=None):
    """Prefill forward (README "Usage"): o [B,T,HQ,V] (and lse [B,T,HQ] fp32, natural log).

    cache: optional KVCache (capacity >= T); the prefill then also writes its decode
    cache rows 0 .. T-1 (k_tilde, anchors, P at row T-1) and sets cache.length = T.
    Value rows are the caller's (copy v into cache.v).
    """
    lib = load_library()
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    dt = q.dtype
    code = _dtype_code(q)
    if out is None:
        out = torch.empty((B, T, HQ, V), dtype=dt, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, T, HQ), dtype=torch.float32, device=q.device)
    need = wall_attn_fwd_workspace_size(B, T, HQ, H, K, V, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cache is not None:
        # the prefill also fills the decode cache (rows 0 .. T-1); no packed documents
        if cu_seqlens is not None:
            raise ValueError("cache output needs one sequence per batch row (no cu_seqlens)")
        st = lib.wall_attn_fwd_with_cache(
            _dev(q, "q", dt), _dev(k, "k", dt, (B, T, H, K)), _dev(v, "v", dt, (B, T, H, V)),
            _dev(g, "g", dt, (B, T, HQ, K)), _dev(g_scalar, "g_scalar", dt, (B, T, HQ)),
            _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), int(window or 0),
            B, T, HQ, H, K, V, code, float(scale) if scale else 0.0,
            _dev(out, "out", dt, (B, T, HQ, V)), _dev(lse, "lse", torch.float32, (B, T, HQ)),
            _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
            cache.cap, cache.chunk, _dev(cache.k_tilde, "k_tilde", dt, (B, cache.cap, HQ, K)),
            _dev(cache.r_cache, "r_cache", torch.float32), _dev(cache.p, "p_last", torch.float32),
            _stream(q.device))
        _check(st, "wall_attn_fwd_with_cache")
        cache.length = T
        return (out, lse) if return_lse else out
    st = lib.wall_attn_fwd(
        _dev(q, "q", dt), _dev(k, "k", dt, (B, T, H, K)), _dev(v, "v", dt, (B, T, H, V)),
        _dev(g, "g", dt, (B, T, HQ, K)), _dev(g_scalar, "g_scalar", dt, (B, T, HQ)),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), int(window or 0),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), nseq, B, T, HQ, H, K, V, code,
        float(scale) if scale else 0.0, _dev(out, "out", dt, (B, T, HQ, V)),
        _dev(lse, "lse", torch.float32, (B, T, HQ)), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "wall_attn_fwd")
    return (out, lse) if return_lse else out


def wall_attn_bwd_workspace_size(B, T, HQ, H, K, V, dtype) -> int:
    code = WALL_DTYPE_BF16 if dtype == torch.bfloat16 else WALL_DTYPE_F32
    return int(load_library().wall_attn_bwd_workspace_size(B, T, HQ, H, K, V, code))


def wall_attn_bwd(q, k, v, g, o, lse, do, g_scalar=None, sink_bias=None, window=0,
                  cu_seqlens=None, scale=None, dlse=None, workspace=None, grads=None):
    """Prefill backward: gradients of a loss through o (and optionally lse).

    o, lse: the forward's outputs for the same inputs; do [B,T,HQ,V] = dL/do;
    dlse [B,T,HQ] fp32 or None.  Returns a dict with dq, dk, dv, dg (input dtype),
    dg_scalar (with g_scalar) and dsink (fp32 [HQ], with sink_bias).  ``grads``: an
    optional dict of preallocated outputs with those keys.
    """
    lib = load_library()
    B, T, HQ, K = q.shape
    H, V = k.shape[2], v.shape[3]
    dt = q.dtype
    code = _dtype_code(q)
    dev = q.device
    out = dict(grads or {})
    shapes = dict(dq=(B, T, HQ, K), dk=(B, T, H, K), dv=(B, T, H, V), dg=(B, T, HQ, K))
    if g_scalar is not None:
        shapes["dg_scalar"] = (B, T, HQ)
    for name, shp in shapes.items():
        if out.get(name) is None:
            out[name] = torch.empty(shp, dtype=dt, device=dev)
    if sink_bias is not None and out.get("dsink") is None:
        out["dsink"] = torch.empty((HQ,), dtype=torch.float32, device=dev)
    need = wall_attn_bwd_workspace_size(B, T, HQ, H, K, V, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    st = lib.wall_attn_bwd(
        _dev(q, "q", dt), _dev(k, "k", dt, (B, T, H, K)), _dev(v, "v", dt, (B, T, H, V)),
        _dev(g, "g", dt, (B, T, HQ, K)), _dev(g_scalar, "g_scalar", dt, (B, T, HQ)),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), int(window or 0),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), nseq, B, T, HQ, H, K, V, code,
        float(scale) if scale else 0.0, _dev(o, "o", dt, (B, T, HQ, V)),
        _dev(lse, "lse", torch.float32, (B, T, HQ)), _dev(do, "do", dt, (B, T, HQ, V)),
        _dev(dlse, "dlse", torch.float32, (B, T, HQ)),
        *(_dev(out[n], n, dt, shapes[n]) for n in ("dq", "dk", "dv", "dg")),
        _dev(out.get("dg_scalar"), "dg_scalar", dt, (B, T, HQ)),
        _dev(out.get("dsink"), "dsink", torch.float32, (HQ,)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(dev))
    _check(st, "wall_attn_bwd")
    out.setdefault("dg_scalar", None)
    out.setdefault("dsink", None)
    return out


# ----------------------------------------------------------------- decode
def wall_build_kv_cache(k_new, g_new, k_tilde, r_cache, p_last, t_start=0, p_prev=None,
                        chunk=64):
    """Build (t_start=0) or append to the pre-rescaled key cache (README "Decode")."""
    lib = load_library()
    B, T_new, H, K = k_new.shape
    HQ = g_new.shape[2]
    cap = k_tilde.shape[1]
    dt = k_new.dtype
    st = lib.wall_build_kv_cache(
        _dev(k_new, "k_new", dt), _dev(g_new, "g_new", dt, (B, T_new, HQ, K)),
        _dev(p_prev, "p_prev", torch.float32), B, int(t_start), T_new, cap, HQ, H, K, int(chunk),
        _dtype_code(k_new), _dev(k_tilde, "k_tilde", dt, (B, cap, HQ, K)),
        _dev(r_cache, "r_cache", torch.float32, (B, (cap + chunk - 1) // chunk, HQ, K)),
        _dev(p_last, "p_last", torch.float32), _stream(k_new.device))
    _check(st, "wall_build_kv_cache")
    return p_last


def wall_append_kv_cache_varlen(k_new, g_new, k_tilde, r_cache, p_last, t_pos, p_prev=None,
                                chunk=64):
    """Append one token per batch row at row b's own position t_pos[b] (device int32 [B]).

    k_new [B,1,H,K], g_new [B,1,HQ,K]; p_prev [B,HQ,K] fp32 (defaults to p_last, updated in
    place) holds P at row t_pos[b] - 1.
    """
    lib = load_library()
    B, _, H, K = k_new.shape
    HQ = g_new.shape[2]
    cap = k_tilde.shape[1]
    dt = k_new.dtype
    if p_prev is None:
        p_prev = p_last
    st = lib.wall_append_kv_cache_varlen(
        _dev(k_new, "k_new", dt, (B, 1, H, K)), _dev(g_new, "g_new", dt, (B, 1, HQ, K)),
        _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)), _dev(t_pos, "t_pos", torch.int32, (B,)),
        B, cap, HQ, H, K, int(chunk), _dtype_code(k_new),
        _dev(k_tilde, "k_tilde", dt, (B, cap, HQ, K)),
        _dev(r_cache, "r_cache", torch.float32, (B, (cap + chunk - 1) // chunk, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)), _stream(k_new.device))
    _check(st, "wall_append_kv_cache_varlen")
    return p_last


def wall_attn_decode_workspace_size(B, T_kv, HQ, H, V, chunk=64) -> int:
    return int(load_library().wall_attn_decode_workspace_size(B, T_kv, HQ, H, V, chunk))


def wall_attn_decode(q, p_curr, v, k_tilde, r_cache, T_kv, sink_bias=None, scale=None, chunk=64,
                     out=None, lse=None, workspace=None, seqlens=None):
    """One decode step over cache rows [0, T_kv): o [B,1,HQ,V] (lse [B,1,HQ] if given).

    seqlens: optional device int32 [B]; batch row b then attends rows
    [0, seqlens[b]) (each in [1, T_kv]; T_kv is then the largest length).
    """
    lib = load_library()
    B, cap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    dt = k_tilde.dtype
    if out is None:
        out = torch.empty((B, 1, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(wall_attn_decode_workspace_size(B, T_kv, HQ, H, V, chunk), 1),
                                dtype=torch.uint8, device=q.device)
    if seqlens is not None:
        st = lib.wall_attn_decode_varlen(
            _dev(q, "q", dt), _dev(p_curr, "p_curr", torch.float32),
            _dev(v, "v", dt, (B, cap, H, V)), _dev(k_tilde, "k_tilde", dt),
            _dev(r_cache, "r_cache", torch.float32),
            _dev(sink_bias, "sink_bias", torch.float32, (HQ,)),
            _dev(seqlens, "seqlens", torch.int32, (B,)), B, int(T_kv), cap, HQ, H, K, V,
            int(chunk), _dtype_code(k_tilde), float(scale) if scale else 0.0,
            _dev(out, "out", dt), _dev(lse, "lse", torch.float32), _dev(workspace, "workspace"),
            workspace.numel() * workspace.element_size(), _stream(q.device))
        _check(st, "wall_attn_decode_varlen")
        return out
    st = lib.wall_attn_decode(
        _dev(q, "q", dt), _dev(p_curr, "p_curr", torch.float32), _dev(v, "v", dt, (B, cap, H, V)),
        _dev(k_tilde, "k_tilde", dt), _dev(r_cache, "r_cache", torch.float32),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), B, int(T_kv), cap, HQ, H, K, V,
        int(chunk), _dtype_code(k_tilde), float(scale) if scale else 0.0,
        _dev(out, "out", dt), _dev(lse, "lse", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "wall_attn_decode")
    return out


# ----------------------------------------------------------------- paged caches
def _pool_dims(k_tilde_pool, block_table, chunk):
    nblk, bs = k_tilde_pool.shape[0], k_tilde_pool.shape[1]
    return nblk, bs, block_table.shape[1], bs // chunk


def wall_build_kv_cache_paged(k_new, g_new, block_table, k_tilde_pool, r_pool, p_last, t_start=0,
                              p_prev=None, chunk=64):
    """wall_build_kv_cache into a paged pool: rows t_start .. t_start+T_new-1 of each batch row,
    addressed through block_table [B, max_blocks] (int32, device)."""
    lib = load_library()
    B, T_new, H, K = k_new.shape
    HQ = g_new.shape[2]
    dt = k_new.dtype
    nblk, bs, maxblk, cpb = _pool_dims(k_tilde_pool, block_table, chunk)
    st = lib.wall_build_kv_cache_paged(
        _dev(k_new, "k_new", dt), _dev(g_new, "g_new", dt, (B, T_new, HQ, K)),
        _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)),
        _dev(block_table, "block_table", torch.int32, (B, maxblk)), maxblk, B, int(t_start), T_new,
        nblk, bs, HQ, H, K, int(chunk), _dtype_code(k_new),
        _dev(k_tilde_pool, "k_tilde_pool", dt, (nblk, bs, HQ, K)),
        _dev(r_pool, "r_pool", torch.float32, (nblk, cpb, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)), _stream(k_new.device))
    _check(st, "wall_build_kv_cache_paged")
    return p_last


def wall_append_kv_cache_paged(k_new, g_new, block_table, k_tilde_pool, r_pool, p_last, t_pos,
                               p_prev=None, chunk=64):
    """One token per batch row at row b's own position t_pos[b], into a paged pool."""
    lib = load_library()
    B, _, H, K = k_new.shape
    HQ = g_new.shape[2]
    dt = k_new.dtype
    nblk, bs, maxblk, cpb = _pool_dims(k_tilde_pool, block_table, chunk)
    if p_prev is None:
        p_prev = p_last
    st = lib.wall_append_kv_cache_paged(
        _dev(k_new, "k_new", dt, (B, 1, H, K)), _dev(g_new, "g_new", dt, (B, 1, HQ, K)),
        _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)), _dev(t_pos, "t_pos", torch.int32, (B,)),
        _dev(block_table, "block_table", torch.int32, (B, maxblk)), maxblk, B, nblk, bs, HQ, H, K,
        int(chunk), _dtype_code(k_new), _dev(k_tilde_pool, "k_tilde_pool", dt, (nblk, bs, HQ, K)),
        _dev(r_pool, "r_pool", torch.float32, (nblk, cpb, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)), _stream(k_new.device))
    _check(st, "wall_append_kv_cache_paged")
    return p_last


def wall_attn_decode_paged(q, p_curr, v_pool, k_tilde_pool, r_pool, seqlens, block_table,
                           sink_bias=None, scale=None, chunk=64, out=None, lse=None,
                           workspace=None):
    """One decode step over paged caches: batch row b attends its rows [0, seqlens[b])."""
    lib = load_library()
    B = q.shape[0]
    nblk, bs, HQ, K = k_tilde_pool.shape
    H, V = v_pool.shape[2], v_pool.shape[3]
    maxblk = block_table.shape[1]
    dt = k_tilde_pool.dtype
    if out is None:
        out = torch.empty((B, 1, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(
            max(wall_attn_decode_workspace_size(B, maxblk * bs, HQ, H, V, chunk), 1),
            dtype=torch.uint8, device=q.device)
    st = lib.wall_attn_decode_paged(
        _dev(q, "q", dt), _dev(p_curr, "p_curr", torch.float32),
        _dev(v_pool, "v_pool", dt, (nblk, bs, H, V)), _dev(k_tilde_pool, "k_tilde_pool", dt),
        _dev(r_pool, "r_pool", torch.float32, (nblk, bs // chunk, HQ, K)),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)),
        _dev(seqlens, "seqlens", torch.int32, (B,)),
        _dev(block_table, "block_table", torch.int32, (B, maxblk)), maxblk, B, nblk, bs, HQ, H, K,
        V, int(chunk), _dtype_code(k_tilde_pool), float(scale) if scale else 0.0,
        _dev(out, "out", dt), _dev(lse, "lse", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "wall_attn_decode_paged")
    return out


def wall_attn_decode_step(q, k_new, g_new, v_new, k_tilde, r_cache, v_cache, p_prev, p_last,
                          T_kv=None, seqlens=None, block_table=None, sink_bias=None, scale=None,
                          chunk=64, out=None, lse=None, workspace=None):
    """One decode step with the append fused in: the new token of batch row b (k_new, g_new,
    v_new [B,1,...]) joins the cache at row T_b - 1 (T_b = seqlens[b], else T_kv) and its
    query attends rows 0 .. T_b - 1.  Dense caches [B,cap,...] (block_table None) or pools
    [num_blocks,block_size,...] with a block table (seqlens required).  p_prev is P at the
    previous row; P at the new row is written to p_last (a different buffer)."""
    lib = load_library()
    B, _, HQ, K = q.shape
    H, V = k_new.shape[2], v_new.shape[3]
    dt = k_tilde.dtype
    if block_table is None:
        cap = k_tilde.shape[1]
        maxblk = nblk = bs = 0
        rows = cap
        if T_kv is None:
            raise ValueError("dense caches need T_kv")
        r_shape = (B, (cap + chunk - 1) // chunk, HQ, K)
        kv_shape, v_shape = (B, cap, HQ, K), (B, cap, H, V)
    else:
        nblk, bs = k_tilde.shape[0], k_tilde.shape[1]
        maxblk = block_table.shape[1]
        cap = rows = maxblk * bs
        if seqlens is None:
            raise ValueError("paged caches need seqlens")
        T_kv = rows if T_kv is None else T_kv
        r_shape = (nblk, bs // chunk, HQ, K)
        kv_shape, v_shape = (nblk, bs, HQ, K), (nblk, bs, H, V)
    if out is None:
        out = torch.empty((B, 1, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(wall_attn_decode_workspace_size(B, rows if block_table is not None
                                                                    else T_kv, HQ, H, V, chunk), 1),
                                dtype=torch.uint8, device=q.device)
    st = lib.wall_attn_decode_step(
        _dev(q, "q", dt, (B, 1, HQ, K)), _dev(k_new, "k_new", dt, (B, 1, H, K)),
        _dev(g_new, "g_new", dt, (B, 1, HQ, K)), _dev(v_new, "v_new", dt, (B, 1, H, V)),
        _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)),
        _dev(seqlens, "seqlens", torch.int32, (B,)),
        _dev(block_table, "block_table", torch.int32), maxblk, nblk, bs, B, int(T_kv), cap, HQ, H,
        K, V, int(chunk), _dtype_code(k_tilde), float(scale) if scale else 0.0,
        _dev(k_tilde, "k_tilde", dt, kv_shape), _dev(r_cache, "r_cache", torch.float32, r_shape),
        _dev(v_cache, "v_cache", dt, v_shape), _dev(out, "out", dt, (B, 1, HQ, V)),
        _dev(lse, "lse", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "wall_attn_decode_step")
    return out


def wall_attn_decode_step_gated(q, k_new, g_new, v_new, gs_new, k_tilde, r_cache, v_cache, p_prev,
                                p_last, gs_cache, gs_prev, gs_last, T_kv=None, seqlens=None,
                                block_table=None, sink_bias=None, scale=None, chunk=64, out=None,
                                lse=None, workspace=None):
    """wall_attn_decode_step with the scalar gate: gs_new [B,1,HQ] is the new token's g_scalar;
    gs_prev / gs_last [B,HQ] fp32 are PS at the previous / new row (different buffers); the
    gate cache row of the new token is written.  Other arguments as wall_attn_decode_step."""
    lib = load_library()
    B, _, HQ, K = q.shape
    H, V = k_new.shape[2], v_new.shape[3]
    dt = k_tilde.dtype
    if block_table is None:
        cap = k_tilde.shape[1]
        maxblk = nblk = bs = 0
        rows = cap
        if T_kv is None:
            raise ValueError("dense caches need T_kv")
        r_shape = (B, (cap + chunk - 1) // chunk, HQ, K)
        kv_shape, v_shape, g_shape = (B, cap, HQ, K), (B, cap, H, V), (B, cap, HQ)
    else:
        nblk, bs = k_tilde.shape[0], k_tilde.shape[1]
        maxblk = block_table.shape[1]
        cap = rows = maxblk * bs
        if seqlens is None:
            raise ValueError("paged caches need seqlens")
        T_kv = rows if T_kv is None else T_kv
        r_shape = (nblk, bs // chunk, HQ, K)
        kv_shape, v_shape, g_shape = (nblk, bs, HQ, K), (nblk, bs, H, V), (nblk, bs, HQ)
    if out is None:
        out = torch.empty((B, 1, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(wall_attn_decode_workspace_size(B, rows if block_table is not None
                                                                    else T_kv, HQ, H, V, chunk), 1),
                                dtype=torch.uint8, device=q.device)
    st = lib.wall_attn_decode_step_gated(
        _dev(q, "q", dt, (B, 1, HQ, K)), _dev(k_new, "k_new", dt, (B, 1, H, K)),
        _dev(g_new, "g_new", dt, (B, 1, HQ, K)), _dev(v_new, "v_new", dt, (B, 1, H, V)),
        _dev(gs_new, "gs_new", dt, (B, 1, HQ)),
        _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)),
        _dev(gs_prev, "gs_prev", torch.float32, (B, HQ)),
        _dev(gs_last, "gs_last", torch.float32, (B, HQ)),
        _dev(gs_cache, "gs_cache", torch.float32, g_shape),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)),
        _dev(seqlens, "seqlens", torch.int32, (B,)),
        _dev(block_table, "block_table", torch.int32), maxblk, nblk, bs, B, int(T_kv), cap, HQ, H,
        K, V, int(chunk), _dtype_code(k_tilde), float(scale) if scale else 0.0,
        _dev(k_tilde, "k_tilde", dt, kv_shape), _dev(r_cache, "r_cache", torch.float32, r_shape),
        _dev(v_cache, "v_cache", dt, v_shape), _dev(out, "out", dt, (B, 1, HQ, V)),
        _dev(lse, "lse", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "wall_attn_decode_step_gated")
    return out


# ----------------------------------------------------------------- scalar gate in decode
def _gate_table(gs_cache, block_table):
    """(block_table, max_blocks, num_blocks, block_size, cap) for a dense or paged gate cache."""
    if block_table is None:
        return None, 0, 0, 0, gs_cache.shape[1]
    return block_table, block_table.shape[1], gs_cache.shape[0], gs_cache.shape[1], 0


def wall_build_gate_cache(gs_new, gs_cache, gs_last, t_start=0, gs_prev=None, block_table=None):
    """PS rows t_start .. t_start+T_new-1 of the scalar-gate cache from gs_new [B,T_new,HQ]."""
    lib = load_library()
    B, T_new, HQ = gs_new.shape
    bt, mb, nb, bs, cap = _gate_table(gs_cache, block_table)
    st = lib.wall_build_gate_cache(
        _dev(gs_new, "gs_new", gs_new.dtype), _dev(gs_prev, "gs_prev", torch.float32, (B, HQ)),
        _dev(bt, "block_table", torch.int32), mb, nb, bs, B, int(t_start), T_new, cap, HQ,
        _dtype_code(gs_new), _dev(gs_cache, "gs_cache", torch.float32),
        _dev(gs_last, "gs_last", torch.float32, (B, HQ)), _stream(gs_new.device))
    _check(st, "wall_build_gate_cache")
    return gs_last


def wall_append_gate_cache(gs_new, gs_cache, gs_last, t_pos, gs_prev=None, block_table=None):
    """One gate row per batch row at t_pos[b] from gs_new [B,1,HQ] (gs_prev defaults to gs_last)."""
    lib = load_library()
    B, _, HQ = gs_new.shape
    bt, mb, nb, bs, cap = _gate_table(gs_cache, block_table)
    if gs_prev is None:
        gs_prev = gs_last
    st = lib.wall_append_gate_cache(
        _dev(gs_new, "gs_new", gs_new.dtype, (B, 1, HQ)),
        _dev(gs_prev, "gs_prev", torch.float32, (B, HQ)), _dev(t_pos, "t_pos", torch.int32, (B,)),
        _dev(bt, "block_table", torch.int32), mb, nb, bs, B, cap, HQ, _dtype_code(gs_new),
        _dev(gs_cache, "gs_cache", torch.float32), _dev(gs_last, "gs_last", torch.float32, (B, HQ)),
        _stream(gs_new.device))
    _check(st, "wall_append_gate_cache")
    return gs_last


def wall_attn_decode_gated(q, p_curr, gs_curr, v, k_tilde, r_cache, gs_cache, T_kv=None,
                           seqlens=None, block_table=None, sink_bias=None, scale=None, chunk=64,
                           out=None, lse=None, workspace=None):
    """wall_attn_decode (dense; T_kv rows or per-row seqlens) or wall_attn_decode_paged
    (block_table + seqlens) with the scalar gate: gs_curr [B,HQ] = PS at the current row."""
    lib = load_library()
    B = q.shape[0]
    dt = k_tilde.dtype
    if block_table is None:
        _, cap, HQ, K = k_tilde.shape
        H, V = v.shape[2], v.shape[3]
        mb = nb = bs = 0
        rows = int(T_kv)
    else:
        nb, bs, HQ, K = k_tilde.shape
        H, V = v.shape[2], v.shape[3]
        mb = block_table.shape[1]
        cap = rows = mb * bs
    if out is None:
        out = torch.empty((B, 1, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(wall_attn_decode_workspace_size(B, rows, HQ, H, V, chunk), 1),
                                dtype=torch.uint8, device=q.device)
    st = lib.wall_attn_decode_gated(
        _dev(q, "q", dt), _dev(p_curr, "p_curr", torch.float32),
        _dev(gs_curr, "gs_curr", torch.float32), _dev(v, "v", dt), _dev(k_tilde, "k_tilde", dt),
        _dev(r_cache, "r_cache", torch.float32), _dev(gs_cache, "gs_cache", torch.float32),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)),
        _dev(seqlens, "seqlens", torch.int32, (B,)), _dev(block_table, "block_table", torch.int32),
        mb, nb, bs, B, rows, cap, HQ, H, K, V, int(chunk), _dtype_code(k_tilde),
        float(scale) if scale else 0.0, _dev(out, "out", dt), _dev(lse, "lse", torch.float32),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(q.device))
    _check(st, "wall_attn_decode_gated")
    return out


# ----------------------------------------------------------------- chunked prefill
def wall_attn_chunk_workspace_size(B, M, cap, HQ, H, K, V, chunk=64,
                                   dtype=torch.bfloat16) -> int:
    code = WALL_DTYPE_F32 if dtype == torch.float32 else WALL_DTYPE_BF16
    return int(load_library().wall_attn_chunk_workspace_size(B, M, cap, HQ, H, K, V, chunk, code))


def wall_attn_chunk(q, k_new, g_new, k_tilde, r_cache, p_last, v_cache, t_start, p_prev=None,
                    sink_bias=None, window=0, scale=None, chunk=64, out=None, lse=None,
                    workspace=None, gs_new=None, gs_cache=None, gs_last=None, gs_prev=None):
    """M new tokens at rows t_start.. of the cache: append their keys, then attend rows
    0 .. t_start + i.  q [B,M,HQ,K]; v_cache rows of the chunk must already hold its values.
    Returns o [B,M,HQ,V].  p_prev defaults to p_last (updated in place).  With the scalar
    gate: gs_new [B,M,HQ] (the chunk's g_scalar), gs_cache [B,cap,HQ] fp32, gs_last [B,HQ]
    (PS at the last row; gs_prev defaults to it, updated in place)."""
    lib = load_library()
    B, M, HQ, K = q.shape
    H = k_new.shape[2]
    cap, V = v_cache.shape[1], v_cache.shape[3]
    dt = q.dtype
    if p_prev is None and t_start > 0:
        p_prev = p_last
    if out is None:
        out = torch.empty((B, M, HQ, V), dtype=dt, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(wall_attn_chunk_workspace_size(B, M, cap, HQ, H, K, V,
                                                                   chunk, dt), 1),
                                dtype=torch.uint8, device=q.device)
    if gs_new is not None:
        if gs_prev is None and t_start > 0:
            gs_prev = gs_last
        st = lib.wall_attn_chunk_gated(
            _dev(q, "q", dt), _dev(k_new, "k_new", dt, (B, M, H, K)),
            _dev(g_new, "g_new", dt, (B, M, HQ, K)), _dev(gs_new, "gs_new", dt, (B, M, HQ)),
            _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)),
            _dev(gs_prev, "gs_prev", torch.float32, (B, HQ)),
            _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), int(window or 0), B, int(t_start),
            M, cap, HQ, H, K, V, int(chunk), _dtype_code(q), float(scale) if scale else 0.0,
            _dev(k_tilde, "k_tilde", dt, (B, cap, HQ, K)),
            _dev(r_cache, "r_cache", torch.float32, (B, (cap + chunk - 1) // chunk, HQ, K)),
            _dev(p_last, "p_last", torch.float32, (B, HQ, K)),
            _dev(gs_cache, "gs_cache", torch.float32, (B, cap, HQ)),
            _dev(gs_last, "gs_last", torch.float32, (B, HQ)), _dev(v_cache, "v_cache", dt),
            _dev(out, "out", dt, (B, M, HQ, V)), _dev(lse, "lse", torch.float32, (B, M, HQ)),
            _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
            _stream(q.device))
        _check(st, "wall_attn_chunk_gated")
        return out
    st = lib.wall_attn_chunk(
        _dev(q, "q", dt), _dev(k_new, "k_new", dt, (B, M, H, K)),
        _dev(g_new, "g_new", dt, (B, M, HQ, K)), _dev(p_prev, "p_prev", torch.float32, (B, HQ, K)),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), int(window or 0), B, int(t_start), M,
        cap, HQ, H, K, V, int(chunk), _dtype_code(q), float(scale) if scale else 0.0,
        _dev(k_tilde, "k_tilde", dt, (B, cap, HQ, K)),
        _dev(r_cache, "r_cache", torch.float32, (B, (cap + chunk - 1) // chunk, HQ, K)),
        _dev(p_last, "p_last", torch.float32, (B, HQ, K)), _dev(v_cache, "v_cache", dt),
        _dev(out, "out", dt, (B, M, HQ, V)), _dev(lse, "lse", torch.float32, (B, M, HQ)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(q.device))
    _check(st, "wall_attn_chunk")
    return out


def wall_attn_decode_noalloc(q, p_curr, v, k_tilde, r_cache, T_kv, out, lse=None,
                             sink_bias=None, scale=None, chunk=64):
    """wall_attn_decode without a workspace: the split partials live in a fixed
    4 MiB device array inside the library (for callers that cannot allocate at
    decode time).  `out` (and `lse`) must be allocated by the caller."""
    lib = load_library()
    B, cap, HQ, K = k_tilde.shape
    H, V = v.shape[2], v.shape[3]
    dt = k_tilde.dtype
    st = lib.wall_attn_decode_noalloc(
        _dev(q, "q", dt), _dev(p_curr, "p_curr", torch.float32), _dev(v, "v", dt, (B, cap, H, V)),
        _dev(k_tilde, "k_tilde", dt), _dev(r_cache, "r_cache", torch.float32),
        _dev(sink_bias, "sink_bias", torch.float32, (HQ,)), B, int(T_kv), cap, HQ, H, K, V,
        int(chunk), _dtype_code(k_tilde), float(scale) if scale else 0.0,
        _dev(out, "out", dt, (B, 1, HQ, V)), _dev(lse, "lse", torch.float32), _stream(q.device))
    _check(st, "wall_attn_decode_noalloc")
    return out


def wall_device_error(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error status."""
    return int(load_library().wall_device_error(_stream(device)))


def wall_debug_set_stage_events(before=None, between=None, after=None):
    """Profiling hook: torch.cuda.Event objects recorded at kernel boundaries (None clears)."""
    h = [ctypes.c_void_p(e.cuda_event) if e is not None else None for e in (before, between, after)]
    load_library().wall_debug_set_stage_events(*h)


def wall_debug_set_fault(mode: int, wait_ms: int = 0):
    """Testing hook: mode 1 starves the prefill consumers so their bounded waits expire."""
    load_library().wall_debug_set_fault(int(mode), int(wait_ms))


class KVCache:
    """Device tensors of a streaming decode: k_tilde, r_cache, v cache and the running prefix P.

    The caller writes value rows into ``v``; ``append`` folds the decay of new
    keys into ``k_tilde`` (README "Decode": build once, then append token by
    token) and returns P at the last appended row, which is the ``p_curr`` of
    the next decode step.
    """

    def __init__(self, B, cap, HQ, H, K, V, dtype=torch.bfloat16, chunk=64, device="cuda",
                 gate=False):
        self.B, self.cap, self.HQ, self.H, self.K, self.V, self.chunk = B, cap, HQ, H, K, V, chunk
        # scalar gate (models with g_scalar): PS per row and head, and PS at the last row
        self.gs_cache = torch.empty((B, cap, HQ), dtype=torch.float32, device=device) if gate else None
        self.gs = torch.zeros((B, HQ), dtype=torch.float32, device=device) if gate else None
        self._gs_next = torch.zeros_like(self.gs) if gate else None  # PS out of a fused step
        nc = (cap + chunk - 1) // chunk
        self.k_tilde = torch.empty((B, cap, HQ, K), dtype=dtype, device=device)
        self.r_cache = torch.empty((B, nc, HQ, K), dtype=torch.float32, device=device)
        self.v = torch.empty((B, cap, H, V), dtype=dtype, device=device)
        self.p = torch.zeros((B, HQ, K), dtype=torch.float32, device=device)
        self._p_next = torch.zeros_like(self.p)  # P_last of a fused step (must not be p_prev)
        self.length = 0
        self.workspace = torch.empty(max(wall_attn_decode_workspace_size(B, cap, HQ, H, V, chunk), 1),
                                     dtype=torch.uint8, device=device)

    def append(self, k_new, g_new, v_new=None, gs_new=None):
        T_new = k_new.shape[1]
        if v_new is not None:
            self.v[:, self.length:self.length + T_new].copy_(v_new)
        wall_build_kv_cache(k_new, g_new, self.k_tilde, self.r_cache, self.p,
                            t_start=self.length, p_prev=self.p if self.length > 0 else None,
                            chunk=self.chunk)
        if self.gs_cache is not None:
            if gs_new is None:
                raise ValueError("this cache carries the scalar gate: pass gs_new")
            wall_build_gate_cache(gs_new, self.gs_cache, self.gs, t_start=self.length,
                                  gs_prev=self.gs if self.length > 0 else None)
        self.length += T_new
        return self.p

    def decode(self, q, sink_bias=None, scale=None, out=None, lse=None):
        if self.gs_cache is not None:
            return wall_attn_decode_gated(q, self.p, self.gs, self.v, self.k_tilde, self.r_cache,
                                          self.gs_cache, T_kv=self.length, sink_bias=sink_bias,
                                          scale=scale, chunk=self.chunk, out=out, lse=lse,
                                          workspace=self.workspace)
        return wall_attn_decode(q, self.p, self.v, self.k_tilde, self.r_cache, self.length,
                                sink_bias=sink_bias, scale=scale, chunk=self.chunk, out=out,
                                lse=lse, workspace=self.workspace)

    def step(self, q, k_new, g_new, v_new, sink_bias=None, scale=None, out=None, lse=None,
             gs_new=None):
        """append(k_new, g_new, v_new) then decode(q), fused into the decode's launches
        (with the scalar gate, gs_new [B,1,HQ] joins the gate cache the same way).

        The kernel reads P (and PS) from one buffer and writes the new value to another, so
        after the call ``self.p`` / ``self.gs`` are the other tensors: read them afresh.
        """
        if self.gs_cache is not None:
            if gs_new is None:
                raise ValueError("this cache carries the scalar gate: pass gs_new")
            o = wall_attn_decode_step_gated(q, k_new, g_new, v_new, gs_new, self.k_tilde,
                                            self.r_cache, self.v, self.p, self._p_next,
                                            self.gs_cache, self.gs, self._gs_next,
                                            T_kv=self.length + 1, sink_bias=sink_bias,
                                            scale=scale, chunk=self.chunk, out=out, lse=lse,
                                            workspace=self.workspace)
            self.gs, self._gs_next = self._gs_next, self.gs
        else:
            o = wall_attn_decode_step(q, k_new, g_new, v_new, self.k_tilde, self.r_cache, self.v,
                                      self.p, self._p_next, T_kv=self.length + 1,
                                      sink_bias=sink_bias, scale=scale, chunk=self.chunk, out=out,
                                      lse=lse, workspace=self.workspace)
        self.p, self._p_next = self._p_next, self.p
        self.length += 1
        return o


class PagedKVCache:
    """A paged decode cache: pools of fixed-size blocks plus one block table per sequence.

    Blocks are handed out from a free list on the host as sequences grow
    (``reserve``) and returned when a sequence is dropped (``release``); the
    device block table is refreshed from the host copy after each change.  Value
    rows are written by ``append`` (a scatter through the table) or by the caller.
    """

    def __init__(self, B, num_blocks, block_size, max_blocks, HQ, H, K, V, dtype=torch.bfloat16,
                 chunk=64, device="cuda", gate=False):
        if block_size % chunk:
            raise ValueError("block_size must be a multiple of chunk")
        self.B, self.HQ, self.H, self.K, self.V, self.chunk = B, HQ, H, K, V, chunk
        self.num_blocks, self.block_size, self.max_blocks = num_blocks, block_size, max_blocks
        self.k_tilde = torch.empty((num_blocks, block_size, HQ, K), dtype=dtype, device=device)
        self.r_cache = torch.empty((num_blocks, block_size // chunk, HQ, K), dtype=torch.float32,
                                   device=device)
        self.v = torch.zeros((num_blocks, block_size, H, V), dtype=dtype, device=device)
        self.p = torch.zeros((B, HQ, K), dtype=torch.float32, device=device)
        self._p_next = torch.zeros_like(self.p)  # P_last of a fused step (must not be p_prev)
        self.gs_cache = (torch.empty((num_blocks, block_size, HQ), dtype=torch.float32,
                                     device=device) if gate else None)
        self.gs = torch.zeros((B, HQ), dtype=torch.float32, device=device) if gate else None
        self._gs_next = torch.zeros_like(self.gs) if gate else None  # PS out of a fused step
        self.free = list(range(num_blocks))
        self.host_table = [[] for _ in range(B)]
        self.block_table = torch.zeros((B, max_blocks), dtype=torch.int32, device=device)
        self.lengths = [0] * B
        self.workspace = torch.empty(
            max(wall_attn_decode_workspace_size(B, max_blocks * block_size, HQ, H, V, chunk), 1),
            dtype=torch.uint8, device=device)

    def _sync_table(self):
        t = torch.zeros((self.B, self.max_blocks), dtype=torch.int32)
        for b, blocks in enumerate(self.host_table):
            if blocks:
                t[b, :len(blocks)] = torch.tensor(blocks, dtype=torch.int32)
        self.block_table.copy_(t)

    def reserve(self, b, rows):
        """Make batch row b hold at least `rows` rows (allocates blocks)."""
        need = (rows + self.block_size - 1) // self.block_size
        if need > self.max_blocks:
            raise ValueError("sequence longer than max_blocks * block_size")
        changed = False
        while len(self.host_table[b]) < need:
            if not self.free:
                raise MemoryError("paged cache pool exhausted")
            self.host_table[b].append(self.free.pop(0))
            changed = True
        if changed:
            self._sync_table()

    def release(self, b):
        self.free.extend(self.host_table[b])
        self.host_table[b] = []
        self.lengths[b] = 0
        self._sync_table()

    def rows_of(self, b, t0, t1):
        """Physical pool rows of logical rows [t0, t1) of batch row b (host list)."""
        bs = self.block_size
        return [self.host_table[b][t // bs] * bs + t % bs for t in range(t0, t1)]

    def prefill(self, k, g, v, gs=None):
        """Build rows 0 .. T-1 of every batch row (all rows start empty)."""
        B, T = k.shape[0], k.shape[1]
        for b in range(B):
            self.reserve(b, T)
        wall_build_kv_cache_paged(k, g, self.block_table, self.k_tilde, self.r_cache, self.p,
                                  t_start=0, chunk=self.chunk)
        if self.gs_cache is not None:
            if gs is None:
                raise ValueError("this cache carries the scalar gate: pass gs")
            wall_build_gate_cache(gs, self.gs_cache, self.gs, block_table=self.block_table)
        for b in range(B):
            rows = torch.tensor(self.rows_of(b, 0, T), device=self.v.device)
            self.v.view(-1, self.H, self.V)[rows] = v[b]
            self.lengths[b] = T
        return self.p

    def append(self, k_new, g_new, v_new, t_pos, gs_new=None):
        """One token per batch row at t_pos (host list of ints) = each row's current length."""
        for b, t in enumerate(t_pos):
            self.reserve(b, t + 1)
        tp = torch.tensor(t_pos, dtype=torch.int32, device=k_new.device)
        wall_append_kv_cache_paged(k_new, g_new, self.block_table, self.k_tilde, self.r_cache,
                                   self.p, tp, chunk=self.chunk)
        if self.gs_cache is not None:
            if gs_new is None:
                raise ValueError("this cache carries the scalar gate: pass gs_new")
            wall_append_gate_cache(gs_new, self.gs_cache, self.gs, tp, block_table=self.block_table)
        rows = torch.tensor([self.rows_of(b, t, t + 1)[0] for b, t in enumerate(t_pos)],
                            device=self.v.device)
        self.v.view(-1, self.H, self.V)[rows] = v_new[:, 0]
        for b, t in enumerate(t_pos):
            self.lengths[b] = t + 1
        return self.p

    def decode(self, q, sink_bias=None, scale=None, out=None, lse=None):
        seqlens = torch.tensor(self.lengths, dtype=torch.int32, device=q.device)
        if self.gs_cache is not None:
            return wall_attn_decode_gated(q, self.p[:, None], self.gs, self.v, self.k_tilde,
                                          self.r_cache, self.gs_cache, seqlens=seqlens,
                                          block_table=self.block_table, sink_bias=sink_bias,
                                          scale=scale, chunk=self.chunk, out=out, lse=lse,
                                          workspace=self.workspace)
        return wall_attn_decode_paged(q, self.p[:, None], self.v, self.k_tilde, self.r_cache,
                                      seqlens, self.block_table, sink_bias=sink_bias, scale=scale,
                                      chunk=self.chunk, out=out, lse=lse, workspace=self.workspace)

    def step(self, q, k_new, g_new, v_new, t_pos, sink_bias=None, scale=None, out=None, lse=None,
             gs_new=None):
        """append(k_new, g_new, v_new, t_pos) then decode(q), fused into the decode's launches;
        t_pos (host list) = each row's current length, where its new token goes.  As for
        KVCache.step, ``self.p`` (and ``self.gs``) are different tensors after the call."""
        for b, t in enumerate(t_pos):
            self.reserve(b, t + 1)
        seqlens = torch.tensor([t + 1 for t in t_pos], dtype=torch.int32, device=q.device)
        if self.gs_cache is not None:
            if gs_new is None:
                raise ValueError("this cache carries the scalar gate: pass gs_new")
            o = wall_attn_decode_step_gated(q, k_new, g_new, v_new, gs_new, self.k_tilde,
                                            self.r_cache, self.v, self.p, self._p_next,
                                            self.gs_cache, self.gs, self._gs_next,
                                            seqlens=seqlens, block_table=self.block_table,
                                            sink_bias=sink_bias, scale=scale, chunk=self.chunk,
                                            out=out, lse=lse, workspace=self.workspace)
            self.gs, self._gs_next = self._gs_next, self.gs
        else:
            o = wall_attn_decode_step(q, k_new, g_new, v_new, self.k_tilde, self.r_cache, self.v,
                                      self.p, self._p_next, seqlens=seqlens,
                                      block_table=self.block_table, sink_bias=sink_bias,
                                      scale=scale, chunk=self.chunk, out=out, lse=lse,
                                      workspace=self.workspace)
        self.p, self._p_next = self._p_next, self.p
        for b, t in enumerate(t_pos):
            self.lengths[b] = t + 1
        return o
