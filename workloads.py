"""Seeded synthetic inputs for Wall attention (decayed softmax attention).

This module only draws random numbers in the shapes and distributions of the
workloads named on the Wall Attention README page (sections "Usage /
Training-Prefill" and "Decode"): q, k, v ~ N(0, 1); per-channel log-decay g in
[B, T, HQ, K]; optional scalar gate g_scalar [B, T, HQ]; per-head sink_bias
[HQ]; varlen document lengths for cu_seqlens packing.  It holds none of the
method's arithmetic, so both the CPU oracle (tests only) and the CUDA path can
consume the very same tensors.

Values are drawn in fp32 and rounded once to the workload dtype; every
consumer (oracle included) reads those rounded values.  Generation uses a
torch.Generator on the requested device, so the very large decode workload can
be drawn directly in device memory; the oracle then receives host copies of
the slices it checks.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch

__all__ = [
    "PrefillSpec", "DecodeSpec", "PREFILL", "DECODE", "gen_prefill", "gen_decode",
    "doc_lengths", "random_prefill_spec",
]


@dataclass(frozen=True)
class PrefillSpec:
    """One prefill workload: shapes plus value distributions."""
    name: str
    B: int
    T: int                      # total tokens per batch row (sum of docs when varlen)
    HQ: int
    H: int
    K: int
    V: int
    dtype: str                  # "f32" | "bf16"
    g_kind: str = "normal002"   # "normal002": 0.02*N(0,1); "negsoftplus": -softplus(N(0,1)-4); "zero";
                                # strong decay: "strong", "strong_cache", "strong_all", "spike" (_decay)
    g_scalar: bool = False      # draw g_scalar = -softplus(N(0,1)-4) [B,T,HQ]
    sink: bool = False          # draw sink_bias ~ N(0,1) [HQ]
    window: int = 0             # <=0: no window
    docs: Optional[tuple] = None  # document lengths (B must be 1) -> cu_seqlens
    scale: Optional[float] = None  # None -> K**-0.5
    seed: int = 1000

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else self.K ** -0.5


@dataclass(frozen=True)
class DecodeSpec:
    """Decode workload: prefix of T0 tokens built into the cache, then `steps` appends."""
    name: str
    B: int
    T0: int
    steps: int
    HQ: int
    H: int
    K: int
    V: int
    C: int = 64
    dtype: str = "bf16"
    g_kind: str = "negsoftplus"
    sink: bool = False
    seed: int = 1005

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def cap(self) -> int:
        return self.T0 + self.steps


def doc_lengths(n_docs: int, lo: int, hi: int, seed: int) -> tuple:
    """Document lengths uniform on the integers [lo, hi], seeded (CPU generator)."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n_docs,), generator=gen))


_VARLEN_DOCS = doc_lengths(16, 256, 4096, seed=1003)

# The five workloads: tiny fp32, GQA bf16, long T=8K bf16 (headline prefill),
# packed varlen + window + sink, decode (headline decode).
PREFILL = {
    "tiny": PrefillSpec("tiny", B=1, T=256, HQ=2, H=2, K=64, V=64, dtype="f32",
                        g_kind="normal002", seed=1000),
    "tiny_g0": PrefillSpec("tiny_g0", B=1, T=256, HQ=2, H=2, K=64, V=64, dtype="f32",
                           g_kind="zero", seed=1000),
    "gqa": PrefillSpec("gqa", B=2, T=1024, HQ=8, H=4, K=64, V=64, dtype="bf16",
                       g_kind="normal002", seed=1001),
    "long": PrefillSpec("long", B=1, T=8192, HQ=32, H=8, K=128, V=128, dtype="bf16",
                        g_kind="negsoftplus", g_scalar=True, seed=1002),
    "varlen_window": PrefillSpec("varlen_window", B=1, T=sum(_VARLEN_DOCS), HQ=16, H=4,
                                 K=128, V=128, dtype="bf16", g_kind="normal002",
                                 sink=True, window=2048, docs=_VARLEN_DOCS, seed=1003),
}

DECODE = {
    "decode": DecodeSpec("decode", B=32, T0=32768, steps=64, HQ=32, H=8, K=128, V=128,
                         C=64, dtype="bf16", g_kind="negsoftplus", seed=1005),
}


def _gen(device, seed):
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    return gen


def _normal(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _decay(kind, shape, gen, device):
    if kind == "zero":
        return torch.zeros(shape, device=device, dtype=torch.float32)
    z = _normal(shape, gen, device)
    if kind == "normal002":
        return 0.02 * z
    if kind == "negsoftplus":
        return -torch.nn.functional.softplus(z - 4.0)
    # Strong per-channel decay (the method's g = -softplus(.) is unbounded below): a few
    # channels forget within a handful of tokens while the rest keep a long memory.
    sp = torch.nn.functional.softplus
    K = shape[-1]
    quarter = max(3, K // 4)
    if kind == "strong":        # channels 0..2 constant -0.5, -2, -8; next quarter
        g = -sp(z - 4.0)        # -softplus(N+2) (~2.1 per token); the rest -softplus(N-4)
        g[..., 3:quarter] = -sp(z[..., 3:quarter] + 2.0)
        g[..., 0], g[..., 1], g[..., 2] = -0.5, -2.0, -8.0
        return g
    if kind == "strong_cache":  # strong, yet inside one 32-row cache chunk's range:
        g = -sp(z - 4.0)        # channels 0, 1 constant -0.5, -2; next quarter -softplus(N+1)
        g[..., 2:quarter] = -sp(z[..., 2:quarter] + 1.0)
        g[..., 0], g[..., 1] = -0.5, -2.0
        return g
    if kind == "strong_all":    # every channel -softplus(N(0,1)+2)
        return -sp(z + 2.0)
    if kind == "spike":         # mild everywhere except a decay of 100 in channel 5 at two
        g = -sp(z - 4.0)        # rows (T/3 and 2T/3): only the blocks holding them are wide
        T = shape[1]
        for t in (T // 3, (2 * T) // 3):
            g[:, t, ..., 5] = -100.0
        return g
    raise ValueError(f"unknown decay distribution {kind!r}")


def gen_prefill(spec: PrefillSpec, device="cpu") -> dict:
    """Draw one prefill workload. Returns tensors in the workload dtype plus metadata.

    Keys: q [B,T,HQ,K], k [B,T,H,K], v [B,T,H,V], g [B,T,HQ,K], g_scalar [B,T,HQ] or None,
    sink_bias [HQ] fp32 or None, cu_seqlens int32 [N+1] or None, window, scale.
    Draw order is fixed: q, k, v, g, g_scalar, sink.
    """
    gen = _gen(device, spec.seed)
    B, T, HQ, H, K, V = spec.B, spec.T, spec.HQ, spec.H, spec.K, spec.V
    dt = spec.torch_dtype
    q = _normal((B, T, HQ, K), gen, device).to(dt)
    k = _normal((B, T, H, K), gen, device).to(dt)
    v = _normal((B, T, H, V), gen, device).to(dt)
    g = _decay(spec.g_kind, (B, T, HQ, K), gen, device).to(dt)
    gs = None
    if spec.g_scalar:
        gs = (-torch.nn.functional.softplus(_normal((B, T, HQ), gen, device) - 4.0)).to(dt)
    sink = _normal((HQ,), gen, device) if spec.sink else None
    cu = None
    if spec.docs is not None:
        assert B == 1 and sum(spec.docs) == T
        cu = torch.tensor([0] + list(_cumsum(spec.docs)), dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, g=g, g_scalar=gs, sink_bias=sink, cu_seqlens=cu,
                window=spec.window, scale=spec.softmax_scale)


def _cumsum(xs):
    s = 0
    for x in xs:
        s += x
        yield s


def gen_decode(spec: DecodeSpec, device="cpu") -> dict:
    """Draw the decode workload for all cap = T0 + steps positions.

    Keys: q [B,steps,HQ,K] (one query per generated token), k [B,cap,H,K],
    v [B,cap,H,V], g [B,cap,HQ,K], sink_bias or None, scale.
    Draw order is fixed: per batch row k, v, g; then q, sink.
    """
    gen = _gen(device, spec.seed)
    B, cap, HQ, H, K, V = spec.B, spec.cap, spec.HQ, spec.H, spec.K, spec.V
    dt = spec.torch_dtype
    # Drawn one batch row at a time so the fp32 temporaries stay small
    # (the full decode workload is ~13 GB once rounded to bf16).
    k = torch.empty((B, cap, H, K), dtype=dt, device=device)
    v = torch.empty((B, cap, H, V), dtype=dt, device=device)
    g = torch.empty((B, cap, HQ, K), dtype=dt, device=device)
    for b in range(B):
        k[b] = _normal((cap, H, K), gen, device).to(dt)
        v[b] = _normal((cap, H, V), gen, device).to(dt)
        g[b] = _decay(spec.g_kind, (cap, HQ, K), gen, device).to(dt)
    q = _normal((B, spec.steps, HQ, K), gen, device).to(dt)
    sink = _normal((HQ,), gen, device) if spec.sink else None
    return dict(q=q, k=k, v=v, g=g, sink_bias=sink, scale=K ** -0.5)


def random_prefill_spec(seed: int, dtype="bf16", **over) -> PrefillSpec:
    """A small randomized shape for parity sweeps (ragged T, GQA, optional pieces)."""
    gen = torch.Generator(device="cpu").manual_seed(seed)

    def pick(xs):
        return xs[int(torch.randint(0, len(xs), (1,), generator=gen))]

    K = pick([64, 128])
    HQ, H = pick([(2, 2), (4, 1), (4, 2), (6, 3)])
    T = int(torch.randint(1, 700, (1,), generator=gen))
    spec = PrefillSpec(f"rand{seed}", B=pick([1, 2]), T=T, HQ=HQ, H=H, K=K, V=pick([64, 128]),
                       dtype=dtype, g_kind=pick(["normal002", "negsoftplus"]),
                       g_scalar=bool(pick([0, 1])), sink=bool(pick([0, 1])),
                       window=pick([0, 0, 1, 37, 200]), seed=5000 + seed)
    return replace(spec, **over)
