"""Helpers shared by the GPU parity tests: tolerance checks against the oracle."""
import os

import numpy as np
import torch

# Wall attention parity tolerances: bf16 inputs |d| <= 2e-2 + 2e-2 |ref|;
# fp32 inputs |d| <= 1e-4 + 1e-4 |ref|.
TOL = {torch.bfloat16: (2e-2, 2e-2), torch.float32: (1e-4, 1e-4)}

ORACLE_THREADS = int(os.environ.get("WALL_ORACLE_THREADS", "0"))


def assert_close(got, ref, dtype, what):
    """Element-wise |got - ref| <= atol + rtol |ref| (ref from the oracle, float64)."""
    atol, rtol = TOL[dtype]
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    err = np.abs(g - r)
    bound = atol + rtol * np.abs(r)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside |d| <= {atol} + {rtol}|ref|; "
            f"max err {float(np.nanmax(err)):.3e}; first bad {idx.tolist()} "
            f"got {[float(g[tuple(i)]) for i in idx]} ref {[float(r[tuple(i)]) for i in idx]}")


def sample_rows(B, T, extra=(), n_random=16, seed=0):
    """Flattened b*T + t rows: ragged tail, block edges, both ends, plus a seeded sample."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(B):
        for t in (0, 1, 63, 64, 127, 128, 129, T // 2, T - 129, T - 128, T - 2, T - 1, *extra):
            if 0 <= t < T:
                rows.add(b * T + t)
        for t in rng.integers(0, T, n_random):
            rows.add(b * T + int(t))
    return np.array(sorted(rows), dtype=np.int64)
