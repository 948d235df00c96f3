"""The benchmark's work counts against brute force (CPU only).

`value` is prefill FLOP over time, with the FLOP taken as 2*(K+V) per admitted
(query, key) pair; the admitted set is causal attention inside each packed
document, cut to a sliding window of the last `window` keys when one is given
(the Wall Attention README's usage section: causal, window, cu_seqlens).  These
tests count that set pair by pair and compare with the closed form the bench
uses, and check the bench's whole-job rate arithmetic.
"""
import itertools

import numpy as np
import pytest

import bench
import workloads as W


def brute_pairs(T, docs, window):
    """Admitted (i, j): same document, j <= i, and i - j < window when window > 0."""
    doc = np.repeat(np.arange(len(docs)), docs)
    assert doc.size == T
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    ok = (doc[:, None] == doc[None, :]) & (j <= i)
    if window > 0:
        ok &= (i - j) < window
    return int(ok.sum())


CASES = [
    (257, None, 0),
    (257, None, 1),
    (257, None, 64),
    (300, (90, 210), 0),
    (518, (100, 37, 250, 1, 130), 96),
    (518, (100, 37, 250, 1, 130), 300),
    (40, (1,) * 40, 5),
    (129, (128, 1), 128),
]


@pytest.mark.parametrize("T,docs,window", CASES)
def test_prefill_pairs_equals_brute_force(T, docs, window):
    spec = W.PrefillSpec("count", B=1, T=T, HQ=1, H=1, K=64, V=64, dtype="bf16",
                         window=window, docs=docs)
    assert bench.prefill_pairs(spec) == brute_pairs(T, docs or (T,), window)


def test_prefill_flops_scale_with_heads_batch_and_width():
    base = W.PrefillSpec("count", B=1, T=200, HQ=1, H=1, K=64, V=64, dtype="bf16")
    pairs = brute_pairs(200, (200,), 0)
    for B, HQ, K, V in itertools.product((1, 3), (1, 4), (64, 128), (64, 128)):
        spec = W.PrefillSpec("count", B=B, T=200, HQ=HQ, H=1, K=K, V=V, dtype="bf16")
        assert bench.prefill_flops(spec) == B * HQ * pairs * 2 * (K + V)
    assert bench.prefill_flops(base) == pairs * 256


def test_long_prefill_flops_match_the_quoted_figure():
    # the long prefill: B=1, T=8192, HQ=32, K=V=128, causal: 8192*8193/2 pairs per head
    spec = W.PREFILL["long"]
    assert bench.prefill_flops(spec) == 32 * (8192 * 8193 // 2) * 2 * 256
    assert abs(bench.prefill_flops(spec) - 5.498e11) / 5.498e11 < 1e-3


def test_weak_scaling_rate_is_whole_job_units_over_slowest_rank():
    # 3 ranks, each 5 units per step over 4 steps, slowest rank 2 s -> 30 units/s
    assert bench.weak_scaling_rate(5, 4, 3, 2000.0) == pytest.approx(30.0)
