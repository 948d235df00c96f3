"""Paged decode caches (block tables) on the GPU.

The pages describe PagedAttention: a pool of fixed-size physical KV blocks,
each sequence listing the blocks that hold its logical rows.  Checks:
  - a paged cache built through a shuffled block table holds, row for row,
    exactly the dense cache's k_tilde and anchors (bit-identical), and the
    paged decode equals the dense per-sequence-length decode bit for bit;
  - the paged decode of each sequence's last token equals the oracle's
    prefill row (Wall Attention README "Tests": decode == prefill);
  - streaming: per-row appends through the table at each row's own position,
    then a decode, equal the prefill row of the token just appended, for every
    sequence, with blocks handed out as sequences grow.
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


def _inputs(B, T, HQ, H, K, V, dtype, seed, sink=False):
    spec = W.PrefillSpec("paged", B=B, T=T, HQ=HQ, H=H, K=K, V=V, dtype=dtype,
                         g_kind="negsoftplus", sink=sink, seed=seed)
    return spec, W.gen_prefill(spec, device="cuda")


def _shuffled_tables(B, maxblk, nblk, seed):
    """Each batch row gets maxblk distinct pool blocks, in a random order."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(nblk)[:B * maxblk].reshape(B, maxblk)
    return torch.tensor(perm, dtype=torch.int32, device="cuda")


CASES = [
    dict(B=3, lens=(300, 517, 64), HQ=8, H=2, K=128, V=128, dtype="bf16", bs=64, chunk=64),
    dict(B=2, lens=(700, 129), HQ=4, H=1, K=64, V=128, dtype="bf16", bs=256, chunk=64),
    dict(B=2, lens=(200, 97), HQ=2, H=2, K=128, V=64, dtype="f32", bs=128, chunk=32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"bs{c['bs']}C{c['chunk']}{c['dtype']}")
def test_paged_cache_and_decode_equal_dense(wall, case):
    B, lens, HQ, H, K, V = case["B"], case["lens"], case["HQ"], case["H"], case["K"], case["V"]
    bs, C = case["bs"], case["chunk"]
    T = max(lens)
    spec, d = _inputs(B, T, HQ, H, K, V, case["dtype"], seed=71, sink=True)
    dt = spec.torch_dtype
    maxblk = (T + bs - 1) // bs
    nblk = B * maxblk + 3                      # spare blocks stay untouched
    cap = maxblk * bs
    table = _shuffled_tables(B, maxblk, nblk, seed=72)
    # dense reference cache (GPU), one build per row through a one-row view
    kt = torch.zeros((B, cap, HQ, K), dtype=dt, device="cuda")
    rc = torch.zeros((B, cap // C, HQ, K), dtype=torch.float32, device="cuda")
    p = torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda")
    vc = torch.zeros((B, cap, H, V), dtype=dt, device="cuda")
    # paged pools: filled with NaN so any row read past a sequence's end would show
    ktp = torch.full((nblk, bs, HQ, K), float("nan"), dtype=dt, device="cuda")
    rp = torch.full((nblk, bs // C, HQ, K), float("nan"), dtype=torch.float32, device="cuda")
    vp = torch.full((nblk, bs, H, V), float("nan"), dtype=dt, device="cuda")
    pp = torch.zeros((B, HQ, K), dtype=torch.float32, device="cuda")
    for b, L in enumerate(lens):
        kb, gb = d["k"][b:b + 1, :L].contiguous(), d["g"][b:b + 1, :L].contiguous()
        wall.wall_build_kv_cache(kb, gb, kt[b:b + 1], rc[b:b + 1], p[b:b + 1], chunk=C)
        wall.wall_build_kv_cache_paged(kb, gb, table[b:b + 1].contiguous(), ktp, rp, pp[b:b + 1],
                                       chunk=C)
        vc[b, :L].copy_(d["v"][b, :L])
        phys = table[b].long()[torch.arange(L, device="cuda") // bs] * bs + \
            torch.arange(L, device="cuda") % bs
        vp.view(-1, H, V)[phys] = d["v"][b, :L]
    torch.cuda.synchronize()
    tab = table.cpu().numpy()
    for b, L in enumerate(lens):
        rows = np.arange(L)
        phys = tab[b][rows // bs] * bs + rows % bs
        assert torch.equal(ktp.view(-1, HQ, K)[torch.tensor(phys, device="cuda")], kt[b, :L])
        ch = np.arange((L + C - 1) // C)
        pch = tab[b][(ch * C) // bs] * (bs // C) + ((ch * C) % bs) // C
        assert torch.equal(rp.view(-1, HQ, K)[torch.tensor(pch, device="cuda")],
                           rc[b, :len(ch)])
    assert torch.equal(pp, p)
    q = torch.stack([d["q"][b, L - 1] for b, L in enumerate(lens)])[:, None].contiguous()
    seqlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o_dense = wall.wall_attn_decode(q, p[:, None].contiguous(), vc, kt, rc, cap,
                                    sink_bias=d["sink_bias"], scale=d["scale"], chunk=C,
                                    seqlens=seqlens)
    o_paged = wall.wall_attn_decode_paged(q, pp[:, None].contiguous(), vp, ktp, rp, seqlens, table,
                                          sink_bias=d["sink_bias"], scale=d["scale"], chunk=C)
    torch.cuda.synchronize()
    assert torch.isfinite(o_paged.float()).all()
    assert torch.equal(o_paged, o_dense)
    rows = [b * T + L - 1 for b, L in enumerate(lens)]
    ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                            scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
    assert_close(o_paged[:, 0], ro, dt, "paged decode vs oracle")


@pytest.mark.parametrize("bs", [64, 128])
def test_paged_streaming_append_and_decode(wall, bs):
    """Blocks are taken from the pool as each sequence grows; every step equals the
    prefill row of the token just appended."""
    start, steps = (150, 63, 1), 70
    B, HQ, H, K, V, C = len(start), 8, 2, 128, 128, 64
    T = max(start) + steps
    spec, d = _inputs(B, T, HQ, H, K, V, "bf16", seed=81, sink=True)
    maxblk = (T + bs - 1) // bs
    cache = wall.PagedKVCache(B, num_blocks=B * maxblk + 2, block_size=bs, max_blocks=maxblk,
                              HQ=HQ, H=H, K=K, V=V, chunk=C)
    for b, L in enumerate(start):  # prefixes of different lengths, one row at a time
        cache.reserve(b, L)
    for b, L in enumerate(start):
        kb, gb = d["k"][b:b + 1, :L].contiguous(), d["g"][b:b + 1, :L].contiguous()
        wall.wall_build_kv_cache_paged(kb, gb, cache.block_table[b:b + 1].contiguous(),
                                       cache.k_tilde, cache.r_cache, cache.p[b:b + 1], chunk=C)
        rows = torch.tensor(cache.rows_of(b, 0, L), device="cuda")
        cache.v.view(-1, H, V)[rows] = d["v"][b, :L]
        cache.lengths[b] = L
    lens = list(start)
    for s_ in range(steps):
        k_new = torch.stack([d["k"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        g_new = torch.stack([d["g"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        v_new = torch.stack([d["v"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        cache.append(k_new, g_new, v_new, lens)
        q = torch.stack([d["q"][b, L] for b, L in enumerate(lens)])[:, None].contiguous()
        o = cache.decode(q, sink_bias=d["sink_bias"], scale=d["scale"])
        if s_ % 7 == 0 or s_ == steps - 1:
            rows = [b * T + L for b, L in enumerate(lens)]
            ro, _ = oracle.wall_fwd(d["q"], d["k"], d["v"], d["g"], sink_bias=d["sink_bias"],
                                    scale=d["scale"], rows=rows, threads=ORACLE_THREADS)
            assert_close(o[:, 0], ro, torch.bfloat16, f"paged step {s_}")
        lens = [L + 1 for L in lens]
    assert wall.wall_device_error() == 0
    # dropping a sequence returns its blocks to the pool
    n_free = len(cache.free)
    cache.release(0)
    assert len(cache.free) == n_free + (lens[0] + bs - 1) // bs
