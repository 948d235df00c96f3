"""C-ABI checks that need no GPU: the library loads, exports every function the
public header declares, and rejects bad arguments on the host before any
CUDA call (status codes, no crash)."""
import ctypes
import os
import re

import pytest

import decayed_softmax_attention_b200 as wall
from decayed_softmax_attention_b200 import build as wall_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wall_attn.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 5
BF16, F32 = 1, 0


@pytest.fixture(scope="module")
def lib():
    wall_build.build()
    return wall.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wall_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = _declared_functions()
    for n in ("wall_attn_fwd", "wall_build_kv_cache", "wall_attn_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert set(names) == set(wall.EXPORTED_SYMBOLS)
    for n in names:
        assert hasattr(lib, n), f"{n} missing from {wall.lib_path()}"


def test_status_strings(lib):
    for code in range(6):
        s = lib.wall_status_string(code).decode()
        assert s.startswith("WALL_")


def _fake(addr=0x1000):
    return ctypes.c_void_p(addr)


def _fwd(lib, **kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), g=_fake(), gs=None, sink=None, window=0, cu=None,
             nseq=0, B=1, T=64, HQ=4, H=2, K=64, V=64, dt=BF16, scale=0.0, o=_fake(), lse=None,
             ws=_fake(0x100000), wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.wall_attn_fwd(a["q"], a["k"], a["v"], a["g"], a["gs"], a["sink"], a["window"],
                             a["cu"], a["nseq"], a["B"], a["T"], a["HQ"], a["H"], a["K"], a["V"],
                             a["dt"], a["scale"], a["o"], a["lse"], a["ws"], a["wsb"], a["stream"])


def test_fwd_host_validation(lib):
    assert _fwd(lib, HQ=6, H=4) == INVALID            # HQ % H != 0
    assert _fwd(lib, K=96) == UNSUPPORTED
    assert _fwd(lib, V=32) == UNSUPPORTED
    assert _fwd(lib, dt=7) == INVALID
    assert _fwd(lib, B=-1) == INVALID
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, o=None) == INVALID
    assert _fwd(lib, q=_fake(0x1008)) == INVALID      # not 16-byte aligned
    assert _fwd(lib, ws=_fake(0x100010)) == INVALID   # workspace not 256-byte aligned
    assert _fwd(lib, cu=_fake(), nseq=2, B=2) == INVALID  # packing needs B == 1
    assert _fwd(lib, cu=_fake(), nseq=0) == INVALID
    assert _fwd(lib, wsb=16) == WORKSPACE
    assert _fwd(lib, T=0) == 0                        # empty input: no-op
    assert _fwd(lib, B=0) == 0


def _fwd_cache(lib, **kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), g=_fake(), gs=None, sink=None, window=0,
             B=1, T=64, HQ=4, H=2, K=64, V=64, dt=BF16, scale=0.0, o=_fake(), lse=None,
             ws=_fake(0x100000), wsb=1 << 40, cap=64, C=64, kt=_fake(0x2000), r=_fake(0x3000),
             p=_fake(0x4000), stream=None)
    a.update(kw)
    return lib.wall_attn_fwd_with_cache(
        a["q"], a["k"], a["v"], a["g"], a["gs"], a["sink"], a["window"], a["B"], a["T"],
        a["HQ"], a["H"], a["K"], a["V"], a["dt"], a["scale"], a["o"], a["lse"], a["ws"],
        a["wsb"], a["cap"], a["C"], a["kt"], a["r"], a["p"], a["stream"])


def test_fwd_with_cache_host_validation(lib):
    assert _fwd_cache(lib, C=48) == UNSUPPORTED
    assert _fwd_cache(lib, cap=32) == INVALID             # cache smaller than the prefill
    assert _fwd_cache(lib, kt=None) == INVALID
    assert _fwd_cache(lib, r=_fake(0x3004)) == INVALID    # anchors not 16-byte aligned
    assert _fwd_cache(lib, p=None) == INVALID
    assert _fwd_cache(lib, HQ=6, H=4) == INVALID          # the forward's own checks still apply
    assert _fwd_cache(lib, K=96) == UNSUPPORTED
    assert _fwd_cache(lib, wsb=16) == WORKSPACE
    assert _fwd_cache(lib, T=0, cap=0) == 0               # empty input: no-op


def test_fwd_workspace_size(lib):
    small = lib.wall_attn_fwd_workspace_size(1, 128, 2, 2, 64, 64, BF16)
    big = lib.wall_attn_fwd_workspace_size(1, 8192, 32, 8, 128, 128, BF16)
    f32 = lib.wall_attn_fwd_workspace_size(1, 128, 2, 2, 64, 64, F32)
    assert 0 < small < f32
    # anchored q and k dominate: 2 * B*HQ*T*K elements
    assert big >= 2 * 32 * 8192 * 128 * 2
    assert lib.wall_attn_fwd_workspace_size(0, 128, 2, 2, 64, 64, BF16) == 0


def _cache(lib, **kw):
    a = dict(k=_fake(), g=_fake(), p_prev=None, B=2, t0=0, Tn=64, cap=128, HQ=4, H=2, K=128,
             C=64, dt=BF16, kt=_fake(), r=_fake(), pl=_fake(), stream=None)
    a.update(kw)
    return lib.wall_build_kv_cache(a["k"], a["g"], a["p_prev"], a["B"], a["t0"], a["Tn"], a["cap"],
                                   a["HQ"], a["H"], a["K"], a["C"], a["dt"], a["kt"], a["r"],
                                   a["pl"], a["stream"])


def test_cache_host_validation(lib):
    assert _cache(lib, t0=100, Tn=64) == INVALID          # beyond capacity
    assert _cache(lib, t0=10, p_prev=None) == INVALID      # append needs the previous prefix
    assert _cache(lib, t0=0, p_prev=_fake()) == INVALID    # fresh build takes none
    assert _cache(lib, C=48) == UNSUPPORTED
    assert _cache(lib, K=80) == UNSUPPORTED
    assert _cache(lib, HQ=3) == INVALID
    assert _cache(lib, kt=None) == INVALID
    assert _cache(lib, r=_fake(0x1004)) == INVALID
    assert _cache(lib, Tn=0) == 0


def _dec(lib, **kw):
    a = dict(q=_fake(), pc=_fake(), v=_fake(), kt=_fake(), r=_fake(), sink=None, B=2, Tkv=100,
             cap=128, HQ=8, H=2, K=128, V=128, C=64, dt=BF16, scale=0.0, o=_fake(), lse=None,
             ws=_fake(), wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.wall_attn_decode(a["q"], a["pc"], a["v"], a["kt"], a["r"], a["sink"], a["B"],
                                a["Tkv"], a["cap"], a["HQ"], a["H"], a["K"], a["V"], a["C"],
                                a["dt"], a["scale"], a["o"], a["lse"], a["ws"], a["wsb"],
                                a["stream"])


def test_decode_host_validation(lib):
    assert _dec(lib, Tkv=0) == INVALID
    assert _dec(lib, Tkv=200) == INVALID                  # more rows than the cache holds
    assert _dec(lib, HQ=96, H=3) == UNSUPPORTED           # group of 32 query heads
    assert _dec(lib, K=32) == UNSUPPORTED
    assert _dec(lib, C=50) == UNSUPPORTED
    assert _dec(lib, kt=None) == INVALID
    assert _dec(lib, o=_fake(0x1002)) == INVALID
    assert _dec(lib, wsb=8) == WORKSPACE


def test_noalloc_decode_host_validation(lib):
    def call(**kw):
        a = dict(q=_fake(), pc=_fake(), v=_fake(), kt=_fake(), r=_fake(), sink=None, B=2, Tkv=100,
                 cap=128, HQ=8, H=2, K=128, V=128, C=64, dt=BF16, scale=0.0, o=_fake(), lse=None,
                 stream=None)
        a.update(kw)
        return lib.wall_attn_decode_noalloc(a["q"], a["pc"], a["v"], a["kt"], a["r"], a["sink"],
                                            a["B"], a["Tkv"], a["cap"], a["HQ"], a["H"], a["K"],
                                            a["V"], a["C"], a["dt"], a["scale"], a["o"], a["lse"],
                                            a["stream"])
    assert call(Tkv=0) == INVALID
    assert call(o=None) == INVALID
    assert call(K=96) == UNSUPPORTED
    # one split per (batch row, query head) no longer fits the fixed 4 MiB scratch
    assert call(B=512, HQ=16, H=4, Tkv=64, cap=64) == WORKSPACE
    assert call(B=0) == 0


def test_decode_workspace_monotone_in_length(lib):
    prev = 0
    for T in (1, 63, 64, 65, 640, 6400, 32768, 32832):
        ws = lib.wall_attn_decode_workspace_size(32, T, 32, 8, 128, 64)
        assert ws >= prev
        prev = ws


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, ImportError)):
        wall.wall_attn_fwd(q, torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16),
                           torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16), q)


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "decayed_softmax_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower().replace("oracle/", ""), f


def test_decode_varlen_host_validation(lib):
    def dv(**kw):
        a = dict(q=_fake(), pc=_fake(), v=_fake(), kt=_fake(), r=_fake(), sink=None,
                 lens=_fake(0x5000), B=2, Tkv=100, cap=128, HQ=8, H=2, K=128, V=128, C=64,
                 dt=BF16, scale=0.0, o=_fake(), lse=None, ws=_fake(), wsb=1 << 40, stream=None)
        a.update(kw)
        return lib.wall_attn_decode_varlen(
            a["q"], a["pc"], a["v"], a["kt"], a["r"], a["sink"], a["lens"], a["B"], a["Tkv"],
            a["cap"], a["HQ"], a["H"], a["K"], a["V"], a["C"], a["dt"], a["scale"], a["o"],
            a["lse"], a["ws"], a["wsb"], a["stream"])
    assert dv(lens=None) == INVALID                       # the lengths are required
    assert dv(lens=_fake(0x5002)) == INVALID              # int32 alignment
    assert dv(Tkv=200) == INVALID                         # largest length beyond the cache
    assert dv(HQ=96, H=3) == UNSUPPORTED
    assert dv(wsb=16) == WORKSPACE
    assert dv(B=0, lens=None) == 0                        # empty batch: no-op


def test_append_varlen_host_validation(lib):
    def av(**kw):
        a = dict(k=_fake(), g=_fake(), pp=_fake(), tp=_fake(0x6000), B=2, cap=64, HQ=4, H=2,
                 K=64, C=64, dt=BF16, kt=_fake(), r=_fake(), pl=_fake(), stream=None)
        a.update(kw)
        return lib.wall_append_kv_cache_varlen(a["k"], a["g"], a["pp"], a["tp"], a["B"], a["cap"],
                                               a["HQ"], a["H"], a["K"], a["C"], a["dt"], a["kt"],
                                               a["r"], a["pl"], a["stream"])
    assert av(tp=None) == INVALID
    assert av(pp=None) == INVALID
    assert av(C=48) == UNSUPPORTED
    assert av(K=80) == UNSUPPORTED
    assert av(HQ=3) == INVALID
    assert av(r=_fake(0x1004)) == INVALID
    assert av(B=0) == 0


def _bwd(lib, **kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), g=_fake(), gs=None, sink=None, window=0, cu=None,
             nseq=0, B=1, T=256, HQ=4, H=2, K=64, V=64, dt=BF16, scale=0.0, o=_fake(),
             lse=_fake(), do=_fake(), dlse=None, dq=_fake(), dk=_fake(), dv=_fake(), dg=_fake(),
             dgs=None, dsink=None, ws=_fake(0x100000), wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.wall_attn_bwd(a["q"], a["k"], a["v"], a["g"], a["gs"], a["sink"], a["window"],
                             a["cu"], a["nseq"], a["B"], a["T"], a["HQ"], a["H"], a["K"], a["V"],
                             a["dt"], a["scale"], a["o"], a["lse"], a["do"], a["dlse"], a["dq"],
                             a["dk"], a["dv"], a["dg"], a["dgs"], a["dsink"], a["ws"], a["wsb"],
                             a["stream"])


def test_bwd_host_validation(lib):
    assert _bwd(lib, lse=None) == INVALID                 # the forward's lse is required
    assert _bwd(lib, do=None) == INVALID
    assert _bwd(lib, dg=None) == INVALID
    assert _bwd(lib, gs=_fake()) == INVALID               # g_scalar without dg_scalar
    assert _bwd(lib, dgs=_fake()) == INVALID              # dg_scalar without g_scalar
    assert _bwd(lib, sink=_fake()) == INVALID             # sink without dsink
    assert _bwd(lib, dq=_fake(0x1008)) == INVALID         # misaligned output
    assert _bwd(lib, HQ=6, H=4) == INVALID
    assert _bwd(lib, cu=_fake(), nseq=2, B=2) == INVALID  # packing needs B == 1
    assert _bwd(lib, K=96) == UNSUPPORTED
    assert _bwd(lib, dt=7) == INVALID
    assert _bwd(lib, wsb=16) == WORKSPACE
    assert _bwd(lib, T=0) == 0                            # empty input: no-op


def test_bwd_workspace_size(lib):
    fwd = lib.wall_attn_fwd_workspace_size(1, 1024, 8, 4, 64, 64, BF16)
    bwd = lib.wall_attn_bwd_workspace_size(1, 1024, 8, 4, 64, 64, BF16)
    # the prepass's workspace plus fp32 accumulators of dq, dk_h and dv_h
    assert bwd >= fwd + 3 * 8 * 1024 * 64 * 4
    assert lib.wall_attn_bwd_workspace_size(0, 1024, 8, 4, 64, 64, BF16) == 0


def test_paged_host_validation(lib):
    def dec(**kw):
        a = dict(q=_fake(), p=_fake(), vp=_fake(), kp=_fake(), rp=_fake(), sink=None,
                 sl=_fake(0x7000), bt=_fake(0x8000), maxblk=4, B=2, nblk=8, bs=64, HQ=4, H=2,
                 K=128, V=128, C=64, dt=BF16, scale=0.0, o=_fake(), lse=None, ws=_fake(),
                 wsb=1 << 30, stream=None)
        a.update(kw)
        return lib.wall_attn_decode_paged(a["q"], a["p"], a["vp"], a["kp"], a["rp"], a["sink"],
                                          a["sl"], a["bt"], a["maxblk"], a["B"], a["nblk"], a["bs"],
                                          a["HQ"], a["H"], a["K"], a["V"], a["C"], a["dt"],
                                          a["scale"], a["o"], a["lse"], a["ws"], a["wsb"],
                                          a["stream"])
    assert dec(bt=None) == INVALID            # the block table is required
    assert dec(sl=None) == INVALID            # so are the per-sequence lengths
    assert dec(bs=96) == UNSUPPORTED          # block size not a multiple of the chunk
    assert dec(bs=32) == UNSUPPORTED          # smaller than the chunk
    assert dec(maxblk=0) == INVALID
    assert dec(nblk=0) == INVALID
    assert dec(bt=_fake(0x8002)) == INVALID   # misaligned table
    assert dec(wsb=16) == WORKSPACE
    assert dec(B=0) == 0

    def app(**kw):
        a = dict(k=_fake(), g=_fake(), pp=_fake(), tp=_fake(0x6000), bt=_fake(0x8000), maxblk=4,
                 B=2, nblk=8, bs=64, HQ=4, H=2, K=64, C=64, dt=BF16, kp=_fake(), rp=_fake(),
                 pl=_fake(), stream=None)
        a.update(kw)
        return lib.wall_append_kv_cache_paged(a["k"], a["g"], a["pp"], a["tp"], a["bt"], a["maxblk"],
                                              a["B"], a["nblk"], a["bs"], a["HQ"], a["H"], a["K"],
                                              a["C"], a["dt"], a["kp"], a["rp"], a["pl"], a["stream"])
    assert app(bt=None) == INVALID
    assert app(tp=None) == INVALID
    assert app(bs=100) == UNSUPPORTED
    assert app(B=0) == 0

    def build(**kw):
        a = dict(k=_fake(), g=_fake(), pp=None, bt=_fake(0x8000), maxblk=4, B=2, t0=0, Tn=100,
                 nblk=8, bs=64, HQ=4, H=2, K=128, C=64, dt=BF16, kp=_fake(), rp=_fake(),
                 pl=_fake(), stream=None)
        a.update(kw)
        return lib.wall_build_kv_cache_paged(a["k"], a["g"], a["pp"], a["bt"], a["maxblk"], a["B"],
                                             a["t0"], a["Tn"], a["nblk"], a["bs"], a["HQ"], a["H"],
                                             a["K"], a["C"], a["dt"], a["kp"], a["rp"], a["pl"],
                                             a["stream"])
    assert build(Tn=300) == INVALID           # more rows than max_blocks * block_size
    assert build(t0=64) == INVALID            # appending needs p_prev
    assert build(bt=None) == INVALID
    assert build(bs=48) == UNSUPPORTED
    assert build(Tn=0) == 0


def test_gate_host_validation(lib):
    def build(**kw):
        a = dict(gs=_fake(), gp=None, bt=None, mb=0, nb=0, bs=0, B=2, t0=0, Tn=10, cap=64, HQ=4,
                 dt=BF16, gc=_fake(), gl=_fake(), stream=None)
        a.update(kw)
        return lib.wall_build_gate_cache(a["gs"], a["gp"], a["bt"], a["mb"], a["nb"], a["bs"], a["B"],
                                         a["t0"], a["Tn"], a["cap"], a["HQ"], a["dt"], a["gc"],
                                         a["gl"], a["stream"])
    assert build(Tn=100) == INVALID          # beyond cap
    assert build(t0=5) == INVALID            # appending needs gs_prev
    assert build(gc=None) == INVALID
    assert build(bt=_fake(0x8000), mb=0, nb=4, bs=16) == INVALID
    assert build(Tn=0) == 0

    def dec(**kw):
        a = dict(q=_fake(), p=_fake(), gcur=_fake(), v=_fake(), kt=_fake(), r=_fake(), gc=_fake(),
                 sink=None, sl=None, bt=None, mb=0, nb=0, bs=0, B=2, T=64, cap=64, HQ=4, H=2,
                 K=128, V=128, C=64, dt=BF16, scale=0.0, o=_fake(), lse=None, ws=_fake(),
                 wsb=1 << 30, stream=None)
        a.update(kw)
        return lib.wall_attn_decode_gated(a["q"], a["p"], a["gcur"], a["v"], a["kt"], a["r"],
                                          a["gc"], a["sink"], a["sl"], a["bt"], a["mb"], a["nb"],
                                          a["bs"], a["B"], a["T"], a["cap"], a["HQ"], a["H"], a["K"],
                                          a["V"], a["C"], a["dt"], a["scale"], a["o"], a["lse"],
                                          a["ws"], a["wsb"], a["stream"])
    assert dec(gcur=None) == INVALID
    assert dec(gc=None) == INVALID
    assert dec(bt=_fake(0x8000), mb=2, nb=4, bs=64) == INVALID   # paged needs seqlens
    assert dec(K=96) == UNSUPPORTED
    assert dec(B=0) == 0


def _step(lib, **kw):
    a = dict(q=_fake(), kn=_fake(0x2000), gn=_fake(0x3000), vn=_fake(0x4000), pp=_fake(0x10000),
             pl=_fake(0x20000), sink=None, seqlens=None, bt=None, maxblk=0, nblk=0, bs=0, B=2,
             T=100, cap=128, HQ=8, H=2, K=128, V=128, chunk=64, dt=BF16, scale=0.0,
             kt=_fake(0x40000), rc=_fake(0x50000), vc=_fake(0x60000), o=_fake(0x70000), lse=None,
             ws=_fake(0x100000), wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.wall_attn_decode_step(
        a["q"], a["kn"], a["gn"], a["vn"], a["pp"], a["pl"], a["sink"], a["seqlens"], a["bt"],
        a["maxblk"], a["nblk"], a["bs"], a["B"], a["T"], a["cap"], a["HQ"], a["H"], a["K"], a["V"],
        a["chunk"], a["dt"], a["scale"], a["kt"], a["rc"], a["vc"], a["o"], a["lse"], a["ws"],
        a["wsb"], a["stream"])


def test_decode_step_host_validation(lib):
    # P_last must not overlap p_prev (other CTAs read p_prev while one writes P_last)
    assert _step(lib, pl=_fake(0x10000)) == INVALID
    assert _step(lib, pl=_fake(0x10000 + 2 * 8 * 128 * 4 - 16)) == INVALID
    assert _step(lib, kn=None) == INVALID
    assert _step(lib, vn=_fake(0x4008)) == INVALID           # misaligned
    assert _step(lib, T=129) == INVALID                      # more rows than the cache holds
    assert _step(lib, chunk=48) == UNSUPPORTED
    assert _step(lib, HQ=6, H=2) == UNSUPPORTED              # group of 3
    assert _step(lib, wsb=16) == WORKSPACE
    # paged: the per-row lengths are required
    assert _step(lib, bt=_fake(0x80000), maxblk=4, nblk=16, bs=64) == INVALID
    assert _step(lib, B=0) == 0


def test_chunk_workspace_size(lib):
    BF, F32 = wall.WALL_DTYPE_BF16, wall.WALL_DTYPE_F32
    # invalid shapes: 0
    assert lib.wall_attn_chunk_workspace_size(0, 4, 1024, 32, 8, 128, 128, 64, BF) == 0
    assert lib.wall_attn_chunk_workspace_size(2, 4, 1024, 6, 4, 128, 128, 64, BF) == 0  # HQ % H
    # a few tokens per sequence (group 4: up to 8) also hold the split-KV partials, which
    # grow with the cache capacity; longer chunks need only the anchored queries
    small = [lib.wall_attn_chunk_workspace_size(32, 4, cap, 32, 8, 128, 128, 64, BF)
             for cap in (64, 1024, 32832)]
    assert small[0] <= small[1] <= small[2]
    prep4 = 32 * 32 * 4 * 128 * 2
    assert small[2] > prep4 + 32 * 4 * 32 * 130 * 4   # at least one split's partials
    big = [lib.wall_attn_chunk_workspace_size(1, 1024, cap, 32, 8, 128, 128, 64, BF)
           for cap in (1024, 32832)]
    assert big[0] == big[1]
    # the bound: 2 * 16 / group tokens (group 16: 2 tokens; 3 take the tensor-core tiles)
    g16 = [lib.wall_attn_chunk_workspace_size(1, m, 32832, 16, 1, 128, 128, 64, BF)
           for m in (2, 3)]
    assert g16[0] > g16[1]
    # fp32 chunks of any length take the split pass: fp32 anchored queries plus one
    # partial (V + 2 floats) per token, query head and split, at least one split
    for M in (3, 1024):
        f = lib.wall_attn_chunk_workspace_size(1, M, 32832, 16, 1, 128, 128, 64, F32)
        assert f >= 16 * M * 128 * 4 + 16 * M * 130 * 4
        assert f > lib.wall_attn_chunk_workspace_size(1, M, 32832, 16, 1, 128, 128, 64, BF)


def test_new_calls_fail_loudly_without_cuda_tensors():
    import torch
    bf = torch.bfloat16
    with pytest.raises((ValueError, ImportError)):
        wall.wall_attn_chunk(torch.zeros(1, 4, 4, 64, dtype=bf), torch.zeros(1, 4, 2, 64, dtype=bf),
                             torch.zeros(1, 4, 4, 64, dtype=bf),
                             torch.zeros(1, 64, 4, 64, dtype=bf),
                             torch.zeros(1, 1, 4, 64), torch.zeros(1, 4, 64),
                             torch.zeros(1, 64, 2, 64, dtype=bf), 0, workspace=torch.zeros(1 << 20,
                                                                                          dtype=torch.uint8))
    with pytest.raises((ValueError, ImportError)):
        wall.wall_attn_decode_step(torch.zeros(1, 1, 4, 64, dtype=bf),
                                   torch.zeros(1, 1, 2, 64, dtype=bf),
                                   torch.zeros(1, 1, 4, 64, dtype=bf),
                                   torch.zeros(1, 1, 2, 64, dtype=bf),
                                   torch.zeros(1, 64, 4, 64, dtype=bf), torch.zeros(1, 1, 4, 64),
                                   torch.zeros(1, 64, 2, 64, dtype=bf), torch.zeros(1, 4, 64),
                                   torch.zeros(1, 4, 64), T_kv=1,
                                   workspace=torch.zeros(1 << 20, dtype=torch.uint8))


def test_paged_cache_block_allocation_on_the_host():
    """PagedKVCache's free list and block tables (host logic; no kernel runs)."""
    import torch
    c = wall.PagedKVCache(2, num_blocks=5, block_size=64, max_blocks=3, HQ=4, H=2, K=64, V=64,
                          chunk=32, device="cpu")
    c.reserve(0, 65)                  # two blocks
    c.reserve(1, 1)                   # one block
    assert [len(t) for t in c.host_table] == [2, 1]
    assert sorted(c.host_table[0] + c.host_table[1] + c.free) == list(range(5))
    assert c.block_table[0, :2].tolist() == c.host_table[0]
    # logical row t of a sequence lives in row t % 64 of its (t // 64)-th block
    rows = c.rows_of(0, 62, 66)
    b0, b1 = c.host_table[0]
    assert rows == [b0 * 64 + 62, b0 * 64 + 63, b1 * 64, b1 * 64 + 1]
    c.reserve(0, 65)                  # already held: nothing changes
    assert len(c.free) == 2
    with pytest.raises(ValueError):
        c.reserve(1, 3 * 64 + 1)      # longer than max_blocks * block_size
    c.reserve(1, 3 * 64)              # takes the last two free blocks
    with pytest.raises(MemoryError):
        c.reserve(0, 3 * 64)          # the pool is exhausted
    c.release(1)
    assert len(c.free) == 3 and c.lengths[1] == 0 and c.host_table[1] == []
    assert c.block_table[1].tolist() == [0, 0, 0]
    with pytest.raises(ValueError):
        wall.PagedKVCache(1, 4, 48, 2, 4, 2, 64, 64, chunk=32, device="cpu")  # 48 % 32 != 0
