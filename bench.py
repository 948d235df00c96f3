#!/usr/bin/env python
"""Wall attention benchmark on B200.

One step is one pass of the whole hot path over synthetic inputs:
  * prefill forward on the long workload (B=1, T=8192, HQ=32, H=8, K=V=128,
    bf16, g = -softplus(N(0,1)-4) per channel, g_scalar likewise): prepass +
    tcgen05 attention kernel;
  * a 64-token streaming decode on the decode workload (B=32, prefix
    T_kv=32768 built once in set-up, HQ=32, H=8, K=V=128, C=64): per token,
    one decode step that appends the token to the pre-rescaled cache inside
    the split-KV decode, then the combine.

Printed (rank 0, one JSON line): prefill TFLOP/s (the headline `value`),
decode KV GB/s (`decode`), each with its roofline fraction against the
measured B200 peaks; an end-to-end prefill number through host buffers
(`e2e`); the CPU oracle's throughput on a bounded sample (`cpu_baseline`).

Multi-GPU (torchrun): every rank runs its own independent shard (its own
prefill sequence and its own decode batch, seeded by rank) -- the method has
no exchange step -- and `value` is all ranks' work over the slowest rank's
device time (weak scaling).

`--impl reference` times the CPU oracle on bounded samples of the same
prefill workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import replace

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of the prefill attention kernel per launch on the long workload
# (dram__bytes_read.sum + dram__bytes_write.sum from one ncu capture) and the
# hash of the kernel source it was taken on; reported as null once the kernel
# source changes.  Filled in after each capture.
TRAFFIC = {
    # full capture on the long prefill: 318.078976 MB read + 44.150016 MB written
    "prefill_main": {"bytes": 362228992, "source_sha": "bbdfce647d9e4ec6"},
    # capture of the decode step at batch 4, scaled by 8 to batch 32 (traffic is
    # proportional to the batch): (1.376312 GB + 4.968448 MB) * 8
    "decode_split": {"bytes": 11050243584, "source_sha": "abf8446f86c17272"},
    # full-size capture of the cache build (batch 32, 1-pass DRAM metrics):
    # 10738862336 B read + 8820070400 B written
    "cache_build": {"bytes": 19558932736, "source_sha": "ef8c7faf6102f370"},
}
KERNEL_SOURCES = {
    "prefill_main": "decayed_softmax_attention_b200/csrc/wall_fwd_tc.cu",
    "decode_split": "decayed_softmax_attention_b200/csrc/wall_split_mma.cu",
    "cache_build": "decayed_softmax_attention_b200/csrc/wall_cache.cu",
}


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def source_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(name):
    t = TRAFFIC[name]
    if t["bytes"] is None or t["source_sha"] != source_sha(KERNEL_SOURCES[name]):
        return None
    return t["bytes"]


def prefill_pairs(spec):
    """Admitted (query, key) pairs per (batch row, query head): causal, window, documents."""
    W_ = spec.window
    docs = spec.docs if spec.docs is not None else (spec.T,)
    total = 0
    for L in docs:
        if W_ <= 0 or L <= W_:
            total += L * (L + 1) // 2
        else:
            total += W_ * (W_ + 1) // 2 + (L - W_) * W_
    return total


def prefill_flops(spec):
    """2*(K+V) FLOPs per admitted pair (QK^T and PV), all batch rows and query heads."""
    return float(spec.B * spec.HQ * prefill_pairs(spec) * 2 * (spec.K + spec.V))


def decode_bytes(spec, T_kv):
    """Algorithmic HBM bytes of one decode step attending T_kv cache rows."""
    esz = 2 if spec.dtype == "bf16" else 4
    B, HQ, H, K, V, C = spec.B, spec.HQ, spec.H, spec.K, spec.V, spec.C
    ktilde = B * T_kv * HQ * K * esz
    vals = B * T_kv * H * V * esz
    anchors = B * ((T_kv + C - 1) // C) * HQ * K * 4
    small = B * HQ * (K * esz + K * 4 + V * esz + 4)  # q, p_curr, o, lse
    return ktilde + vals + anchors + small


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            fd, self.path = tempfile.mkstemp(prefix="wall_clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, power, reasons = [], None, [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax = float(parts[1])
                    power.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names[1:], parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        loaded = [s for s in sm if smax and s > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "power_w_max": max(power) if power else None, "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(x, world, device):
    """Max over ranks of a host float (timing only; no data-path collective).

    `device` is the rank's CUDA device under NCCL, or "cpu" under gloo."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank, steps, world, max_ms):
    """Whole-job rate: the units every rank processed over the slowest rank's time (per s)."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def shard_specs(rank):
    """This rank's independent shard: the long prefill and the decode batch, seeded by rank."""
    p = W.PREFILL["long"]
    d = W.DECODE["decode"]
    return replace(p, seed=p.seed + 100 * rank), replace(d, seed=d.seed + 100 * rank)


# ----------------------------------------------------------------- CPU oracle timing
def oracle_sample_rows(spec, n_rows):
    """n_rows query rows spread evenly over the sequence (all heads), batch row 0."""
    import numpy as np
    return np.unique(np.linspace(0, spec.T - 1, n_rows).round().astype(np.int64))


def time_oracle(spec, host, n_rows, threads):
    import oracle
    rows = oracle_sample_rows(spec, n_rows)
    t0 = time.perf_counter()
    oracle.wall_fwd(host["q"], host["k"], host["v"], host["g"], host["g_scalar"],
                    host["sink_bias"], window=spec.window, scale=spec.softmax_scale, rows=rows,
                    threads=threads)
    dt = time.perf_counter() - t0
    flops = float(sum(spec.HQ * (int(t) + 1) * 2 * (spec.K + spec.V) for t in rows))
    return dt, flops, rows


def cpu_baseline(spec, host, budget_s=15.0):
    import oracle
    threads = oracle.max_threads()
    n = 8
    dt, flops, rows = time_oracle(spec, host, n, threads)
    # grow the sample until it takes at least half the budget (10-30 s of oracle work)
    for _ in range(3):
        if dt >= budget_s / 2 or n >= spec.T:
            break
        n = int(min(spec.T, max(n + 1, n * budget_s / max(dt, 1e-3) * 0.9)))
        dt, flops, rows = time_oracle(spec, host, n, threads)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} query rows evenly spaced over T={spec.T}, all {spec.HQ} heads "
                      f"of the long prefill workload (batch row 0), double precision; "
                      f"{dt:.1f} s"}


def rows_flops(spec, rows):
    """Algorithmic FLOPs of the given query rows (batch row 0): admitted keys x 2(K+V) x HQ."""
    cu = [0]
    for L in (spec.docs if spec.docs is not None else (spec.T,)):
        cu.append(cu[-1] + L)
    total = 0
    for t in rows:
        t = int(t)
        start = max(c for c in cu[:-1] if c <= t)
        lo = max(start, t - spec.window + 1) if spec.window > 0 else start
        total += t - lo + 1
    return float(total * spec.HQ * 2 * (spec.K + spec.V))


def cpu_per_config(decode_rows):
    """The oracle on the host cores for the other workloads (reported baselines only):
    the tiny and GQA prefills in full, the packed varlen + window prefill on 512 evenly
    spaced rows, and the decode workload's direct decode oracle (each step = the prefill
    row of the appended token) for batch rows 0 and 31 over the timed steps."""
    import numpy as np
    import oracle
    threads = oracle.max_threads()
    out = {}
    for name, n_rows in (("tiny", None), ("gqa", None), ("varlen_window", 512)):
        spec = W.PREFILL[name]
        host = host_inputs(W.gen_prefill(spec, device="cpu"))
        rows = None if n_rows is None else oracle_sample_rows(spec, n_rows)
        t0 = time.perf_counter()
        oracle.wall_fwd(host["q"], host["k"], host["v"], host["g"], host["g_scalar"],
                        host["sink_bias"], window=spec.window, cu_seqlens=host["cu_seqlens"],
                        scale=spec.softmax_scale, rows=rows, threads=threads)
        dt = time.perf_counter() - t0
        flops = prefill_flops(spec) if rows is None else rows_flops(spec, rows)
        out[name] = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "seconds": dt,
                     "sample": ("all rows" if rows is None else
                                f"{len(rows)} query rows evenly spaced over T={spec.T}, all heads")}
    if decode_rows is not None:
        dspec, rows_by_b = decode_rows
        t0 = time.perf_counter()
        nbytes = 0
        for b, (qf, kb, vb, gb, rows) in rows_by_b.items():
            oracle.wall_fwd(qf, kb, vb, gb, scale=dspec.K ** -0.5, rows=rows, threads=threads)
            for t in rows:
                one = replace(dspec, B=1)
                nbytes += decode_bytes(one, int(t) + 1)
        dt = time.perf_counter() - t0
        nb = len(rows_by_b)
        steps = len(next(iter(rows_by_b.values()))[4])
        out["decode"] = {
            "value": nbytes / dt / 1e9, "unit": "GB/s", "seconds": dt,
            "sample": f"batch rows {sorted(rows_by_b)} of B={dspec.B}, {steps} streaming steps each "
                      f"(T_kv {dspec.T0 + 1}..{dspec.T0 + steps}), all {dspec.HQ} heads",
            "extrapolated_ms_per_token_all_batch_rows": 1e3 * dt / steps * dspec.B / nb,
            "extrapolation": f"per-step time of the {nb} sampled rows x B/{nb} (label: extrapolated)"}
    return out


def host_inputs(d):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


# ----------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import oracle
    spec, dspec = shard_specs(0)
    dspec = replace(dspec, steps=args.decode_steps)
    host = host_inputs(W.gen_prefill(spec, device="cpu"))
    threads = oracle.max_threads()
    # size the per-step sample to about 2 s of oracle work
    dt, _, _ = time_oracle(spec, host, 4, threads)
    n_rows = int(max(4, min(spec.T, 4 * 2.0 / max(dt, 1e-3))))
    for _ in range(args.warmup):
        time_oracle(spec, host, n_rows, threads)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, fl, rows = time_oracle(spec, host, n_rows, threads)
        times.append(dt)
        flops += fl
    total = sum(times)
    value = flops / total / 1e12
    sample = (f"{n_rows} query rows evenly spaced over T={spec.T}, all {spec.HQ} heads of the "
              f"long prefill workload per step, double precision")
    line = {
        "impl": "reference", "metric": "wall_attn_fwd TFLOP/s @ T=8K (long prefill)",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(spec, dspec, args.gpus),  # the same config line as our arm
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(pspec, dspec, n):
    c = {
        "workload": (f"prefill: long B={pspec.B} T={pspec.T} HQ={pspec.HQ} H={pspec.H} "
                     f"K={pspec.K} V={pspec.V} {pspec.dtype} causal, g=-softplus(N(0,1)-4), "
                     f"g_scalar=-softplus(N(0,1)-4)"),
        "global_batch": pspec.B * n,
        "seq_len": pspec.T,
        "parallelism": f"dp{n} (independent shards, no collective)",
        "l2": "inputs larger than L2: each step streams the 11 GB decode cache 64 times "
              "between prefill passes (126 MB L2)",
    }
    if dspec is not None:
        c["workload"] += (f"; decode: B={dspec.B} T_kv={dspec.T0}->{dspec.cap} HQ={dspec.HQ} "
                          f"H={dspec.H} K={dspec.K} V={dspec.V} C={dspec.C} {dspec.dtype}, "
                          f"{dspec.steps} streaming steps (wall_attn_decode_step: append fused into the decode)")
    return c


# ----------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import decayed_softmax_attention_b200 as wall
    from decayed_softmax_attention_b200 import build as wall_build
    if not os.path.exists(wall.lib_path()):
        wall_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    pspec, dspec = shard_specs(rank)
    dspec = replace(dspec, steps=args.decode_steps)
    if args.decode_batch:
        dspec = replace(dspec, B=args.decode_batch)
    do_prefill = args.only in (None, "prefill")
    do_decode = args.only in (None, "decode")
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    # ---- prefill set-up
    if do_prefill:
        pd = W.gen_prefill(pspec, device=dev)
        B, T, HQ, H, K, V = pspec.B, pspec.T, pspec.HQ, pspec.H, pspec.K, pspec.V
        o = torch.empty((B, T, HQ, V), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, T, HQ), dtype=torch.float32, device=dev)
        ws = torch.empty(wall.wall_attn_fwd_workspace_size(B, T, HQ, H, K, V, torch.bfloat16),
                         dtype=torch.uint8, device=dev)

    def prefill():
        wall.wall_attn_fwd(pd["q"], pd["k"], pd["v"], pd["g"], pd["g_scalar"], pd["sink_bias"],
                           window=pd["window"], scale=pd["scale"], out=o, lse=lse, workspace=ws,
                           return_lse=True)

    # ---- decode set-up: build the prefix cache once (timed as a side number)
    T0, S = dspec.T0, (dspec.steps if do_decode else 0)
    build_ms = build_bytes = build1_ms = build1_bytes = None
    if do_decode:
        dd = W.gen_decode(dspec, device=dev)
        cache = wall.KVCache(dspec.B, dspec.cap, dspec.HQ, dspec.H, dspec.K, dspec.V,
                             dtype=torch.bfloat16, chunk=dspec.C, device=dev)
        cache.v.copy_(dd["v"])                   # value cache is the caller's; preload all rows
        k_pre = dd["k"][:, :T0].contiguous()
        g_pre = dd["g"][:, :T0].contiguous()
        k_steps = [dd["k"][:, T0 + s:T0 + s + 1].contiguous() for s in range(S)]
        g_steps = [dd["g"][:, T0 + s:T0 + s + 1].contiguous() for s in range(S)]
        q_steps = [dd["q"][:, s:s + 1].contiguous() for s in range(S)]
        v_steps = [dd["v"][:, T0 + s:T0 + s + 1].contiguous() for s in range(S)]
        decode_rows = None
        if world == 1 and not args.no_cpu_baseline:
            import numpy as np
            rows_by_b = {}
            for b_ in sorted({0, dspec.B - 1}):
                qf = torch.zeros((1, T0 + S, dspec.HQ, dspec.K), dtype=torch.bfloat16)
                qf[0, T0:T0 + S] = dd["q"][b_].cpu()
                rows_by_b[b_] = (qf, dd["k"][b_:b_ + 1].cpu(), dd["v"][b_:b_ + 1].cpu(),
                                 dd["g"][b_:b_ + 1].cpu(),
                                 np.arange(T0, T0 + S, dtype=np.int64))
            decode_rows = (dspec, rows_by_b)
        del dd
        dout = torch.empty((dspec.B, 1, dspec.HQ, dspec.V), dtype=torch.bfloat16, device=dev)
        dlse = torch.empty((dspec.B, 1, dspec.HQ), dtype=torch.float32, device=dev)
        p_prefix = torch.empty_like(cache.p)
        e0, e1 = ev(), ev()
        cache.length = 0
        cache.append(k_pre, g_pre)     # first launch loads the kernel module: untimed
        torch.cuda.synchronize()
        e0.record()
        cache.length = 0
        cache.append(k_pre, g_pre)     # timed rebuild (writes the same values)
        e1.record()
        torch.cuda.synchronize()
        build_ms = e0.elapsed_time(e1)
        esz = 2
        build_bytes = (dspec.B * T0 * (dspec.H * dspec.K + dspec.HQ * dspec.K) * esz  # read k, g
                       + dspec.B * T0 * dspec.HQ * dspec.K * esz                       # k_tilde
                       + dspec.B * (T0 // dspec.C) * dspec.HQ * dspec.K * 4)            # anchors
        p_prefix.copy_(cache.p)
        # the same build for one batch row (segment-parallel path), warm
        one = wall.KVCache(1, T0, dspec.HQ, dspec.H, dspec.K, dspec.V, dtype=torch.bfloat16,
                           chunk=dspec.C, device=dev)
        k1, g1 = k_pre[:1].contiguous(), g_pre[:1].contiguous()
        one.append(k1, g1)
        torch.cuda.synchronize()
        e0.record()
        one.length = 0
        one.append(k1, g1)
        e1.record()
        torch.cuda.synchronize()
        build1_ms = e0.elapsed_time(e1)
        build1_bytes = build_bytes // dspec.B
        del one, k1, g1
        del k_pre, g_pre

    pre_ev = [[ev() for _ in range(3)] for _ in range(args.steps)] if do_prefill else []
    dec_ev = [[[ev() for _ in range(3)] for _ in range(S)] for _ in range(args.steps)]
    # torch creates the underlying cudaEvent_t on first record: record every
    # event once here so the library receives valid handles to re-record.
    for trio in pre_ev + [t for row in dec_ev for t in row]:
        for e in trio:
            e.record()
    torch.cuda.synchronize()

    def step(i=None):
        if do_prefill:
            if i is not None:
                wall.wall_debug_set_stage_events(*pre_ev[i])
            prefill()
            if i is not None:
                wall.wall_debug_set_stage_events()
        if do_decode:
            cache.length = T0
            cache.p.copy_(p_prefix)
            for s in range(S):  # one decode step per token, the append fused in
                if i is not None:
                    wall.wall_debug_set_stage_events(*dec_ev[i][s])
                cache.step(q_steps[s], k_steps[s], g_steps[s], v_steps[s], scale=dspec.K ** -0.5,
                           out=dout, lse=dlse)
                if i is not None:
                    wall.wall_debug_set_stage_events()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert wall.wall_device_error(dev) == 0

    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = ev(), ev()
    t_start.record()
    for i in range(args.steps):
        step(i)
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    status = wall.wall_device_error(dev)
    if status != 0:
        raise RuntimeError(f"device error status {status} during the timed region")
    total_ms = reduce_max(t_start.elapsed_time(t_end), world, dev)

    line = {
        "metric": "wall_attn_fwd TFLOP/s @ T=8K (long prefill)",
        "value": None, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_block(pspec, dspec if do_decode else None, world),
    }
    side = {}
    bf16_peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    if do_prefill:
        pre_ms = [e[0].elapsed_time(e[2]) for e in pre_ev]
        pre_prep_ms = [e[0].elapsed_time(e[1]) for e in pre_ev]
        pre_main_ms = [e[1].elapsed_time(e[2]) for e in pre_ev]
        flops = prefill_flops(pspec)
        pre_total_ms = reduce_max(sum(pre_ms), world, dev)
        value = weak_scaling_rate(flops, args.steps, world, pre_total_ms) / 1e12
        main_avg = statistics.mean(pre_main_ms)
        achieved = flops / (main_avg * 1e-3) / 1e12
        line["value"] = value
        # timed inside a long step (the decode loop runs the GPU at its power
        # cap), so the denominator is the sustained bf16 peak
        bf16_sus = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
        line["roofline"] = {
            "kernel": "wall_fwd_tc_kernel (prefill attention)", "bound": "tensor",
            "achieved": achieved, "peak": bf16_sus, "unit": "TFLOP/s", "frac": achieved / bf16_sus,
            "traffic": traffic_for("prefill_main"),
            "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
            "algorithmic_flops_per_launch": flops,
            "share_of_step": sum(pre_main_ms) / total_ms}
        # the prefill alone (no decode between launches): burst conditions
        alone = [[ev() for _ in range(3)] for _ in range(args.steps)]
        for trio in alone:
            for e in trio:
                e.record()
        for i in range(args.steps):
            wall.wall_debug_set_stage_events(*alone[i])
            prefill()
            wall.wall_debug_set_stage_events()
        torch.cuda.synchronize()
        alone_main = statistics.mean(e[1].elapsed_time(e[2]) for e in alone)
        alone_all = statistics.mean(e[0].elapsed_time(e[2]) for e in alone)
        side.update({"prefill_alone_ms": alone_all, "prefill_alone_main_ms": alone_main,
                     "prefill_alone_main_TFLOPs": flops / (alone_main * 1e-3) / 1e12,
                     "prefill_alone_main_frac_of_burst_peak":
                         flops / (alone_main * 1e-3) / 1e12 / bf16_peak})
        # secondary bound of the attention kernel: one exponential per admitted score on
        # the MUFU, 16 per clock per SM (at the maximum SM clock)
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        mufu_peak = 16.0 * n_sm * peaks.get("sm_max_mhz", 1965.0) * 1e6
        exps = float(pspec.B * pspec.HQ * prefill_pairs(pspec))
        side["mufu"] = {"exps_per_launch": exps, "achieved_per_s": exps / (alone_main * 1e-3),
                        "peak_per_s": mufu_peak,
                        "frac": exps / (alone_main * 1e-3) / mufu_peak,
                        "note": "kernel timed alone; 16 MUFU ops per clock per SM x SMs x max clock"}
        # the other prefill workloads (GQA; packed varlen + window + sink), timed alone
        for name in ("gqa", "varlen_window"):
            ospec = W.PREFILL[name]
            od = W.gen_prefill(ospec, device=dev)
            oo = torch.empty((ospec.B, ospec.T, ospec.HQ, ospec.V), dtype=torch.bfloat16, device=dev)
            ol = torch.empty((ospec.B, ospec.T, ospec.HQ), dtype=torch.float32, device=dev)
            ows = torch.empty(wall.wall_attn_fwd_workspace_size(ospec.B, ospec.T, ospec.HQ, ospec.H,
                                                                ospec.K, ospec.V, torch.bfloat16),
                              dtype=torch.uint8, device=dev)

            def run_other():
                wall.wall_attn_fwd(od["q"], od["k"], od["v"], od["g"], od["g_scalar"], od["sink_bias"],
                                   window=od["window"], cu_seqlens=od["cu_seqlens"],
                                   scale=od["scale"], out=oo, lse=ol, workspace=ows,
                                   return_lse=True)
            run_other()
            oev = [[ev() for _ in range(3)] for _ in range(args.steps)]
            for trio in oev:
                for e in trio:
                    e.record()
            for i in range(args.steps):
                wall.wall_debug_set_stage_events(*oev[i])
                run_other()
                wall.wall_debug_set_stage_events()
            torch.cuda.synchronize()
            om = statistics.mean(e[1].elapsed_time(e[2]) for e in oev)
            oa = statistics.mean(e[0].elapsed_time(e[2]) for e in oev)
            of = prefill_flops(ospec)
            side.update({f"prefill_{name}_ms": oa, f"prefill_{name}_main_ms": om,
                         f"prefill_{name}_main_TFLOPs": of / (om * 1e-3) / 1e12,
                         f"prefill_{name}_main_frac_of_burst_peak": of / (om * 1e-3) / 1e12 / bf16_peak})
            del od, oo, ol, ows
        # prefill that also emits its decode cache, against prefill + a separate build
        pc = wall.KVCache(B, T, HQ, H, K, V, dtype=torch.bfloat16, chunk=64, device=dev)

        def prefill_cache():
            wall.wall_attn_fwd(pd["q"], pd["k"], pd["v"], pd["g"], pd["g_scalar"],
                               pd["sink_bias"], window=pd["window"], scale=pd["scale"], out=o,
                               lse=lse, workspace=ws, return_lse=True, cache=pc)

        def build_only():
            pc.length = 0
            pc.append(pd["k"], pd["g"])

        def time_fn(fn, n):
            fn()
            a, z = ev(), ev()
            torch.cuda.synchronize()
            a.record()
            for _ in range(n):
                fn()
            z.record()
            torch.cuda.synchronize()
            return a.elapsed_time(z) / n

        n_rep = max(args.steps, 5)
        cev = [[ev() for _ in range(3)] for _ in range(n_rep)]
        for trio in cev:
            for e in trio:
                e.record()
        for i in range(n_rep):
            wall.wall_debug_set_stage_events(*cev[i])
            prefill_cache()
            wall.wall_debug_set_stage_events()
        torch.cuda.synchronize()
        side.update({
            "prefill_with_cache_prepass_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in cev),
            "prefill_with_cache_main_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in cev)})
        side.update({"prefill_with_cache_ms": time_fn(prefill_cache, n_rep),
                     "prefill_plain_ms": time_fn(prefill, n_rep),
                     "cache_build_of_prefill_ms": time_fn(build_only, n_rep)})
        del pc
        # the same prefill fed as 8 chunks of 1024 tokens against the decode cache
        # (chunked prefill: each chunk's keys appended, its queries over the cache
        # rows before them); no gate term on this path, so g_scalar is left out
        nchk = 8
        Mc = T // nchk
        cc = wall.KVCache(B, T, HQ, H, K, V, dtype=torch.bfloat16, chunk=64, device=dev)
        cc.v.copy_(pd["v"])
        co = torch.empty((B, Mc, HQ, V), dtype=torch.bfloat16, device=dev)
        cws = torch.empty(wall.wall_attn_chunk_workspace_size(B, Mc, T, HQ, H, K, V, 64), dtype=torch.uint8,
                          device=dev)
        chunks = [(pd["q"][:, i * Mc:(i + 1) * Mc].contiguous(),
                   pd["k"][:, i * Mc:(i + 1) * Mc].contiguous(),
                   pd["g"][:, i * Mc:(i + 1) * Mc].contiguous()) for i in range(nchk)]

        def chunked():
            for i, (qc, kc, gc) in enumerate(chunks):
                wall.wall_attn_chunk(qc, kc, gc, cc.k_tilde, cc.r_cache, cc.p, cc.v, i * Mc,
                                     scale=pd["scale"], chunk=64, out=co, workspace=cws)

        chk_ms = time_fn(chunked, n_rep)
        side.update({"chunked_prefill_8x1024_ms": chk_ms,
                     "chunked_prefill_TFLOPs": flops / (chk_ms * 1e-3) / 1e12})
        del cc, co, cws, chunks
        # prefill backward on the same workload: gradients of sum(o * dO)
        gdo = torch.Generator(device=dev).manual_seed(pspec.seed + 7)
        dO = torch.randn((B, T, HQ, V), generator=gdo, device=dev).to(torch.bfloat16)
        bws = torch.empty(wall.wall_attn_bwd_workspace_size(B, T, HQ, H, K, V, torch.bfloat16),
                          dtype=torch.uint8, device=dev)
        grads = {}

        def backward():
            grads.update(wall.wall_attn_bwd(pd["q"], pd["k"], pd["v"], pd["g"], o, lse, dO,
                                            pd["g_scalar"], pd["sink_bias"], pd["window"], None,
                                            pd["scale"], workspace=bws, grads=grads))

        backward()
        bev = [[ev() for _ in range(3)] for _ in range(n_rep)]
        for trio in bev:
            for e in trio:
                e.record()
        for i in range(n_rep):
            wall.wall_debug_set_stage_events(*bev[i])
            backward()
            wall.wall_debug_set_stage_events()
        torch.cuda.synchronize()
        bwd_ms = time_fn(backward, n_rep)
        kv_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in bev)
        q_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in bev)
        pairs = float(B * HQ * prefill_pairs(pspec))
        algo = 2.5 * flops   # five pair-products: QK^T, dO V^T, P^T dO, dS^T Q, dS K
        side.update({
            "bwd_ms": bwd_ms, "bwd_TFLOPs_algorithmic": algo / (bwd_ms * 1e-3) / 1e12,
            "bwd_frac_of_burst_peak": algo / (bwd_ms * 1e-3) / 1e12 / bf16_peak,
            "bwd_dkdv_kernel_ms": kv_ms, "bwd_dq_kernel_ms": q_ms,
            # executed tensor work: key-block 4 products per pair, query-block 3
            "bwd_dkdv_kernel_TFLOPs": pairs * 2 * (2 * K + 2 * V) / (kv_ms * 1e-3) / 1e12,
            "bwd_dq_kernel_TFLOPs": pairs * 2 * (2 * K + V) / (q_ms * 1e-3) / 1e12,
            "bwd_outside_contractions_ms": bwd_ms - kv_ms - q_ms})
        del bws, grads, dO
        side.update({"prefill_ms": statistics.mean(pre_ms),
                     "prefill_prepass_ms": statistics.mean(pre_prep_ms),
                     "prefill_main_ms": main_avg,
                     "frac_of_measured_peak_whole_prefill": value / world / bf16_peak})
    if do_decode:
        dec_ms = [[e[0].elapsed_time(e[2]) for e in row] for row in dec_ev]
        dec_split_ms = [[e[0].elapsed_time(e[1]) for e in row] for row in dec_ev]
        step_bytes = [decode_bytes(dspec, T0 + s + 1) for s in range(S)]
        dec_total_ms = reduce_max(sum(sum(r) for r in dec_ms), world, dev)
        dec_value = weak_scaling_rate(sum(step_bytes), args.steps, world, dec_total_ms) / 1e9
        split_avg = statistics.mean(x for r in dec_split_ms for x in r)
        dec_achieved = statistics.mean(step_bytes) / (split_avg * 1e-3) / 1e9
        line["decode"] = {
            "metric": f"wall_attn_decode KV GB/s (B={dspec.B}, T_kv {T0 + 1}..{T0 + S})",
            "value": dec_value, "unit": "GB/s",
            "ms_per_token": statistics.mean(x for r in dec_ms for x in r),
            "roofline": {"kernel": "split_mma_kernel (decode split pass, fused append)",
                         "bound": "hbm", "achieved": dec_achieved,
                         "peak": hbm_peak, "unit": "GB/s", "frac": dec_achieved / hbm_peak,
                         "traffic": traffic_for("decode_split"),
                         "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic_bytes_per_launch": statistics.mean(step_bytes),
                         "share_of_step": sum(sum(r) for r in dec_split_ms) / total_ms},
            "frac_of_hbm_incl_combine": dec_value / world / hbm_peak,
        }
        build_gbps = build_bytes / (build_ms * 1e-3) / 1e9
        # per-sequence lengths: row b attends rows [0, len_b), len_b ~ U[T0/2, T0] (seeded)
        gl = torch.Generator().manual_seed(4242)
        lens = torch.randint(T0 // 2, T0 + 1, (dspec.B,), generator=gl, dtype=torch.int32)
        seqlens = lens.to(dev)
        cache.length = T0
        cache.p.copy_(p_prefix)
        qv = q_steps[0] if S else torch.zeros((dspec.B, 1, dspec.HQ, dspec.K),
                                               dtype=torch.bfloat16, device=dev)

        def dec_varlen():
            wall.wall_attn_decode(qv, cache.p[:, None], cache.v, cache.k_tilde, cache.r_cache, T0,
                                  scale=dspec.K ** -0.5, chunk=dspec.C, out=dout, seqlens=seqlens)

        dec_varlen()
        va, vz = ev(), ev()
        torch.cuda.synchronize()
        va.record()
        for _ in range(10):
            dec_varlen()
        vz.record()
        torch.cuda.synchronize()
        var_ms = va.elapsed_time(vz) / 10
        var_bytes = sum(int(L) * (dspec.HQ * dspec.K + dspec.H * dspec.V) * 2
                        + ((int(L) + dspec.C - 1) // dspec.C) * dspec.HQ * dspec.K * 4 for L in lens)
        side.update({"decode_varlen_ms": var_ms,
                     "decode_varlen_GBps": var_bytes / (var_ms * 1e-3) / 1e9,
                     "decode_varlen_frac_of_hbm": var_bytes / (var_ms * 1e-3) / 1e9 / hbm_peak})
        # the same decode over a paged cache: 256-row blocks of the same rows, scattered
        # through the pool by a seeded permutation (block tables)
        pbs = 256
        pmax = (cache.cap + pbs - 1) // pbs
        nblk = dspec.B * pmax
        perm = torch.randperm(nblk, generator=torch.Generator().manual_seed(4343))
        ptable = perm.view(dspec.B, pmax).to(torch.int32).to(dev)
        kt_pool = torch.empty((nblk, pbs, dspec.HQ, dspec.K), dtype=torch.bfloat16, device=dev)
        v_pool = torch.empty((nblk, pbs, dspec.H, dspec.V), dtype=torch.bfloat16, device=dev)
        r_pool = torch.empty((nblk, pbs // dspec.C, dspec.HQ, dspec.K), dtype=torch.float32,
                             device=dev)
        n = (cache.cap // pbs) * pbs   # whole blocks; the lengths above never exceed T0 <= n
        nb_full = n // pbs
        for b in range(dspec.B):   # setup only: copy each row's blocks into their pool slots
            idx = ptable[b, :nb_full].long()
            kt_pool[idx] = cache.k_tilde[b, :n].reshape(-1, pbs, dspec.HQ, dspec.K)
            v_pool[idx] = cache.v[b, :n].reshape(-1, pbs, dspec.H, dspec.V)
            r_pool[idx] = cache.r_cache[b, :n // dspec.C].reshape(-1, pbs // dspec.C, dspec.HQ,
                                                                 dspec.K)
        if n >= T0:
            pws = torch.empty(wall.wall_attn_decode_workspace_size(
                dspec.B, pmax * pbs, dspec.HQ, dspec.H, dspec.V, dspec.C), dtype=torch.uint8,
                device=dev)

            def dec_paged():
                wall.wall_attn_decode_paged(qv, cache.p[:, None], v_pool, kt_pool, r_pool, seqlens,
                                            ptable, scale=dspec.K ** -0.5, chunk=dspec.C,
                                            out=dout, workspace=pws)

            dec_paged()
            pa, pz = ev(), ev()
            torch.cuda.synchronize()
            pa.record()
            for _ in range(10):
                dec_paged()
            pz.record()
            torch.cuda.synchronize()
            pg_ms = pa.elapsed_time(pz) / 10
            side.update({"decode_paged_ms": pg_ms, "decode_paged_block_rows": pbs,
                         "decode_paged_GBps": var_bytes / (pg_ms * 1e-3) / 1e9,
                         "decode_paged_frac_of_hbm": var_bytes / (pg_ms * 1e-3) / 1e9 / hbm_peak})
            del pws
        del kt_pool, v_pool, r_pool
        # the same per-sequence-length decode with the scalar gate (a gate cache of PS rows)
        gsd = (-torch.nn.functional.softplus(
            torch.randn((dspec.B, T0, dspec.HQ), generator=torch.Generator(device=dev).manual_seed(77),
                        device=dev) - 4.0)).to(torch.bfloat16)
        gs_cache = torch.empty((dspec.B, cache.cap, dspec.HQ), dtype=torch.float32, device=dev)
        gs_last = torch.empty((dspec.B, dspec.HQ), dtype=torch.float32, device=dev)
        wall.wall_build_gate_cache(gsd, gs_cache, gs_last)
        gws = torch.empty(wall.wall_attn_decode_workspace_size(
            dspec.B, T0, dspec.HQ, dspec.H, dspec.V, dspec.C), dtype=torch.uint8, device=dev)

        def dec_gated():
            wall.wall_attn_decode_gated(qv, cache.p[:, None], gs_last, cache.v, cache.k_tilde,
                                        cache.r_cache, gs_cache, T_kv=T0, seqlens=seqlens,
                                        scale=dspec.K ** -0.5, chunk=dspec.C, out=dout,
                                        workspace=gws)

        dec_gated()
        ga, gz = ev(), ev()
        torch.cuda.synchronize()
        ga.record()
        for _ in range(10):
            dec_gated()
        gz.record()
        torch.cuda.synchronize()
        gt_ms = ga.elapsed_time(gz) / 10
        gate_bytes = var_bytes + sum(int(L) for L in lens) * dspec.HQ * 4
        side.update({"decode_gated_ms": gt_ms,
                     "decode_gated_GBps": gate_bytes / (gt_ms * 1e-3) / 1e9,
                     "decode_gated_frac_of_hbm": gate_bytes / (gt_ms * 1e-3) / 1e9 / hbm_peak})
        del gs_cache, gs_last, gws, gsd
        # multi-token decode: 4 new tokens per sequence against the T0-row cache in one
        # chunk call (append + attend); timing only (the rows after T0 are overwritten);
        # needs room for the 4 rows after T0
        Mt = 4
        if dspec.cap >= T0 + Mt:
            g4 = torch.Generator(device=dev).manual_seed(78)
            q4 = torch.randn((dspec.B, Mt, dspec.HQ, dspec.K), generator=g4, device=dev).to(torch.bfloat16)
            k4 = torch.randn((dspec.B, Mt, dspec.H, dspec.K), generator=g4, device=dev).to(torch.bfloat16)
            gg4 = (-torch.nn.functional.softplus(torch.randn((dspec.B, Mt, dspec.HQ, dspec.K),
                                                             generator=g4, device=dev) - 4.0)).to(torch.bfloat16)
            p4 = cache.p.clone()
            o4 = torch.empty((dspec.B, Mt, dspec.HQ, dspec.V), dtype=torch.bfloat16, device=dev)
            w4 = torch.empty(wall.wall_attn_chunk_workspace_size(dspec.B, Mt, dspec.cap, dspec.HQ,
                                                             dspec.H, dspec.K, dspec.V, dspec.C),
                             dtype=torch.uint8, device=dev)

            def dec_multi():
                wall.wall_attn_chunk(q4, k4, gg4, cache.k_tilde, cache.r_cache, cache.p, cache.v, T0,
                                     p_prev=p4, scale=dspec.K ** -0.5, chunk=dspec.C, out=o4,
                                     workspace=w4)

            dec_multi()
            ma, mz = ev(), ev()
            torch.cuda.synchronize()
            ma.record()
            for _ in range(10):
                dec_multi()
            mz.record()
            torch.cuda.synchronize()
            mt_ms = ma.elapsed_time(mz) / 10
            mt_bytes = decode_bytes(dspec, T0 + Mt)
            side.update({"decode_4tokens_chunk_ms": mt_ms,
                         "decode_4tokens_chunk_GBps": mt_bytes / (mt_ms * 1e-3) / 1e9,
                         "decode_4tokens_chunk_frac_of_hbm": mt_bytes / (mt_ms * 1e-3) / 1e9 / hbm_peak})
            del q4, k4, gg4, p4, o4, w4
        # the same token as append + decode (two calls), against the main loop's fused step;
        # timing only (row T0 is rewritten with the same values)
        if dspec.cap >= T0 + 1:
            def split_step():
                cache.length = T0
                cache.append(k_steps[0], g_steps[0])
                cache.decode(q_steps[0], scale=dspec.K ** -0.5, out=dout, lse=dlse)

            split_step()
            fa, fz = ev(), ev()
            torch.cuda.synchronize()
            fa.record()
            for _ in range(10):
                split_step()
            fz.record()
            torch.cuda.synchronize()
            sp_ms = fa.elapsed_time(fz) / 10
            side.update({"decode_append_then_decode_ms": sp_ms,
                         "decode_append_then_decode_frac_of_hbm":
                             decode_bytes(dspec, T0 + 1) / (sp_ms * 1e-3) / 1e9 / hbm_peak})
        side.update({"cache_build_prefix_ms": build_ms,
                     "cache_build_prefix_GBps": build_gbps,
                     "cache_build_roofline": {
                         "kernel": "cache_build_kernel", "bound": "hbm", "achieved": build_gbps,
                         "peak": hbm_peak, "unit": "GB/s", "frac": build_gbps / hbm_peak,
                         "algorithmic_bytes_per_launch": build_bytes,
                         "traffic": (traffic_for("cache_build")
                                     if dspec.B == 32 and T0 == 32768 else None)},
                     "cache_build_prefix_b1_ms": build1_ms,
                     "cache_build_prefix_b1_GBps": build1_bytes / (build1_ms * 1e-3) / 1e9})
        if not do_prefill:
            line["metric"] = line["decode"]["metric"]
            line["value"], line["unit"] = dec_value, "GB/s"
            line["roofline"] = line["decode"]["roofline"]
    line["side"] = side

    # ---- end to end through host buffers (pinned), prefill headline metric
    if do_prefill and not args.no_e2e:
        names = ["q", "k", "v", "g", "g_scalar"]
        host = {n: pd[n].cpu().pin_memory() for n in names}
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(host[n].numel() * host[n].element_size() for n in names)
        d2h = o_host.numel() * o_host.element_size()

        def e2e_step():
            for n in names:
                pd[n].copy_(host[n], non_blocking=True)
            prefill()
            o_host.copy_(o, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b_ = ev(), ev()
        a.record()
        for _ in range(args.steps):
            e2e_step()
        b_.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = reduce_max(a.elapsed_time(b_), world, dev)
        line["e2e"] = {"value": weak_scaling_rate(prefill_flops(pspec), args.steps, world, e2e_ms) / 1e12,
                       "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    # per timed step: prefill = prepass (2) + attention (1) + the wide-block pass (1, which
    # exits at once on these inputs); each decode token = the fused decode split (append
    # inside) + the combine (2)
    line["gpu_launches"] = args.steps * ((4 if do_prefill else 0) + (2 * S if do_decode else 0))
    line["clocks"] = clk
    if rank != 0:
        return 0
    if world == 1 and do_prefill and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(pspec, host_inputs(pd))
        line["cpu_baseline"]["per_config"] = cpu_per_config(decode_rows if do_decode else None)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="profiling runs: time one half of the step only")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="profiling runs: smaller decode batch (default: the workload's B=32)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
