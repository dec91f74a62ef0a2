#!/usr/bin/env python
"""Benchmark of the causal sliding-window attention hot path on B200.

One step = the whole hot path over one batch of synthetic input:
  * the depth-24 shape (B=32, T=2048, H=12, D=128) through the "SSSL" window
    pattern (three layers at W=512, one at W=2048): forward (O, lse) and
    backward (dQ, dK, dV) per layer;
  * single-token decode over the KV-cache workload (32 sequences, H=12,
    D=128, capacity 2048, cache_len ~ U[1, 2048]) at W=2048 and W=1024.
value = unmasked fwd+bwd FLOPs of the step / step time (decode time included).
FLOPs count only (i, j) pairs inside the band: 4*D per pair forward, 10*D per
pair backward (five matmuls with the recomputed scores).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run; every rank
runs its own independent batch (weak scaling, no data-path collective) and
the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd+bwd TFLOP/s (unmasked FLOPs) & % BF16 peak; decode HBM GB/s"
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def band_pairs(T: int, W: int) -> int:
    """Number of (i, j) pairs with i - W < j <= i, 0 <= j <= i < T."""
    if W >= T:
        return T * (T + 1) // 2
    return W * (W + 1) // 2 + (T - W) * W


def fwd_flops(B, T, H, D, W):
    return 4 * D * B * H * band_pairs(T, W)


def bwd_flops(B, T, H, D, W):
    return 10 * D * B * H * band_pairs(T, W)


def decode_bytes(cache_len, H, D, W):
    n = np.minimum(cache_len.astype(np.int64), W)
    B = len(cache_len)
    return int(n.sum()) * H * D * 2 * 2 + 2 * B * H * D * 2


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank_step * world * steps / (max_ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


PROFILE_FOR_KERNEL = {
    "swa_bwd_dkdv_kernel<128>": "swa_bwd_dkdv_kernel_d24shape_b8.md",
    "swa_bwd_dq_kernel<128>": "swa_bwd_dq_kernel_d24shape_b8.md",
    # the forward runs swa_fwd_short_kernel for W < T and swa_fwd_kernel otherwise; one summary
    # covers both, per window
    "swa_fwd_short_kernel<128> (W < T) / swa_fwd_kernel<128>": "swa_fwd_kernel_d24shape_b8.md",
    "swa_decode_kernel<128>": "swa_decode_kernel_decode_workload.md",
}


def measured_traffic(kernel, windows, batch):
    """DRAM bytes per launch (read + write) of `kernel` from its committed ncu summary, scaled from
    the captured batch to `batch` and averaged over the step's launches (one per window); None when
    there is no summary or the kernel's sources changed since the capture (fingerprint mismatch)."""
    import hashlib
    import re

    name = PROFILE_FOR_KERNEL.get(kernel)
    path = os.path.join(ROOT, "profiles", name) if name else None
    if not path or not os.path.exists(path):
        return None
    m = re.search(r"^traffic_bytes: (.*); batch (\d+); source_sha256 ([0-9a-f]{64}) \((.*)\)$",
                  open(path).read(), flags=re.M)
    if not m:
        return None
    per_w = {int(w): int(b) for w, b in re.findall(r"W=(\d+) (\d+)", m.group(1))}
    h = hashlib.sha256()
    for f in m.group(4).split(" + "):
        with open(os.path.join(ROOT, "causal_sliding_window_b200", "csrc", f.strip()), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != m.group(3) or any(w not in per_w for w in windows):
        return None
    return sum(per_w[w] for w in windows) / len(windows) * batch / int(m.group(2))


class ClockSampler:
    """nvidia-smi clock / throttle sampling of one GPU while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, path: str | None):
        self.proc = None
        self.path = path
        try:
            self.out = open(path, "w") if path else subprocess.PIPE
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.out, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            text = ""
        if self.path:
            self.out.close()
            text = open(self.path).read()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (text or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [s for s in sm if smax and s > 0.3 * max(smax)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_uuid(dev) -> str:
    import torch

    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


def make_inputs(rank: int):
    from causal_sliding_window_b200 import inputs

    cfg = inputs.WORKLOADS["d24"]
    att = inputs.attention_inputs(cfg["B"], cfg["T"], cfg["H"], cfg["D"], seed=cfg["seed"] + 1000 * rank)
    dc = inputs.DECODE_WORKLOAD
    dec = inputs.decode_inputs(dc["B"], dc["cap"], dc["H"], dc["D"], seed=dc["seed"] + 1000 * rank)
    return cfg, att, dc, dec


def to_bf16(bits, device, pin=False):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    if pin:
        return t.pin_memory()
    return t.to(device)


def cpu_baseline_sample(cfg, att, heads=None):
    """The oracle, as it stands, on sequence 0 (first `heads` heads) of the d24 SSSL step (fwd + bwd)."""
    from oracle import oracle_bwd, oracle_fwd, oracle_threads

    heads = cfg["H"] if heads is None else heads
    q, k, v, do = (np.ascontiguousarray(att[n][:1, :, :heads]) for n in ("q", "k", "v", "do"))
    B, T, H, D = 1, cfg["T"], heads, cfg["D"]
    t0 = time.perf_counter()
    flops = 0
    for W in cfg["windows"]:
        oracle_fwd(q, k, v, W)
        oracle_bwd(q, k, v, do, W)
        flops += fwd_flops(B, T, H, D, W) + bwd_flops(B, T, H, D, W)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"sequence 0 of the d24 batch (1 x {T} x {H} x {D}), SSSL windows {list(cfg['windows'])}, "
                      f"fwd+bwd in fp64; {dt:.1f} s",
            "seconds": dt}


def run_reference(args, rank, world):
    """--impl reference: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    from causal_sliding_window_b200 import inputs

    cfg = inputs.WORKLOADS["d24"]
    att = inputs.attention_inputs(1, cfg["T"], cfg["H"], cfg["D"], seed=cfg["seed"])
    heads = 2   # bounded sample per step: sequence 0, heads 0-1 (a few seconds of fp64 work)
    for _ in range(args.warmup):
        cpu_baseline_sample(cfg, att, heads)
    times, flops = [], 0.0
    for _ in range(args.steps):
        cb = cpu_baseline_sample(cfg, att, heads)
        times.append(cb["seconds"])
        flops = cb["value"] * 1e12 * cb["seconds"]
    total = sum(times)
    value = flops * len(times) / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"d24 SSSL fwd+bwd, bounded sample: sequence 0 of 32, heads 0-{heads - 1} of 12",
                   "global_batch": 1, "seq_len": cfg["T"], "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_case(args):
    """Profiling helper: `--warmup` untimed then `--steps` calls of one entry point on the d24
    shape with a reduced batch (inputs still larger than L2), for ncu captures."""
    import torch

    from causal_sliding_window_b200 import inputs, ops

    dev = torch.device("cuda", 0)
    cfg = inputs.WORKLOADS["d24"]
    B, T, H, D, W = args.batch, cfg["T"], cfg["H"], cfg["D"], args.window
    if args.case == "decode":
        dc = inputs.DECODE_WORKLOAD
        x = inputs.decode_inputs(dc["B"], dc["cap"], dc["H"], dc["D"], seed=dc["seed"])
        q, kc, vc = to_bf16(x["q"], dev), to_bf16(x["k_cache"], dev), to_bf16(x["v_cache"], dev)
        cl = torch.from_numpy(x["cache_len"]).to(dev)
        ws = ops.decode_workspace(dc["B"], dc["cap"], dc["H"], dc["D"], dev)
        call = lambda: ops.decode(q, kc, vc, cl, W, workspace=ws)  # noqa: E731
    elif args.case == "fp8":
        x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"], with_do=False)
        # e4m3 inputs by torch's conversion of the bf16 values (unit descales: |x| stays far below 448)
        q8, k8, v8 = (to_bf16(x[n], dev).float().to(torch.float8_e4m3fn) for n in ("q", "k", "v"))
        ds = torch.ones((B, H), dtype=torch.float32, device=dev)
        o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
        ws = torch.empty(ops.attn_fwd_fp8_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=dev)
        call = lambda: ops.attn_fwd_fp8(q8, k8, v8, ds, ds, ds, o, lse, ws, W)  # noqa: E731
    else:
        x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"])
        q, k, v, do = (to_bf16(x[n], dev) for n in ("q", "k", "v", "do"))
        o, lse = ops.forward(q, k, v, W)
        ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=dev)
        if args.case == "fwd":
            call = lambda: ops.attn_fwd(q, k, v, o, lse, W)  # noqa: E731
        else:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
            call = lambda: ops.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, W)  # noqa: E731
    for _ in range(args.warmup + args.steps):
        call()
    torch.cuda.synchronize()
    status = ops.attn_device_status(clear=True)
    print(json.dumps({"case": args.case, "batch": B, "window": W, "calls": args.warmup + args.steps,
                      "status": status}))
    return 0 if status == 0 else 1


def timed_median(fn, reps=20, warmup=3, before=None):
    """Median device time (ms) of `reps` calls of fn, each between its own pair of CUDA events on
    the current stream, after `warmup` untimed calls.  `before(i)` (optional, untimed) runs ahead
    of call i, e.g. to pick the next of several rotated input sets."""
    import torch

    for i in range(warmup):
        if before:
            before(i)
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        if before:
            before(warmup + i)
        ev[i][0].record()
        fn()
        ev[i][1].record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def run_configs(args):
    """Standalone timing of every configuration row (one JSON line each): the depth-12/24/26 shapes
    at each of their windows (forward and backward), the decode workload at both windows, and the
    widened rows (grouped K/V heads, the RoPE + QK-norm op, chunked prefill, decode with the
    prologue).  Protocol: median of `--reps` (default 20) CUDA-event-timed calls after 3 warm-ups,
    seeded synthetic inputs; every attention input is larger than L2, and decode rotates 3
    independently filled cache sets so that no call finds its cache in L2."""
    import torch

    from causal_sliding_window_b200 import inputs, ops

    dev = torch.device("cuda", 0)
    reps = max(20, args.reps)
    peaks, peak_src = load_peaks()
    pt = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    pts = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    ph = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])

    def emit(**kw):
        kw.update(protocol=f"median of {reps} CUDA-event calls after 3 warm-ups", peak_source=peak_src)
        print(json.dumps(kw), flush=True)

    def tensor_row(row, W, kind, flops, ms):
        tf = flops / ms / 1e9
        # FP8 rows against the FP8 peaks: twice the bf16 ones (the nominal dense ratio, 4.5 / 2.25 PF)
        mult = 2.0 if kind == "fwd-fp8" else 1.0
        emit(row=row, W=W, kind=kind, ms=round(ms, 4), tflops=round(tf, 1),
             frac_spec=round(tf / (mult * SPEC_BF16_TFLOPS), 4), frac_burst=round(tf / (mult * pt), 4),
             frac_sustained=round(tf / (mult * pts), 4))

    def attention_rows(name, Hkv=None, label=None):
        cfg = inputs.WORKLOADS[name]
        B, T, H, D = cfg["B"], cfg["T"], cfg["H"], cfg["D"]
        hk = Hkv or H
        x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"], peaky=cfg["peaky"])
        q, do = to_bf16(x["q"], dev), to_bf16(x["do"], dev)
        k = to_bf16(np.ascontiguousarray(x["k"][:, :, :hk]), dev)
        v = to_bf16(np.ascontiguousarray(x["v"][:, :, :hk]), dev)
        del x
        o, lse = torch.empty_like(q), torch.empty((B, H, T), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=dev)
        out = {}
        for W in sorted(set(cfg["windows"]), reverse=True):
            tf = timed_median(lambda: ops.attn_fwd(q, k, v, o, lse, W), reps)
            tb = timed_median(lambda: ops.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, W), reps)
            row = label or f"{name} B={B} T={T} H={H} D={D}" + (" peaky Q/K" if cfg["peaky"] else "")
            tensor_row(row, W, "fwd", fwd_flops(B, T, H, D, W), tf)
            tensor_row(row, W, "bwd", bwd_flops(B, T, H, D, W), tb)
            out[W] = (tf, tb)
        if name == "d24" and Hkv is None:   # the SSSL layer pattern from the per-window medians
            wins = cfg["windows"]
            f = sum(fwd_flops(B, T, H, D, W) for W in wins)
            tensor_row("d24 SSSL (3 x W512 + W2048), sum of per-window medians", list(wins), "fwd", f,
                       sum(out[W][0] for W in wins))
            tensor_row("d24 SSSL (3 x W512 + W2048), sum of per-window medians", list(wins), "bwd", 2.5 * f,
                       sum(out[W][1] for W in wins))
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()

    for name in ("d12", "d24", "d26"):
        attention_rows(name)
    attention_rows("d24", Hkv=4, label="d24 shape with 4 K/V heads (grouped)")

    # FP8 forward on the depth-24 shape: e4m3 by torch's conversion of the seeded bf16 values
    cfg = inputs.WORKLOADS["d24"]
    B, T, H, D = cfg["B"], cfg["T"], cfg["H"], cfg["D"]
    x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"], with_do=False)
    q8, k8, v8 = (to_bf16(x[n], dev).float().to(torch.float8_e4m3fn) for n in ("q", "k", "v"))
    del x
    ds = torch.ones((B, H), dtype=torch.float32, device=dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    ws8 = torch.empty(ops.attn_fwd_fp8_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=dev)
    for W in (2048, 512):
        tensor_row(f"d24 B={B} T={T} H={H} D={D}, FP8 (e4m3) forward", W, "fwd-fp8", fwd_flops(B, T, H, D, W),
                   timed_median(lambda: ops.attn_fwd_fp8(q8, k8, v8, ds, ds, ds, o, lse, ws8, W), reps))
    del q8, k8, v8, o, lse, ws8
    torch.cuda.empty_cache()

    cfg = inputs.WORKLOADS["d24"]
    B, T, H, D = cfg["B"], cfg["T"], cfg["H"], cfg["D"]
    x = inputs.attention_inputs(B, T, H, D, seed=cfg["seed"], with_do=True)
    q, dy = to_bf16(x["q"], dev), to_bf16(x["do"], dev)
    del x
    cos, sin = ops.rope_tables(4096, D, dev)
    y = torch.empty_like(q)
    t = timed_median(lambda: ops.attn_rope_qknorm(q, y, cos, sin, 1e-6), reps)
    gbs = 2 * q.numel() * 2 / t / 1e6
    emit(row="rope + qk norm, d24-shaped q", kind="hbm", ms=round(t, 4), gbs=round(gbs, 1),
         frac_spec=round(gbs / SPEC_HBM_GBS, 4), frac_measured=round(gbs / ph, 4))
    t = timed_median(lambda: ops.attn_rope_qknorm_bwd(q, dy, y, cos, sin, 1e-6), reps)
    gbs = 3 * q.numel() * 2 / t / 1e6
    emit(row="rope + qk norm backward, d24-shaped q", kind="hbm", ms=round(t, 4), gbs=round(gbs, 1),
         frac_spec=round(gbs / SPEC_HBM_GBS, 4), frac_measured=round(gbs / ph, 4))
    del q, dy, y
    torch.cuda.empty_cache()

    # chunked prefill: 32 sequences, a 512-token chunk after U[0, 1536] cached tokens
    Bp, Tn, cap = 32, 512, 2048
    L = inputs.uniform_int(7, "cache_len", Bp, 0, cap - Tn)
    xp = inputs.attention_inputs(Bp, Tn, H, D, seed=7)
    qp, kn, vn = (to_bf16(xp[n], dev) for n in ("q", "k", "v"))
    kc = torch.zeros((Bp, cap, H, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    cl = torch.from_numpy(L).to(dev)
    for W in (2048, 512):
        f = 4 * D * H * sum(min(int(L[b]) + t + 1, W) for b in range(Bp) for t in range(Tn))
        tensor_row("prefill, 32 x 512-token chunks after U[0,1536] cached", W, "prefill", f,
                   timed_median(lambda: ops.prefill(qp, kn, vn, kc, vc, cl, W), reps))
        tensor_row("prefill with the prologue, as above", W, "prefill", f,
                   timed_median(lambda: ops.prefill_rope(qp, kn, vn, kc, vc, cl, cos, sin, 1e-6, W), reps))
    del qp, kn, vn, kc, vc
    torch.cuda.empty_cache()

    # decode, 12 and 4 K/V heads, with and without the prologue; 3 cache sets in rotation
    dc = inputs.DECODE_WORKLOAD
    xd = inputs.decode_inputs(dc["B"], dc["cap"], dc["H"], dc["D"], seed=dc["seed"])
    qd = to_bf16(xd["q"], dev)
    cl = torch.from_numpy(xd["cache_len"]).to(dev)
    for hk in (dc["H"], 4):
        sets = []
        for r in range(3):   # independently filled sets (r = 0 is the seeded workload itself)
            xs = xd if r == 0 else inputs.decode_inputs(dc["B"], dc["cap"], dc["H"], dc["D"], seed=dc["seed"] + 17 * r,
                                                        cache_len=xd["cache_len"])
            sets.append((to_bf16(np.ascontiguousarray(xs["k_cache"][:, :, :hk]), dev),
                         to_bf16(np.ascontiguousarray(xs["v_cache"][:, :, :hk]), dev)))
        cur = [sets[0]]

        def pick(i):
            cur[0] = sets[i % len(sets)]

        kn = torch.zeros((dc["B"], hk, dc["D"]), dtype=torch.bfloat16, device=dev)
        vn = torch.zeros_like(kn)
        wsd = ops.decode_workspace(dc["B"], dc["cap"], dc["H"], dc["D"], dev, Hkv=hk)
        for W in dc["windows"]:
            nbytes = decode_bytes(xd["cache_len"], hk, dc["D"], W) + 2 * dc["B"] * (dc["H"] - hk) * dc["D"] * 2
            for rope in (False, True):
                if rope:
                    fn = lambda: ops.decode_rope(qd, kn, vn, *cur[0], cl, cos, sin, 1e-6, W, workspace=wsd)  # noqa: E731
                else:
                    fn = lambda: ops.decode(qd, *cur[0], cl, W, workspace=wsd)  # noqa: E731
                t = timed_median(fn, reps, before=pick)
                gbs = nbytes / t / 1e6
                emit(row=f"decode workload, {hk} K/V heads" + (", with the prologue" if rope else ""), W=W,
                     kind="hbm", us=round(t * 1e3, 2), gbs=round(gbs, 1), bytes=nbytes,
                     frac_spec=round(gbs / SPEC_HBM_GBS, 4), frac_measured=round(gbs / ph, 4), cache_sets=len(sets))
        del sets, cur
        torch.cuda.empty_cache()
    status = ops.attn_device_status(clear=True)
    emit(row="status", status=status)
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-log", default=None)
    ap.add_argument("--case", default="step", choices=["step", "fwd", "bwd", "decode", "fp8", "configs"],
                    help="fwd / bwd / decode / fp8: run only that call repeatedly on a reduced batch, for profiling "
                         "(no metric line); configs: standalone timing of every configuration row")
    ap.add_argument("--reps", type=int, default=20, help="timed calls per row for --case configs (>= 20)")
    ap.add_argument("--batch", type=int, default=8, help="batch for --case (d24 shape otherwise)")
    ap.add_argument("--window", type=int, default=2048, help="window for --case")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.case == "configs":
        return run_configs(args)
    if args.case != "step":
        return run_case(args)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    from causal_sliding_window_b200 import ops

    cfg, att, dc, dec = make_inputs(rank)
    B, T, H, D = cfg["B"], cfg["T"], cfg["H"], cfg["D"]
    windows = list(cfg["windows"])
    dwins = list(dc["windows"])
    # Device-resident inputs and outputs.
    q, k, v, do = (to_bf16(att[n], dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=dev)
    dB, cap, dH, dD = dc["B"], dc["cap"], dc["H"], dc["D"]
    from causal_sliding_window_b200 import inputs
    dq_in = to_bf16(dec["q"], dev)
    kc, vc = to_bf16(dec["k_cache"], dev), to_bf16(dec["v_cache"], dev)
    # Three independently filled cache sets in rotation, so that no decode launch finds the cache
    # it reads in L2 (a step's two decode launches read different sets).
    cache_sets = [(kc, vc)]
    for r in (1, 2):
        xs = inputs.decode_inputs(dB, cap, dH, dD, seed=dc["seed"] + 17 * r + 1000 * rank,
                                  cache_len=dec["cache_len"])
        cache_sets.append((to_bf16(xs["k_cache"], dev), to_bf16(xs["v_cache"], dev)))
        del xs
    cl = torch.from_numpy(dec["cache_len"]).to(dev)
    d_o = torch.empty((dB, dH, dD), dtype=torch.bfloat16, device=dev)
    d_lse = torch.empty((dB, dH), dtype=torch.float32, device=dev)
    dws = ops.decode_workspace(dB, cap, dH, dD, dev)

    stream = torch.cuda.current_stream()
    step_flops = sum(fwd_flops(B, T, H, D, W) + bwd_flops(B, T, H, D, W) for W in windows)
    step_fwd_flops = sum(fwd_flops(B, T, H, D, W) for W in windows)
    step_bwd_flops = sum(bwd_flops(B, T, H, D, W) for W in windows)
    step_dec_bytes = sum(decode_bytes(dec["cache_len"], dH, dD, W) for W in dwins)
    launches_per_step = 4 * len(windows) + len(dwins)

    def run_step(ev=None, step=0, rotate=True):
        for li, W in enumerate(windows):
            if ev is not None:
                ev["f0"][li].record(stream)
            ops.attn_fwd(q, k, v, o, lse, W, stream=stream)
            if ev is not None:
                ev["f1"][li].record(stream)
                ops.attn_bwd_set_profile_events(ev["bp"][li], ev["bm"][li])
            ops.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, W, stream=stream)
            if ev is not None:
                ops.attn_bwd_set_profile_events(None, None)
                ev["b1"][li].record(stream)
        for di, W in enumerate(dwins):
            if ev is not None:
                ev["d0"][di].record(stream)
            kcs, vcs = cache_sets[(step * len(dwins) + di) % len(cache_sets)] if rotate else cache_sets[0]
            ops.attn_decode(dq_in, kcs, vcs, cl, d_o, d_lse, dws, W, stream=stream)
            if ev is not None:
                ev["d1"][di].record(stream)

    for w in range(args.warmup):
        run_step(step=w)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0, "device wait timed out during warm-up"

    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]  # noqa: E731
    evs = [{"f0": mk(len(windows)), "f1": mk(len(windows)), "bp": mk(len(windows)), "bm": mk(len(windows)),
            "b1": mk(len(windows)), "d0": mk(len(dwins)), "d1": mk(len(dwins))} for _ in range(args.steps)]
    # torch creates the CUDA event lazily at its first record(); the library records the
    # backward's inner events by handle, so make every handle exist before the timed region.
    for e in evs:
        for lst in e.values():
            for ev in lst:
                ev.record(stream)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_uuid(dev), args.clock_log if rank == 0 else None)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for s in range(args.steps):
        run_step(evs[s], step=s)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    status = ops.attn_device_status(clear=True)
    assert status == 0, "device wait timed out during the timed region"
    t_fwd = sum(e["f0"][i].elapsed_time(e["f1"][i]) for e in evs for i in range(len(windows)))
    t_pre = sum(e["f1"][i].elapsed_time(e["bp"][i]) for e in evs for i in range(len(windows)))
    t_dkdv = sum(e["bp"][i].elapsed_time(e["bm"][i]) for e in evs for i in range(len(windows)))
    t_dqk = sum(e["bm"][i].elapsed_time(e["b1"][i]) for e in evs for i in range(len(windows)))
    t_dec = sum(e["d0"][i].elapsed_time(e["d1"][i]) for e in evs for i in range(len(dwins)))
    ms_max = max_over_ranks(ms, dev)
    finite = bool(torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()
                  and torch.isfinite(d_o.float()).all())

    # ---- end to end: host buffers in, results out, every step ----
    host = {n: to_bf16(att[n], None, pin=True) for n in ("q", "k", "v", "do")}
    host_dec = {"q": to_bf16(dec["q"], None, pin=True), "k": to_bf16(dec["k_cache"], None, pin=True),
                "v": to_bf16(dec["v_cache"], None, pin=True),
                "cl": torch.from_numpy(dec["cache_len"]).pin_memory()}
    out_host = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in
                (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("d_o", d_o), ("d_lse", d_lse))}
    h2d = sum(t.numel() * t.element_size() for t in list(host.values()) + list(host_dec.values()))
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())

    def e2e_step():
        for n, dst in (("q", q), ("k", k), ("v", v), ("do", do)):
            dst.copy_(host[n], non_blocking=True)
        dq_in.copy_(host_dec["q"], non_blocking=True)
        kc.copy_(host_dec["k"], non_blocking=True)
        vc.copy_(host_dec["v"], non_blocking=True)
        cl.copy_(host_dec["cl"], non_blocking=True)
        run_step(rotate=False)   # both decode launches read the cache set copied in this step
        for n, src in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("d_o", d_o),
                       ("d_lse", d_lse)):
            out_host[n].copy_(src, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)

    if rank == 0:
        peaks, peak_src = load_peaks()
        K = args.steps
        value = weak_scaling_value(step_flops, world, K, ms_max)
        fwd_tf = step_fwd_flops * K / (t_fwd * 1e-3) / 1e12
        # Per-kernel algorithmic work: the dK/dV kernel needs S, dP, dV, dK (8*D flops per in-band
        # pair), the dQ kernel S, dP, dQ (6*D); the backward as a whole counts 10*D.
        dkdv_tf = step_bwd_flops * 0.8 * K / (t_dkdv * 1e-3) / 1e12
        dqk_tf = step_bwd_flops * 0.6 * K / (t_dqk * 1e-3) / 1e12
        bwd_tf = step_bwd_flops * K / ((t_pre + t_dkdv + t_dqk) * 1e-3) / 1e12
        dec_gbs = step_dec_bytes * K / (t_dec * 1e-3) / 1e9
        parts = {"fwd_ms": t_fwd / K, "bwd_pre_ms": t_pre / K, "bwd_dkdv_ms": t_dkdv / K,
                 "bwd_dq_ms": t_dqk / K, "decode_ms": t_dec / K}
        dominant = max(parts, key=parts.get)
        # Burst or sustained bf16 peak, from this run's own clock record: a timed region that kept
        # the SM clock at its maximum ran at burst clocks, so the burst GEMM figure applies.
        at_max = bool(clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.97 * clk["sm_max_mhz"])
        peak_kind = "bf16_tflops" if at_max else "bf16_tflops_sustained"
        peak_t = peaks.get(peak_kind, FALLBACK_PEAKS[peak_kind])
        peak_h = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        if dominant == "fwd_ms":
            roof = {"kernel": "swa_fwd_short_kernel<128> (W < T) / swa_fwd_kernel<128>", "bound": "tensor",
                    "achieved": fwd_tf, "peak": peak_t,
                    "unit": "TFLOP/s"}
        elif dominant == "decode_ms":
            roof = {"kernel": "swa_decode_kernel<128>", "bound": "hbm", "achieved": dec_gbs, "peak": peak_h,
                    "unit": "GB/s"}
        elif dominant == "bwd_dq_ms":
            roof = {"kernel": "swa_bwd_dq_kernel<128>", "bound": "tensor", "achieved": dqk_tf, "peak": peak_t,
                    "unit": "TFLOP/s"}
        else:
            roof = {"kernel": "swa_bwd_dkdv_kernel<128>", "bound": "tensor", "achieved": dkdv_tf, "peak": peak_t,
                    "unit": "TFLOP/s"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = (measured_traffic(roof["kernel"], dwins, dB) if roof["kernel"].startswith("swa_decode")
                           else measured_traffic(roof["kernel"], windows, B))
        roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
        roof["peak_source"] = (f"{peak_src} ({'burst' if at_max else 'sustained'} bf16: median SM clock "
                               f"{clk.get('sm_mhz')} of {clk.get('sm_max_mhz')} MHz in the timed region)"
                               if roof["unit"] == "TFLOP/s" else f"{peak_src} (copy)")
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline_sample(cfg, att)
            cb.pop("seconds")
            cpu = cb
        e2e_val = weak_scaling_value(step_flops, world, 1, e2e_ms)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "d24 SSSL fwd+bwd (B=32,T=2048,H=12,D=128; W=512,512,512,2048) "
                                   "+ decode (32 seqs, cap 2048, H=12, D=128; W=2048,1024)",
                       "global_batch": B * world, "seq_len": T, "heads": H, "head_dim": D,
                       "windows": windows, "decode_windows": dwins,
                       "l2": "inputs larger than L2 (q,k,v,dO 201 MB each; decode caches 403 MB each, "
                             "3 cache sets in rotation)",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "parts": {
                **{k2: round(v2, 4) for k2, v2 in parts.items()},
                "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf, "bwd_dkdv_tflops": dkdv_tf, "bwd_dq_tflops": dqk_tf, "decode_gbs": dec_gbs,
                "fwd_frac_spec_2250": fwd_tf / SPEC_BF16_TFLOPS, "bwd_frac_spec_2250": bwd_tf / SPEC_BF16_TFLOPS,
                "decode_frac_spec_8000": dec_gbs / SPEC_HBM_GBS,
                "fwd_frac_measured": fwd_tf / peak_t, "bwd_frac_measured": bwd_tf / peak_t,
                "decode_frac_measured": dec_gbs / peak_h,
            },
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": args.e2e_steps},
            "gpu_launches": launches_per_step * K,
            "clocks": clk,
            "outputs_finite": finite,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
