#!/usr/bin/env python
"""Benchmark of the Mamba-2 selective-scan hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

Headline (one JSON line on rank 0): SSD prefill tokens/s/layer on the 8k-token prefill
workload (B1 L8192 H128 P64 N128 G8 chunk 128, bf16 inputs, fp32 state, conv window 4 +
SiLU, output + final state), inputs resident in HBM, L2 flushed between timed steps, CUDA
events on the launching stream.  The same line carries:
  - "roofline": the dominant kernel's algorithmic GB/s against the measured HBM copy peak;
  - "e2e": the same metric with host (pinned) inputs copied in and outputs copied back
    inside the timed region;
  - "clocks": nvidia-smi SM clocks and throttle reasons sampled during the timed region
    (extended by one second of the same step when the region is shorter than that);
  - "decode": the 16384-step decode workload (B64 H128, fp32 state of 256 MiB), state-update
    GB/s with the steps replayed from CUDA graphs;
  - "long_context": 131072 tokens in 4 segments of 32768 with state and conv-cache carry,
    chunk 256, gated RMSNorm;
  - "mixer": the whole mixer layer at the 12B width (d_model 5120, 160 heads, B8 L8192),
    tensor-core roofline of its dominant GEMM;
  - "cpu_baseline": the fp64 oracle timed on a bounded sample of the prefill workload;
    "parity": the library's prefill on that sample against the oracle's result (max|err|/RMS).
Multi-GPU (torchrun): one process per GPU, each an independent replica (weak scaling), time
= max over ranks.  --impl reference times the fp64 CPU oracle on the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mamba_ssd_scan_02_b200 import datagen  # noqa: E402

L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "SSD prefill tokens/s/layer"
HEADLINE_CONFIG = {"workload": "prefill_8k", "batch": 1, "seqlen": 8192, "nheads": 128,
                   "headdim": 64, "dstate": 128, "ngroups": 8, "chunk": 128, "conv_width": 4,
                   "state_dtype": "f32",
                   "l2": "flushed between timed steps: 256 MiB written, then a second 256 MiB "
                         "buffer read, so the step starts with no dirty lines in L2"}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's sources are still
    the ones that were captured (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
    except (OSError, ValueError, KeyError):
        return None
    h = hashlib.sha256()
    for rel in rec["sources"]:
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    return rec["bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None


# ---------------------------------------------------------------------------------------------
# algorithmic byte counts (each required input once, each output once, state in/out once,
# parameters once)
def scan_bytes(cfg, state_in=False) -> int:
    """Tensors the scan itself must move: x, B, C, dt in, y out, final (and initial) state."""
    Bn, L, H, P, N, G = (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                         cfg["ngroups"])
    e = 2 if cfg["dtype"] == "bf16" else 4
    b = Bn * L * (H * P + 2 * G * N + H) * e + Bn * L * H * P * e
    b += Bn * H * P * N * 4 * (2 if state_in else 1)
    return b


def prefill_bytes(cfg, state_in=False) -> int:
    """The whole prefill call: scan_bytes plus z (gated norm), conv cache, parameters."""
    Bn, L, H, P = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"]
    e = 2 if cfg["dtype"] == "bf16" else 4
    cd, W = datagen.conv_dim(cfg), cfg["conv_width"]
    b = scan_bytes(cfg, state_in)
    if cfg.get("norm_groups"):
        b += Bn * L * H * P * e + H * P * e        # z, norm weight
    b += cd * W * e + 3 * H * 4                    # conv weight, A, D, dt_bias
    b += Bn * W * cd * e * (2 if state_in else 1)  # conv cache out (and in)
    return b


def gated_norm_bytes(cfg) -> int:
    Bn, L, d = cfg["batch"], cfg["seqlen"], cfg["nheads"] * cfg["headdim"]
    return 3 * Bn * L * d * 2 + d * 2              # y in, z in, out (bf16), weight


def decode_bytes(cfg) -> int:
    Bn, H, P, N = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    cd = datagen.conv_dim(cfg)
    d_inner = H * P
    W = cfg["conv_width"]
    b = 2 * Bn * H * P * N * 4                   # state read + write
    b += Bn * (cd + H + d_inner) * 2             # xBC_t, dt_t, z_t
    b += Bn * d_inner * 2                        # y_t
    b += Bn * (W - 1) * cd * 2 + Bn * W * cd * 2  # conv cache: W-1 rows read, W rows written
    b += cd * W * 2 + 3 * H * 4 + d_inner * 2    # parameters
    return b


def mixer_flops(cfg) -> dict:
    T = cfg["batch"] * cfg["seqlen"]
    H, P, N, G, Q = cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["ngroups"], 128
    d_inner, dm = H * P, cfg["d_model"]
    proj = 2 * d_inner + 2 * G * N + H
    ssd = T * (H * (2 * Q * P + 4 * N * P) + G * 2 * Q * N)
    return {"in_proj": 2 * T * proj * dm, "out_proj": 2 * T * dm * d_inner, "ssd": ssd}


# ---------------------------------------------------------------------------------------------
# multi-GPU accounting: every rank runs an independent replica of the workload (weak scaling)
def max_over_ranks(torch, dist, value: float, device) -> float:
    """The job's time is the slowest rank's: all-reduce MAX (identity on one process)."""
    if not dist:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, steps: int, total_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the (max-over-ranks) time."""
    return world * units_per_rank * steps / (total_ms * 1e-3)


# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock/throttle sampling every 100 ms in a reader thread; each sample is
    stamped with the host's monotonic clock when it arrives."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.samples = []
        self.lock = threading.Lock()

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        threading.Thread(target=self._read, daemon=True).start()
        t0 = time.monotonic()
        while time.monotonic() - t0 < 10 and not self.samples and self.proc.poll() is None:
            time.sleep(0.05)
        return self

    def _read(self):
        for ln in self.proc.stdout:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                s = (time.monotonic(), float(f[1]), float(f[2]),
                     {n for n, v in zip(self.NAMES, f[5:9]) if v.lower() == "active"})
            except ValueError:
                continue
            with self.lock:
                self.samples.append(s)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float, window: str):
        with self.lock:
            sel = [s for s in self.samples if t0 <= s[0] <= t1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": window}
        reasons = set().union(*(s[3] for s in sel))
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": sel[-1][2],
                "reasons": sorted(reasons), "samples": len(sel), "window": window}


def smi_gpu_id(torch, dev: int) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except (AttributeError, RuntimeError):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[dev] if vis else str(dev)


class Ctx:
    """What every workload needs: torch, the binding, the process group, the clock sampler."""

    def __init__(self, args, torch, ssd, dist, rank, world, clk):
        self.args, self.torch, self.ssd, self.dist = args, torch, ssd, dist
        self.rank, self.world, self.clk = rank, world, clk
        self.dev = torch.device("cuda")
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=self.dev)
        self.flush_rd = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=self.dev)

    def flush_l2(self, i: int):
        """Evicts the previous step's data from L2: a write of a buffer larger than L2, then a
        read of a second one, which writes back the dirty lines outside the timed region."""
        self.flush.fill_(float(i))
        self.flush_rd.sum()

    def max_over_ranks(self, v: float) -> float:
        return max_over_ranks(self.torch, self.dist, v, self.dev)

    def timed(self, step, steps, flush=True, trace=True):
        """Times `steps` calls of step() with CUDA events on the current stream (barrier and
        synchronize on both sides), then keeps the GPU on the same step for one more second
        when the timed region was shorter, so that the clock sampler sees it under load.
        With `trace`, a second pass of the same steps records each library launch with CUDA
        events (for the per-kernel breakdown); the timed pass itself runs untraced.
        Returns (total ms, max over ranks), the traced kernel records, and the clocks."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        if self.dist:
            self.dist.barrier()
        torch.cuda.synchronize()
        t0 = time.monotonic()
        for i in range(steps):
            if flush:
                self.flush_l2(i)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t1 = time.monotonic()
        window = "timed region"
        if t1 - t0 < 1.0:
            while time.monotonic() - t1 < 1.0:
                for _ in range(4):
                    if flush:
                        self.flush_l2(0)
                    step()
                torch.cuda.synchronize()
            window = "timed region + 1 s of the same step right after it"
        t2 = time.monotonic()
        if self.dist:
            self.dist.barrier()
        ms = self.max_over_ranks(float(sum(a.elapsed_time(b) for a, b in ev)))
        recs = []
        if trace:
            self.ssd.trace_enable(True)
            self.ssd.trace_read()
            for i in range(steps):
                if flush:
                    self.flush_l2(i)
                step()
            torch.cuda.synchronize()
            self.ssd.trace_enable(False)
            recs = self.ssd.trace_read()
        return ms, recs, self.clk.summary(t0, t2, window)


# Kernels that the library runs on its side stream, concurrently with the stream's own work:
# their time is not on the step's critical path, so they take no share and are never the
# dominant kernel.
OVERLAPPED = {"ssd_state_tail": "side stream, concurrent with ssd_scan_tc"}


def kernel_table(recs):
    per = {}
    for name, ms in recs:
        per.setdefault(name, []).append(ms)
    serial = {k: v for k, v in per.items() if k not in OVERLAPPED}
    total = sum(sum(v) for v in serial.values()) or 1.0
    table = {}
    for k, v in per.items():
        row = {"launches": len(v), "mean_ms": round(statistics.mean(v), 5)}
        if k in OVERLAPPED:
            row.update(share=None, overlapped=OVERLAPPED[k])
        else:
            row["share"] = round(sum(v) / total, 4)
        table[k] = row
    dom = max(serial, key=lambda k: sum(serial[k])) if serial else None
    return per, table, dom


def hbm_roofline(kernel, ms, algo_bytes, workload):
    pk, src = peaks()
    ach = algo_bytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / pk["hbm_gbs"], 4),
            "traffic": recorded_traffic(kernel, workload), "kernel": kernel,
            "kernel_ms": round(ms, 5), "algorithmic_bytes": algo_bytes,
            "peak_source": f"{src} HBM copy (burst)"}


# ---------------------------------------------------------------------------------------------
def bench_prefill(c: Ctx):
    torch, ssd, args = c.torch, c.ssd, c.args
    cfg = datagen.config(1)
    inp = datagen.make_inputs(1)
    d = {k: ssd.to_device(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    Bn, L, H, P, N = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    y = torch.empty((Bn, L, H * P), dtype=torch.bfloat16, device=c.dev)
    hf = torch.empty((Bn, H, P, N), dtype=torch.float32, device=c.dev)
    cso = torch.empty((Bn, 4, datagen.conv_dim(cfg)), dtype=torch.bfloat16, device=c.dev)
    ws = ssd.alloc_workspace(ssd.workspace_size(cfg), c.dev)

    def step():
        ssd.prefill(cfg, d["xBC"], d["dt"], d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None,
                    None, None, None, y=y, h_final=hf, conv_state_out=cso, workspace=ws)

    for _ in range(args.warmup):
        step()
    total_ms, recs, clocks = c.timed(step, args.steps)
    per, table, dom = kernel_table(recs)
    tokens = Bn * L
    res = {
        "value": job_throughput(tokens, c.world, args.steps, total_ms),
        "ms_per_step": total_ms / args.steps,
        "gpu_launches": len(recs),
        "clocks": clocks,
        "kernels": table,
        # ssd_scan_tc moves every tensor of scan_bytes (x, B|C, dt in; y, state out)
        "roofline": hbm_roofline(dom, statistics.mean(per[dom]), scan_bytes(cfg), "prefill_8k"),
        "path_bytes_per_step": prefill_bytes(cfg),
    }
    # end to end: pinned host inputs in, results out, inside the timed region
    res["e2e"] = e2e_prefill(c, cfg, d, ws, tokens)
    return res


def e2e_prefill(c: Ctx, cfg, d, ws, tokens):
    """Throughput through the public call with host buffers: every step copies its inputs
    (xBC, dt) from pinned host memory to the device, runs ssd.prefill and copies its results
    (y, h_final) back to pinned host memory.  Device inputs and outputs are double-buffered, so
    step i+1's host-to-device copy (copy stream) overlaps step i's compute (current stream) and
    its device-to-host copy (a third stream); PCIe carries both directions at once.  Timed on
    the device as one span from before the first copy to after the last one, max over ranks."""
    torch, ssd, args = c.torch, c.ssd, c.args
    hx = torch.empty(d["xBC"].shape, dtype=torch.bfloat16, pin_memory=True)
    hx.copy_(d["xBC"].cpu())
    hdt = torch.empty(d["dt"].shape, dtype=torch.bfloat16, pin_memory=True)
    hdt.copy_(d["dt"].cpu())
    Bn, L = d["xBC"].shape[0], d["xBC"].shape[1]
    H, P, N = cfg["nheads"], cfg["headdim"], cfg["dstate"]
    hy = torch.empty((Bn, L, H * P), dtype=torch.bfloat16, pin_memory=True)
    hh = torch.empty((Bn, H, P, N), dtype=torch.float32, pin_memory=True)
    xdev = [torch.empty_like(d["xBC"]) for _ in range(2)]
    dtdev = [torch.empty_like(d["dt"]) for _ in range(2)]
    ydev = [torch.empty((Bn, L, H * P), dtype=torch.bfloat16, device=c.dev) for _ in range(2)]
    hdev = [torch.empty((Bn, H, P, N), dtype=torch.float32, device=c.dev) for _ in range(2)]
    cso = torch.empty((Bn, 4, datagen.conv_dim(cfg)), dtype=torch.bfloat16, device=c.dev)
    main = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    consumed = [ev(), ev()]  # the inputs of buffer k have been read by its prefill
    drained = [ev(), ev()]   # the outputs of buffer k have reached the host
    loaded, done = [ev(), ev()], [ev(), ev()]
    for k in range(2):
        consumed[k].record(main)
        drained[k].record(main)

    def step(i):
        k = i % 2
        h2d.wait_event(consumed[k])
        with torch.cuda.stream(h2d):
            xdev[k].copy_(hx, non_blocking=True)
            dtdev[k].copy_(hdt, non_blocking=True)
        loaded[k].record(h2d)
        main.wait_event(loaded[k])
        main.wait_event(drained[k])
        ssd.prefill(cfg, xdev[k], dtdev[k], d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None,
                    None, None, None, y=ydev[k], h_final=hdev[k], conv_state_out=cso, workspace=ws)
        consumed[k].record(main)
        done[k].record(main)
        d2h.wait_event(done[k])
        with torch.cuda.stream(d2h):
            hy.copy_(ydev[k], non_blocking=True)
            hh.copy_(hdev[k], non_blocking=True)
        drained[k].record(d2h)

    def span(n):
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t_start.record(main)
        h2d.wait_event(t_start)
        d2h.wait_event(t_start)
        for i in range(n):
            step(i)
        main.wait_stream(h2d)
        main.wait_stream(d2h)
        t_end.record(main)
        torch.cuda.synchronize()
        return t_start.elapsed_time(t_end)

    span(max(3, args.warmup))
    if c.dist:
        c.dist.barrier()
    e_ms = c.max_over_ranks(span(args.steps))
    return {"value": job_throughput(tokens, c.world, args.steps, e_ms), "unit": "tokens/s",
            "h2d_bytes_per_step": hx.numel() * 2 + hdt.numel() * 2,
            "d2h_bytes_per_step": hy.numel() * 2 + hh.numel() * 4,
            "ms_per_step": round(e_ms / args.steps, 4),
            "pipeline": "inputs and outputs double-buffered: step i+1's host-to-device copy overlaps "
                        "step i's compute and device-to-host copy"}


def bench_decode(c: Ctx, steps_total=16384, graph_steps=256):
    torch, ssd = c.torch, c.ssd
    steps_total = c.args.decode_steps or steps_total
    cfg = datagen.config(2)
    Bn, H, P = cfg["batch"], cfg["nheads"], cfg["headdim"]
    pcfg = dict(cfg, seqlen=c.args.decode_prefill_len or cfg["prefill_len"], norm_groups=0)
    pin = datagen.make_inputs(2, pcfg)
    dp = {k: ssd.to_device(pin[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    _, state, cache = ssd.prefill(pcfg, ssd.to_device(pin["xBC"]), ssd.to_device(pin["dt"]),
                                  dp["A"], dp["D"], dp["dt_bias"], dp["conv_w"])
    del pin
    torch.cuda.synchronize()
    torch.cuda.empty_cache()  # the 8192-token prefill at batch 64 used ~20 GB; give it back
    pool = {k: ssd.to_device(v) for k, v in datagen.decode_pool(cfg).items()}
    npool = pool["xBC"].shape[0]
    norm_w = torch.ones(H * P, dtype=torch.bfloat16, device=c.dev)
    caches = [cache, torch.empty_like(cache)]
    y = torch.empty((Bn, H * P), dtype=torch.bfloat16, device=c.dev)

    def run(n, offset=0):
        for s in range(n):
            i = (offset + s) % npool
            ssd.decode_step(cfg, pool["xBC"][i], pool["dt"][i], dp["A"], dp["D"], dp["dt_bias"],
                            dp["conv_w"], None, state, caches[s % 2], caches[(s + 1) % 2],
                            pool["z"][i], norm_w, y=y)

    run(8)
    torch.cuda.synchronize()
    # kernel-only timing of individual launches (traced)
    ssd.trace_enable(True)
    ssd.trace_read()
    run(64)
    torch.cuda.synchronize()
    ssd.trace_enable(False)
    recs = ssd.trace_read()
    kms = statistics.mean(ms for _, ms in recs)
    launches_per_step = len(recs) / 64
    # graph of graph_steps steps (even count: the cache ping-pong returns to buffer 0)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(2)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            run(graph_steps)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, steps_total // graph_steps)

    def replay_all():
        for _ in range(reps):
            g.replay()

    # the 256 MiB state stream exceeds L2 by itself: no flush needed
    ms, _, clocks = c.timed(replay_all, 1, flush=False, trace=False)
    del g
    nsteps = reps * graph_steps
    per_step_ms = ms / nsteps
    # A step is one kernel launch: its average duration over the timed region is the replayed
    # graph's time per launch (a CUDA event pair around each single launch adds a few us).
    kernel_ms = per_step_ms if launches_per_step == 1 else kms
    algo = decode_bytes(cfg)
    gbs = c.world * algo / (per_step_ms * 1e-3) / 1e9
    return {"metric": "decode state-update GB/s", "value": round(gbs, 1), "unit": "GB/s",
            "workload": "decode_16k", "steps": nsteps, "ms_per_step": round(per_step_ms, 5),
            "tokens_per_s": round(c.world * Bn / (per_step_ms * 1e-3), 1),
            "algorithmic_bytes_per_step": algo, "graph_steps": graph_steps, "clocks": clocks,
            "roofline": dict(hbm_roofline("ssd_decode", kernel_ms, algo, "decode_16k"),
                             kernel_timing="CUDA events around the timed graph replays, "
                                           f"{nsteps} launches back to back" if launches_per_step == 1
                                           else "CUDA events around each launch",
                             kernel_ms_single_launch_events=round(kms, 5))}


def bench_long_context(c: Ctx):
    """131072 tokens as 4 prefill calls of 32768 tokens; each call's final state and conv
    cache are the next call's initial state and cache (chunk 256, gated RMSNorm)."""
    torch, ssd, args = c.torch, c.ssd, c.args
    cfg = datagen.config(3)
    inp = datagen.make_inputs(3)
    d = {k: ssd.to_device(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    del inp
    Bn, L, H, P, N = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    nseg = cfg["segments"]
    Ls = L // nseg
    scfg = dict(cfg, seqlen=Ls)
    cd = datagen.conv_dim(cfg)
    y = torch.empty((Bn, L, H * P), dtype=torch.bfloat16, device=c.dev)
    states = [torch.empty((Bn, H, P, N), dtype=torch.float32, device=c.dev) for _ in range(2)]
    caches = [torch.empty((Bn, 4, cd), dtype=torch.bfloat16, device=c.dev) for _ in range(2)]
    ws = ssd.alloc_workspace(ssd.workspace_size(scfg), c.dev)

    def step():
        for s in range(nseg):
            sl = slice(s * Ls, (s + 1) * Ls)
            ssd.prefill(scfg, d["xBC"][:, sl], d["dt"][:, sl], d["A"], d["D"], d["dt_bias"],
                        d["conv_w"], None, d["z"][:, sl], d["norm_w"],
                        states[(s + 1) % 2] if s else None, caches[(s + 1) % 2] if s else None,
                        y=y[:, sl], h_final=states[s % 2], conv_state_out=caches[s % 2],
                        workspace=ws)

    for _ in range(args.warmup):
        step()
    # the 2.7 GB of xBC per step exceed L2 many times over: no flush needed
    total_ms, recs, clocks = c.timed(step, args.steps, flush=False)
    per, table, dom = kernel_table(recs)
    algo = scan_bytes(scfg, state_in=True) if dom.startswith("ssd_scan") else gated_norm_bytes(scfg)
    return {"metric": METRIC, "workload": "long_context_128k",
            "value": round(job_throughput(Bn * L, c.world, args.steps, total_ms), 1),
            "unit": "tokens/s", "ms_per_step": round(total_ms / args.steps, 4),
            "segments": nseg, "segment_len": Ls, "chunk": cfg["chunk"],
            "path_bytes_per_step": nseg * prefill_bytes(scfg, state_in=True),
            "gpu_launches": len(recs), "kernels": table, "clocks": clocks,
            "l2": "not flushed (inputs 2.7 GB per step)",
            "roofline": hbm_roofline(dom, statistics.mean(per[dom]), algo, "long_context_128k")}


def bench_mixer(c: Ctx):
    """mamba2_mixer_forward at the 12B width: B8 L8192 d_model 5120, 160 heads."""
    torch, ssd, args = c.torch, c.ssd, c.args
    cfg = dict(datagen.config(4), batch=args.mixer_batch)
    inp = datagen.make_inputs(4, cfg)
    d = {k: ssd.to_device(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    del inp
    Bn, L = cfg["batch"], cfg["seqlen"]
    out = torch.empty((Bn, L, cfg["d_model"]), dtype=torch.bfloat16, device=c.dev)
    ws = ssd.alloc_workspace(ssd.mixer_workspace_size(cfg), c.dev)

    def step():
        ssd.mixer_forward(cfg, d["hidden"], d["rms_w"], d["W_in"], d["W_out"], d["A"], d["D"],
                          d["dt_bias"], d["conv_w"], None, d["norm_w"], out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    total_ms, recs, clocks = c.timed(step, args.steps, flush=False)
    per, table, dom = kernel_table(recs)
    fl = mixer_flops(cfg)
    pk, src = peaks()
    sus, sus_src = pk.get("bf16_tflops_sustained"), src
    if not sus:
        sus, sus_src = FALLBACK_PEAKS["bf16_tflops_sustained"], "fallback"
    gemm_ms = statistics.mean(per["gemm_in_proj"])
    ach = fl["in_proj"] / (gemm_ms * 1e-3) / 1e12
    step_ms = total_ms / args.steps
    return {"metric": "mixer layer tokens/s", "workload": "mixer_12b", "batch": Bn,
            "value": round(job_throughput(Bn * L, c.world, args.steps, total_ms), 1),
            "unit": "tokens/s", "ms_per_step": round(step_ms, 4),
            "layer_tflops": round(sum(fl.values()) / (step_ms * 1e-3) / 1e12, 1),
            "flops_per_step": fl, "gpu_launches": len(recs), "kernels": table, "clocks": clocks,
            "l2": "not flushed (hidden 671 MB per step)",
            # the GEMM runs inside a long step under the power cap: the sustained peak is its
            # roof (the burst fraction is reported beside it)
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": sus,
                         "unit": "TFLOP/s", "frac": round(ach / sus, 4),
                         "frac_of_burst": round(ach / pk["bf16_tflops"], 4),
                         "traffic": recorded_traffic("gemm_tc_kernel", "mixer_12b_in_proj"),
                         "kernel": "gemm_in_proj (gemm_tc_kernel)", "kernel_ms": round(gemm_ms, 4),
                         "algorithmic_flops": fl["in_proj"],
                         "peak_source": f"{sus_src} cuBLAS bf16 (sustained, seconds-long loop under the power cap)"},
            "dominant_kernel": dom}


def bench_varlen(c: Ctx, nseq=128):
    """A packed batch of many short sequences (the 8k layer's shape: 128 heads, 8 groups), each
    with its own state and conv cache: ssd_prefill_varlen (one pass) against one ssd_prefill
    call per sequence on the same stream."""
    torch, ssd, args = c.torch, c.ssd, c.args
    rng = np.random.default_rng(datagen.SEED_BASE + 128)
    lens = rng.integers(64, 1025, nseq)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int)
    T = int(cu[-1])
    cfg = dict(datagen.config(1), batch=1, seqlen=T)
    inp = datagen.make_inputs(1, cfg)
    H, P, N, W = cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["conv_width"]
    d = {k: ssd.to_device(inp[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    x, dtt = ssd.to_device(inp["xBC"][0]), ssd.to_device(inp["dt"][0])
    del inp
    seed = datagen.SEED_BASE + 129
    h0 = ssd.to_device(datagen.random_state(seed, (nseq, H, P, N)))
    csi = ssd.to_device(datagen.random_conv_state(seed, (nseq, W, datagen.conv_dim(cfg))))

    vws = ssd.alloc_workspace(ssd.varlen_workspace_size(cfg, cu), c.dev)

    def one_pass():
        ssd.prefill_varlen(cfg, cu, x, dtt, d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None,
                           None, h0, csi, workspace=vws)

    def one_pass_no_state():
        ssd.prefill_varlen(cfg, cu, x, dtt, d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None,
                           None, h0, csi, workspace=vws, want_state=False)

    ws = ssd.alloc_workspace(max(ssd.workspace_size(dict(cfg, seqlen=int(L))) for L in lens), c.dev)

    def per_sequence():
        for i in range(nseq):
            a, b = int(cu[i]), int(cu[i + 1])
            ssd.prefill(dict(cfg, seqlen=b - a), x[None, a:b], dtt[None, a:b], d["A"], d["D"],
                        d["dt_bias"], d["conv_w"], None, None, None, h0[i:i + 1], csi[i:i + 1],
                        workspace=ws)

    res = {}
    for name, fn in (("one_pass", one_pass), ("one_pass_without_final_states", one_pass_no_state),
                     ("per_sequence_calls", per_sequence)):
        for _ in range(args.warmup):
            fn()
        ms, recs, _ = c.timed(fn, args.steps, flush=True, trace=(name == "one_pass"))
        res[name] = {"ms_per_step": round(ms / args.steps, 4),
                     "tokens_per_s": round(job_throughput(T, c.world, args.steps, ms), 1)}
        if name == "one_pass":
            res[name]["gpu_launches_per_step"] = len(recs) / args.steps
    return {"metric": METRIC, "workload": "varlen_128_short", "sequences": nseq, "tokens": T,
            "lengths": "uniform 64..1024 (seeded)", "value": res["one_pass"]["tokens_per_s"],
            "unit": "tokens/s", **res}


def summarize(rec):
    """The figures of a workload record that a reader needs first (None stays None)."""
    if not rec:
        return rec
    out = {k: rec[k] for k in ("workload", "metric", "value", "unit", "ms_per_step") if k in rec}
    rf = rec.get("roofline")
    if rf:
        out["roofline"] = {k: rf[k] for k in ("bound", "kernel", "kernel_ms", "achieved", "peak",
                                              "unit", "frac", "traffic") if k in rf}
    for k in ("layer_tflops", "tokens", "sequences"):
        if k in rec:
            out[k] = rec[k]
    for k in ("one_pass", "per_sequence_calls"):
        if k in rec:
            out[k] = rec[k]
    if "clocks" in rec:
        out["clocks"] = {k: rec["clocks"][k] for k in ("sm_mhz", "reasons") if k in rec["clocks"]}
    return out


def cpu_baseline(target_s: float = 10.0):
    """fp64 oracle on a bounded sample of the prefill workload (a token prefix of whole norm
    groups of heads), scaled to tokens/s of the whole layer."""
    import oracle
    o = oracle.get()
    cfg = datagen.config(1)
    inp = datagen.make_inputs(1)
    cores = os.cpu_count() or 1
    tok, groups, reps = 512, 1, 1
    hpg = cfg["nheads"] // cfg["ngroups"]
    while True:
        t0 = time.time()
        for _ in range(reps):
            ref = o.ssd_prefill(dict(cfg, seqlen=tok), inp["xBC"][:, :tok], inp["dt"][:, :tok],
                                inp["A"], inp["D"], inp["dt_bias"], conv_w=inp["conv_w"],
                                heads=(0, groups * hpg), threads=cores)
        dt = time.time() - t0
        if dt >= target_s:
            break
        grow = max(2.0, min(8.0, target_s / max(dt, 1e-3)))
        if tok < cfg["seqlen"]:
            tok = min(cfg["seqlen"], int(tok * grow))
        elif groups < cfg["ngroups"]:
            groups = min(cfg["ngroups"], int(groups * grow))
        else:
            reps = int(reps * grow) + 1
    frac = groups / cfg["ngroups"]
    # the same oracle on one thread, on a sample sized for a few seconds
    tok1 = max(64, min(tok, int(tok * 3.0 / max(dt / reps * cores, 1e-3))))
    t0 = time.time()
    o.ssd_prefill(dict(cfg, seqlen=tok1), inp["xBC"][:, :tok1], inp["dt"][:, :tok1], inp["A"], inp["D"],
                  inp["dt_bias"], conv_w=inp["conv_w"], heads=(0, hpg), threads=1)
    dt1 = time.time() - t0
    parity = sample_parity(cfg, inp, tok, groups * hpg, ref)
    return {"value": round(reps * tok * frac / dt, 2), "unit": "tokens/s", "cores": cores,
            "parity": parity,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"prefill_8k inputs, first {tok} tokens x heads 0-{groups * hpg - 1} "
                      f"({groups}/{cfg['ngroups']} of the layer) x {reps} run(s), fp64, "
                      f"{dt:.1f} s",
            "single_thread": {"value": round(tok1 / cfg["ngroups"] / dt1, 2), "unit": "tokens/s",
                              "cores": 1,
                              "sample": f"first {tok1} tokens x heads 0-{hpg - 1} (1/{cfg['ngroups']} "
                                        f"of the layer), fp64, {dt1:.1f} s"}}


def sample_parity(cfg, inp, tok, nh, ref):
    """The library's prefill on the oracle's timing sample (the first `tok` tokens of the
    prefill_8k inputs, all heads on the GPU) against the oracle's result for heads 0..nh-1:
    max|err|/RMS of y and h_final, and of y's error beyond its bf16 storage rounding."""
    import torch
    from mamba_ssd_scan_02_b200 import ssd
    c = dict(cfg, seqlen=tok)
    d = {k: ssd.to_device(np.ascontiguousarray(inp[k][:, :tok])) for k in ("xBC", "dt")}
    p = {k: ssd.to_device(inp[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    y, hf, _ = ssd.prefill(c, d["xBC"], d["dt"], p["A"], p["D"], p["dt_bias"], p["conv_w"])
    torch.cuda.synchronize()
    P = cfg["headdim"]
    yg = y.float().cpu().numpy()[:, :, :nh * P].astype(np.float64)
    yw = ref["y"].reshape(ref["y"].shape[0], ref["y"].shape[1], -1)
    hg = ssd.to_numpy(hf)[:, :nh].astype(np.float64)
    hw = ref["h_final"]
    rms_y, rms_h = float(np.sqrt(np.mean(yw * yw))), float(np.sqrt(np.mean(hw * hw)))
    return {"y_max_err_rms": float(np.max(np.abs(yg - yw)) / rms_y),
            "y_excess_over_bf16_rounding": float(np.max(np.abs(yg - yw) - 2.0 ** -8 * np.abs(yw)) / rms_y),
            "h_final_max_err_rms": float(np.max(np.abs(hg - hw)) / rms_h),
            "bound": 2e-2, "oracle": "fp64",
            "sample": f"prefill_8k inputs, first {tok} tokens x heads 0-{nh - 1}",
            "device_status": int(ssd.get_device_error())}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def reference_arm(args):
    """The fp64 oracle as the reference implementation, on bounded samples per step."""
    import oracle
    o = oracle.get()
    cfg = datagen.config(1)
    inp = datagen.make_inputs(1)
    cores = os.cpu_count() or 1
    heads = (0, 16)
    tok = 1024
    run = lambda: o.ssd_prefill(dict(cfg, seqlen=tok), inp["xBC"][:, :tok], inp["dt"][:, :tok],
                                inp["A"], inp["D"], inp["dt_bias"], conv_w=inp["conv_w"],
                                heads=heads, threads=cores)
    for _ in range(args.warmup):
        run()
    t0 = time.time()
    for _ in range(args.steps):
        run()
    el = time.time() - t0
    frac = (heads[1] - heads[0]) / cfg["nheads"]
    val = tok * frac * args.steps / el
    sample = f"per step: first {tok} tokens x heads 0-15 (1/8 of the layer) of prefill_8k, fp64"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(val, 2),
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(HEADLINE_CONFIG, parallelism=f"replicas x{args.gpus}"),
        "cpu_baseline": {"value": round(val, 2), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(val, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true",
                    help="headline prefill only (no decode, long-context, mixer or CPU legs)")
    ap.add_argument("--workload", choices=["all", "prefill", "decode", "long_context", "mixer", "varlen"],
                    default="all", help="run one workload alone (for profiling); prints its object")
    ap.add_argument("--mixer-batch", type=int, default=8,
                    help="batch of the mixer workload (smaller only for profiling captures)")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="decode steps timed (0: the workload's 16384; fewer only for profiling "
                         "captures)")
    ap.add_argument("--decode-prefill-len", type=int, default=0,
                    help="tokens of the prefill that gives the decode its starting state (0: the "
                         "workload's 8192; shorter only for profiling captures, whose device "
                         "memory it bounds)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            reference_arm(args)
        return

    import torch
    from mamba_ssd_scan_02_b200 import ssd
    torch.cuda.set_device(local_rank)
    ssd.load()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    clk = ClockSampler(smi_gpu_id(torch, local_rank)).start()
    c = Ctx(args, torch, ssd, dist, rank, world, clk)
    if args.workload != "all":
        fn = {"prefill": bench_prefill, "decode": bench_decode, "long_context": bench_long_context,
              "mixer": bench_mixer, "varlen": bench_varlen}[args.workload]
        try:
            r = fn(c)
            r["device_status"] = ssd.get_device_error()
        finally:
            clk.stop()
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"workload": args.workload, "result": r}))
        return
    try:
        res = bench_prefill(c)
        dec = lng = mix = vln = None
        if not args.quick:
            dec = bench_decode(c)
            torch.cuda.empty_cache()
            lng = bench_long_context(c)
            torch.cuda.empty_cache()
            mix = bench_mixer(c)
            torch.cuda.empty_cache()
            vln = bench_varlen(c)
        status = ssd.get_device_error()
    finally:
        clk.stop()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None if (args.quick or world > 1) else cpu_baseline()
    parity = cpu.pop("parity", None) if cpu else None  # the GPU path on the oracle's sample
    line = {
        "metric": METRIC, "value": round(res["value"], 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(res["ms_per_step"], 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(HEADLINE_CONFIG, parallelism=f"replicas x{world}"),
        "roofline": res["roofline"], "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
        "clocks": res["clocks"], "kernels": res["kernels"],
        "path_bytes_per_step": res["path_bytes_per_step"], "cpu_baseline": cpu, "parity": parity,
        "device_status": status,
    }
    # The other workloads: their full records on stderr, a short summary of each at the end
    # of the line (where a truncated tail of the output still shows them).
    detail = {"decode": dec, "long_context": lng, "mixer": mix, "varlen": vln}
    print(json.dumps({"detail": detail}), file=sys.stderr, flush=True)
    line.update({k: summarize(v) for k, v in detail.items()})
    print(json.dumps(line))


if __name__ == "__main__":
    main()
