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
  - "decode": the 16384-step decode workload (B64 H128, fp32 state of 256 MiB), state-update
    GB/s with the steps replayed from CUDA graphs;
  - "cpu_baseline": the fp64 oracle timed on a bounded sample of the prefill workload.
Multi-GPU (torchrun): one process per GPU, each an independent replica (weak scaling), time
= max over ranks.  --impl reference times the fp64 CPU oracle on the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mamba_ssd_scan_02_b200 import datagen  # noqa: E402

L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------------------------
# algorithmic byte counts (each required input once, each output once, state in/out once)
def prefill_bytes(cfg) -> int:
    Bn, L, H, P, N, G = (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                         cfg["ngroups"])
    e = 2 if cfg["dtype"] == "bf16" else 4
    cd = datagen.conv_dim(cfg)
    d_inner = H * P
    b = Bn * L * (cd + H) * e          # xBC + dt
    b += Bn * L * d_inner * e          # y
    if cfg.get("norm_groups"):
        b += Bn * L * d_inner * e      # z
    b += Bn * H * P * N * 4            # final state out
    b += cd * cfg["conv_width"] * e + 3 * H * 4  # parameters
    b += Bn * cfg["conv_width"] * cd * e  # conv cache out
    return b


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


# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
def bench_prefill(args, rank, world, torch, ssd, dist):
    cfg = datagen.config(1)
    inp = datagen.make_inputs(1)
    dev = torch.device("cuda")
    d = {k: ssd.to_device(v) for k, v in inp.items() if isinstance(v, np.ndarray)}
    Bn, L, H, P, N = cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    y = torch.empty((Bn, L, H * P), dtype=torch.bfloat16, device=dev)
    hf = torch.empty((Bn, H, P, N), dtype=torch.float32, device=dev)
    cso = torch.empty((Bn, 4, datagen.conv_dim(cfg)), dtype=torch.bfloat16, device=dev)
    ws = ssd.alloc_workspace(ssd.workspace_size(cfg), dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ssd.prefill(cfg, d["xBC"], d["dt"], d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None,
                    None, None, None, y=y, h_final=hf, conv_state_out=cso, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ssd.trace_enable(True)
    ssd.trace_read()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))            # evict the previous step's data from L2
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ssd.trace_enable(False)
    recs = ssd.trace_read()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = float(sum(step_ms))
    if dist:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    # dominant kernel: largest total traced time
    per = {}
    for name, ms in recs:
        per.setdefault(name, []).append(ms)
    dom = max(per, key=lambda k: sum(per[k]))
    dom_ms = statistics.mean(per[dom])
    pk, pk_src = peaks()
    algo = prefill_bytes(cfg)
    achieved = algo / (dom_ms * 1e-3) / 1e9
    tokens = Bn * L
    res = {
        "value": world * tokens * args.steps / (total_ms * 1e-3),
        "ms_per_step": total_ms / args.steps,
        "gpu_launches": len(recs),
        "clocks": clk.summary(),
        "kernels": {k: {"launches": len(v), "mean_ms": round(statistics.mean(v), 5),
                        "share": round(sum(v) / sum(sum(x) for x in per.values()), 4)}
                    for k, v in per.items()},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": None,
                     "kernel": dom, "kernel_ms": round(dom_ms, 5), "algorithmic_bytes": algo,
                     "peak_source": pk_src},
    }
    # end to end: pinned host inputs in, results out, inside the timed region
    hx = torch.empty(d["xBC"].shape, dtype=torch.bfloat16, pin_memory=True)
    hx.copy_(d["xBC"].cpu())
    hdt = torch.empty(d["dt"].shape, dtype=torch.bfloat16, pin_memory=True)
    hdt.copy_(d["dt"].cpu())
    hy = torch.empty(y.shape, dtype=torch.bfloat16, pin_memory=True)
    hh = torch.empty(hf.shape, dtype=torch.float32, pin_memory=True)
    xdev = torch.empty_like(d["xBC"])
    dtdev = torch.empty_like(d["dt"])

    def e2e_step():
        xdev.copy_(hx, non_blocking=True)
        dtdev.copy_(hdt, non_blocking=True)
        ssd.prefill(cfg, xdev, dtdev, d["A"], d["D"], d["dt_bias"], d["conv_w"], None, None, None,
                    None, None, y=y, h_final=hf, conv_state_out=cso, workspace=ws)
        hy.copy_(y, non_blocking=True)
        hh.copy_(hf, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(float(i))
        e2[i][0].record(stream)
        e2e_step()
        e2[i][1].record(stream)
    torch.cuda.synchronize()
    e_ms = sum(a.elapsed_time(b) for a, b in e2)
    if dist:
        t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_ms = float(t.item())
    res["e2e"] = {"value": world * tokens * args.steps / (e_ms * 1e-3), "unit": "tokens/s",
                  "h2d_bytes_per_step": hx.numel() * 2 + hdt.numel() * 2,
                  "d2h_bytes_per_step": hy.numel() * 2 + hh.numel() * 4}
    return res


def bench_decode(args, rank, world, torch, ssd, dist, steps_total=16384, graph_steps=256):
    cfg = datagen.config(2)
    Bn, H, P, N = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]
    dev = torch.device("cuda")
    pcfg = dict(cfg, seqlen=cfg["prefill_len"], norm_groups=0)
    pin = datagen.make_inputs(2, pcfg)
    dp = {k: ssd.to_device(pin[k]) for k in ("A", "D", "dt_bias", "conv_w")}
    _, state, cache = ssd.prefill(pcfg, ssd.to_device(pin["xBC"]), ssd.to_device(pin["dt"]),
                                  dp["A"], dp["D"], dp["dt_bias"], dp["conv_w"])
    del pin
    pool = {k: ssd.to_device(v) for k, v in datagen.decode_pool(cfg).items()}
    npool = pool["xBC"].shape[0]
    norm_w = torch.ones(H * P, dtype=torch.bfloat16, device=dev)
    caches = [cache, torch.empty_like(cache)]
    y = torch.empty((Bn, H * P), dtype=torch.bfloat16, device=dev)

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
    kms = statistics.mean(ms for _, ms in ssd.trace_read())
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
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if dist:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    del g
    nsteps = reps * graph_steps
    per_step_ms = ms / nsteps
    algo = decode_bytes(cfg)
    pk, pk_src = peaks()
    gbs = world * algo / (per_step_ms * 1e-3) / 1e9
    kach = algo / (kms * 1e-3) / 1e9
    return {"metric": "decode state-update GB/s", "value": round(gbs, 1), "unit": "GB/s",
            "steps": nsteps, "ms_per_step": round(per_step_ms, 5),
            "tokens_per_s": round(world * Bn / (per_step_ms * 1e-3), 1),
            "algorithmic_bytes_per_step": algo, "graph_steps": graph_steps,
            "roofline": {"bound": "hbm", "achieved": round(kach, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(kach / pk["hbm_gbs"], 4), "traffic": None,
                         "kernel": "ssd_decode", "kernel_ms": round(kms, 5), "peak_source": pk_src}}


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
            o.ssd_prefill(dict(cfg, seqlen=tok), inp["xBC"][:, :tok], inp["dt"][:, :tok],
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
    return {"value": round(reps * tok * frac / dt, 2), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"prefill_8k inputs, first {tok} tokens x heads 0-{groups * hpg - 1} "
                      f"({groups}/{cfg['ngroups']} of the layer) x {reps} run(s), fp64, "
                      f"{dt:.1f} s"}


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
        "impl": "reference", "metric": "SSD prefill tokens/s/layer", "value": round(val, 2),
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_8k", "batch": 1, "seqlen": 8192, "nheads": 128,
                   "headdim": 64, "dstate": 128, "ngroups": 8, "chunk": 128},
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
    ap.add_argument("--quick", action="store_true", help="skip the decode and CPU-baseline legs")
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
    res = bench_prefill(args, rank, world, torch, ssd, dist)
    dec = None if args.quick else bench_decode(args, rank, world, torch, ssd, dist)
    status = ssd.get_device_error()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None if args.quick else cpu_baseline()
    line = {
        "metric": "SSD prefill tokens/s/layer", "value": round(res["value"], 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(res["ms_per_step"], 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "prefill_8k", "batch": 1, "seqlen": 8192, "nheads": 128,
                   "headdim": 64, "dstate": 128, "ngroups": 8, "chunk": 128, "conv_width": 4,
                   "state_dtype": "f32", "l2": "flushed between timed steps (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "roofline": res["roofline"], "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
        "clocks": res["clocks"], "kernels": res["kernels"], "decode": dec, "cpu_baseline": cpu,
        "device_status": status,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
