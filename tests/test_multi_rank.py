"""The benchmark's multi-process accounting on CPU: two gloo ranks, each an independent
replica (the path has no exchange step), the job timed as the slowest rank."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        t = bench.max_over_ranks(torch, dist, ms, "cpu")
        out[rank] = (t, bench.job_throughput(8192, world, 4, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 replicas x 8192 tokens x 4 steps in 15 ms
    assert res[0][1] == pytest.approx(2 * 8192 * 4 / 15e-3)


def test_single_process_is_the_identity():
    import torch
    import bench
    assert bench.max_over_ranks(torch, None, 3.5, "cpu") == 3.5
    assert bench.job_throughput(100, 1, 10, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` launched as 2 ranks: rank 0 alone times the oracle and
    prints one JSON line; the other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_kernel_table_keeps_side_stream_kernels_off_the_critical_path():
    """A kernel the library runs on its side stream (concurrently with the scan) is listed but
    takes no share of the step and is never the dominant kernel, even when its own traced
    time is the largest."""
    import bench
    recs = [("ssd_front", 0.03), ("ssd_state_tail", 0.5), ("ssd_scan_tc", 0.2), ("ssd_tail_fold", 0.01)] * 2
    per, table, dom = bench.kernel_table(recs)
    assert dom == "ssd_scan_tc"
    assert table["ssd_state_tail"]["share"] is None and "overlapped" in table["ssd_state_tail"]
    assert table["ssd_scan_tc"]["share"] == pytest.approx(0.2 / 0.24, abs=1e-4)
    assert sum(r["share"] for r in table.values() if r["share"] is not None) == pytest.approx(1.0, abs=1e-3)
