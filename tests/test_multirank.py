"""The N>1 path on CPU: two gloo ranks.

The attention path has no exchange step, so a multi-GPU run is N independent
replicas: each rank times its own copy of the workload, the job's time is the
slowest rank's (a MAX all-reduce), and its throughput is all ranks' work over
that time.  These tests run that host logic as real world-size-2 process
groups over gloo, and run the reference arm under torchrun with two ranks
(rank 0 alone works and prints; the other exits 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        # per-rank step times that differ in each slot, so a sum, a min or a
        # rank-0 shortcut would all give a different answer than the max
        mine = [1.0 + rank, 10.0 - rank, 0.25 * (rank + 1)]
        got = bench.replica_max(mine, dist, "cpu")
        rate = bench.whole_job_rate(world, 2.0e12, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_replica_max_and_whole_job_rate_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_replica_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r, got, rate = q.get(timeout=120)
            res[r] = (got, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in range(world):
        got, rate = res[r]
        assert got == [2.0, 10.0, 0.5]                  # every rank sees the slowest rank
        # 2 replicas x 2e12 flops over the slowest rank's 2 ms = 2000 TFLOP/s
        assert rate == pytest.approx(2000.0)


def test_replica_max_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.replica_max([3.5, 1.25]) == [3.5, 1.25]
    assert bench.whole_job_rate(1, 1.0e12, 1.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "3", "--ref-seconds", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout                    # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("prefill_prefix")
