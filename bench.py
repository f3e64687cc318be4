"""Benchmark: paged fused inference attention on B200.

Headline workload (the metric's configuration): prefix-encoder prefill with a
causal mask over cached prefixes, B=4, new=[128,256,512,1024],
prefix=[0,512,1024,3072], H=32, KVH=8 (GQA), D=128, blockSize=128, bf16.
A step is one full fia_run (plan upload + prefill kernel) over that batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  value = TFLOP/s counting only unmasked
(query, key) pairs (4*D flops each), whole job; the decode workloads are
reported under "configs" (c1, c3, c4a/c4b, c5, each with its own roofline
fraction; c3 and c5 last) and the secondary workloads under "extra".  L2 is flushed (512 MiB
write) between timed steps.  Multi-GPU runs are independent replicas (the
path has no exchange step), reported as weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

_ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, _ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

SPEC_TFLOPS = 2250.0
SPEC_GBS = 8000.0


def measured_peaks():
    path = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return (float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m["bf16_tflops_sustained"]),
                "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def unmasked_pairs(p) -> int:
    """Sum over sequences and query heads of visible (query, key) pairs."""
    tot = 0
    for b in range(p.batch):
        ql, kl = int(p.seq_len[b]), int(p.kv_seq_len[b])
        if p.band is not None:
            # band: keys qpos - pre .. qpos + next, clipped to [0, kvSeqLen)
            qpos = np.arange(kl - ql, kl, dtype=np.int64)
            lo = np.maximum(0, qpos - p.band[0])
            hi = np.minimum(kl - 1, qpos + p.band[1])
            tot += int(np.maximum(0, hi - lo + 1).sum())
        elif p.mask_type in (W.MASK_CAUSAL, W.MASK_ALIBI):
            pre = kl - ql
            tot += ql * pre + ql * (ql + 1) // 2
        else:
            tot += ql * kl
    return tot * p.head_num


def flops(p) -> float:
    return 4.0 * p.head_size * unmasked_pairs(p)


def kv_bytes(p) -> int:
    """K+V bytes a decode pass must read once per KV head, plus the per-token
    dequantisation scales / offsets (fp32, one per cached token) once."""
    es = 1 if p.kv_is_int8 else 2
    tokens = int(sum(int(k) for k in p.kv_seq_len))
    per_token = 0
    if p.kv_is_int8:
        for mode, arrs in ((p.k_antiquant_mode, (p.k_scale, p.k_offset)),
                           (p.v_antiquant_mode, (p.v_scale, p.v_offset))):
            if mode == 1:
                per_token += tokens * 4 * sum(a is not None for a in arrs)
    return tokens * p.kv_head_num * p.head_size * es * 2 + per_token


def io_bytes(p) -> int:
    q = p.query.numel() * 2
    lse = p.n_tokens * p.head_num * 4
    return 2 * q + lse + p.block_tables.numel() * 4


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 20 ms from before the
    warm-up to after the timed region; each line is stamped with host time so
    the samples inside the timed window can be picked out."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def _parse(self, lines):
        sm, mx, reasons = [], None, set()
        for _, ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return sm, mx, reasons

    def summary(self):
        inside = self.lines
        scope = "timed region"
        if self.window is not None:
            t0, t1 = self.window
            inside = [x for x in self.lines if t0 <= x[0] <= t1 + 0.025]
            if not inside:
                inside = self.lines
                scope = "warm-up + timed region (timed region shorter than the 20 ms sample period)"
        sm, mx, reasons = self._parse(inside)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "scope": scope}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def to_dev(p, dev):
    d = lambda t: None if t is None else t.to(dev).contiguous()
    return dict(query=d(p.query), key=d(p.key_cache), value=d(p.value_cache),
                block_tables=d(p.block_tables), slopes=d(p.slopes), pse=d(p.pse), sink=d(p.sink),
                k_scale=d(p.k_scale), k_offset=d(p.k_offset), v_scale=d(p.v_scale),
                v_offset=d(p.v_offset))


def make_op(p, t):
    import paged_attention_02_b200 as fia
    return fia.FiaOp(t["query"], t["key"], t["value"], t["block_tables"],
                     [int(x) for x in p.seq_len], [int(x) for x in p.kv_seq_len], p.head_num,
                     p.kv_head_num, p.qk_scale, mask_type=p.mask_type, slopes=t["slopes"],
                     pse=t["pse"], sink=t["sink"], k_scale=t["k_scale"], k_offset=t["k_offset"],
                     v_scale=t["v_scale"], v_offset=t["v_offset"], want_lse=p.want_lse,
                     kv_layout=p.kv_layout, k_antiquant_mode=p.k_antiquant_mode,
                     v_antiquant_mode=p.v_antiquant_mode, band=p.band)


def time_op(op, steps, warmup, flush):
    """Per-step device times (ms) of fia_run and of its kernels alone, with
    an L2 flush between steps (outside the timed events)."""
    for _ in range(warmup):
        flush.zero_()
        op.run()
    torch.cuda.synchronize()
    run_ms, kern_ms = [], []
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b, ka, kb in evs:
        flush.zero_()
        op.set_timing_events(ka, kb)
        a.record()
        op.run()
        b.record()
    torch.cuda.synchronize()
    op.set_timing_events(None, None)
    for a, b, ka, kb in evs:
        run_ms.append(a.elapsed_time(b))
        kern_ms.append(ka.elapsed_time(kb))
    return run_ms, kern_ms


def time_e2e(p, steps, warmup, dev):
    """Same metric through the public API with HOST inputs: every step copies
    all of its inputs host->device (pinned), runs, and copies out + lse back.
    Two device buffer sets (each with its own op) and three streams let step
    i's upload, step i-1's run and step i-2's download overlap, as a serving
    loop would; events order the reuse of each set."""
    host = {k: (v.pin_memory() if v is not None else None) for k, v in
            dict(query=p.query, key=p.key_cache, value=p.value_cache,
                 block_tables=p.block_tables, slopes=p.slopes, pse=p.pse, sink=p.sink,
                 k_scale=p.k_scale, k_offset=p.k_offset, v_scale=p.v_scale,
                 v_offset=p.v_offset).items()}
    sets = []
    for _ in range(2):
        devt = {k: (torch.empty_like(v, device=dev) if v is not None else None)
                for k, v in host.items()}
        sets.append(dict(devt=devt, op=make_op(p, devt),
                         out_h=torch.empty_like(p.query).pin_memory(),
                         lse_h=torch.empty((p.n_tokens, p.head_num),
                                           dtype=torch.float32).pin_memory()))
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = sets[0]["out_h"].numel() * sets[0]["out_h"].element_size() + sets[0]["lse_h"].numel() * 4
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "run", "out")}
    for lst in ev.values():
        for e in lst:
            e.record(torch.cuda.current_stream(dev))

    def step(i):
        k = i % 2
        st = sets[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["run"][k])          # set k's last run has read its inputs
            for name, v in host.items():
                if v is not None:
                    st["devt"][name].copy_(v, non_blocking=True)
            ev["in"][k].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev["in"][k])
            s_run.wait_event(ev["out"][k])         # set k's last result has been read back
            out, lse = st["op"].run(s_run)
            ev["run"][k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][k])
            st["out_h"].copy_(out, non_blocking=True)
            st["lse_h"].copy_(lse, non_blocking=True)
            ev["out"][k].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    a.record(cur)
    for s in (s_in, s_run, s_out):
        s.wait_event(a)
    for i in range(steps):
        step(i)
    for s in (s_in, s_run, s_out):
        cur.wait_stream(s)
    b.record(cur)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps, h2d, d2h


def cpu_baseline(p, budget_s=12.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    rows of the same workload; returns (TFLOP/s-equivalent rate, cores, desc)."""
    import oracle
    cores = oracle.max_threads()
    rng = np.random.Generator(np.random.PCG64(123))
    cu = p.cu_seq()
    # rows are weighted by their visible keys; sample uniformly over (token, head)
    n = 64
    elapsed, done_flops, done_rows = 0.0, 0.0, 0
    while elapsed < budget_s and done_rows < p.n_tokens * p.head_num:
        rows = [(int(rng.integers(p.n_tokens)), int(rng.integers(p.head_num))) for _ in range(n)]
        t0 = time.perf_counter()
        oracle.attention(p, rows=rows, threads=cores)
        elapsed += time.perf_counter() - t0
        for t, _ in rows:
            b = int(np.searchsorted(cu, t, side="right") - 1)
            i = t - int(cu[b])
            kl, ql = int(p.kv_seq_len[b]), int(p.seq_len[b])
            vis = (kl - ql + i + 1) if p.mask_type in (W.MASK_CAUSAL, W.MASK_ALIBI) else kl
            done_flops += 4.0 * p.head_size * vis
        done_rows += n
        n = min(n * 2, 4096)
    return done_flops / elapsed / 1e12, cores, "%d sampled (token, head) rows, %.1f s" % (done_rows, elapsed)


# ---------------------------------------------------------------------------
# replicas: every rank runs the same workload on its own GPU; the job's time
# is the slowest rank's, its throughput all ranks' work over that time
# ---------------------------------------------------------------------------
def replica_max(vals, dist=None, dev=None):
    """Element-wise max of per-rank floats over all ranks (identity alone)."""
    if dist is None:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(world, flops_per_replica, ms):
    """TFLOP/s of the whole job: N replicas' flops over the slowest rank's ms."""
    return world * flops_per_replica / (ms * 1e-3) / 1e12


def reference_line(args, world):
    """The oracle timed as it stands on this host's cores: --warmup short
    untimed samples, then --steps samples that share --ref-seconds of work."""
    p = W.prefill_prefix()
    warm_s = min(1.0, args.ref_seconds / 10.0)
    step_s = max(0.2, args.ref_seconds / max(args.steps, 1))
    for _ in range(args.warmup):
        cpu_baseline(p, budget_s=warm_s)
    rates = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        r, cores, desc = cpu_baseline(p, budget_s=step_s)
        rates.append(r)
    val = statistics.mean(rates)
    return {"metric": "prefill attention TFLOP/s", "value": val, "unit": "TFLOP/s",
            "impl": "reference", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": p.name, "batch": 4, "seq_len": [128, 256, 512, 1024],
                       "prefix": [0, 512, 1024, 3072], "head_num": 32, "kv_head_num": 8,
                       "head_size": 128, "block_size": 128, "mask": "causal"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": time.perf_counter() - t_all}


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="reference arm: CPU seconds of oracle work spread over the timed steps")
    ap.add_argument("--profile", default=None, metavar="WORKLOAD",
                    help="run --warmup + --steps plain fia_run calls of one named workload "
                         "(%s) and exit: the command profiled by ncu" % ", ".join(W.NAMED))
    args = ap.parse_args()
    if not args.profile:
        args.warmup = max(args.warmup, 3)

    if args.profile:
        import paged_attention_02_b200  # noqa: F401
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        q = W.NAMED[args.profile]()
        op = make_op(q, to_dev(q, dev))
        for _ in range(args.warmup + args.steps):
            op.run()
        torch.cuda.synchronize()
        assert op.error_word() == 0
        print(json.dumps({"profile": args.profile, "launches": args.warmup + args.steps,
                          "plan": op.plan_info()}))
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle arm runs on rank 0 alone; the other ranks do no work and
        # join no process group
        if rank == 0:
            print(json.dumps(reference_line(args, world)), flush=True)
        return

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    hbm, tfl, tfl_sus, peak_src = measured_peaks()
    p = W.prefill_prefix()
    F = flops(p)

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import paged_attention_02_b200 as fia  # noqa: F401  (fails loudly without libfia.so)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    t = to_dev(p, dev)
    op = make_op(p, t)
    info = op.plan_info()
    with ClockSampler(local) as clk:
        clk.wait_first()
        # warm-up + timed steps, bracketed by barrier + synchronize
        for _ in range(args.warmup):
            flush.zero_()
            op.run()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t_start = time.time()
        run_ms, kern_ms = time_op(op, args.steps, 0, flush)
        torch.cuda.synchronize()
        clk.window = (t_start, time.time())
        if dist is not None:
            dist.barrier()
    ms, kms = replica_max([statistics.mean(run_ms), statistics.mean(kern_ms)], dist, dev)
    value = whole_job_rate(world, F, ms)
    achieved = F / (kms * 1e-3) / 1e12

    e2e_ms, h2d, d2h = time_e2e(p, max(3, args.steps // 4), 2, dev)
    (e2e_ms,) = replica_max([e2e_ms], dist, dev)
    e2e_val = whole_job_rate(world, F, e2e_ms)

    extra = {}
    if not args.no_extra:
        # the five named configurations are timed last and printed last (the
        # large-batch and int8 decodes at the very end of the line)
        for name, fn in (("decode_large_batch_bnnbsd", W.decode_large_batch_bnnbsd),
                         ("prefill_prefix_bnnbsd", W.prefill_prefix_bnnbsd),
                         ("mtp_decode", W.mtp_decode),
                         ("int8_per_token_decode", W.int8_per_token_decode),
                         ("sliding_window_prefill", W.sliding_window_prefill),
                         ("int8_prefix_prefill", W.int8_prefix_prefill),
                         ("int8_mtp_decode", W.int8_mtp_decode),
                         ("c1_tiny_decode", W.tiny_decode),
                         ("c4a_alibi_prefill", lambda: W.alibi_prefill(False)),
                         ("c4b_alibi_prefill_pse", lambda: W.alibi_prefill(True)),
                         ("c3_decode_large_batch", W.decode_large_batch),
                         ("c5_int8_long_decode", W.int8_long_decode)):
            q = fn()
            td = to_dev(q, dev)
            o2 = make_op(q, td)
            r2, k2 = time_op(o2, max(5, args.steps // 2), 3, flush)
            m2, km2 = statistics.mean(r2), statistics.mean(k2)
            ent = {"kernel_ms": round(km2, 5), "ms_per_call": round(m2, 5)}
            # decode shapes are bound by the cache read, whichever kernel runs
            # them (multi-token int8 decode with 24 rows per KV head takes the
            # tensor-core kernel)
            if o2.plan_info()["path"] == 1 or name.endswith("_decode"):
                byts = kv_bytes(q) + io_bytes(q)
                gbs = byts / (km2 * 1e-3) / 1e9
                ent.update({"value": round(gbs, 1), "unit": "GB/s", "bound": "hbm",
                            "frac": round(gbs / hbm, 4), "frac_of_spec": round(gbs / SPEC_GBS, 4),
                            "bytes": byts})
            else:
                f2 = flops(q)
                tf = f2 / (km2 * 1e-3) / 1e12
                ent.update({"value": round(tf, 1), "unit": "TFLOP/s", "bound": "tensor",
                            "frac": round(tf / tfl, 4), "frac_of_spec": round(tf / SPEC_TFLOPS, 4),
                            "flops": f2})
                if q.pse is not None:
                    pse_b = unmasked_pairs(q) * 2
                    floor_ms = max(f2 / (tfl * 1e9), (pse_b + kv_bytes(q)) / (hbm * 1e6))
                    ent["frac_of_floor"] = round(floor_ms / km2, 4)
            extra[name] = ent
            del o2, td

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc = cpu_baseline(p)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}

    traffic = None
    tr_path = os.path.join(_ROOT, "profiles", "traffic.json")
    if os.path.exists(tr_path):
        try:
            with open(tr_path) as f:
                traffic = json.load(f).get(p.name)
        except Exception:
            traffic = None

    line = {
        "metric": "prefill attention TFLOP/s", "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": p.name, "batch": 4, "seq_len": [128, 256, 512, 1024],
                   "prefix": [0, 512, 1024, 3072], "head_num": 32, "kv_head_num": 8,
                   "head_size": 128, "block_size": 128, "mask": "causal",
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "flushed between steps (512 MiB write)", "flops_per_step": F},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": tfl, "unit": "TFLOP/s",
                     "frac": achieved / tfl, "peak_source": peak_src + " burst bf16",
                     "frac_of_spec": achieved / SPEC_TFLOPS, "traffic": traffic,
                     "kernel_ms": kms},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * int(info["kernels_per_run"]),
        "plan": info,
        "clocks": clk.summary(),
        # secondary workloads, then the named configurations (c1..c5; c2 is
        # the headline above), each with its own roofline fraction
        "extra": {k: v for k, v in extra.items() if not k.startswith("c")},
        "configs": {k: v for k, v in extra.items() if k.startswith("c")},
    }
    if cpu is not None:
        # keep the named configurations at the end of the printed line
        configs = line.pop("configs")
        line["cpu_baseline"] = cpu
        line["configs"] = configs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
