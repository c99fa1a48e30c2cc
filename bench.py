#!/usr/bin/env python
"""Forward-pass throughput of the LSH-attention library on B200.

One step is one whole forward pass (hash, sort + gather, chunked attention,
un-sort + round merge) over the long-text workload: batch 1, 8 heads,
n = 65536, d = 128, 1024 buckets, chunk 64, 4 rounds, causal, bf16, seeded
synthetic inputs resident in HBM. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas: the forward pass has no exchange step); the time is
the max over ranks and the value counts every rank's tokens.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lsh_attention_b200 import binding as lb  # noqa: E402
from lsh_attention_b200 import inputs as I  # noqa: E402

METRIC = "LSH-attn fwd tokens/sec at n=64K, 4 rounds; % of HBM / tensor-pipe roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ("hash", "sort_gather", "chunk_attention", "unsort_merge")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=I.LONG_64K.name, choices=sorted(I.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# ----------------------------------------------------------------------------
# algorithmic bytes and flops per forward pass, per stage
def algorithmic(w: I.Workload) -> dict:
    E = 2 if w.dtype == "bf16" else 4
    T = w.batch * w.heads * w.n  # (token, head) units
    Rn = w.rounds
    X = T * w.d * E  # bytes of x (and of v)
    m = min(w.chunk, w.n)
    return {
        "hash": {"bytes": X + Rn * w.d * (w.n_buckets // 2) * E + 4 * T * Rn,
                 "flops": 2 * T * w.d * (w.n_buckets // 2) * Rn},
        "sort_gather": {"bytes": 4 * T * Rn + 2 * X * Rn + 2 * X * Rn + 8 * T * Rn, "flops": 0},
        "chunk_attention": {"bytes": 2 * X * Rn + 4 * T * Rn + T * Rn * w.d * 4 + 4 * T * Rn,
                            "flops": 8 * m * w.d * T * Rn},
        "unsort_merge": {"bytes": T * Rn * (4 * w.d + 8) + X, "flops": 0},
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while it runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", uuid], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, RuntimeError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.file.flush()
        self.file.seek(0)
        sm, smax, reasons = [], [], set()
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.file.name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
def dist_setup(backend: str):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(w: I.Workload, heads: int, threads: int):
    """Run the CPU oracle on `heads` heads of batch 0, all rounds, full length."""
    import oracle
    x, v = I.make_qkv(w.with_(batch=1))
    R = I.make_rotations(w)
    xs, vs = x[:, :heads].contiguous(), v[:, :heads].contiguous()
    t0 = time.perf_counter()
    oracle.forward(xs, vs, R, w.chunk, w.causal, nthreads=threads)
    return time.perf_counter() - t0


def cpu_baseline(w: I.Workload, min_seconds: float = 10.0) -> dict:
    cores = os.cpu_count() or 1
    heads = max(1, min(w.heads, cores // w.rounds))
    times = []
    while sum(times) < min_seconds and len(times) < 10:
        times.append(oracle_sample(w, heads, cores))
    t = statistics.mean(times)
    frac = heads / (w.heads * w.batch)
    return {"value": w.tokens * frac / t, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"C fp64 oracle, {heads} of {w.heads * w.batch} (batch, head) pairs, all "
                      f"{w.rounds} rounds, full n={w.n}, hash included; tokens counted as "
                      f"{frac:.4g} x B*n; mean of {len(times)} runs ({sum(times):.1f} s)"}


# ----------------------------------------------------------------------------
def run_reference(args, w):
    world, rank, _ = dist_setup("gloo")
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    heads = max(1, min(w.heads, cores // w.rounds))
    for _ in range(args.warmup):
        oracle_sample(w, heads, cores)
    times = [oracle_sample(w, heads, cores) for _ in range(args.steps)]
    t = statistics.mean(times)
    frac = heads / (w.heads * w.batch)
    value = w.tokens * frac / t
    sample = (f"C fp64 oracle per step: {heads} of {w.heads * w.batch} (batch, head) pairs, all "
              f"{w.rounds} rounds, full n={w.n}; tokens counted as {frac:.4g} x B*n")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def config_of(w):
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "n": w.n, "d_head": w.d,
            "n_buckets": w.n_buckets, "chunk": w.chunk, "rounds": w.rounds, "causal": w.causal,
            "clustered": w.clustered,
            "l2": "inputs larger than L2: x+v and the per-step workspace exceed 126 MB"}


def run_ours(args, w):
    world, rank, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lb.load()
    stream = torch.cuda.current_stream(dev)

    x_h, v_h = I.make_qkv(w)
    R_h = I.make_rotations(w)
    x, v, R = x_h.to(dev), v_h.to(dev), R_h.to(dev)
    out = torch.empty_like(x)
    lse = torch.empty((w.batch, w.heads, w.rounds, w.n), dtype=torch.float32, device=dev)
    desc = lb.make_desc(w.batch, w.heads, w.n, w.d, w.n_buckets, w.chunk, w.rounds, w.causal,
                        x.dtype)
    ws = lb.workspace(desc, dev)

    def fwd(events=None):
        lb.lsh_attn_forward(x, v, R, n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal,
                            out=out, lse=lse, ws=ws, events=events)

    def new_event():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)  # materialise the handle; the library re-records it
        return e

    K, W = args.steps, args.warmup
    ev = [[new_event() for _ in range(5)] for _ in range(K)]
    clocks = ClockSampler(local)
    for _ in range(W):
        fwd()
    torch.cuda.synchronize()
    status = lb.lsh_attn_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    # ---- device-resident timed region
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for k in range(K):
        fwd(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    local_ms = start.elapsed_time(end)
    total_ms = max_over_ranks(local_ms, world, dev)
    stage_ms = {}
    for i, name in enumerate(STAGES):
        stage_ms[name] = statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(K))
    value = world * w.tokens * K / (total_ms / 1e3)

    # ---- end to end through the public API: pinned host in, host out
    xp, vp, Rp = x_h.pin_memory(), v_h.pin_memory(), R_h.pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    K2 = max(3, min(K, 20))

    def e2e_step():
        x.copy_(xp, non_blocking=True)
        v.copy_(vp, non_blocking=True)
        R.copy_(Rp, non_blocking=True)
        fwd()
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(K2):
        e2e_step()
    e2.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (x_h, v_h, R_h))
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    if rank != 0:
        return
    alg = algorithmic(w)
    pk, pk_kind = peaks()
    dom = max(STAGES, key=lambda s: stage_ms[s])
    timed_s = total_ms / 1e3
    tensor_bound = {"hash": w.n_buckets // 2 >= 256, "chunk_attention": False}
    stages = {}
    for s in STAGES:
        t = stage_ms[s] / 1e3
        gbs = alg[s]["bytes"] / t / 1e9
        tfs = alg[s]["flops"] / t / 1e12
        stages[s] = {"ms": round(stage_ms[s], 4), "GB/s": round(gbs, 1),
                     "hbm_frac": round(gbs / pk["hbm_gbs"], 4),
                     "TFLOP/s": round(tfs, 2)}
    if tensor_bound.get(dom, False):
        peak = pk["bf16_tflops_sustained"] if timed_s > 1.0 else pk["bf16_tflops"]
        achieved = alg[dom]["flops"] / (stage_ms[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "unit": "TFLOP/s"}
    else:
        peak = pk["hbm_gbs"]
        achieved = alg[dom]["bytes"] / (stage_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "unit": "GB/s"}
    roof.update({"kernel": dom, "achieved": round(achieved, 2), "peak": peak,
                 "frac": round(achieved / peak, 4), "traffic": None,
                 "peak_source": f"{pk_kind} (MEASURED_PEAKS.json)" if pk_kind == "measured"
                 else "fallback"})
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1))",
        "config": config_of(w),
        "e2e": {"value": world * w.tokens * K2 / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K * launches_per_forward(buckets_given=False),
        "roofline": roof,
        "stages": stages,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


def launches_per_forward(buckets_given: bool) -> int:
    # hash (1) + sort: histogram, scan, rank/scatter/gather (3) + attention (1) + merge (1)
    return (0 if buckets_given else 1) + 3 + 1 + 1


def main():
    args = parse_args()
    w = I.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
