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
# kernels between consecutive profiling events, and the stage each belongs to
KERNELS = lb.PROFILE_KERNELS
KERNEL_STAGE = {"hash_prep": "hash", "hash_mma": "hash", "hash_refine": "hash",
                "sort_hist": "sort_gather", "sort_scan": "sort_gather",
                "sort_rank": "sort_gather", "row_gather": "sort_gather",
                "chunk_attention": "chunk_attention",
                "unsort_merge": "unsort_merge"}
# the kernel that carries a stage's algorithmic work
STAGE_KERNEL = {"hash": "hash_mma", "sort_gather": "row_gather",
                "chunk_attention": "chunk_attention", "unsort_merge": "unsort_merge"}
# DRAM bytes (read + write) per launch from one ncu capture of the long-64k
# workload, valid only while the kernel's source file is unchanged (sha256
# of the file at capture time); see profiles/.
NCU_WORKLOAD = I.LONG_64K.name
NCU_TRAFFIC = {
    "hash_prep": {"bytes": 532000, "file": "hash_tc.cuh",
        "sha256": "37f57d7a8e89a1eeafa3c2e622f96c5a6d2ad920cdf54cb8c39cddab6f44948e"},
    "hash_mma": {"bytes": 150716200, "file": "hash_tc.cuh",
        "sha256": "37f57d7a8e89a1eeafa3c2e622f96c5a6d2ad920cdf54cb8c39cddab6f44948e"},
    "hash_refine": {"bytes": 2748000, "file": "hash_tc.cuh",
        "sha256": "37f57d7a8e89a1eeafa3c2e622f96c5a6d2ad920cdf54cb8c39cddab6f44948e"},
    "sort_scan": {"bytes": 4204000, "file": "sort.cuh",
        "sha256": "e031792086f8fef697f441014adf16e9a9b36d922f1a623610bc2e5e46c4b5ab"},
    "sort_rank": {"bytes": 12598000, "file": "sort.cuh",
        "sha256": "e031792086f8fef697f441014adf16e9a9b36d922f1a623610bc2e5e46c4b5ab"},
    "row_gather": {"bytes": 1513671000, "file": "gather.cuh",
        "sha256": "e6ed6996ab9b55d7b4ab341085d7fa0a4c9c38b1532727b5bb8fad26bde2238a"},
    "chunk_attention": {"bytes": 1656132536, "file": "attn_tc.cuh",
        "sha256": "ef34b0f22a208e36832902dd14b8d51dc86fdddd67df14426033343ba0d3c0df"},
    "unsort_merge": {"bytes": 672942000, "file": "merge.cuh",
        "sha256": "f313dd4622da3353060cb7b84324a099bfef2be35a4e693135b8674f34cd17db"},
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=I.LONG_64K.name, choices=sorted(I.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--ref-seconds", type=float, default=120.0,
                   help="reference arm: seconds that warm-up plus timed steps should take")
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
        # the row gather, which carries the stage: perm in, x and v once per
        # (batch, head) (the rounds share them through L2), xs and vs rows
        # out, 1/||x|| out (ranks and histograms: ~1% more)
        "sort_gather": {"bytes": 4 * T * Rn + 2 * X + 2 * X * Rn + 4 * T * Rn, "flops": 0},
        "chunk_attention": {"bytes": 2 * X * Rn + 4 * T * Rn + T * Rn * w.d * E + 4 * T * Rn,
                            "flops": 8 * m * w.d * T * Rn},
        "unsort_merge": {"bytes": T * Rn * (E * w.d + 8) + X, "flops": 0},
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML every 20 ms
    in a background thread; only samples inside [start(), stop()) count."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index: int):
        import threading
        self.samples, self.window, self.handle = [], None, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
        except Exception:  # no NVML on this host: report no samples
            self.handle = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            self._stop.wait(0.02)

    def start(self):
        self.t0 = time.perf_counter()

    def stop(self) -> dict:
        t1 = time.perf_counter()
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "unavailable"}
        self._stop.set()
        self.thread.join(timeout=2)
        inside = [(m, r) for (t, m, r) in self.samples if self.t0 <= t < t1]
        reasons = sorted({name for (_, r) in inside for name, bit in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in inside) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "source": "NVML every 20 ms during the timed region"}


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
    """The oracle on the host cores, as the reference arm: each step runs the
    C fp64 oracle (hash, sort, chunk attention, merge) on `hs` heads x `rs`
    rounds of batch 0 over the first `n_s` positions, one OpenMP thread per
    (head, round) unit; n_s is calibrated so warm-up plus steps take about two
    minutes (--ref-seconds). Tokens are counted pro rata: B*n * (n_s/n) * (hs/H) * (rs/R)."""
    world, rank, _ = dist_setup("gloo")
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    x, v = I.make_qkv(w.with_(batch=1))
    R = I.make_rotations(w)
    rs = min(w.rounds, cores)
    hs = max(1, min(w.heads, cores // rs))
    m = min(w.chunk, w.n)

    def step(n_s):
        xs = x[:, :hs, :n_s].contiguous()
        vs = v[:, :hs, :n_s].contiguous()
        t0 = time.perf_counter()
        oracle.forward(xs, vs, R[:rs], m, w.causal, nthreads=hs * rs)
        return time.perf_counter() - t0

    budget = args.ref_seconds / max(1, args.steps + args.warmup)  # seconds per step
    n_s = min(w.n, 4096)
    t0 = step(n_s)  # calibration
    n_s = int(min(w.n, max(m, (n_s * budget / max(t0, 1e-3)) // m * m)))
    for _ in range(args.warmup):
        step(n_s)
    times = [step(n_s) for _ in range(args.steps)]
    t = statistics.mean(times)
    frac = (n_s / w.n) * (hs / w.heads) * (rs / w.rounds) / w.batch
    value = w.tokens * frac / t
    sample = (f"C fp64 oracle per step: {hs} of {w.heads * w.batch} (batch, head) pairs x {rs} "
              f"of {w.rounds} rounds over the first {n_s} of n={w.n} positions, "
              f"{hs * rs} threads; tokens counted as {frac:.4g} x B*n")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": hs * rs, "kind": "oracle",
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
    NE = lb.PROFILE_EVENTS
    ev = [[new_event() for _ in range(NE)] for _ in range(K)]
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
    clocks.start()
    start.record(stream)
    for k in range(K):
        fwd(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    local_ms = start.elapsed_time(end)
    total_ms = max_over_ranks(local_ms, world, dev)
    kernel_ms = {}
    for i, name in enumerate(KERNELS):
        kernel_ms[name] = statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(K))
    stage_ms = {st: sum(t for kn, t in kernel_ms.items() if KERNEL_STAGE[kn] == st)
                for st in STAGES}
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
    timed_s = total_ms / 1e3
    stages = {}
    for st in STAGES:
        t = stage_ms[st] / 1e3
        stages[st] = {"ms": round(stage_ms[st], 4),
                      "GB/s": round(alg[st]["bytes"] / t / 1e9, 1),
                      "hbm_frac": round(alg[st]["bytes"] / t / 1e9 / pk["hbm_gbs"], 4),
                      "TFLOP/s": round(alg[st]["flops"] / t / 1e12, 2)}
    kernels = {kn: round(t, 4) for kn, t in kernel_ms.items()}
    # roofline of the dominant kernel, against its own launch time
    dom = max(KERNELS, key=lambda kn: kernel_ms[kn])
    dst = KERNEL_STAGE[dom]
    dsec = kernel_ms[dom] / 1e3
    carries = STAGE_KERNEL[dst] == dom
    tensor = dst in ("hash", "chunk_attention") and alg[dst]["flops"] / max(1, alg[dst]["bytes"]) > \
        1e3 * pk["bf16_tflops"] / pk["hbm_gbs"]
    if carries and tensor:
        peak = pk["bf16_tflops_sustained"] if timed_s > 1.0 else pk["bf16_tflops"]
        roof = {"bound": "tensor", "unit": "TFLOP/s",
                "achieved": round(alg[dst]["flops"] / dsec / 1e12, 2), "peak": peak}
    else:
        roof = {"bound": "hbm", "unit": "GB/s",
                "achieved": round((alg[dst]["bytes"] if carries else 0) / dsec / 1e9, 1),
                "peak": pk["hbm_gbs"]}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["kernel"] = dom
    roof["traffic"] = traffic_of(dom, w.name)
    roof["peak_source"] = "of measured (MEASURED_PEAKS.json)" if pk_kind == "measured" else \
        "of fallback"
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
        "kernels_ms": kernels,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


def launches_per_forward(buckets_given: bool) -> int:
    # hash: rotation transpose, projection/argmax (which also counts the sort's
    # histograms), fp64 re-decision (3); sort: histogram (caller buckets only),
    # scan, ranks, row gather; attention (1); merge (1)
    return (4 if buckets_given else 3 + 3) + 1 + 1


def traffic_of(kernel: str, workload: str):
    """ncu DRAM bytes per launch of `kernel`, if the capture was of this
    workload and the kernel's source is unchanged since."""
    import hashlib
    rec = NCU_TRAFFIC.get(kernel)
    if rec is None or workload != NCU_WORKLOAD:
        return None
    path = os.path.join(ROOT, "lsh_attention_b200", "csrc", rec["file"])
    with open(path, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
            return None
    return rec["bytes"]


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
