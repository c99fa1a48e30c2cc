#!/usr/bin/env python
"""Forward-pass throughput of the LSH-attention library on B200.

One step is one whole forward pass (hash, sort, chunked attention with the
rows read by the sort's permutation, un-sort + round merge) over the
long-text workload: batch 1, 8 heads, n = 65536, d = 128, 1024 buckets,
chunk 64, 4 rounds, causal, bf16, seeded synthetic inputs resident in HBM.
Prints one JSON line (rank 0), which also carries a block per other workload
(image-shaped, short bf16, two sweep points) measured the same way.

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
STAGES = ("hash", "sort", "chunk_attention", "unsort_merge")
# kernels between consecutive profiling events, and the stage each belongs to
KERNELS = lb.PROFILE_KERNELS
KERNEL_STAGE = {"hash_prep": "hash", "hash_mma": "hash", "hash_refine": "hash",
                "sort_hist": "sort", "sort_scan": "sort", "sort_rank": "sort",
                "gather_or_norm": "chunk_attention", "chunk_attention": "chunk_attention",
                "unsort_merge": "unsort_merge"}
# the kernel that carries a stage's algorithmic work
STAGE_KERNEL = {"hash": "hash_mma", "sort": "sort_rank",
                "chunk_attention": "chunk_attention", "unsort_merge": "unsort_merge"}
# other workloads measured in the same run (one block each in the JSON line)
EXTRA_WORKLOADS = ("image-12k", "bf16-short", "sweep-n131072-r8-iso", "sweep-n2048-r1-iso")
# DRAM bytes (read + write) per launch from one ncu capture of the long-64k
# workload, valid only while the kernel's source file is unchanged (sha256
# of the file at capture time); see profiles/.
NCU_WORKLOAD = I.LONG_64K.name
NCU_TRAFFIC: dict = {
    "hash_mma": {"file": "hash_tc.cuh", "bytes": 150568448,
                 "sha256": "12d5a1b8c7fa8d801e4068aa78d84d763a93a54e65660f0779ff448a785ab33d"},
    "chunk_attention": {"file": "attn_tc.cuh", "bytes": 839529728,
                 "sha256": "d9137349f2a4744965edacb7179a784ccd709fedbc7c1c0817532d3ace81986e"},
    "unsort_merge": {"file": "merge.cuh", "bytes": 673624320,
                 "sha256": "f313dd4622da3353060cb7b84324a099bfef2be35a4e693135b8674f34cd17db"},
    "hash_refine": {"file": "hash_tc.cuh", "bytes": 1661184,
                 "sha256": "12d5a1b8c7fa8d801e4068aa78d84d763a93a54e65660f0779ff448a785ab33d"},
    "sort_rank": {"file": "sort.cuh", "bytes": 12597760,
                 "sha256": "e031792086f8fef697f441014adf16e9a9b36d922f1a623610bc2e5e46c4b5ab"},
    "hash_prep": {"file": "hash_tc.cuh", "bytes": 533760,
                 "sha256": "12d5a1b8c7fa8d801e4068aa78d84d763a93a54e65660f0779ff448a785ab33d"},
    "sort_scan": {"file": "sort.cuh", "bytes": 4203776,
                 "sha256": "e031792086f8fef697f441014adf16e9a9b36d922f1a623610bc2e5e46c4b5ab"},
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=I.LONG_64K.name, choices=sorted(I.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the other workloads' blocks")
    p.add_argument("--ref-seconds", type=float, default=120.0,
                   help="reference arm: seconds that warm-up plus timed steps should take")
    return p.parse_args()


# ----------------------------------------------------------------------------
# algorithmic bytes and flops per forward pass, per stage
def algorithmic(w: I.Workload) -> dict:
    """Bytes each stage must move and flops it must do, as the method is
    specified (T = B*H*n (token, head) units, R rounds, X = bytes of x)."""
    E = 2 if w.dtype == "bf16" else 4
    T = w.batch * w.heads * w.n  # (token, head) units
    Rn = w.rounds
    X = T * w.d * E  # bytes of x (and of v)
    m = min(w.chunk, w.n)
    return {
        # x once, R, bucket ids out, 1/||x|| out (by position)
        "hash": {"bytes": X + Rn * w.d * (w.n_buckets // 2) * E + 4 * T * Rn + 4 * T,
                 "flops": 2 * T * w.d * (w.n_buckets // 2) * Rn},
        # ranks, which carry the stage: bucket ids in, perm and inv out
        "sort": {"bytes": 4 * T * Rn + 8 * T * Rn, "flops": 0},
        # rows of x and v read by perm: every round reads every row, but a
        # row need come from HBM only once (the rounds of a (batch, head) run
        # together); perm and key scales in; each round's output (input type)
        # and lse out. Flops: m queries against 2m keys, QK^T and PV.
        "chunk_attention": {"bytes": 2 * X + 4 * T + 4 * T * Rn + T * Rn * w.d * E + 4 * T * Rn,
                            "flops": 8 * m * w.d * T * Rn},
        # every round's row (input type) and (lse, slot), one output row
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
    """SM clock and clock-event (throttle) reasons read through NVML every 2 ms
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
            self._stop.wait(0.002)

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
                "source": "NVML every 2 ms during the timed region"}


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


def new_event(stream):
    e = torch.cuda.Event(enable_timing=True)
    e.record(stream)  # materialise the handle; the library re-records it
    return e


def measure(w: I.Workload, dev, K: int, W: int, world: int = 1, clocks=None) -> dict:
    """Time K forward passes (after W untimed ones) on device-resident seeded
    inputs, with CUDA events on the launching stream around the whole run and
    at every kernel boundary of every pass (lsh_attn_forward_profiled)."""
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

    NE = lb.PROFILE_EVENTS
    ev = [[new_event(stream) for _ in range(NE)] for _ in range(K)]
    for _ in range(W):
        fwd()
    torch.cuda.synchronize()
    status = lb.lsh_attn_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status} after warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
    start.record(stream)
    for k in range(K):
        fwd(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks is not None else None
    if lb.lsh_attn_get_device_status(ws) != 0:
        raise RuntimeError(f"{w.name}: device status after the timed passes")
    total_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    kernel_ms = {name: statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(K))
                 for i, name in enumerate(KERNELS)}
    return {"w": w, "total_ms": total_ms, "K": K, "kernel_ms": kernel_ms, "clocks": clk,
            "host": (x_h, v_h, R_h), "dev": (x, v, R, out, lse), "fwd": fwd}


def roofline_block(w: I.Workload, kernel_ms: dict, timed_s: float) -> tuple[dict, dict]:
    """Per-stage achieved rates, and the roofline of the dominant kernel
    against its own mean launch time."""
    alg = algorithmic(w)
    pk, pk_kind = peaks()
    stage_ms = {st: sum(t for kn, t in kernel_ms.items() if KERNEL_STAGE[kn] == st)
                for st in STAGES}
    stages = {}
    for st in STAGES:
        t = max(stage_ms[st], 1e-9) / 1e3
        stages[st] = {"ms": round(stage_ms[st], 4),
                      "GB/s": round(alg[st]["bytes"] / t / 1e9, 1),
                      "hbm_frac": round(alg[st]["bytes"] / t / 1e9 / pk["hbm_gbs"], 4),
                      "TFLOP/s": round(alg[st]["flops"] / t / 1e12, 2)}
    dom = max(KERNELS, key=lambda kn: kernel_ms[kn])
    dst = KERNEL_STAGE[dom]
    dsec = kernel_ms[dom] / 1e3
    carries = STAGE_KERNEL[dst] == dom
    tensor = dst in ("hash", "chunk_attention") and \
        alg[dst]["flops"] / max(1, alg[dst]["bytes"]) > 1e3 * pk["bf16_tflops"] / pk["hbm_gbs"]
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
    if "chunk_attention" in kernel_ms and kernel_ms["chunk_attention"] > 0:
        t = kernel_ms["chunk_attention"] / 1e3
        stages["chunk_attention"]["tensor_frac"] = round(
            alg["chunk_attention"]["flops"] / t / 1e12 / pk["bf16_tflops"], 4)
    return stages, roof


def e2e_overlapped(m: dict, dev, K2: int, world: int) -> tuple[float, int, int]:
    """The same forward through the public API with every step's inputs
    copied in from pinned host memory and its outputs read back, each step's
    copies overlapping the neighbouring steps' compute: inputs and outputs are
    double-buffered on the device, the host->device copies run on one stream,
    the forward on another and the device->host copies on a third, ordered
    by events. Returns (ms for K2 steps, h2d bytes per step, d2h bytes per step)."""
    w = m["w"]
    x_h, v_h, R_h = m["host"]
    xp, vp, Rp = x_h.pin_memory(), v_h.pin_memory(), R_h.pin_memory()
    x0, v0, R0, out0, lse0 = m["dev"]
    slots = [(x0, v0, R0, out0, lse0),
             (torch.empty_like(x0), torch.empty_like(v0), torch.empty_like(R0),
              torch.empty_like(out0), torch.empty_like(lse0))]
    outs_h = [(torch.empty(out0.shape, dtype=out0.dtype, pin_memory=True),
               torch.empty(lse0.shape, dtype=lse0.dtype, pin_memory=True)) for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    desc = lb.make_desc(w.batch, w.heads, w.n, w.d, w.n_buckets, w.chunk, w.rounds, w.causal,
                        x0.dtype)
    ws = lb.workspace(desc, dev, s_cmp)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(k):
        b = k % 2
        x, v, R, out, lse = slots[b]
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_cmp[b])  # the forward of step k-2 has read slot b
            x.copy_(xp, non_blocking=True)
            v.copy_(vp, non_blocking=True)
            R.copy_(Rp, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if k >= 2:
                s_cmp.wait_event(ev_out[b])  # step k-2's outputs have left slot b
            lb.lsh_attn_forward(x, v, R, n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal,
                                out=out, lse=lse, ws=ws, stream=s_cmp)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            outs_h[b][0].copy_(out, non_blocking=True)
            outs_h[b][1].copy_(lse, non_blocking=True)
            ev_out[b].record(s_out)

    main = torch.cuda.current_stream(dev)
    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    barrier(world)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(main)
    for st in (s_in, s_cmp, s_out):
        st.wait_event(s2)
    for k in range(K2):
        step(k)
    for st in (s_in, s_cmp, s_out):
        main.wait_stream(st)
    e2.record(main)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s2.elapsed_time(e2), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (x_h, v_h, R_h))
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0])
    return ms, h2d, d2h


DENSE_16K = I.Workload("dense-16k", 1, 8, 16384, 64, 2, 16384, 1, True, "bf16")


def dense_comparison(dev, K: int = 20, W: int = 3) -> dict:
    """Dense shared-QK causal attention against the LSH forward at n = 16K
    (8 heads, d = 64; LSH with n/64 buckets, chunk 64, 1 to 8 rounds), each
    timed with CUDA events over K passes after W, on the same seeded inputs."""
    w = DENSE_16K
    stream = torch.cuda.current_stream(dev)
    x_h, v_h = I.make_qkv(w)
    x, v = x_h.to(dev), v_h.to(dev)
    out = torch.empty_like(x)
    lse = torch.empty((w.batch, w.heads, w.n), dtype=torch.float32, device=dev)
    for _ in range(W):
        lb.lsh_attn_dense_forward(x, v, causal=True, out=out, lse=lse)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s0.record(stream)
    for _ in range(K):
        lb.lsh_attn_dense_forward(x, v, causal=True, out=out, lse=lse)
    s1.record(stream)
    torch.cuda.synchronize()
    dense_ms = s0.elapsed_time(s1) / K
    # visible (query, key) pairs under the causal mask, QK^T and PV
    flops = 2 * 2 * (w.n * (w.n + 1) // 2) * w.d * w.heads * w.batch
    pk, _ = peaks()
    res = {"config": config_of(w), "dense_ms": round(dense_ms, 4),
           "dense_TFLOP/s": round(flops / dense_ms / 1e9, 1),
           "dense_tensor_frac": round(flops / dense_ms / 1e9 / pk["bf16_tflops"], 4),
           "lsh_ms": {}, "dense_over_lsh": {}}
    for rounds in (1, 2, 4, 8):
        wl = I.Workload(f"lsh-16k-r{rounds}", 1, 8, 16384, 64, 256, 64, rounds, True, "bf16")
        m = measure(wl, dev, K, W)
        ms = m["total_ms"] / m["K"]
        res["lsh_ms"][rounds] = round(ms, 4)
        res["dense_over_lsh"][rounds] = round(dense_ms / ms, 2)
    return res


def time_calls(fn, dev, K: int, W: int) -> float:
    """Mean ms of fn() over K calls after W, CUDA events on the current stream."""
    stream = torch.cuda.current_stream(dev)
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(K):
        fn()
    s1.record(stream)
    torch.cuda.synchronize()
    return s0.elapsed_time(s1) / K


def backward_block(w: I.Workload, dev, K: int = 20, W: int = 3) -> dict:
    """The backward pass on the main workload (bucket ids from the library's
    hash, the forward's out and lse, a seeded upstream gradient)."""
    x_h, v_h = I.make_qkv(w)
    x, v, R = x_h.to(dev), v_h.to(dev), I.make_rotations(w).to(dev)
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    bk = lb.lsh_attn_hash(x, R, w.n_buckets)
    out, lse = lb.lsh_attn_forward(x, v, None, buckets=bk, **kw)
    g = torch.Generator(device="cpu").manual_seed(4)
    dout = torch.randn(x.shape, generator=g).to(x.dtype).to(dev)
    dx, dv = torch.empty_like(x), torch.empty_like(x)
    ms = time_calls(lambda: lb.lsh_attn_backward(x, v, bk, out, lse, dout, dx=dx, dv=dv, **kw),
                    dev, K, W)
    T = w.batch * w.heads * w.n
    m = min(w.chunk, w.n)
    # five products of m queries against 2m keys per chunk and round
    # (QK^T recomputed, dO V^T, dQ, dK, dV)
    flops = 5 * 4 * m * w.d * T * w.rounds
    pk, _ = peaks()
    return {"config": config_of(w), "ms": round(ms, 4),
            "tokens_per_s": w.tokens / (ms / 1e3),
            "TFLOP/s": round(flops / ms / 1e9, 1),
            "tensor_frac": round(flops / ms / 1e9 / pk["bf16_tflops"], 4),
            "flops_counted": "5 products of m x 2m x d per chunk and round"}


REV_CONFIG = dict(batch=1, n=16384, heads=8, d_head=128, d_ff=4096, rounds=4, n_buckets=256,
                  ffn_chunk=4096)


def reversible_block(dev, K: int = 10, W: int = 3) -> dict:
    """One reversible layer forward (projections, LSH attention with its own
    hash, output projection, chunked feed-forward) at d_model 1024."""
    c = REV_CONFIG
    dm = c["heads"] * c["d_head"]
    Wt = {k: v.to(dev) for k, v in I.make_rev_weights(dm, c["d_ff"]).items()}
    x1, x2 = (t.to(dev) for t in I.make_rev_inputs(c["batch"], c["n"], dm))
    wl = I.Workload("rev", c["batch"], c["heads"], c["n"], c["d_head"], c["n_buckets"], 64,
                    c["rounds"], True, "bf16")
    R = I.make_rotations(wl).to(dev)
    kw = dict(heads=c["heads"], n_buckets=c["n_buckets"], rounds=c["rounds"], causal=True,
              ffn_chunk=c["ffn_chunk"])
    y1, y2 = torch.empty_like(x1), torch.empty_like(x2)
    ms = time_calls(lambda: lb.lsh_rev_block(x1, x2, Wt, R=R, out1=y1, out2=y2, **kw), dev, K, W)
    rows = c["batch"] * c["n"]
    gemm_flops = 2 * rows * dm * dm * 3 + 2 * 2 * rows * dm * c["d_ff"]
    return {"config": dict(c, d_model=dm, chunk=64, causal=True), "ms": round(ms, 4),
            "tokens_per_s": rows / (ms / 1e3),
            "gemm_GFLOP": round(gemm_flops / 1e9, 1),
            "gemm_TFLOP/s_if_all_time": round(gemm_flops / ms / 1e9, 1)}


def run_ours(args, w):
    world, rank, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lb.load()
    K, W = args.steps, args.warmup
    clocks = ClockSampler(local)
    m = measure(w, dev, K, W, world, clocks)
    total_ms = m["total_ms"]
    value = world * w.tokens * K / (total_ms / 1e3)
    K2 = max(3, min(K, 20))
    e2e_ms, h2d, d2h = e2e_overlapped(m, dev, K2, world)
    extra = {}
    if world == 1 and not args.no_extra:
        sweep = {s.name: s for s in I.sweep_workloads()}
        for name in EXTRA_WORKLOADS:
            wx = I.WORKLOADS.get(name) or sweep[name]
            mx = measure(wx, dev, 20, 3)
            st, rf = roofline_block(wx, mx["kernel_ms"], mx["total_ms"] / 1e3)
            extra[name] = {"config": config_of(wx), "ms_per_step": mx["total_ms"] / mx["K"],
                           "value": wx.tokens * mx["K"] / (mx["total_ms"] / 1e3), "unit": UNIT,
                           "roofline": rf, "stages": st,
                           "kernels_ms": {kn: round(t, 4) for kn, t in mx["kernel_ms"].items()}}
            del mx
        extra["dense_baseline"] = dense_comparison(dev)
        extra["backward"] = backward_block(w, dev)
        extra["reversible_layer"] = reversible_block(dev)
    if rank != 0:
        return
    stages, roof = roofline_block(w, m["kernel_ms"], total_ms / 1e3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1))",
        "config": config_of(w),
        "e2e": {"value": world * w.tokens * K2 / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "each step's copies overlap the neighbouring steps' compute"},
        "gpu_launches": K * launches_per_forward(buckets_given=False),
        "roofline": roof,
        "stages": stages,
        "kernels_ms": {kn: round(t, 4) for kn, t in m["kernel_ms"].items()},
        "clocks": m["clocks"],
    }
    if extra:
        line["workloads"] = extra
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))


def launches_per_forward(buckets_given: bool) -> int:
    """Kernels one bf16 chunk-64 forward launches. Internal hash: rotation
    transpose, projection/argmax (which also counts the sort's histograms and
    writes the key norms), fp64 re-decision, scan, ranks, attention, merge.
    Caller buckets: histograms, scan, ranks, key norms, attention, merge."""
    return 6 if buckets_given else 7


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
