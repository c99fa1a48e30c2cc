"""bench.py's host-side bookkeeping on the CPU: the algorithmic bytes and
flops behind the roofline fractions, the launch count per forward, and the
rule that ncu traffic is reported only for the workload it was captured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from lsh_attention_b200 import binding as lb  # noqa: E402
from lsh_attention_b200 import inputs as I  # noqa: E402


def test_algorithmic_work_of_the_long_sequence_workload():
    w = I.LONG_64K
    T = w.batch * w.heads * w.n  # (token, head) units
    R, d, half, m = w.rounds, w.d, w.n_buckets // 2, w.chunk
    X = T * d * 2  # bytes of x (bf16)
    a = bench.algorithmic(w)
    # hash: one projection of every token onto nb/2 columns per round
    assert a["hash"]["flops"] == 2 * T * d * half * R == 274_877_906_944
    assert a["hash"]["bytes"] == X + R * d * half * 2 + 4 * T * R + 4 * T
    # sort: ids in, perm and inv out
    assert a["sort"]["bytes"] == 12 * T * R
    # attention: m queries against 2m keys, QK^T and PV, per chunk and round;
    # x and v once, perm and key scales in, bf16 rows and lse out
    assert a["chunk_attention"]["flops"] == 2 * 2 * (2 * m) * d * T * R
    assert a["chunk_attention"]["bytes"] == 2 * X + 4 * T + 4 * T * R + T * R * d * 2 + 4 * T * R
    # merge: every round's bf16 row and (lse, slot), one output row
    assert a["unsort_merge"]["bytes"] == T * R * (2 * d + 8) + X


def test_launches_per_forward_match_the_kernel_boundaries():
    # the profiled entry point marks one event per kernel boundary
    assert lb.PROFILE_EVENTS == len(lb.PROFILE_KERNELS) + 1
    # internal hash: every kernel but the separate histogram pass and the
    # norm pass (the hash counts the histograms and writes the norms)
    assert bench.launches_per_forward(buckets_given=False) == len(lb.PROFILE_KERNELS) - 2
    # caller buckets: histograms, scan, ranks, key norms, attention, merge
    assert bench.launches_per_forward(buckets_given=True) == 6


def test_traffic_is_reported_only_for_the_captured_workload():
    for kernel in bench.NCU_TRAFFIC:
        assert bench.traffic_of(kernel, I.IMAGE_12K.name) is None
    assert bench.traffic_of("no-such-kernel", bench.NCU_WORKLOAD) is None
    every_stage_kernel = set(bench.STAGE_KERNEL.values())
    assert every_stage_kernel <= set(bench.KERNEL_STAGE)
