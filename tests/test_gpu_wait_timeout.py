"""Bounded waits. Every wait of the tcgen05 kernels on an mbarrier gives up
after a time limit and records LSH_ERR_TIMEOUT in the workspace status word.
The self-test entry point runs that path for real with a short limit: one CTA
waits on an mbarrier that nothing arrives at. The wait ends by itself (no
fault, no hang), the status reaches the host, and the stream keeps working."""
import time

import pytest
import torch

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu

LSH_ERR_TIMEOUT = 5


def test_wait_that_nothing_completes_gives_up_and_reports_it():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lb.lsh_attn_selftest_wait_timeout(ws, 20000)  # 20 ms
    status = lb.lsh_attn_get_device_status(ws)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == LSH_ERR_TIMEOUT
    assert elapsed >= 0.019  # the wait ran to its limit
    assert elapsed < 2.0     # and no longer than the kernels' own limit


def test_stream_is_usable_after_a_timeout():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    lb.lsh_attn_selftest_wait_timeout(ws, 1000)
    assert lb.lsh_attn_get_device_status(ws) == LSH_ERR_TIMEOUT
    w = I.BF16_SHORT.with_(batch=1, heads=2)
    x, v = (t.cuda() for t in I.make_qkv(w))
    R = I.make_rotations(w).cuda()
    out, lse = lb.lsh_attn_forward(x, v, R, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=w.causal)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    desc = lb.make_desc(w.batch, w.heads, w.n, w.d, w.n_buckets, w.chunk, w.rounds, w.causal,
                        x.dtype)
    assert lb.lsh_attn_get_device_status(lb.workspace(desc, x.device)) == 0
