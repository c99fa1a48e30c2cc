"""Dense shared-QK attention (the full-attention baseline) through the C ABI
against the oracle. The oracle's dense attention is its forward pass with one
round and one chunk spanning the sequence, which the CPU pins tie to a
textbook dense softmax attention. Bar as for the LSH forward: bf16 max abs
<= 2e-2 and mean abs <= 2e-3 on out and lse."""
import numpy as np
import pytest
import torch

import oracle
from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu


def check(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    assert np.isfinite(gpu).all(), what
    assert err.max() <= 2e-2, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= 2e-3, f"{what}: mean abs {err.mean():.3e}"


CASES = [  # name, B, H, n, d, causal, clustered
    ("n1000-d64-causal", 1, 2, 1000, 64, True, False),   # ragged last tile
    ("n384-d128-noncausal", 2, 1, 384, 128, False, False),
    ("n1-d64", 1, 1, 1, 64, True, False),                # one query that sees only itself
    ("n129-d64-noncausal", 1, 2, 129, 64, False, False),
    ("n2048-d64-clustered", 1, 2, 2048, 64, True, True),
    ("n640-d128-causal", 1, 3, 640, 128, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_dense_full(case):
    name, B, H, n, d, causal, clu = case
    w = I.Workload(name, B, H, n, d, 2, n, 1, causal, "bf16", clustered=clu)
    x, v = I.make_qkv(w)
    pos = np.arange(n, dtype=np.int32)
    ro, rl = oracle.dense_sampled(x, v, causal, pos)
    out, lse = lb.lsh_attn_dense_forward(x.cuda(), v.cuda(), causal=causal)
    check(out.float().cpu().numpy(), ro, f"{name} out")
    check(lse.cpu().numpy(), rl, f"{name} lse")


@pytest.mark.parametrize("causal", [True, False])
def test_dense_sampled_16k(causal):
    """The size the pages quote their speed ratio at: n = 16K, 8 heads."""
    w = I.Workload("dense-16k", 1, 8, 16384, 64, 2, 16384, 1, causal, "bf16")
    x, v = I.make_qkv(w)
    out, lse = lb.lsh_attn_dense_forward(x.cuda(), v.cuda(), causal=causal)
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    pos = np.unique(np.concatenate([[0, 1, 127, 128, 16383],
                                    np.random.default_rng(4).integers(0, 16384, 160)]))
    pos = pos.astype(np.int32)
    for h in (0, 7):
        ro, rl = oracle.dense_sampled(x[:, h:h + 1], v[:, h:h + 1], causal, pos)
        check(out[:, h:h + 1][:, :, pos], ro, f"h{h} out")
        check(lse[:, h:h + 1][:, :, pos], rl, f"h{h} lse")


def test_dense_equals_one_chunk_lsh():
    """One round whose single chunk spans the sequence is dense attention."""
    w = I.Workload("one-chunk", 1, 2, 128, 64, 16, 128, 1, True, "bf16")
    x, v = I.make_qkv(w)
    xg, vg = x.cuda(), v.cuda()
    bk = I.make_buckets(w).cuda()
    lo, ll = lb.lsh_attn_forward(xg, vg, None, n_buckets=16, chunk=128, causal=True, buckets=bk)
    do, dl = lb.lsh_attn_dense_forward(xg, vg, causal=True)
    check(do.float().cpu().numpy(), lo.float().cpu().numpy().astype(np.float64), "out")
    check(dl.cpu().numpy(), ll[:, :, 0].cpu().numpy().astype(np.float64), "lse")


def test_dense_rows_beyond_the_one_pass_bound_are_exact():
    """Vectors with norm ~500 put the stabiliser ||q|| log2(e)/sqrt(d) above its
    one-pass limit: those rows are recomputed with their exact maximum."""
    w = I.Workload("big-norm", 1, 2, 512, 64, 2, 512, 1, True, "bf16")
    x, v = I.make_qkv(w)
    x = (x.float() * 64).to(torch.bfloat16)
    pos = np.arange(512, dtype=np.int32)
    ro, rl = oracle.dense_sampled(x, v, True, pos)
    out, lse = lb.lsh_attn_dense_forward(x.cuda(), v.cuda(), causal=True)
    check(out.float().cpu().numpy(), ro, "out")
    check(lse.cpu().numpy(), rl, "lse")


def test_dense_deterministic():
    w = I.Workload("det", 1, 4, 4096, 128, 2, 4096, 1, True, "bf16")
    x, v = I.make_qkv(w)
    xg, vg = x.cuda(), v.cuda()
    a = [t.clone() for t in lb.lsh_attn_dense_forward(xg, vg, causal=True)]
    b = lb.lsh_attn_dense_forward(xg, vg, causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
