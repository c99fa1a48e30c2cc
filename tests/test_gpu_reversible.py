"""Reversible layer (LSH attention + chunked feed-forward) through the C ABI
against the oracle (oracle/reversible.py, float64; its pins are on the CPU).

Bar for the forward against the oracle: max abs <= 5e-2, mean abs <= 4e-3.
The GPU keeps qk, v, the attention output, y1, the feed-forward hidden layer
and y2 in bf16; the oracle's arithmetic with exactly those roundings (and
nothing else) differs from its float64 result by at most 1.9e-2 (mean 2e-3)
on these configurations, and the attention's own bf16 probabilities and fp32
sums add a little more. Round trips (inverse of forward) are held to the same
bar against the input: each step rounds its result to bf16 once more."""
import numpy as np
import pytest
import torch

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I
from oracle import reversible as rv

pytestmark = pytest.mark.gpu

CASES = [  # name, B, n, heads, d_head, d_ff, rounds, n_buckets, ffn_chunk
    ("d128-h2", 1, 512, 2, 128, 512, 2, 16, 256),
    ("d64-h4-b2", 2, 256, 4, 64, 1024, 2, 8, 128),
]


def check(gpu, ref, what, mx=5e-2, mean=4e-3):
    gpu = gpu.float().cpu().double().numpy()
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    print(f"{what}: max {err.max():.3e} mean {err.mean():.3e}")
    assert np.isfinite(gpu).all(), what
    assert err.max() <= mx, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= mean, f"{what}: mean abs {err.mean():.3e}"


def setup(B, n, H, dh, dff, rounds, nb):
    dm = H * dh
    W = I.make_rev_weights(dm, dff)
    x1, x2 = I.make_rev_inputs(B, n, dm)
    bk = I.make_buckets(I.Workload("rev", B, H, n, dh, nb, 64, rounds, True, "bf16"))
    return W, x1, x2, bk


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_rev_forward_matches_oracle(case):
    name, B, n, H, dh, dff, rounds, nb, fc = case
    W, x1, x2, bk = setup(B, n, H, dh, dff, rounds, nb)
    Wg = {k: v.cuda() for k, v in W.items()}
    y1, y2, _ = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, heads=H, n_buckets=nb, rounds=rounds,
                                 causal=True, ffn_chunk=fc, buckets=bk.cuda())
    r1, r2 = rv.block(x1, x2, {k: v.double().numpy() for k, v in W.items()}, bk.numpy(), H, 64,
                      True, fc)
    check(y1, r1, f"{name} y1")
    check(y2, r2, f"{name} y2")


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_rev_inverse_recovers_input(case):
    """Forward with the layer's own hash, then the inverse with those bucket
    ids: the halves of the input come back."""
    name, B, n, H, dh, dff, rounds, nb, fc = case
    W, x1, x2, _ = setup(B, n, H, dh, dff, rounds, nb)
    Wg = {k: v.cuda() for k, v in W.items()}
    R = I.make_rotations(I.Workload("rev", B, H, n, dh, nb, 64, rounds, True, "bf16")).cuda()
    kw = dict(heads=H, n_buckets=nb, rounds=rounds, causal=True, ffn_chunk=fc)
    y1, y2, bk = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, R=R, **kw)
    y1, y2 = y1.clone(), y2.clone()
    z1, z2, _ = lb.lsh_rev_block(y1, y2, Wg, buckets=bk, inverse=True, **kw)
    check(z1, x1.double().numpy(), f"{name} x1 back")
    check(z2, x2.double().numpy(), f"{name} x2 back")
    assert (y1 - x1.cuda()).abs().max() > 0.1  # the layer changed its input


def test_rev_feed_forward_chunks_give_the_same_bits():
    name, B, n, H, dh, dff, rounds, nb, fc = CASES[1]
    W, x1, x2, bk = setup(B, n, H, dh, dff, rounds, nb)
    Wg = {k: v.cuda() for k, v in W.items()}
    kw = dict(heads=H, n_buckets=nb, rounds=rounds, causal=True, buckets=bk.cuda())
    a1, a2, _ = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, ffn_chunk=128, **kw)
    a1, a2 = a1.clone(), a2.clone()
    b1, b2, _ = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, ffn_chunk=B * n, **kw)
    assert torch.equal(a1, b1) and torch.equal(a2, b2)


def test_rev_hashed_buckets_are_the_layers_own():
    """Forward that hashes equals forward fed the ids it produced."""
    name, B, n, H, dh, dff, rounds, nb, fc = CASES[0]
    W, x1, x2, _ = setup(B, n, H, dh, dff, rounds, nb)
    Wg = {k: v.cuda() for k, v in W.items()}
    R = I.make_rotations(I.Workload("rev", B, H, n, dh, nb, 64, rounds, True, "bf16")).cuda()
    kw = dict(heads=H, n_buckets=nb, rounds=rounds, causal=True, ffn_chunk=fc)
    a1, a2, bk = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, R=R, **kw)
    a1, a2, bk = a1.clone(), a2.clone(), bk.clone()
    b1, b2, _ = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, buckets=bk, **kw)
    assert torch.equal(a1, b1) and torch.equal(a2, b2)
    assert 0 <= int(bk.min()) and int(bk.max()) < nb


def test_rev_full_size_matches_oracle():
    """The layer the benchmark times (B1 n16384, 8 heads of 128, d_ff 4096,
    4 rounds, nb 256, feed-forward chunk 4096), against the oracle, then its
    inverse against the input."""
    B, n, H, dh, dff, rounds, nb, fc = 1, 16384, 8, 128, 4096, 4, 256, 4096
    W, x1, x2, bk = setup(B, n, H, dh, dff, rounds, nb)
    Wg = {k: v.cuda() for k, v in W.items()}
    kw = dict(heads=H, n_buckets=nb, rounds=rounds, causal=True, ffn_chunk=fc, buckets=bk.cuda())
    y1, y2, _ = lb.lsh_rev_block(x1.cuda(), x2.cuda(), Wg, **kw)
    y1, y2 = y1.clone(), y2.clone()
    z1, z2, _ = lb.lsh_rev_block(y1, y2, Wg, inverse=True, **kw)
    r1, r2 = rv.block(x1, x2, {k: v.double().numpy() for k, v in W.items()}, bk.numpy(), H, 64,
                      True, fc)
    check(y1, r1, "full-size y1")
    check(y2, r2, "full-size y2")
    check(z1, x1.double().numpy(), "full-size x1 back")
    check(z2, x2.double().numpy(), "full-size x2 back")
