"""Pins of the backward-pass oracle (oracle/backward.py), on the CPU.

The backward oracle restates the forward in float64 torch operations and
differentiates it. These tests tie it to things other than itself: its
forward equals the C oracle's; its derivatives equal finite differences; with
one round and one chunk (dense attention) its gradients equal those of a
textbook dense attention written separately; identical rounds give the one-
round gradient."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob


def _case(B, H, n, d, nb, R, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, H, n, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, n, d, generator=g, dtype=torch.float64)
    bk = torch.randint(0, nb, (B, H, R, n), generator=g, dtype=torch.int32)
    return x, v, bk


@pytest.mark.parametrize("n,chunk,R,causal", [(16, 4, 2, True), (16, 4, 2, False),
                                              (12, 4, 3, True), (8, 16, 1, True),
                                              (24, 8, 2, False)])
def test_forward_equals_the_c_oracle(n, chunk, R, causal):
    x, v, bk = _case(1, 2, n, 8, 8, R, seed=n + R)
    out, lse = ob.forward_torch(x, v, bk, chunk, causal)
    Rz = np.zeros((R, 8, 4))
    ref_out, ref_lse, ref_bk = oracle.forward(x.numpy(), v.numpy(), Rz, chunk, causal,
                                              buckets=bk.numpy())
    assert np.array_equal(ref_bk, bk.numpy())
    # the C oracle forms logsumexp_r lse_r before the weights; where every
    # round of a position sees only the token itself (lse = -1e5), the fp64
    # spacing of that sum (1.5e-11) scales its weights by 1 +- 1.5e-11, while
    # this restatement normalises the weights directly (exactly v there)
    np.testing.assert_allclose(out.numpy(), ref_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse.numpy(), ref_lse, rtol=0, atol=1e-10)
    sees_others = ~(ref_lse <= -99999.0).all(axis=2)  # [B, H, n]
    assert np.abs(out.numpy() - ref_out)[sees_others].max() <= 1e-13


@pytest.mark.parametrize("chunk,causal", [(2, True), (4, False), (8, True)])
def test_derivatives_equal_finite_differences(chunk, causal):
    x, v, bk = _case(1, 1, 8, 3, 4, 2, seed=chunk)
    x.requires_grad_(True)
    v.requires_grad_(True)

    def f(x_, v_):
        return ob.forward_torch(x_, v_, bk, chunk, causal)

    assert torch.autograd.gradcheck(f, (x, v), eps=1e-6, atol=1e-6, rtol=1e-4)


def _dense_attention(x, v, causal):
    """Textbook dense shared-QK attention of one head: keys x_j / ||x_j||,
    logits scaled by 1/sqrt(d), self logit -1e5, optional causal mask."""
    n, d = x.shape
    keys = x / x.norm(dim=1, keepdim=True)
    logits = (x @ keys.T) / math.sqrt(d)
    eye = torch.eye(n, dtype=torch.bool)
    logits = logits.masked_fill(eye, -1.0e5)
    if causal:
        logits = logits.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
    return torch.softmax(logits, dim=1) @ v


@pytest.mark.parametrize("causal", [True, False])
def test_dense_case_equals_textbook_attention_gradients(causal):
    x, v, bk = _case(1, 1, 12, 5, 2, 1, seed=3)
    g = torch.Generator().manual_seed(9)
    dout = torch.randn(1, 1, 12, 5, generator=g, dtype=torch.float64)
    dx, dv = ob.backward(x, v, bk, chunk=64, causal=causal, dout=dout)  # one chunk = dense
    xr = x[0, 0].clone().requires_grad_(True)
    vr = v[0, 0].clone().requires_grad_(True)
    ref_dx, ref_dv = torch.autograd.grad(_dense_attention(xr, vr, causal), (xr, vr), dout[0, 0])
    torch.testing.assert_close(dx[0, 0], ref_dx, rtol=0, atol=1e-10)
    torch.testing.assert_close(dv[0, 0], ref_dv, rtol=0, atol=1e-10)


def test_identical_rounds_give_the_one_round_gradient():
    x, v, bk1 = _case(1, 2, 16, 6, 4, 1, seed=5)
    bk3 = bk1.repeat(1, 1, 3, 1)
    dout = torch.randn(1, 2, 16, 6, generator=torch.Generator().manual_seed(2),
                       dtype=torch.float64)
    dx1, dv1 = ob.backward(x, v, bk1, chunk=4, causal=True, dout=dout)
    dx3, dv3 = ob.backward(x, v, bk3, chunk=4, causal=True, dout=dout)
    torch.testing.assert_close(dx3, dx1, rtol=0, atol=1e-12)
    torch.testing.assert_close(dv3, dv1, rtol=0, atol=1e-12)
