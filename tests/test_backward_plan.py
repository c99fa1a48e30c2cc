"""The backward-pass plan, written out by hand in numpy (no autograd), agrees
with the backward oracle (autograd of the restated forward). This checks the
derivation a GPU backward pass will follow:

  merge:     dL/do_r = w_r g,  dL/dlse_r = w_r g.(o_r - out) (+ given dL/dlse)
  attention: D = rowsum(dO o), dS = P (dO V^T - D + dlse) (0 at self and
             masked keys), dV = P^T dO, dQ = dS K^ / sqrt(d), dK^ = dS^T Q / sqrt(d),
             dx_key = (I - k^ k^T) dK^ / ||x||
  un-sort:   sum the query and key roles of every round per position."""
import math

import numpy as np
import pytest
import torch

from oracle import backward as ob

SELF = -1.0e5


def planned_backward(x, v, bk, m, causal, g, dlse_in):
    n, d = x.shape
    R = bk.shape[0]
    rounds = []
    for r in range(R):  # forward per round, keeping what the backward needs
        perm = np.argsort(bk[r].astype(np.int64) * n + np.arange(n), kind="stable")
        xs, vs = x[perm], v[perm]
        nrm = np.linalg.norm(xs, axis=1)
        kh = xs / nrm[:, None]
        o = np.zeros((n, d))
        lse = np.zeros(n)
        P = {}
        for c in range(n // m):
            q0, q1, k0 = c * m, (c + 1) * m, max(0, (c - 1) * m)
            l = xs[q0:q1] @ kh[k0:q1].T / math.sqrt(d)
            pq, pk = perm[q0:q1][:, None], perm[k0:q1][None, :]
            l = np.where(pk == pq, SELF, l)
            if causal:
                l = np.where(pk > pq, -np.inf, l)
            M = l.max(axis=1)
            e = np.exp(l - M[:, None])
            Z = e.sum(axis=1)
            P[c] = (e / Z[:, None], (pk == pq) | (causal & (pk > pq)))
            o[q0:q1] = P[c][0] @ vs[k0:q1]
            lse[q0:q1] = M + np.log(Z)
        inv = np.argsort(perm)
        rounds.append(dict(perm=perm, xs=xs, vs=vs, nrm=nrm, kh=kh, P=P, o=o[inv], lse=lse[inv]))
    lse_all = np.stack([rd["lse"] for rd in rounds])
    w = np.exp(lse_all - lse_all.max(0))
    w /= w.sum(0)
    out = sum(w[r][:, None] * rounds[r]["o"] for r in range(R))
    dx = np.zeros_like(x)
    dv = np.zeros_like(v)
    for r, rd in enumerate(rounds):
        perm = rd["perm"]
        dO = (w[r][:, None] * g)[perm]  # slot order
        dl = (w[r] * np.sum(g * (rd["o"] - out), axis=1) + dlse_in[r])[perm]
        os_ = rd["o"][perm]
        dxs = np.zeros((n, d))
        dkh = np.zeros((n, d))
        dvs = np.zeros((n, d))
        for c in range(n // m):
            q0, q1, k0 = c * m, (c + 1) * m, max(0, (c - 1) * m)
            p, dead = rd["P"][c]
            D = np.sum(dO[q0:q1] * os_[q0:q1], axis=1)
            dS = p * (dO[q0:q1] @ rd["vs"][k0:q1].T - D[:, None] + dl[q0:q1][:, None])
            dS = np.where(dead, 0.0, dS)
            dvs[k0:q1] += p.T @ dO[q0:q1]
            dxs[q0:q1] += dS @ rd["kh"][k0:q1] / math.sqrt(d)
            dkh[k0:q1] += dS.T @ rd["xs"][q0:q1] / math.sqrt(d)
        kh = rd["kh"]
        dxs += (dkh - kh * np.sum(kh * dkh, axis=1, keepdims=True)) / rd["nrm"][:, None]
        dx[perm] += dxs
        dv[perm] += dvs
    return dx, dv


@pytest.mark.parametrize("n,chunk,R,causal", [(16, 4, 2, True), (12, 4, 3, False),
                                              (8, 8, 1, True), (24, 8, 2, True)])
def test_planned_backward_equals_the_oracle(n, chunk, R, causal):
    g_ = torch.Generator().manual_seed(n * 10 + R)
    d = 6
    x = torch.randn(1, 1, n, d, generator=g_, dtype=torch.float64)
    v = torch.randn(1, 1, n, d, generator=g_, dtype=torch.float64)
    bk = torch.randint(0, 4, (1, 1, R, n), generator=g_, dtype=torch.int32)
    dout = torch.randn(1, 1, n, d, generator=g_, dtype=torch.float64)
    dlse = torch.randn(1, 1, R, n, generator=g_, dtype=torch.float64)
    ref_dx, ref_dv = ob.backward(x, v, bk, chunk, causal, dout, dlse)
    dx, dv = planned_backward(x[0, 0].numpy(), v[0, 0].numpy(), bk[0, 0].numpy(),
                              min(chunk, n), causal, dout[0, 0].numpy(), dlse[0, 0].numpy())
    np.testing.assert_allclose(dx, ref_dx[0, 0].numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dv, ref_dv[0, 0].numpy(), rtol=0, atol=1e-10)
