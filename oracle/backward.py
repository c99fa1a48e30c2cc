"""Gradients of the LSH-attention forward pass, for a backward pass to be
checked against.

TEST INFRASTRUCTURE ONLY, like the rest of this package: it shares no code
with the CUDA path.

The forward is restated here in float64 torch operations, step by step as
the method defines it (the hash is not differentiated: bucket ids are an
input, as in training, where the sort is piecewise constant):

  * per (batch, head, round), the tokens are ordered by (bucket, position)
    ("Reformer summary" (ttnews.xyz), §局部敏感哈希注意力);
  * the query at sorted slot s, in chunk c = s // m, sees the keys of chunks
    c - 1 and c; the logit against key slot j is (x_s . x_j) / (||x_j|| sqrt(d))
    ("Reformer: LSH attention and reversible layers" (dtcms.com), §二.1), 0 for
    a zero key, removed when causal and pos_j > pos_s, and replaced by -1e5 for
    the token itself ("Reformer summary", §共享QK中的自掩碼);
  * lse_r = log sum exp over the candidates, o_r = softmax-weighted sum of v,
    both by the two-pass form (max, then sum of exponentials);
  * the rounds are merged per position with weights exp(lse_r - logsumexp_r lse_r)
    ("Reformer summary", §多輪LSH哈希 leaves this to the paper; this weighting is
    one softmax over the union of the rounds' candidates).

The gradient is reverse-mode differentiation of exactly this computation
(torch.autograd), so it is the derivative of the definition. The tests pin
the forward to the C oracle and the derivatives to finite differences and to
a separately written dense attention.
"""
from __future__ import annotations

import math

import torch

SELF_LOGIT = -1.0e5


def _round(x: torch.Tensor, v: torch.Tensor, bk: torch.Tensor, m: int, causal: bool):
    """One (batch, head, round): x, v [n, d] float64, bk [n] bucket ids.
    Returns (o [n, d], lse [n]) in position order."""
    n, d = x.shape
    pos = torch.arange(n)
    perm = torch.argsort(bk.long() * n + pos)  # stable order by (bucket, position)
    inv = torch.argsort(perm)
    xs, vs = x[perm], v[perm]
    norm = xs.norm(dim=1)
    # 1 / ||x_j|| with a zero key giving logit 0 (its scale is 0)
    scale = torch.where(norm > 0, 1.0 / torch.where(norm > 0, norm, torch.ones_like(norm)),
                        torch.zeros_like(norm)) / math.sqrt(d)
    o_chunks, l_chunks = [], []
    for c in range(n // m):
        q0, q1 = c * m, (c + 1) * m
        k0 = max(0, (c - 1) * m)
        logits = (xs[q0:q1] @ xs[k0:q1].T) * scale[k0:q1][None, :]
        pq, pk = perm[q0:q1][:, None], perm[k0:q1][None, :]
        logits = torch.where(pk == pq, torch.full_like(logits, SELF_LOGIT), logits)
        if causal:
            logits = torch.where(pk > pq, torch.full_like(logits, -math.inf), logits)
        # two-pass softmax: M = max, Z = sum exp(l - M), lse = M + log Z,
        # o = sum exp(l - M) v / Z (exact for a row that sees only itself)
        M = logits.max(dim=1).values.detach()
        e = torch.exp(logits - M[:, None])
        Z = e.sum(dim=1)
        o_chunks.append((e @ vs[k0:q1]) / Z[:, None])
        l_chunks.append(M + torch.log(Z))
    o = torch.cat(o_chunks)[inv]
    lse = torch.cat(l_chunks)[inv]
    return o, lse


def forward_torch(x: torch.Tensor, v: torch.Tensor, buckets: torch.Tensor, chunk: int,
                  causal: bool):
    """x, v [B, H, n, d] float64 (gradients allowed); buckets [B, H, R, n].
    Returns (out [B, H, n, d], lse [B, H, R, n]) in position order."""
    B, H, n, d = x.shape
    R = buckets.shape[2]
    m = min(chunk, n)
    assert n % m == 0, "n must be a multiple of the chunk length (or chunk >= n)"
    outs, lses = [], []
    for b in range(B):
        for h in range(H):
            os_, ls_ = zip(*[_round(x[b, h], v[b, h], buckets[b, h, r], m, causal)
                             for r in range(R)])
            o = torch.stack(os_)  # [R, n, d]
            lse = torch.stack(ls_)  # [R, n]
            mx = lse.max(dim=0).values.detach()  # exp(lse_r - logsumexp_r lse_r),
            e = torch.exp(lse - mx)               # formed without the logsumexp
            w = e / e.sum(dim=0)
            outs.append((w[:, :, None] * o).sum(0))
            lses.append(lse)
    return (torch.stack(outs).reshape(B, H, n, d), torch.stack(lses).reshape(B, H, R, n))


def backward(x, v, buckets, chunk: int, causal: bool, dout, dlse=None):
    """Gradients of (out, lse) with respect to x and v, for upstream gradients
    dout [B, H, n, d] and (optionally) dlse [B, H, R, n]. Returns (dx, dv) in
    float64."""
    x64 = torch.as_tensor(x, dtype=torch.float64).detach().clone().requires_grad_(True)
    v64 = torch.as_tensor(v, dtype=torch.float64).detach().clone().requires_grad_(True)
    out, lse = forward_torch(x64, v64, torch.as_tensor(buckets), chunk, causal)
    grads = [torch.as_tensor(dout, dtype=torch.float64)]
    outputs = [out]
    if dlse is not None:
        grads.append(torch.as_tensor(dlse, dtype=torch.float64))
        outputs.append(lse)
    dx, dv = torch.autograd.grad(outputs, (x64, v64), grads)
    return dx, dv
