"""Reversible Reformer layer around the LSH attention, in float64 numpy, for
the reversible-block kernels to be checked against.

TEST INFRASTRUCTURE ONLY, like the rest of this package: it shares no code
with the CUDA path.

"Reformer: LSH attention and reversible layers" (dtcms.com), §二.2: the
input is split into two halves x = [x1, x2] and
    y1 = x1 + Attention(x2),   y2 = x2 + FeedForward(y1),
which is undone by
    x2 = y2 - FeedForward(y1),   x1 = y1 - Attention(x2).
§二.3: the feed-forward layer is applied to chunks of the sequence and the
results concatenated; each row is independent of the others, so the chunk
size changes nothing but the memory held at once.

Readings (the pages fix neither): Attention(x) projects x with W_qk (shared
query/key) and W_v into heads of d_head features, runs the LSH attention of
oracle.forward on every head with the given bucket ids, concatenates the
heads and applies W_o; FeedForward(y) = max(y W1^T + b1, 0) W2^T + b2. Weights
are stored out x in, as the CUDA path takes them. matmul is the library
primitive; everything else is written out.
"""
from __future__ import annotations

import numpy as np

from . import forward as lsh_forward


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def attention(x, w_qk, w_v, w_o, buckets, heads: int, chunk: int, causal: bool, R=None):
    """Attention sublayer of x [B, n, d_model] with given bucket ids
    [B, heads, rounds, n]. Returns [B, n, d_model]."""
    x = _f64(x)
    B, n, dm = x.shape
    dh = dm // heads
    qk = (x @ _f64(w_qk).T).reshape(B, n, heads, dh).transpose(0, 2, 1, 3)
    v = (x @ _f64(w_v).T).reshape(B, n, heads, dh).transpose(0, 2, 1, 3)
    bk = np.asarray(buckets)
    rounds = bk.shape[2]
    if R is None:  # only its shape matters (the bucket count): the ids are given
        nb = int(bk.max()) + 1
        R = np.zeros((rounds, dh, (nb + 1) // 2))
    out, _, _ = lsh_forward(np.ascontiguousarray(qk), np.ascontiguousarray(v), R, chunk, causal,
                            buckets=buckets)
    att = out.transpose(0, 2, 1, 3).reshape(B, n, dm)
    return att @ _f64(w_o).T


def feed_forward(y, w1, b1, w2, b2, ffn_chunk: int):
    """Feed-forward sublayer of y [B, n, d_model], ffn_chunk rows at a time
    (rows of all sequences, in order)."""
    y = _f64(y)
    B, n, dm = y.shape
    rows = y.reshape(B * n, dm)
    out = np.empty_like(rows)
    b1 = np.zeros(_f64(w1).shape[0]) if b1 is None else _f64(b1)
    b2 = np.zeros(dm) if b2 is None else _f64(b2)
    for r0 in range(0, B * n, ffn_chunk):
        h = rows[r0:r0 + ffn_chunk] @ _f64(w1).T + b1
        h = np.maximum(h, 0.0)
        out[r0:r0 + ffn_chunk] = h @ _f64(w2).T + b2
    return out.reshape(B, n, dm)


def block(x1, x2, W, buckets, heads: int, chunk: int, causal: bool, ffn_chunk: int):
    """y1 = x1 + Attention(x2), y2 = x2 + FeedForward(y1). W: dict with w_qk,
    w_v, w_o, w1, b1, w2, b2."""
    y1 = _f64(x1) + attention(x2, W["w_qk"], W["w_v"], W["w_o"], buckets, heads, chunk, causal)
    y2 = _f64(x2) + feed_forward(y1, W["w1"], W["b1"], W["w2"], W["b2"], ffn_chunk)
    return y1, y2


def inverse(y1, y2, W, buckets, heads: int, chunk: int, causal: bool, ffn_chunk: int):
    """x2 = y2 - FeedForward(y1), x1 = y1 - Attention(x2)."""
    x2 = _f64(y2) - feed_forward(y1, W["w1"], W["b1"], W["w2"], W["b2"], ffn_chunk)
    x1 = _f64(y1) - attention(x2, W["w_qk"], W["w_v"], W["w_o"], buckets, heads, chunk, causal)
    return x1, x2
