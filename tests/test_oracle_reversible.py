"""Pins of the reversible-block oracle (oracle/reversible.py), each against
something other than itself: the round trip of the reversible residual, the
chunk-size independence of the feed-forward layer, special weights that
reduce a sublayer to a known map, and a direct evaluation of one row."""
import numpy as np
import pytest

import oracle
from oracle import reversible as rv


def setup(seed=0, B=1, n=32, heads=2, dh=8, dff=24, rounds=2, nb=4):
    g = np.random.default_rng(seed)
    dm = heads * dh
    W = {"w_qk": g.standard_normal((dm, dm)) / 4, "w_v": g.standard_normal((dm, dm)) / 4,
         "w_o": g.standard_normal((dm, dm)) / 4, "w1": g.standard_normal((dff, dm)) / 4,
         "b1": g.standard_normal(dff) / 10, "w2": g.standard_normal((dm, dff)) / 4,
         "b2": g.standard_normal(dm) / 10}
    x1 = g.standard_normal((B, n, dm))
    x2 = g.standard_normal((B, n, dm))
    bk = g.integers(0, nb, (B, heads, rounds, n)).astype(np.int32)
    return W, x1, x2, bk


@pytest.mark.parametrize("causal", [True, False])
def test_inverse_recovers_the_input(causal):
    W, x1, x2, bk = setup()
    y1, y2 = rv.block(x1, x2, W, bk, 2, 8, causal, 16)
    r1, r2 = rv.inverse(y1, y2, W, bk, 2, 8, causal, 16)
    np.testing.assert_allclose(r1, x1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r2, x2, rtol=0, atol=1e-12)
    assert np.abs(y1 - x1).max() > 1e-2 and np.abs(y2 - x2).max() > 1e-2  # the layer did something


def test_feed_forward_chunking_changes_nothing():
    W, x1, x2, bk = setup(B=2, n=24)
    a = rv.feed_forward(x1, W["w1"], W["b1"], W["w2"], W["b2"], 48)
    for c in (1, 5, 16):  # the library matmul may block differently: equal to rounding
        np.testing.assert_allclose(rv.feed_forward(x1, W["w1"], W["b1"], W["w2"], W["b2"], c), a,
                                   rtol=0, atol=1e-13)


def test_feed_forward_one_row_by_hand():
    W, x1, _, _ = setup()
    row = x1[0, 3]
    h = [max(0.0, sum(W["w1"][j, k] * row[k] for k in range(row.size)) + W["b1"][j])
         for j in range(W["w1"].shape[0])]
    want = [sum(W["w2"][i, j] * h[j] for j in range(len(h))) + W["b2"][i]
            for i in range(W["w2"].shape[0])]
    got = rv.feed_forward(x1, W["w1"], W["b1"], W["w2"], W["b2"], 7)[0, 3]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_zero_output_weights_leave_the_halves():
    W, x1, x2, bk = setup()
    W = dict(W, w_o=np.zeros_like(W["w_o"]), w2=np.zeros_like(W["w2"]), b2=np.zeros(16))
    y1, y2 = rv.block(x1, x2, W, bk, 2, 8, True, 16)
    np.testing.assert_array_equal(y1, x1)
    np.testing.assert_array_equal(y2, x2)


def test_identity_projections_give_the_lsh_attention_of_each_head():
    """W_qk = W_v = W_o = I: the attention sublayer is the LSH forward of the
    heads of x2, concatenated."""
    W, _, x2, bk = setup(heads=2, dh=8)
    eye = np.eye(16)
    att = rv.attention(x2, eye, eye, eye, bk, 2, 8, True)
    heads = np.ascontiguousarray(x2.reshape(1, 32, 2, 8).transpose(0, 2, 1, 3))
    out, _, _ = oracle.forward(heads, heads, np.zeros((2, 8, 2)), 8, True, buckets=bk)
    np.testing.assert_allclose(att, out.transpose(0, 2, 1, 3).reshape(1, 32, 16), rtol=0, atol=1e-13)


def test_projections_and_head_split_by_hand():
    """W_o = I: the features [h dh, (h + 1) dh) of the attention sublayer are
    the LSH attention of head h, whose shared-QK and value rows are
    qk_i[k] = sum_j W_qk[h dh + k, j] x_i[j] (and likewise v), written out."""
    W, _, x2, bk = setup(heads=2, dh=8)
    att = rv.attention(x2, W["w_qk"], W["w_v"], np.eye(16), bk, 2, 8, True)
    n, dm, dh = 32, 16, 8
    for h in range(2):
        qk = np.array([[sum(W["w_qk"][h * dh + k, j] * x2[0, i, j] for j in range(dm))
                        for k in range(dh)] for i in range(n)])
        v = np.array([[sum(W["w_v"][h * dh + k, j] * x2[0, i, j] for j in range(dm))
                       for k in range(dh)] for i in range(n)])
        pos = np.arange(n, dtype=np.int32)
        o, _ = oracle.forward_sampled(qk[None, None], v[None, None], bk[:, h:h + 1], 4, 8, True, pos)
        np.testing.assert_allclose(att[0, :, h * dh:(h + 1) * dh], o[0, 0], rtol=0, atol=1e-12)


def test_block_wiring():
    """y1 - x1 is the attention of x2 and y2 - x2 the feed-forward of y1."""
    W, x1, x2, bk = setup()
    y1, y2 = rv.block(x1, x2, W, bk, 2, 8, True, 16)
    np.testing.assert_allclose(y1 - x1, rv.attention(x2, W["w_qk"], W["w_v"], W["w_o"], bk, 2, 8,
                                                     True), rtol=0, atol=1e-12)
    np.testing.assert_allclose(y2 - x2, rv.feed_forward(y1, W["w1"], W["b1"], W["w2"], W["b2"], 32),
                               rtol=0, atol=1e-12)
    # and not of the other half
    assert np.abs(y2 - x2 - rv.feed_forward(x1, W["w1"], W["b1"], W["w2"], W["b2"], 32)).max() > 1e-3
