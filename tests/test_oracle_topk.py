"""Pins of the top-k variant's oracle (oracle/topk_variant.py), each against
something other than itself: the SimHash collision rate the page states,
the binary code for K = 2^m, the ordering property of a top-k set, the
union of identical rounds, and dense attention when one bucket holds
everything and k covers it."""
import numpy as np
import pytest

from oracle import topk_variant as tv

from test_oracle_pins import dense_attention


def test_simhash_bit_collision_rate_is_one_minus_angle_over_pi():
    """"Reformer re-reading", §2.2: for one projection, two vectors share the
    bit with probability 1 - theta/pi. Monte Carlo over 20000 projections."""
    g = np.random.default_rng(1)
    d = 16
    for theta in (0.3, 1.1, 2.4):
        u = np.zeros(d); u[0] = 1.0
        w = np.zeros(d); w[0] = np.cos(theta); w[1] = np.sin(theta)
        proj = g.standard_normal((d, 20000))
        bu = (u @ proj > 0)
        bw = (w @ proj > 0)
        rate = (bu == bw).mean()
        assert abs(rate - (1 - theta / np.pi)) < 4 * np.sqrt(0.25 / 20000), (theta, rate)
        # and simhash_buckets takes exactly that bit for m = 1, K = 2
        for t in range(5):
            assert tv.simhash_buckets(u[None], proj[:, t:t + 1], 2)[0] == int(bu[t])


def test_code_is_the_binary_number_of_the_bits_for_K_a_power_of_two():
    g = np.random.default_rng(2)
    x = g.standard_normal((50, 8))
    proj = g.standard_normal((8, 5))
    b = tv.simhash_buckets(x, proj, 32)
    p = x @ proj
    want = sum((p[:, t] > 0).astype(int) << t for t in range(5))
    np.testing.assert_array_equal(b, want)
    # modulo K: K = 3 folds the same codes
    np.testing.assert_array_equal(tv.simhash_buckets(x, proj, 3), want % 3)


@pytest.mark.parametrize("causal", [True, False])
def test_topk_sets_hold_the_best_keys_of_the_bucket(causal):
    g = np.random.default_rng(3)
    n, d, k = 64, 8, 5
    x = g.standard_normal((n, d))
    bucket = g.integers(0, 4, n)
    sets = tv.topk_round(x, bucket, k, causal)
    for i, s in enumerate(sets):
        pool = [j for j in range(n) if bucket[j] == bucket[i] and (not causal or j <= i)]
        assert len(s) == min(k, len(pool)) and set(s) <= set(pool)
        inside = tv.scores(x, i, s)
        rest = [j for j in pool if j not in set(s)]
        if rest:  # every key left out scores no better than the worst kept one
            assert tv.scores(x, i, rest).max() <= inside.min()


def test_identical_rounds_give_one_rounds_candidates():
    g = np.random.default_rng(4)
    x = g.standard_normal((40, 8))
    proj = g.standard_normal((8, 3))
    one = tv.candidates(x, proj[None], 8, 4, True)
    two = tv.candidates(x, np.stack([proj, proj]), 8, 4, True)
    for a, b in zip(one, two):
        np.testing.assert_array_equal(a, np.sort(b))


@pytest.mark.parametrize("causal", [True, False])
def test_one_bucket_and_large_k_is_dense_attention(causal):
    g = np.random.default_rng(5)
    n, d = 24, 8
    x = g.standard_normal((1, 1, n, d))
    v = g.standard_normal((1, 1, n, d))
    projs = g.standard_normal((2, d, 3))
    out, lse, _ = tv.forward(x, v, projs, K=1, k=n, causal=causal)
    o_ref, l_ref = dense_attention(x[0, 0], v[0, 0], causal)
    np.testing.assert_allclose(out[0, 0], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], l_ref, rtol=0, atol=1e-10)
