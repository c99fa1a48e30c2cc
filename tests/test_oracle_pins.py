"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, an invariant of the hash, a special case that reduces to textbook dense
attention or to a library sort, brute force on tiny inputs, or a hand-worked
example under tests/golden/. CPU only.

Sources (page title, section):
  "Reformer summary" (ttnews.xyz): §局部敏感哈希 (hash definition),
      §局部敏感哈希注意力 (sort by bucket then position, chunks of m),
      §多輪LSH哈希 (several rounds), §共享QK中的自掩碼 (self-mask).
  "Reformer: LSH attention and reversible layers" (dtcms.com): §二.1
      (unit-length keys, softmax(QK^T / sqrt(d_k)) V).
  "Reformer re-reading" (2kiu.com) §2.2: for one random projection the
      collision probability of two vectors at angle theta is 1 - theta/pi.
  "Reformer news article" (xaznjj.net): bucket sizes are similar with high
      probability.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SELF = -1.0e5


# --------------------------------------------------------------------------
# helpers independent of the oracle
def dense_attention(x, v, causal):
    """Textbook dense shared-QK attention (one sequence): unit keys, 1/sqrt(d)
    scale, self logit -1e5, additive causal mask, softmax, weighted sum."""
    n, d = x.shape
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    logits = (x @ k.T) / math.sqrt(d)
    np.fill_diagonal(logits, SELF)
    if causal:
        logits = np.where(np.triu(np.ones((n, n), bool), 1), -np.inf, logits)
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ v, (mx + np.log(z))[:, 0]


def rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# golden, hand-worked cases
def _hash_cases():
    out = []
    with open(os.path.join(GOLDEN, "hash_ties.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, d, nb, R, x, b, _ = [t.strip() for t in line.split("|")]
            d, nb, b = int(d), int(nb), int(b)
            R = np.array([[float(t) for t in row.split(",")] for row in R.split(";")])
            x = np.array([float(t) for t in x.split(",")])
            assert R.shape == (d, nb // 2) and x.shape == (d,)
            out.append((name, x, R, b))
    return out


@pytest.mark.parametrize("name,x,R,expect", _hash_cases(), ids=[c[0] for c in _hash_cases()])
def test_hash_golden(name, x, R, expect):
    b, _ = oracle.hash_rows(x[None, :], R)
    assert b[0] == expect


def _attention_golden():
    env = {"sqrt2": math.sqrt(2.0), "exp": math.exp, "log": math.log}
    vals = {}
    with open(os.path.join(GOLDEN, "attention_3tok.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, expr = line.split("=", 1)
            # the fixture holds plain arithmetic on earlier names only
            vals[key.strip()] = eval(expr, {"__builtins__": {}}, {**env, **vals})
    return vals


@pytest.mark.parametrize("causal", [False, True])
def test_attention_golden(causal):
    g = _attention_golden()
    x = np.array(g["x"], float)
    v = np.array(g["v"], float)
    # one round, a single chunk: every bucket assignment gives the same answer
    for bk in ([0, 0, 0], [1, 0, 1], [2, 1, 0]):
        perm, inv = oracle.sort(np.array(bk), 3)
        out, lse = oracle.attend_slots(x, v, perm, m=4, causal=causal)
        pre = "c_" if causal else ""
        for i in range(3):
            s = inv[i]
            np.testing.assert_allclose(out[s], g[f"{pre}out{i}"], rtol=0, atol=1e-14)
            assert abs(lse[s] - g[f"{pre}lse{i}"]) <= 1e-12


# --------------------------------------------------------------------------
# dense equivalence: one round and m >= n is one chunk holding everything
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("m_over_n", [1, 3])
def test_dense_equivalence(causal, m_over_n):
    r = rng(11)
    B, H, n, d, nb = 2, 3, 40, 16, 8
    x = r.standard_normal((B, H, n, d))
    v = r.standard_normal((B, H, n, d))
    R = r.standard_normal((1, d, nb // 2))
    out, lse, _ = oracle.forward(x, v, R, chunk=m_over_n * n, causal=causal)
    for b in range(B):
        for h in range(H):
            o_ref, l_ref = dense_attention(x[b, h], v[b, h], causal)
            np.testing.assert_allclose(out[b, h], o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h, 0], l_ref, rtol=0, atol=1e-10)


def test_dense_equivalence_any_buckets():
    """With a single chunk the sort cannot change the answer."""
    r = rng(12)
    n, d, nb = 32, 8, 6
    x = r.standard_normal((1, 1, n, d))
    v = r.standard_normal((1, 1, n, d))
    R = r.standard_normal((1, d, nb // 2))
    o_ref, l_ref = dense_attention(x[0, 0], v[0, 0], True)
    for seed in range(4):
        bk = rng(100 + seed).integers(0, nb, (1, 1, 1, n)).astype(np.int32)
        out, lse, _ = oracle.forward(x, v, R, chunk=n, causal=True, buckets=bk)
        np.testing.assert_allclose(out[0, 0], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0, 0], l_ref, rtol=0, atol=1e-10)


# --------------------------------------------------------------------------
# hash invariants
def test_hash_zero_vector_is_bucket_zero():
    R = rng(1).standard_normal((16, 12))
    b, mg = oracle.hash_rows(np.zeros((3, 16)), R)
    assert (b == 0).all() and (mg == 0).all()


def test_hash_basis_vector_selects_row_of_R():
    """x = s e_k projects to row k of R: h is the first argmax of [R_k ; -R_k]."""
    r = rng(2)
    d, nb = 12, 10
    R = r.standard_normal((d, nb // 2))
    for k in range(d):
        for s in (0.5, 3.0):
            x = np.zeros((1, d))
            x[0, k] = s
            b, _ = oracle.hash_rows(x, R)
            assert b[0] == int(np.argmax(np.concatenate([R[k], -R[k]])))


def test_hash_one_projection_is_a_sign_bit():
    """nb = 2: bucket 0 when x.r >= 0, else bucket 1 (angular LSH, one bit)."""
    r = rng(3)
    d = 24
    Rv = r.standard_normal((d, 1))
    x = r.standard_normal((500, d))
    b, _ = oracle.hash_rows(x, Rv)
    expect = np.where(x @ Rv[:, 0] >= 0, 0, 1)
    assert (b == expect).all()


def test_hash_positive_rescaling():
    r = rng(4)
    d, nb = 32, 64
    R = r.standard_normal((d, nb // 2))
    x = r.standard_normal((2000, d))
    b0, mg = oracle.hash_rows(x, R)
    for s in (2.0 ** -7, 0.25, 8.0, 2.0 ** 20):  # exact in binary: identical projections up to scale
        b, _ = oracle.hash_rows(x * s, R)
        assert (b == b0).all()
    for s in (0.3, 1.7, 123.456):
        b, _ = oracle.hash_rows(x * s, R)
        safe = mg > 1e-9 * max(1.0, s)
        assert (b[safe] == b0[safe]).all()


def test_hash_antipodal():
    """h(-x) = (h(x) + nb/2) mod nb whenever the top-2 margin is not zero."""
    r = rng(5)
    d, nb = 16, 20
    R = r.standard_normal((d, nb // 2))
    x = r.standard_normal((3000, d))
    b, mg = oracle.hash_rows(x, R)
    bn, _ = oracle.hash_rows(-x, R)
    ok = mg > 0
    assert ok.mean() > 0.99
    assert (bn[ok] == (b[ok] + nb // 2) % nb).all()


def test_hash_collision_rate_matches_angle():
    """nb = 2 over many independent R: P[h(x) = h(y)] = 1 - theta/pi."""
    d, trials = 16, 4000
    r = rng(6)
    u = r.standard_normal(d)
    u /= np.linalg.norm(u)
    w = r.standard_normal(d)
    w -= (w @ u) * u
    w /= np.linalg.norm(w)
    thetas = [math.pi / 6, math.pi / 3, math.pi / 2, 2 * math.pi / 3]
    xy = np.stack([u] + [math.cos(t) * u + math.sin(t) * w for t in thetas])
    hits = np.zeros(len(thetas))
    for s in range(trials):
        R = np.random.default_rng(10_000 + s).standard_normal((d, 1))
        b, _ = oracle.hash_rows(xy, R)
        hits += b[1:] == b[0]
    for t, h in zip(thetas, hits):
        p = 1 - t / math.pi
        sigma = math.sqrt(p * (1 - p) / trials)
        assert abs(h / trials - p) < 4 * sigma, (t, h / trials, p)


def test_hash_buckets_near_uniform_over_seeds():
    """Isotropic x, pooled over many R seeds: chi-square within 5 sigma of uniform."""
    d, nb, seeds, per = 64, 16, 256, 64
    counts = np.zeros(nb)
    for s in range(seeds):
        g = np.random.default_rng(20_000 + s)
        R = g.standard_normal((d, nb // 2))
        x = g.standard_normal((per, d))
        b, _ = oracle.hash_rows(x, R)
        counts += np.bincount(b, minlength=nb)
    expect = seeds * per / nb
    chi2 = ((counts - expect) ** 2 / expect).sum()
    dof = nb - 1
    assert chi2 < dof + 5 * math.sqrt(2 * dof), chi2


def test_hash_all_matches_rows():
    r = rng(7)
    x = r.standard_normal((2, 3, 50, 8))
    R = r.standard_normal((3, 8, 5))
    b, mg = oracle.hash_all(x, R)
    for bi in range(2):
        for h in range(3):
            for rr in range(3):
                b1, m1 = oracle.hash_rows(x[bi, h], R[rr])
                assert (b[bi, h, rr] == b1).all()
                assert (mg[bi, h, rr] == m1).all()


# --------------------------------------------------------------------------
# sort
@pytest.mark.parametrize("n,nb", [(1, 2), (7, 4), (1000, 16), (4096, 64), (333, 200)])
def test_sort_is_the_stable_bucket_order(n, nb):
    b = rng(n + nb).integers(0, nb, n).astype(np.int32)
    perm, inv = oracle.sort(b, nb)
    assert sorted(perm.tolist()) == list(range(n))
    assert (inv[perm] == np.arange(n)).all()
    keys = b[perm]
    assert (np.diff(keys) >= 0).all()
    same = np.diff(keys) == 0
    assert (np.diff(perm)[same] > 0).all()
    # the unique answer, from the library's stable sort
    assert perm.tolist() == sorted(range(n), key=lambda i: (b[i], i))


def test_sort_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.sort(np.array([0, 5, 1], np.int32), 4)


# --------------------------------------------------------------------------
# chunk membership, one-hot values
def _expected_keys(perm, inv, i, m, causal):
    n = len(perm)
    s = inv[i]
    c = s // m
    lo = max(c - 1, 0) * m
    keys = {int(perm[j]) for j in range(lo, (c + 1) * m)}
    if causal:
        keys = {k for k in keys if k <= i}
    return keys


@pytest.mark.parametrize("m", [4, 8, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_chunk_membership_one_hot(m, causal):
    n, nb = 64, 8
    r = rng(30 + m)
    x = r.standard_normal((n, n))
    v = np.eye(n)  # value j is the one-hot tag of position j (d = n)
    b = r.integers(0, nb, n).astype(np.int32)
    perm, inv = oracle.sort(b, nb)
    out, lse = oracle.attend_slots(x, v, perm, m, causal)
    for i in range(n):
        w = out[inv[i]]
        keys = _expected_keys(perm, inv, i, m, causal)
        others = keys - {i}
        support = set(np.nonzero(w)[0].tolist())
        if others:
            assert support == others, (i, support, others)
        else:  # nothing else available: the token attends to itself
            assert support == {i}
            assert lse[inv[i]] == SELF
        assert abs(w.sum() - 1) < 1e-12


def test_first_position_causal_sees_itself_only():
    r = rng(40)
    B, H, n, d, nb, rounds = 1, 2, 256, 16, 16, 3
    x = r.standard_normal((B, H, n, d))
    v = r.standard_normal((B, H, n, d))
    R = r.standard_normal((rounds, d, nb // 2))
    out, lse, _ = oracle.forward(x, v, R, chunk=32, causal=True)
    assert (lse[:, :, :, 0] == SELF).all()
    # every round gives v_0 with weight 1/rounds after the merge
    np.testing.assert_allclose(out[:, :, 0], v[:, :, 0], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# round merge
def test_identical_rounds_equal_one_round():
    r = rng(50)
    B, H, n, d, nb = 1, 2, 128, 16, 8
    x = r.standard_normal((B, H, n, d))
    v = r.standard_normal((B, H, n, d))
    R1 = r.standard_normal((1, d, nb // 2))
    o1, l1, _ = oracle.forward(x, v, R1, chunk=16, causal=True)
    o4, l4, _ = oracle.forward(x, v, np.repeat(R1, 4, axis=0), chunk=16, causal=True)
    # self-only rows carry lse = -1e5, whose fp64 ulp (~1.5e-11) bounds the
    # rounding of the merge weights exp(lse - logsumexp) = 1/4
    np.testing.assert_allclose(o4, o1, rtol=0, atol=1e-10)
    for k in range(4):
        np.testing.assert_array_equal(l4[:, :, k], l1[:, :, 0])


@pytest.mark.parametrize("causal", [False, True])
def test_merge_is_softmax_over_union_of_candidates(causal):
    """Second formulation: one softmax over the multiset union of every round's
    candidate list (logits from the definition) equals the merged output."""
    r = rng(60)
    n, d, nb, m, rounds = 48, 8, 6, 8, 3
    x = r.standard_normal((1, 1, n, d))
    v = r.standard_normal((1, 1, n, d))
    R = r.standard_normal((rounds, d, nb // 2))
    out, lse, bk = oracle.forward(x, v, R, chunk=m, causal=causal)
    xs, vs = x[0, 0], v[0, 0]
    perms = [oracle.sort(bk[0, 0, k], nb) for k in range(rounds)]
    for i in range(n):
        logits, vals = [], []
        for perm, inv in perms:
            for j in _expected_keys(perm, inv, i, m, causal):
                if j == i:
                    logits.append(SELF)
                else:
                    logits.append(xs[i] @ xs[j] / np.linalg.norm(xs[j]) / math.sqrt(d))
                vals.append(vs[j])
        logits = np.array(logits)
        mx = logits.max()
        w = np.exp(logits - mx)
        ref = (w[:, None] * np.array(vals)).sum(0) / w.sum()
        np.testing.assert_allclose(out[0, 0, i], ref, rtol=0, atol=1e-12)
        L = np.logaddexp.reduce(lse[0, 0, :, i])
        assert abs(L - (mx + math.log(w.sum()))) < 1e-10


def test_merge_weights_closed_form():
    """Two rounds with lse a, b: weights 1/(1+e^(b-a)) and 1/(1+e^(a-b))."""
    o = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    lse = np.array([[0.3], [-1.2]])
    out, L = oracle.merge(o, lse)
    wa = 1 / (1 + math.exp(-1.2 - 0.3))
    np.testing.assert_allclose(out[0], [wa, 1 - wa], rtol=0, atol=1e-15)
    assert abs(L[0] - (0.3 + math.log1p(math.exp(-1.5)))) < 1e-15


# --------------------------------------------------------------------------
# sampled forward agrees with the full forward
def test_sampled_forward_matches_full():
    r = rng(70)
    B, H, n, d, nb, rounds, m = 2, 2, 256, 16, 16, 2, 32
    x = r.standard_normal((B, H, n, d))
    v = r.standard_normal((B, H, n, d))
    R = r.standard_normal((rounds, d, nb // 2))
    out, lse, bk = oracle.forward(x, v, R, chunk=m, causal=True)
    pos = np.array([0, 5, 31, 32, 100, 255], np.int32)
    so, sl = oracle.forward_sampled(x, v, bk, nb, m, True, pos)
    np.testing.assert_array_equal(so, out[:, :, pos])
    np.testing.assert_array_equal(sl, lse[:, :, :, pos])


@pytest.mark.parametrize("causal", [True, False])
def test_dense_sampled_is_textbook_dense_attention(causal):
    """oracle.dense_sampled (the baseline's reference) against the textbook
    dense attention written above, at every position of two heads."""
    g = rng(31)
    x = g.standard_normal((1, 2, 40, 8))
    v = g.standard_normal((1, 2, 40, 8))
    pos = np.arange(40, dtype=np.int32)
    out, lse = oracle.dense_sampled(x, v, causal, pos)
    for h in range(2):
        o_ref, l_ref = dense_attention(x[0, h], v[0, h], causal)
        np.testing.assert_allclose(out[0, h], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], l_ref, rtol=0, atol=1e-10)
