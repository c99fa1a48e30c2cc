"""The in-bucket top-k variant of LSH attention described in "Reformer
re-reading" (2kiu.com), §2.2 and §2.3, as a second workload beside the
chunked attention; float64 numpy, step by step.

TEST INFRASTRUCTURE ONLY, like the rest of this package: it shares no code
with the CUDA path.

Steps, as the page lists them:
  1. Rounds l = 0..L-1, each with m random projections r_t ~ N(0, I_d). Bit
     t of a vector x is [r_t . x > 0]; the m bits form the code
     sum_t bit_t 2^t, and the bucket is the code mod K.
  2. Within its bucket, a query ranks the keys by their score against it and
     keeps the top k.
  3. The candidates of a query are the union of its top-k over the rounds.
Readings taken (the page leaves them open; see also the design notes):
  * shared-QK: keys and queries are the same vectors x, values v;
  * the score is the chunked attention's logit, x_i . x_j / (||x_j|| sqrt(d))
    (0 for a zero key), with -1e5 for the query itself, and under the causal
    mask only keys at positions <= the query's are candidates;
  * ranking: higher score first, the lower position on equal scores; a
    bucket with fewer than k candidates keeps them all;
  * the attention over the union is one softmax of those logits (two-pass:
    maximum, then sums), out = softmax-weighted v, lse = log-normaliser;
  * the page's "bucket shifting" is not restated (its text is garbled) and
    is not part of this workload.
Every score that decides membership is computed in one fixed order (sums
over k in increasing order, no fused multiply-add, then the norm, the
division and the 1/sqrt(d)), so that an implementation taking the same
fp64 steps reaches the same integer decisions.
"""
from __future__ import annotations

import numpy as np

SELF_LOGIT = -1.0e5


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def simhash_buckets(x, proj, K: int):
    """x [n, d], proj [d, m] -> bucket [n] int: sum_t [proj_t . x > 0] 2^t mod K."""
    x, proj = _f64(x), _f64(proj)
    n, d = x.shape
    p = np.zeros((n, proj.shape[1]))
    for k in range(d):  # increasing k, products then sums (no fused multiply-add)
        p = p + x[:, k:k + 1] * proj[k][None, :]
    bits = (p > 0).astype(np.int64)
    code = np.zeros(n, np.int64)
    for t in reversed(range(proj.shape[1])):  # Horner: sum_t bit_t 2^t mod K
        code = (2 * code + bits[:, t]) % K
    return code


def scores(x, i: int, js):
    """Logits of query i against keys js (fixed operation order)."""
    x = _f64(x)
    d = x.shape[1]
    js = np.asarray(js, np.int64)
    dot = np.zeros(js.size)
    nn = np.zeros(js.size)
    for k in range(d):
        dot = dot + x[i, k] * x[js, k]
        nn = nn + x[js, k] * x[js, k]
    nrm = np.sqrt(nn)
    l = np.where(nrm > 0, (dot / np.where(nrm > 0, nrm, 1.0)) / np.sqrt(float(d)), 0.0)
    return np.where(js == i, SELF_LOGIT, l)


def topk_round(x, bucket, k: int, causal: bool):
    """Per query, its top-k keys (positions, ordered best first) in its bucket."""
    n = bucket.shape[0]
    out = []
    for i in range(n):
        js = np.nonzero(bucket == bucket[i])[0]
        if causal:
            js = js[js <= i]
        l = scores(x, i, js)
        order = np.lexsort((js, -l))  # higher score first, then lower position
        out.append(js[order[:k]])
    return out


def candidates(x, projs, K: int, k: int, causal: bool):
    """projs [L, d, m] -> per query the sorted union of its per-round top-k."""
    per_round = [topk_round(x, simhash_buckets(x, projs[l], K), k, causal)
                 for l in range(len(projs))]
    n = _f64(x).shape[0]
    return [np.unique(np.concatenate([pr[i] for pr in per_round])) for i in range(n)]


def attend(x, v, cand):
    """Softmax attention of every query over its candidate positions."""
    x, v = _f64(x), _f64(v)
    n, d = x.shape
    out = np.zeros((n, v.shape[1]))
    lse = np.zeros(n)
    for i in range(n):
        js = cand[i]
        l = scores(x, i, js)
        M = l.max()
        e = np.exp(l - M)
        Z = e.sum()
        out[i] = (e[:, None] * v[js]).sum(0) / Z
        lse[i] = M + np.log(Z)
    return out, lse


def forward(x, v, projs, K: int, k: int, causal: bool):
    """x, v [B, H, n, d]; projs [L, d, m]. Returns (out [B, H, n, d],
    lse [B, H, n], candidates per (b, h) as lists of position arrays)."""
    x, v, projs = _f64(x), _f64(v), _f64(projs)
    B, H, n, d = x.shape
    out = np.zeros_like(v)
    lse = np.zeros((B, H, n))
    cands = []
    for b in range(B):
        for h in range(H):
            c = candidates(x[b, h], projs, K, k, causal)
            out[b, h], lse[b, h] = attend(x[b, h], v[b, h], c)
            cands.append(c)
    return out, lse, cands
