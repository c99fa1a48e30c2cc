"""The in-bucket top-k variant through the C ABI against its oracle
(oracle/topk_variant.py, pinned on the CPU). Bucket codes and top-k sets
are fp64 decisions taken in the same order on both sides: every round's
top-k list must equal the oracle's element for element (position and rank).
Outputs: bf16 bar as for the chunked attention (max abs <= 2e-2, mean abs
<= 2e-3)."""
import numpy as np
import pytest
import torch

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I
from oracle import topk_variant as tv

pytestmark = pytest.mark.gpu

CASES = [  # name, B, H, n, d, K, m, k, rounds, causal, clustered
    ("k8-causal", 1, 2, 512, 64, 8, 3, 8, 2, True, False),
    ("k16-noncausal-d128", 1, 1, 384, 128, 16, 4, 16, 3, False, False),
    ("k32-clustered", 1, 2, 512, 64, 8, 5, 32, 2, True, True),
    ("k5-mod-6", 2, 1, 256, 64, 6, 7, 5, 1, True, False),
]


def run(name, B, H, n, d, K, m, k, R, causal, clu, heads=None):
    w = I.Workload(name, B, H, n, d, K, 64, R, causal, "bf16", clustered=clu)
    x, v = I.make_qkv(w)
    proj = I.make_topk_projections(R, d, m)
    out, lse, cand = lb.lsh_topk_forward(x.cuda(), v.cuda(), proj.cuda(), n_buckets=K, top_k=k,
                                         causal=causal, return_candidates=True)
    out, lse, cand = out.float().cpu().numpy(), lse.cpu().numpy(), cand.cpu().numpy()
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    for b, h in heads:
        xs = x[b, h].double().numpy()
        for r in range(R):
            bucket = tv.simhash_buckets(xs, proj[r].double().numpy(), K)
            ref = tv.topk_round(xs, bucket, k, causal)
            for i in range(n):
                got = cand[b, h, r, i]
                want = np.full(k, -1)
                want[:len(ref[i])] = ref[i]
                assert np.array_equal(got, want), (name, b, h, r, i, got, want)
        c = tv.candidates(xs, proj.double().numpy(), K, k, causal)
        ro, rl = tv.attend(xs, v[b, h].double().numpy(), c)
        for what, g_, r_ in (("out", out[b, h], ro), ("lse", lse[b, h], rl)):
            err = np.abs(g_ - r_)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3, (name, what, err.max(), err.mean())


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_topk_variant_matches_oracle(case):
    run(*case)


def test_topk_variant_page_config_sampled_heads():
    """The page's setting: two rounds, 64 buckets, top 32 (6-bit codes), at
    n = 4096 with 8 heads; two heads checked in full."""
    run("page-config", 1, 8, 4096, 64, 64, 6, 32, 2, True, False, heads=[(0, 0), (0, 5)])
