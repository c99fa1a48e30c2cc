"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: bucket ids and sort permutations bit-exact, except hash disagreements
where the oracle's top-2 margin is below 1e-5 (counted and printed); outputs
compared with identical bucket ids on both sides: fp32 max abs <= 1e-4; bf16
max abs <= 2e-2 and mean abs <= 2e-3. lse is held to the same bounds.

Inputs come from lsh_attention_b200.inputs (seeded); oracle inputs never come
from the GPU. Large workloads are checked on sampled heads and positions.
"""
import numpy as np
import pytest
import torch

import oracle
from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu

TIE_MARGIN = 1e-5


def tol(dtype):
    return (1e-4, None) if dtype == "f32" else (2e-2, 2e-3)


def check_close(gpu, ref, dtype, what):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    mx, mean_lim = tol(dtype)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    assert err.max() <= mx, f"{what}: max abs {err.max():.3e} > {mx}"
    if mean_lim is not None:
        assert err.mean() <= mean_lim, f"{what}: mean abs {err.mean():.3e} > {mean_lim}"
    return float(err.max()), float(err.mean())


def check_buckets(gpu, ref, margin, what):
    gpu = np.asarray(gpu)
    diff = gpu != ref
    bad = diff & (margin >= TIE_MARGIN)
    assert not bad.any(), f"{what}: {int(bad.sum())} bucket ids differ with margin >= {TIE_MARGIN}"
    n_tie = int(diff.sum())
    print(f"{what}: {n_tie} near-tie disagreements of {gpu.size}")
    return n_tie


def to_gpu(*ts):
    return [t.cuda() for t in ts]


def sample_positions(n, k=192, seed=3):
    g = np.random.default_rng(seed)
    pos = set([0, 1, n - 1, n // 2]) | set(g.integers(0, n, k).tolist())
    return np.array(sorted(p for p in pos if 0 <= p < n), np.int32)


SMALL = [I.TINY_F32, I.BF16_SHORT]
# the n x rounds sweep, isotropic and clustered: 16 points with n <= 8K
# checked in full, 16 with n >= 32K checked on sampled heads and positions
SWEEP_SMALL = [w for w in I.sweep_workloads() if w.n <= 8192]
SWEEP_LARGE = [w for w in I.sweep_workloads() if w.n >= 32768]


# --------------------------------------------------------------------------
# hash
@pytest.mark.parametrize("w", SMALL + [I.IMAGE_12K.with_(batch=2)] + SWEEP_SMALL[::3],
                         ids=lambda w: w.name)
def test_hash_full(w):
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    ref, margin = oracle.hash_all(x, R)
    xg, Rg = to_gpu(x, R)
    got = lb.lsh_attn_hash(xg, Rg, w.n_buckets).cpu().numpy()
    check_buckets(got, ref, margin, w.name)


# Epilogue forms of the tensor-core hash: a round of at most 128 projected
# columns (b <= 256) is taken whole by one warp per quadrant, the warps taking
# rounds in turn across tiles; wider rounds are split over the warps. These
# cases cover one and two rounds per tile, rounds spread over several CTA
# groups (16 rounds of resident R do not fit one CTA), and both head sizes.
HASH_FORMS = [
    I.LONG_64K.with_(name="h-d128-b256-R16", heads=2, n=16384, n_buckets=256, rounds=16),
    I.LONG_64K.with_(name="h-d128-b256-R2", heads=2, n=16384, n_buckets=256, rounds=2),
    I.LONG_64K.with_(name="h-d64-b32-R1", heads=3, n=16384, d=64, n_buckets=32, rounds=1),
    I.LONG_64K.with_(name="h-d64-b128-R5", heads=2, n=8192 + 77, d=64, n_buckets=128, rounds=5),
    I.LONG_64K.with_(name="h-d128-b512-R3", heads=2, n=16384, n_buckets=512, rounds=3),
]


@pytest.mark.parametrize("w", HASH_FORMS, ids=lambda w: w.name)
def test_hash_epilogue_forms(w):
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    ref, margin = oracle.hash_all(x, R)
    xg, Rg = to_gpu(x, R)
    got = lb.lsh_attn_hash(xg, Rg, w.n_buckets).cpu().numpy()
    check_buckets(got, ref, margin, w.name)


@pytest.mark.parametrize("w", [I.LONG_64K, I.IMAGE_12K] + SWEEP_LARGE, ids=lambda w: w.name)
def test_hash_sampled_tokens(w):
    """Full-size launch; the oracle re-derives a sample of (b, h, token) rows."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, Rg = to_gpu(x, R)
    got = lb.lsh_attn_hash(xg, Rg, w.n_buckets).cpu().numpy()
    g = np.random.default_rng(5)
    for b in range(w.batch):
        for h in {0, w.heads - 1}:
            tok = np.unique(np.concatenate([[0, w.n - 1], g.integers(0, w.n, 2048)]))
            for r in range(w.rounds):
                ref, margin = oracle.hash_rows(x[b, h, tok], R[r])
                check_buckets(got[b, h, r, tok], ref, margin, f"{w.name} b{b} h{h} r{r}")


# --------------------------------------------------------------------------
# sort and gather
@pytest.mark.parametrize("w", SMALL + [I.IMAGE_12K, I.LONG_64K] + SWEEP_LARGE[:2],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("kind", ["uniform", "skewed"])
def test_sort_bit_exact(w, kind):
    if kind == "uniform":
        bk = I.make_buckets(w)
    else:  # heavy skew: most tokens in a handful of buckets, plus one full bucket
        g = torch.Generator().manual_seed(9)
        bk = torch.randint(0, 4, (w.batch, w.heads, w.rounds, w.n), generator=g,
                           dtype=torch.int64).to(torch.int32)
        bk[..., ::7] = w.n_buckets - 1
        bk[0, 0, 0] = w.n_buckets // 2
    bkg = bk.cuda()
    perm = lb.lsh_attn_sort(bkg, w.n_buckets, d=w.d, dtype=I.torch_dtype(w.dtype)).cpu().numpy()
    bn = bk.numpy()
    for b in range(w.batch):
        for h in range(w.heads):
            for r in range(w.rounds):
                ref, _ = oracle.sort(bn[b, h, r], w.n_buckets)
                np.testing.assert_array_equal(perm[b, h, r], ref)


@pytest.mark.parametrize("w", [I.TINY_F32, I.BF16_SHORT, I.IMAGE_12K.with_(batch=1)],
                         ids=lambda w: w.name)
def test_gather_rows_follow_perm(w):
    x, v = I.make_qkv(w)
    bk = I.make_buckets(w)
    xg, vg, bkg = to_gpu(x, v, bk)
    perm, xs, vs = lb.lsh_attn_sort(bkg, w.n_buckets, x=xg, v=vg)
    bn = bk.numpy()
    for b in range(w.batch):
        for h in range(w.heads):
            for r in range(w.rounds):
                p, _ = oracle.sort(bn[b, h, r], w.n_buckets)
                p = torch.from_numpy(p.astype(np.int64))
                assert torch.equal(xs[b, h, r].cpu(), x[b, h][p])
                assert torch.equal(vs[b, h, r].cpu(), v[b, h][p])


# --------------------------------------------------------------------------
# forward
def oracle_buckets(w, x, R):
    b, _ = oracle.hash_all(x, R)
    return torch.from_numpy(b)


@pytest.mark.parametrize("w", SMALL + SWEEP_SMALL, ids=lambda w: w.name)
def test_forward_full(w):
    """Whole outputs against the oracle, identical buckets on both sides."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    bk = oracle_buckets(w, x, R)
    ref_out, ref_lse, _ = oracle.forward(x, v, R, w.chunk, w.causal, buckets=bk)
    xg, vg, bkg = to_gpu(x, v, bk)
    out, lse = lb.lsh_attn_forward(xg, vg, None, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=w.causal, buckets=bkg)
    mo = check_close(out.float().cpu().numpy(), ref_out, w.dtype, f"{w.name} out")
    ml = check_close(lse.cpu().numpy(), ref_lse, w.dtype, f"{w.name} lse")
    print(f"{w.name}: out max/mean {mo}, lse max/mean {ml}")


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_internal_hash(w):
    """buckets=NULL hashes inside the call: the GPU's bucket ids must equal the
    oracle's bit for bit (no near-tie allowance: the bf16 hash re-decides near
    ties exactly), the output must equal the oracle's own full forward, and
    the GPU forward fed the GPU hash must give the same bits."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, vg, Rg = to_gpu(x, v, R)
    out, lse = lb.lsh_attn_forward(xg, vg, Rg, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=w.causal)
    ref_out, ref_lse, ref_bk = oracle.forward(x, v, R, w.chunk, w.causal)
    gbk = lb.lsh_attn_hash(xg, Rg, w.n_buckets)
    np.testing.assert_array_equal(gbk.cpu().numpy(), ref_bk)
    check_close(out.float().cpu().numpy(), ref_out, w.dtype, f"{w.name} out")
    check_close(lse.cpu().numpy(), ref_lse, w.dtype, f"{w.name} lse")
    out2, lse2 = lb.lsh_attn_forward(xg, vg, None, n_buckets=w.n_buckets, chunk=w.chunk,
                                     causal=w.causal, buckets=gbk)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("w", [I.LONG_64K, I.IMAGE_12K] + SWEEP_LARGE, ids=lambda w: w.name)
def test_forward_timed_path(w):
    """The bench's call at full size: lsh_attn_forward(x, v, R, buckets=NULL),
    where the tensor-core hash also counts the sort's histograms and writes
    the key norms.
      1. The GPU's bucket ids (every batch, head, round and position) equal the
         oracle's hash bit for bit.
      2. The timed call's out and lse equal, bit for bit, the GPU forward fed
         those bucket ids (histograms and norms from their own passes), so the
         fused histograms give the same permutation.
      3. At sampled positions of every (batch, head), out and lse match the
         oracle's forward on the oracle's own ids."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, vg, Rg = to_gpu(x, v, R)
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    out, lse = lb.lsh_attn_forward(xg, vg, Rg, **kw)
    out, lse = out.clone(), lse.clone()
    gbk = lb.lsh_attn_hash(xg, Rg, w.n_buckets)
    out2, lse2 = lb.lsh_attn_forward(xg, vg, None, buckets=gbk, **kw)
    assert torch.equal(out, out2) and torch.equal(lse, lse2), \
        "the fused-histogram forward differs from the caller-bucket forward"
    gbk = gbk.cpu().numpy()
    ref_bk, _ = oracle.hash_all(x, R)
    np.testing.assert_array_equal(gbk, ref_bk, err_msg=f"{w.name}: bucket ids")
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    pos = sample_positions(w.n)
    ro, rl = oracle.forward_sampled(x, v, ref_bk, w.n_buckets, w.chunk, w.causal, pos)
    check_close(out[:, :, pos], ro, w.dtype, f"{w.name} out")
    check_close(lse[:, :, :, pos], rl, w.dtype, f"{w.name} lse")


def test_forward_tie_moves_histogram_count():
    """Tie-built inputs on which the tensor-core screen and the definition pick
    different buckets inside a forward. Column 3 of every rotation is the
    negation of column 2, so p_3 = -p_2 exactly. For tokens near -R_r[:, 2],
    p_2 < 0 has the largest magnitude: the screen takes column 2 with its sign
    (bucket nb/2 + 2) while the first index of [p ; -p] attaining the maximum
    is 3 (+p_3). The fp64 re-decision changes the bucket and moves the token's
    count between the sort's tile histograms; the whole output must then equal
    the oracle's forward, which hashes on its own."""
    w = I.Workload("tie-forward", 1, 2, 4096, 64, 64, 64, 2, True, "bf16")
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    R[:, :, 3] = -R[:, :, 2]
    g = torch.Generator().manual_seed(17)
    for h in range(w.heads):
        r = h % w.rounds  # head h plants its ties in round h % rounds
        idx = torch.arange(h, w.n, 3)
        noise = 0.05 * torch.randn(len(idx), w.d, generator=g)
        x[0, h, idx] = (-R[r, :, 2].float() + noise).to(torch.bfloat16)
    ref_out, ref_lse, ref_bk = oracle.forward(x, v, R, w.chunk, w.causal)
    half = w.n_buckets // 2
    planted = sum(int((ref_bk[0, h, h % w.rounds] == 3).sum()) for h in range(w.heads))
    assert planted >= w.n // 2, "the planted tokens should hash to bucket 3"
    xg, vg, Rg = to_gpu(x, v, R)
    desc = lb.make_desc(1, 2, w.n, w.d, w.n_buckets, w.chunk, w.rounds, True, torch.bfloat16)
    ws = lb.workspace(desc, xg.device)
    out, lse = lb.lsh_attn_forward(xg, vg, Rg, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=True, ws=ws)
    diag = lb.lsh_attn_get_diag(ws)
    assert diag["status"] == 0
    assert diag["hash_refined"] >= planted, diag
    gbk = lb.lsh_attn_hash(xg, Rg, w.n_buckets).cpu().numpy()
    np.testing.assert_array_equal(gbk, ref_bk)
    assert not (gbk == half + 2).all()
    check_close(out.float().cpu().numpy(), ref_out, "bf16", "tie-forward out")
    check_close(lse.cpu().numpy(), ref_lse, "bf16", "tie-forward lse")


# --------------------------------------------------------------------------
# edge cases
EDGE = [
    # name, B, H, n, d, nb, m, rounds, causal, dtype
    ("single-token", 1, 1, 1, 64, 2, 64, 1, True, "f32"),
    ("single-chunk-dense", 1, 2, 96, 128, 8, 128, 1, True, "bf16"),
    ("m-ge-n-noncausal", 2, 1, 64, 64, 4, 256, 1, False, "f32"),
    ("ragged-hash-tail", 1, 2, 320, 64, 16, 64, 2, True, "bf16"),
    ("ragged-sort-tile", 1, 1, 4160, 128, 32, 64, 1, False, "f32"),
    ("two-buckets", 1, 2, 512, 64, 2, 32, 3, True, "bf16"),
    ("chunk-16", 1, 1, 256, 64, 16, 16, 2, False, "bf16"),
    ("chunk-128", 1, 2, 1024, 128, 32, 128, 2, True, "bf16"),
    ("many-rounds", 1, 1, 256, 64, 8, 32, 16, True, "f32"),
    ("max-buckets", 1, 1, 8192, 64, 4096, 64, 1, True, "bf16"),
    ("noncausal-bf16-d128", 1, 2, 1024, 128, 32, 64, 2, False, "bf16"),
    ("noncausal-bf16-d64", 2, 1, 640, 64, 16, 64, 3, False, "bf16"),
    # more rounds than a merge lane group of bf16 d64 has lanes (8), and the most rounds
    ("many-rounds-bf16-d64", 1, 2, 512, 64, 16, 64, 12, True, "bf16"),
    ("max-rounds-bf16-d128", 1, 1, 512, 128, 16, 64, 16, True, "bf16"),
]


@pytest.mark.parametrize("case", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(case):
    name, B, H, n, d, nb, m, rounds, causal, dt = case
    w = I.Workload(name, B, H, n, d, nb, m, rounds, causal, dt)
    x, v = I.make_qkv(w)
    if name == "two-buckets":
        x[0, 0, 5] = 0  # zero key: zero norm
    R = I.make_rotations(w)
    ref_bk, margin = oracle.hash_all(x, R)
    xg, vg, Rg = to_gpu(x, v, R)
    gbk = lb.lsh_attn_hash(xg, Rg, nb).cpu().numpy()
    check_buckets(gbk, ref_bk, margin, name)
    bk = torch.from_numpy(ref_bk)
    ref_out, ref_lse, _ = oracle.forward(x, v, R, m, causal, buckets=bk)
    out, lse = lb.lsh_attn_forward(xg, vg, None, n_buckets=nb, chunk=m, causal=causal,
                                   buckets=bk.cuda())
    check_close(out.float().cpu().numpy(), ref_out, dt, f"{name} out")
    check_close(lse.cpu().numpy(), ref_lse, dt, f"{name} lse")


@pytest.mark.parametrize("causal", [True, False])
def test_reversed_buckets_self_only_rows(causal):
    """Bucket ids that reverse the order: slot s holds position n-1-s, so in
    causal mode the last slot of every chunk sees nothing but itself."""
    n = 2048
    w = I.Workload("reversed", 1, 2, n, 128, n, 64, 1, causal, "bf16")
    x, v = I.make_qkv(w)
    bk = torch.arange(n - 1, -1, -1, dtype=torch.int32).repeat(1, 2, 1, 1)
    ref_out, ref_lse, _ = oracle.forward(x, v, I.make_rotations(w), 64, causal, buckets=bk)
    if causal:
        assert (ref_lse == -1e5).sum() >= 2 * n // 64
    xg, vg = to_gpu(x, v)
    out, lse = lb.lsh_attn_forward(xg, vg, None, n_buckets=n, chunk=64, causal=causal,
                                   buckets=bk.cuda())
    check_close(out.float().cpu().numpy(), ref_out, "bf16", "reversed out")
    check_close(lse.cpu().numpy(), ref_lse, "bf16", "reversed lse")
    if causal:
        self_only = ref_lse == -1e5
        np.testing.assert_array_equal(lse.cpu().numpy()[self_only], -1e5)


def test_all_tokens_one_bucket():
    w = I.Workload("one-bucket", 1, 2, 2048, 64, 64, 64, 2, True, "bf16")
    x, v = I.make_qkv(w)
    bk = torch.full((1, 2, 2, 2048), 17, dtype=torch.int32)
    ref_out, ref_lse, _ = oracle.forward(x, v, I.make_rotations(w), 64, True, buckets=bk)
    xg, vg = to_gpu(x, v)
    out, lse = lb.lsh_attn_forward(xg, vg, None, n_buckets=64, chunk=64, causal=True,
                                   buckets=bk.cuda())
    check_close(out.float().cpu().numpy(), ref_out, "bf16", "one-bucket out")
    check_close(lse.cpu().numpy(), ref_lse, "bf16", "one-bucket lse")


def test_deterministic():
    w = I.BF16_SHORT
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, vg, Rg = to_gpu(x, v, R)
    a = lb.lsh_attn_forward(xg, vg, Rg, n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    a = [t.clone() for t in a]
    b = lb.lsh_attn_forward(xg, vg, Rg, n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_bucket_ids_are_reported_not_fatal():
    w = I.Workload("bad-ids", 1, 1, 256, 64, 8, 64, 1, True, "bf16")
    x, v = I.make_qkv(w)
    bk = I.make_buckets(w)
    bk[0, 0, 0, 3] = 8
    bk[0, 0, 0, 9] = -1
    xg, vg, bkg = to_gpu(x, v, bk)
    desc = lb.make_desc(1, 1, 256, 64, 8, 64, 1, True, torch.bfloat16)
    ws = lb.workspace(desc, xg.device)
    lb.lsh_attn_forward(xg, vg, None, n_buckets=8, chunk=64, causal=True, buckets=bkg, ws=ws)
    diag = lb.lsh_attn_get_diag(ws)
    assert diag["status"] == 6 and diag["bad_bucket_ids"] == 2
    # the next call resets the status
    lb.lsh_attn_forward(xg, vg, None, n_buckets=8, chunk=64, causal=True,
                        buckets=I.make_buckets(w).cuda(), ws=ws)
    assert lb.lsh_attn_get_device_status(ws) == 0


def test_host_errors_write_nothing():
    w = I.BF16_SHORT
    x, v = I.make_qkv(w)
    xg, vg = to_gpu(x, v)
    out = torch.full_like(xg, 7.0)
    with pytest.raises(lb.LshAttnError) as e:  # n % m != 0
        lb.lsh_attn_forward(xg, vg, None, n_buckets=64, chunk=48, causal=True,
                            buckets=I.make_buckets(w).cuda(), out=out)
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert (out == 7.0).all()


# --------------------------------------------------------------------------
# the tensor-core hash on exact ties and its fp64 re-decision queue
@pytest.mark.parametrize("d,nb", [(64, 16), (128, 1024), (64, 2), (64, 192)])
def test_hash_exact_ties_bit_exact(d, nb):
    """Rows built to tie exactly (zero rows, basis vectors against duplicated
    and negated columns of R) must take the first index of [xR ; -xR]."""
    w = I.Workload("ties", 1, 1, 512, d, nb, 64, 2, True, "bf16")
    x, _ = I.make_qkv(w)
    R = I.make_rotations(w)
    half = nb // 2
    if half >= 4:
        R[:, :, 1] = R[:, :, 0]    # duplicate column: p_1 == p_0
        R[:, :, 3] = -R[:, :, 2]   # negated column: p_3 == -p_2
    x[0, 0, :16] = 0                                       # all projections zero
    for i in range(16, 48):
        x[0, 0, i] = 0
        x[0, 0, i, i % d] = 1.0 if i % 2 else -2.0         # basis vectors
    ref, margin = oracle.hash_all(x, R)
    xg, Rg = to_gpu(x, R)
    desc = lb.make_desc(1, 1, 512, d, nb, 64, 2, True, torch.bfloat16)
    ws = lb.workspace(desc, xg.device)
    got = lb.lsh_attn_hash(xg, Rg, nb, ws=ws).cpu().numpy()
    np.testing.assert_array_equal(got, ref)
    diag = lb.lsh_attn_get_diag(ws)
    assert diag["status"] == 0
    assert diag["hash_refined"] >= 16  # at least the zero rows went through fp64


NEAR_TIE_CASES = [(64, 64), (64, 2048), (128, 256), (128, 1024), (64, 4096)]


@pytest.mark.parametrize("d,nb", NEAR_TIE_CASES, ids=[f"d{d}-nb{nb}" for d, nb in NEAR_TIE_CASES])
def test_hash_near_ties_stress(d, nb):
    """Top-two margins planted across the band where an error in the
    tensor-core screen's bound would show: for column pairs (a, b) of R, column
    b equals column a except at one row k*, where it differs by delta. A token
    x = s R[:, a] + noise with x[k*] = t has p_b - p_a = t delta exactly, while
    |p_a| ~ d leads every other column; t is drawn log-uniformly so that the
    relative margin (margin / max|p|) spans about 1e-10 .. 1e-3. Pairs straddle
    16-column batch edges, an MMA chunk edge (192 columns) and the last
    columns. Every bucket id must equal the oracle's bit for bit."""
    n, rounds = 4096, 2
    w = I.Workload("near-ties", 1, 2, n, d, nb, 64, rounds, True, "bf16")
    R = I.make_rotations(w).float()
    half = nb // 2
    pairs = [(a, a + 1) for a in (0, 15, 47, 63, 191, 383, half - 2) if a + 1 < half]
    pairs = sorted(set(pairs))
    g = torch.Generator().manual_seed(23)
    kstar = 5
    for r in range(rounds):
        for a, b in pairs:
            R[r, :, b] = R[r, :, a]
            R[r, kstar, b] = R[r, kstar, a] + 0.25
    R = R.to(torch.bfloat16)
    x = torch.empty(1, 2, n, d)
    for h in range(2):
        r = h  # head h plants its near ties in round h
        pick = torch.randint(0, len(pairs), (n,), generator=g)
        sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0)
        t = 10.0 ** (-7 + 6 * torch.rand(n, generator=g))
        t = t * torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0)
        cols = torch.tensor([a for a, _ in pairs])[pick]
        xh = sign[:, None] * R[r][:, cols].float().T + 0.02 * torch.randn(n, d, generator=g)
        xh[:, kstar] = t
        x[0, h] = xh
    x = x.to(torch.bfloat16)
    ref, margin = oracle.hash_all(x, R)
    xg, Rg = to_gpu(x, R)
    desc = lb.make_desc(1, 2, n, d, nb, 64, rounds, True, torch.bfloat16)
    ws = lb.workspace(desc, xg.device)
    got = lb.lsh_attn_hash(xg, Rg, nb, ws=ws).cpu().numpy()
    # relative margins of the planted rounds cover the band
    p = torch.einsum("hnd,hdj->hnj", x[0].double(), torch.stack([R[0], R[1]]).double())
    rel = np.array([margin[0, h, h] / p[h].abs().max(dim=1).values.numpy() for h in range(2)])
    for lo in (1e-7, 1e-6, 1e-5, 1e-4):
        assert ((rel >= lo) & (rel < 10 * lo)).sum() >= 50, f"few margins in [{lo}, {10 * lo})"
    diag = lb.lsh_attn_get_diag(ws)
    print(f"d{d} nb{nb}: {diag['hash_refined']} re-decided; relative margins "
          f"{np.percentile(rel, [1, 50, 99])}")
    assert diag["status"] == 0
    np.testing.assert_array_equal(got, ref)


def test_hash_refine_count_is_small():
    w = I.LONG_64K
    x, _ = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, Rg = to_gpu(x, R)
    desc = lb.make_desc(w.batch, w.heads, w.n, w.d, w.n_buckets, w.chunk, w.rounds, w.causal,
                        torch.bfloat16)
    ws = lb.workspace(desc, xg.device)
    lb.lsh_attn_hash(xg, Rg, w.n_buckets, ws=ws)
    diag = lb.lsh_attn_get_diag(ws)
    total = w.batch * w.heads * w.n * w.rounds
    print(f"{w.name}: {diag['hash_refined']} of {total} hashes re-decided in fp64")
    assert diag["status"] == 0
    assert 0 < diag["hash_refined"] < 0.02 * total


def test_profiled_forward_matches_and_times_every_kernel():
    w = I.BF16_SHORT
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, vg, Rg = to_gpu(x, v, R)
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    ref = [t.clone() for t in lb.lsh_attn_forward(xg, vg, Rg, **kw)]
    evs = []
    for _ in range(lb.PROFILE_EVENTS):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        evs.append(e)
    out, lse = lb.lsh_attn_forward(xg, vg, Rg, events=evs, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(lb.PROFILE_EVENTS - 1)]
    assert all(t >= 0 for t in times)
    assert times[1] > 0 and times[7] > 0  # projection kernel, attention kernel
