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
SWEEP_SMALL = [w for w in I.sweep_workloads() if w.n <= 8192]
SWEEP_LARGE = [w for w in I.sweep_workloads() if w.n >= 32768 and w.rounds in (1, 4)]


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


@pytest.mark.parametrize("w", SMALL + SWEEP_SMALL[::2], ids=lambda w: w.name)
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
    """buckets=NULL hashes inside the call: equals the oracle's own full forward
    (the hash is bit-exact here), and equals the GPU forward fed the GPU hash."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    xg, vg, Rg = to_gpu(x, v, R)
    out, lse = lb.lsh_attn_forward(xg, vg, Rg, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=w.causal)
    ref_out, ref_lse, ref_bk = oracle.forward(x, v, R, w.chunk, w.causal)
    gbk = lb.lsh_attn_hash(xg, Rg, w.n_buckets)
    _, margin = oracle.hash_all(x, R)
    if check_buckets(gbk.cpu().numpy(), ref_bk, margin, w.name) == 0:
        check_close(out.float().cpu().numpy(), ref_out, w.dtype, f"{w.name} out")
        check_close(lse.cpu().numpy(), ref_lse, w.dtype, f"{w.name} lse")
    out2, lse2 = lb.lsh_attn_forward(xg, vg, None, n_buckets=w.n_buckets, chunk=w.chunk,
                                     causal=w.causal, buckets=gbk)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("w,heads", [(I.IMAGE_12K, [0, 7]), (I.LONG_64K, [0, 5])] +
                         [(s, [0, 7]) for s in SWEEP_LARGE],
                         ids=lambda p: p.name if hasattr(p, "name") else str(p))
def test_forward_sampled(w, heads):
    """Full-size launch in the bench's configuration; the oracle evaluates sampled
    positions of sampled heads with the oracle's own buckets for those heads."""
    x, v = I.make_qkv(w)
    R = I.make_rotations(w)
    bk = I.make_buckets(w)  # other heads: any valid ids
    big = w.n * w.n_buckets * w.rounds > 2 ** 27
    for h in heads:
        xb = x[:1, h:h + 1] if big else x[:, h:h + 1]
        b, _ = oracle.hash_all(xb, R)
        bk[: b.shape[0], h] = torch.from_numpy(b[:, 0])
    xg, vg, bkg = to_gpu(x, v, bk)
    out, lse = lb.lsh_attn_forward(xg, vg, None, n_buckets=w.n_buckets, chunk=w.chunk,
                                   causal=w.causal, buckets=bkg)
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    pos = sample_positions(w.n)
    bsel = [0] if big else list(range(w.batch))
    for h in heads:
        xs, vs = x[bsel][:, h:h + 1], v[bsel][:, h:h + 1]
        ro, rl = oracle.forward_sampled(xs, vs, bk[bsel][:, h:h + 1], w.n_buckets, w.chunk,
                                        w.causal, pos)
        check_close(out[bsel][:, h:h + 1][:, :, pos], ro, w.dtype, f"{w.name} h{h} out")
        check_close(lse[bsel][:, h:h + 1][:, :, :, pos], rl, w.dtype, f"{w.name} h{h} lse")


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
    assert times[1] > 0 and times[6] > 0  # projection kernel, attention kernel
