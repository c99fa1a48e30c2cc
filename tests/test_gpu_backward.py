"""Backward pass through the C ABI against the backward oracle
(oracle/backward.py: the forward restated in float64 torch operations and
differentiated by autograd, pinned on the CPU to the C oracle, to finite
differences and to a textbook dense attention).

The GPU takes the forward's own out and lse (bf16 out, fp32 lse), as a
training step would; the oracle differentiates the exact forward. Bar: for
each gradient, max abs error <= 3e-2 * max(1, max |ref|) and mean abs error
<= 3e-3 * max(1, mean |ref|): the tensor-core products take P w and dS' in bf16
(relative 2^-9), like the forward's P."""
import numpy as np
import pytest
import torch

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I
from oracle import backward as ob

pytestmark = pytest.mark.gpu


def check_grad(gpu, ref, what):
    gpu = gpu.float().cpu().double().numpy()
    ref = ref.numpy()
    err = np.abs(gpu - ref)
    scale_max = max(1.0, float(np.abs(ref).max()))
    scale_mean = max(1.0, float(np.abs(ref).mean()))
    print(f"{what}: max err {err.max():.3e} (ref max {np.abs(ref).max():.3e}), "
          f"mean err {err.mean():.3e} (ref mean {np.abs(ref).mean():.3e})")
    assert np.isfinite(gpu).all(), what
    assert err.max() <= 3e-2 * scale_max, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= 3e-3 * scale_mean, f"{what}: mean abs {err.mean():.3e}"


def run_case(w, with_dlse, seed=5, buckets=None):
    x, v = I.make_qkv(w)
    bk = I.make_buckets(w) if buckets is None else buckets
    g = torch.Generator().manual_seed(seed)
    dout = torch.randn(x.shape, generator=g).to(torch.bfloat16)
    dlse = (torch.randn((w.batch, w.heads, w.rounds, w.n), generator=g)
            if with_dlse else None)
    xg, vg, bkg, dg = x.cuda(), v.cuda(), bk.cuda(), dout.cuda()
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    out, lse = lb.lsh_attn_forward(xg, vg, None, buckets=bkg, **kw)
    dx, dv = lb.lsh_attn_backward(xg, vg, bkg, out, lse, dg,
                                  dlse=None if dlse is None else dlse.cuda(), **kw)
    torch.cuda.synchronize()
    ref_dx, ref_dv = ob.backward(x, v, bk, w.chunk, w.causal, dout.double(),
                                 None if dlse is None else dlse.double())
    return dx, dv, ref_dx, ref_dv


CASES = [  # name, B, H, n, d, nb, rounds, causal, with_dlse
    ("d64-causal-r2", 1, 2, 1024, 64, 16, 2, True, False),
    ("d128-noncausal-r2-dlse", 1, 2, 1024, 128, 16, 2, False, True),
    ("d64-r4-dlse-odd-chunks", 1, 1, 576, 64, 8, 4, True, True),   # 9 chunks: a lone last pair
    ("d128-causal-r1", 2, 1, 512, 128, 8, 1, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(case):
    name, B, H, n, d, nb, R, causal, with_dlse = case
    w = I.Workload(name, B, H, n, d, nb, 64, R, causal, "bf16")
    dx, dv, ref_dx, ref_dv = run_case(w, with_dlse)
    check_grad(dx, ref_dx, f"{name} dx")
    check_grad(dv, ref_dv, f"{name} dv")


def test_backward_self_only_rows():
    """Reversed bucket order: with the causal mask the last slot of every
    chunk sees only itself; its output is its own v, so dv there gets the
    merge-weighted upstream gradient and dx gets nothing through that round."""
    n = 1024
    w = I.Workload("reversed-bwd", 1, 1, n, 64, n, 64, 1, True, "bf16")
    bk = torch.arange(n - 1, -1, -1, dtype=torch.int32).repeat(1, 1, 1, 1)
    dx, dv, ref_dx, ref_dv = run_case(w, True, buckets=bk)
    check_grad(dx, ref_dx, "reversed dx")
    check_grad(dv, ref_dv, "reversed dv")


def test_backward_deterministic():
    w = I.Workload("det-bwd", 1, 4, 2048, 128, 32, 64, 2, True, "bf16")
    x, v = I.make_qkv(w)
    bk = I.make_buckets(w).cuda()
    xg, vg = x.cuda(), v.cuda()
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    out, lse = lb.lsh_attn_forward(xg, vg, None, buckets=bk, **kw)
    dout = torch.randn_like(xg)
    a = [t.clone() for t in lb.lsh_attn_backward(xg, vg, bk, out, lse, dout, **kw)]
    b = lb.lsh_attn_backward(xg, vg, bk, out, lse, dout, **kw)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_backward_rejects_unsupported():
    w = I.Workload("f32-bwd", 1, 1, 256, 64, 8, 64, 1, True, "f32")
    x, v = I.make_qkv(w)
    xg, vg = x.cuda(), v.cuda()
    bk = I.make_buckets(w).cuda()
    out, lse = lb.lsh_attn_forward(xg, vg, None, buckets=bk, n_buckets=8, chunk=64, causal=True)
    with pytest.raises(lb.LshAttnError) as e:
        lb.lsh_attn_backward(xg, vg, bk, out, lse, out, n_buckets=8, chunk=64, causal=True)
    assert e.value.status == 2


def test_backward_full_size_one_head():
    """The long-64k workload (B1 H8 n65536 d128 nb1024 m64 R4, causal) in the
    launch configuration the benchmark times; head 0's gradients against the
    oracle, which differentiates that head alone (the heads are independent).
    Bucket ids are the seeded synthetic ones (an input of the backward)."""
    w = I.LONG_64K
    x, v = I.make_qkv(w)
    bk = I.make_buckets(w)
    g = torch.Generator().manual_seed(5)
    dout = torch.randn(x.shape, generator=g).to(torch.bfloat16)
    kw = dict(n_buckets=w.n_buckets, chunk=w.chunk, causal=w.causal)
    xg, vg, bkg = x.cuda(), v.cuda(), bk.cuda()
    out, lse = lb.lsh_attn_forward(xg, vg, None, buckets=bkg, **kw)
    dx, dv = lb.lsh_attn_backward(xg, vg, bkg, out, lse, dout.cuda(), **kw)
    torch.cuda.synchronize()
    dx0, dv0 = dx[:, :1].cpu(), dv[:, :1].cpu()
    del xg, vg, bkg, out, lse, dx, dv
    ref_dx, ref_dv = ob.backward(x[:, :1], v[:, :1], bk[:, :1], w.chunk, w.causal,
                                 dout[:, :1].double(), None)
    check_grad(dx0, ref_dx, "long-64k head 0 dx")
    check_grad(dv0, ref_dv, "long-64k head 0 dv")
