"""lsh_attn_sort_noalloc: the sort entry point that allocates nothing.

It exists for callers that may not allocate device memory (a plug-in whose
host runtime owns all device memory, a loop that cannot afford the device
synchronisation of cudaMalloc / cudaFree). Its scratch is a fixed array in
the library's device memory, shared by every call and keeping the previous
call's contents, so the tests run it twice in a row, with different bucket
ids, and compare each result with the workspace-based lsh_attn_sort. The
permutation is integer data: the comparison is exact.

This file is collected last so that a run stopping at the first failure has
run every other test before it.
"""
import pytest
import torch

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = [I.BF16_SHORT, I.TINY_F32, I.IMAGE_12K.with_(batch=1),
         I.Workload("many-buckets", 1, 2, 8192, 64, 4096, 64, 2, True, "bf16")]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_sort_matches_workspace_sort_on_consecutive_calls(w):
    first = I.make_buckets(w, seed=11).cuda()
    second = I.make_buckets(w, seed=12).cuda()
    for bk in (first, second):  # the second call starts from the first call's scratch
        ref = lb.lsh_attn_sort(bk, w.n_buckets, d=w.d, dtype=I.torch_dtype(w.dtype))
        got = lb.lsh_attn_sort_noalloc(bk, w.n_buckets)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)


def test_noalloc_sort_rejects_problems_beyond_its_scratch():
    w = I.LONG_64K  # needs more than LSH_ATTN_NOALLOC_SCRATCH_BYTES
    bk = I.make_buckets(w).cuda()
    perm = torch.full_like(bk, -7)
    with pytest.raises(lb.LshAttnError) as e:
        lb.lsh_attn_sort_noalloc(bk, w.n_buckets, perm=perm)
    assert e.value.status == 2  # LSH_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (perm == -7).all()


def test_noalloc_sort_clamps_out_of_range_ids_silently():
    """Ids outside [0, nb) are clamped on this path (no status is readable):
    the permutation is that of the clamped ids."""
    w = I.BF16_SHORT
    bk = I.make_buckets(w, seed=13)
    bk[0, 0, 0, 5] = w.n_buckets + 3
    bk[1, 7, 1, 100] = -4
    bk[0, 3, 1, 0] = 1 << 30
    clamped = bk.clamp(0, w.n_buckets - 1)
    got = lb.lsh_attn_sort_noalloc(bk.cuda(), w.n_buckets)
    ref = lb.lsh_attn_sort(clamped.cuda(), w.n_buckets, d=w.d, dtype=I.torch_dtype(w.dtype))
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
