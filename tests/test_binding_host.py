"""Host-side checks of the Python binding that need no GPU.

The library launches on the current CUDA device and dereferences every
pointer there, so a tensor (or a stream) on another device must be rejected
before anything is launched. These tests stand in CUDA tensors on a second
device by small objects with the attributes the binding reads, make the
current device 0, and make loading the library an error: a call that got as
far as the library would fail the test.
"""
import pytest
import torch

from lsh_attention_b200 import binding as lb


class FakeCudaTensor:
    """What the binding reads of a CUDA tensor: shape, dtype, device."""

    is_cuda = True

    def __init__(self, shape, dtype, index):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True

    def data_ptr(self):
        raise AssertionError("a pointer was taken: the call got past the device check")


class FakeStream:
    def __init__(self, index):
        self.device = torch.device("cuda", index)
        self.cuda_stream = 0


@pytest.fixture
def device0(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)

    def no_load():
        raise AssertionError("the library was loaded: the call got past the device check")

    monkeypatch.setattr(lb, "load", no_load)


def qkv(idx_x=0, idx_v=0, idx_r=0):
    B, H, n, d, nb, R = 1, 2, 256, 64, 16, 2
    return (FakeCudaTensor((B, H, n, d), torch.bfloat16, idx_x),
            FakeCudaTensor((B, H, n, d), torch.bfloat16, idx_v),
            FakeCudaTensor((R, d, nb // 2), torch.bfloat16, idx_r))


@pytest.mark.parametrize("where", ["x", "v", "R"])
def test_forward_rejects_tensor_on_other_device(device0, where):
    x, v, R = qkv(**{f"idx_{where.lower()}": 1})
    with pytest.raises(ValueError, match=f"{where} is on cuda:1"):
        lb.lsh_attn_forward(x, v, R, n_buckets=16, chunk=64, causal=True)


def test_forward_rejects_output_and_workspace_on_other_device(device0):
    x, v, R = qkv()
    out = FakeCudaTensor(x.shape, torch.bfloat16, 1)
    with pytest.raises(ValueError, match="out is on cuda:1"):
        lb.lsh_attn_forward(x, v, R, n_buckets=16, chunk=64, causal=True, out=out)
    ws = FakeCudaTensor((1 << 20,), torch.uint8, 2)
    with pytest.raises(ValueError, match="ws is on cuda:2"):
        lb.lsh_attn_forward(x, v, R, n_buckets=16, chunk=64, causal=True, ws=ws)


def test_stream_on_other_device_is_rejected(device0):
    x, v, R = qkv()
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        lb.lsh_attn_forward(x, v, R, n_buckets=16, chunk=64, causal=True, stream=FakeStream(1))


def test_hash_sort_and_noalloc_sort_reject_other_device(device0):
    x, _, R = qkv(idx_x=1)
    with pytest.raises(ValueError, match="x is on cuda:1"):
        lb.lsh_attn_hash(x, R, 16)
    bk = FakeCudaTensor((1, 2, 2, 256), torch.int32, 3)
    with pytest.raises(ValueError, match="buckets is on cuda:3"):
        lb.lsh_attn_sort(bk, 16)
    with pytest.raises(ValueError, match="buckets is on cuda:3"):
        lb.lsh_attn_sort_noalloc(bk, 16)
    ws = FakeCudaTensor((256,), torch.uint8, 1)
    with pytest.raises(ValueError, match="ws is on cuda:1"):
        lb.lsh_attn_get_diag(ws)
    with pytest.raises(ValueError, match="ws is on cuda:1"):
        lb.lsh_attn_selftest_wait_timeout(ws, 1000)


def test_cpu_tensor_is_rejected(device0):
    _, v, R = qkv()
    x = torch.zeros(v.shape, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        lb.lsh_attn_forward(x, v, R, n_buckets=16, chunk=64, causal=True)
