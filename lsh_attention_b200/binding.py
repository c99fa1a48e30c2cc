"""Thin Python binding of the C ABI in include/lsh_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
library liblshattn.so. PyTorch supplies device memory (inputs, outputs and
the workspace) and the current CUDA stream. There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblshattn.so")

LSH_F32, LSH_BF16 = 0, 1
PROFILE_EVENTS = 10  # LSH_ATTN_PROFILE_EVENTS
#: what ends at each profiling event after the first
PROFILE_KERNELS = ("hash_prep", "hash_mma", "hash_refine", "sort_hist", "sort_scan",
                   "sort_rank", "gather_or_norm", "chunk_attention", "unsort_merge")
_DTYPES = {torch.float32: LSH_F32, torch.bfloat16: LSH_BF16}

#: every symbol the header declares
EXPORTS = ("lsh_attn_workspace_size", "lsh_attn_hash", "lsh_attn_sort", "lsh_attn_forward",
           "lsh_attn_forward_profiled", "lsh_attn_get_device_status", "lsh_attn_get_diag",
           "lsh_attn_sort_noalloc", "lsh_attn_selftest_wait_timeout",
           "lsh_attn_dense_workspace_size", "lsh_attn_dense_forward",
           "lsh_attn_backward_workspace_size", "lsh_attn_backward", "lsh_rev_workspace_size",
           "lsh_rev_block", "lsh_topk_workspace_size", "lsh_topk_forward",
           "lsh_attn_status_string")


class LshAttnDesc(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in
                ("batch", "heads", "n", "d", "n_buckets", "chunk", "rounds", "causal", "dtype")]


class LshAttnDiag(ctypes.Structure):
    _fields_ = [(k, ctypes.c_uint32) for k in
                ("status", "hash_refined", "bad_bucket_ids", "reserved")]


class LshRevDesc(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in
                ("batch", "n", "d_model", "heads", "d_head", "d_ff", "ffn_chunk", "n_buckets",
                 "chunk", "rounds", "causal", "hash_buckets")]


class LshRevWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("w_qk", "w_v", "w_o", "w1", "b1", "w2", "b2")]


class LshTopkDesc(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in
                ("batch", "heads", "n", "d", "n_buckets", "n_bits", "top_k", "rounds", "causal")]


class LshAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load liblshattn.so; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(f"{_LIB_PATH} is missing: build it with "
                                  "`python -m lsh_attention_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, sz = ctypes.c_void_p, ctypes.c_size_t
            dp = ctypes.POINTER(LshAttnDesc)
            lib.lsh_attn_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
            lib.lsh_attn_hash.argtypes = [dp, vp, vp, vp, vp, sz, vp]
            lib.lsh_attn_sort.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.lsh_attn_forward.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.lsh_attn_forward_profiled.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                                      ctypes.POINTER(ctypes.c_void_p)]
            lib.lsh_attn_get_device_status.argtypes = [vp, vp]
            lib.lsh_attn_sort_noalloc.argtypes = [dp, vp, vp, vp]
            lib.lsh_attn_get_diag.argtypes = [vp, vp, ctypes.POINTER(LshAttnDiag)]
            lib.lsh_attn_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
            lib.lsh_attn_dense_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
            lib.lsh_attn_dense_forward.argtypes = [dp, vp, vp, vp, vp, vp, sz, vp]
            lib.lsh_attn_backward_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
            lib.lsh_attn_backward.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.lsh_rev_workspace_size.argtypes = [ctypes.POINTER(LshRevDesc),
                                                   ctypes.POINTER(sz)]
            lib.lsh_rev_block.argtypes = [ctypes.POINTER(LshRevDesc), ctypes.c_int, vp, vp,
                                          ctypes.POINTER(LshRevWeights), vp, vp, vp, vp, vp, sz,
                                          vp]
            lib.lsh_topk_workspace_size.argtypes = [ctypes.POINTER(LshTopkDesc),
                                                    ctypes.POINTER(sz)]
            lib.lsh_topk_forward.argtypes = [ctypes.POINTER(LshTopkDesc), vp, vp, vp, vp, vp, vp,
                                             vp, sz, vp]
            lib.lsh_attn_status_string.argtypes = [ctypes.c_int]
            lib.lsh_attn_status_string.restype = ctypes.c_char_p
            for f in EXPORTS[:-1]:
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _check(status: int) -> None:
    if status != 0:
        msg = load().lsh_attn_status_string(status).decode()
        raise LshAttnError(status, msg)


def make_desc(batch, heads, n, d, n_buckets, chunk, rounds, causal, dtype) -> LshAttnDesc:
    if isinstance(dtype, torch.dtype):
        if dtype not in _DTYPES:
            raise TypeError(f"unsupported dtype {dtype}")
        dtype = _DTYPES[dtype]
    return LshAttnDesc(batch, heads, n, d, n_buckets, chunk, rounds, int(bool(causal)), dtype)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _on_current_device(stream=None, **tensors) -> None:
    """The library launches on the current CUDA device and dereferences every
    pointer there: raise ValueError, before anything is launched, unless every
    given tensor (and the stream, if one is given) lives on that device."""
    cur = torch.cuda.current_device()
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.device.index != cur:
            raise ValueError(f"{name} is on {t.device}, but the current device is cuda:{cur}; "
                             f"call inside `with torch.cuda.device({t.device})`")
    if stream is not None and stream.device.index != cur:
        raise ValueError(f"stream is on {stream.device}, but the current device is cuda:{cur}")


def _require(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def lsh_attn_workspace_size(desc: LshAttnDesc) -> int:
    out = ctypes.c_size_t(0)
    _check(load().lsh_attn_workspace_size(ctypes.byref(desc), ctypes.byref(out)))
    return out.value


_ws_cache: dict = {}


def workspace(desc: LshAttnDesc, device, stream=None) -> torch.Tensor:
    """A cached workspace of at least the size `desc` needs, one per
    (device, stream): calls that may run concurrently must not share one."""
    return _scratch(device, stream, lsh_attn_workspace_size(desc))


def lsh_attn_hash(x, R, n_buckets: int, buckets=None, ws=None, stream=None):
    """Bucket ids [B, H, rounds, n] int32 of x [B, H, n, d] under R [rounds, d, nb/2]."""
    _on_current_device(stream, x=x, R=R, buckets=buckets, ws=ws)
    B, H, n, d = x.shape
    rounds = R.shape[0]
    _require(x, "x", None, None)
    _require(R, "R", x.dtype, (rounds, d, n_buckets // 2))
    desc = make_desc(B, H, n, d, n_buckets, 1, rounds, False, x.dtype)
    if buckets is None:
        buckets = torch.empty((B, H, rounds, n), dtype=torch.int32, device=x.device)
    _require(buckets, "buckets", torch.int32, (B, H, rounds, n))
    if ws is None:
        ws = workspace(desc, x.device, stream)
    _check(load().lsh_attn_hash(ctypes.byref(desc), _ptr(x), _ptr(R), _ptr(buckets), _ptr(ws),
                                ws.numel(), _stream(stream)))
    return buckets


def lsh_attn_sort(buckets, n_buckets: int, x=None, v=None, perm=None, xs=None, vs=None, ws=None,
                  stream=None, d: int = 64, dtype=torch.bfloat16):
    """Stable sort by (bucket, position) of every (batch, head, round).
    Returns perm [B, H, rounds, n] int32, and (xs, vs) sorted row copies when
    x and v are given."""
    _on_current_device(stream, buckets=buckets, x=x, v=v, perm=perm, xs=xs, vs=vs, ws=ws)
    B, H, rounds, n = buckets.shape
    _require(buckets, "buckets", torch.int32, None)
    if x is not None:
        _require(x, "x", None, (B, H, n, x.shape[-1]))
        _require(v, "v", x.dtype, tuple(x.shape))
        d, dtype = x.shape[-1], x.dtype
    desc = make_desc(B, H, n, d, n_buckets, 1, rounds, False, dtype)
    if perm is None:
        perm = torch.empty((B, H, rounds, n), dtype=torch.int32, device=buckets.device)
    _require(perm, "perm", torch.int32, (B, H, rounds, n))
    if x is not None:
        if xs is None:
            xs = torch.empty((B, H, rounds, n, d), dtype=dtype, device=x.device)
        if vs is None:
            vs = torch.empty((B, H, rounds, n, d), dtype=dtype, device=x.device)
        _require(xs, "xs", dtype, (B, H, rounds, n, d))
        _require(vs, "vs", dtype, (B, H, rounds, n, d))
    if ws is None:
        ws = workspace(desc, buckets.device, stream)
    _check(load().lsh_attn_sort(ctypes.byref(desc), _ptr(buckets), _ptr(x), _ptr(v), _ptr(perm),
                                _ptr(xs), _ptr(vs), _ptr(ws), ws.numel(), _stream(stream)))
    return (perm, xs, vs) if x is not None else perm


def lsh_attn_forward(x, v, R=None, *, n_buckets: int, chunk: int, causal: bool, rounds=None,
                     buckets=None, out=None, lse=None, ws=None, stream=None, events=None):
    """LSH-attention forward. x, v [B, H, n, d]; R [rounds, d, nb/2] (or
    caller buckets [B, H, rounds, n]). Returns (out [B, H, n, d], lse
    [B, H, rounds, n] fp32). `events`: PROFILE_EVENTS recorded
    torch.cuda.Event objects marking the kernel boundaries
    (lsh_attn_forward_profiled)."""
    _on_current_device(stream, x=x, v=v, R=R, buckets=buckets, out=out, lse=lse, ws=ws)
    B, H, n, d = x.shape
    _require(x, "x", None, None)
    _require(v, "v", x.dtype, tuple(x.shape))
    if buckets is not None:
        rounds = buckets.shape[2]
        _require(buckets, "buckets", torch.int32, (B, H, rounds, n))
    else:
        if R is None:
            raise ValueError("either R or buckets is required")
        rounds = R.shape[0]
        _require(R, "R", x.dtype, (rounds, d, n_buckets // 2))
    desc = make_desc(B, H, n, d, n_buckets, chunk, rounds, causal, x.dtype)
    if out is None:
        out = torch.empty_like(x)
    if lse is None:
        lse = torch.empty((B, H, rounds, n), dtype=torch.float32, device=x.device)
    _require(out, "out", x.dtype, tuple(x.shape))
    _require(lse, "lse", torch.float32, (B, H, rounds, n))
    if ws is None:
        ws = workspace(desc, x.device, stream)
    args = (ctypes.byref(desc), _ptr(x), _ptr(v), _ptr(R), _ptr(buckets), _ptr(out), _ptr(lse),
            _ptr(ws), ws.numel(), _stream(stream))
    if events is None:
        _check(load().lsh_attn_forward(*args))
    else:
        if len(events) != PROFILE_EVENTS or any(e.cuda_event == 0 for e in events):
            raise ValueError(f"events: {PROFILE_EVENTS} torch.cuda.Event objects, each recorded once")
        ev = (ctypes.c_void_p * PROFILE_EVENTS)(*[e.cuda_event for e in events])
        _check(load().lsh_attn_forward_profiled(*args, ev))
    return out, lse


def lsh_attn_dense_forward(x, v, *, causal: bool, out=None, lse=None, ws=None, stream=None):
    """Dense shared-QK attention (the full-attention baseline) of x, v
    [B, H, n, d] bf16. Returns (out [B, H, n, d], lse [B, H, n] fp32)."""
    _on_current_device(stream, x=x, v=v, out=out, lse=lse, ws=ws)
    B, H, n, d = x.shape
    _require(x, "x", torch.bfloat16, None)
    _require(v, "v", torch.bfloat16, tuple(x.shape))
    desc = make_desc(B, H, n, d, 2, 1, 1, causal, x.dtype)
    if out is None:
        out = torch.empty_like(x)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=x.device)
    _require(out, "out", torch.bfloat16, tuple(x.shape))
    _require(lse, "lse", torch.float32, (B, H, n))
    need = ctypes.c_size_t(0)
    _check(load().lsh_attn_dense_workspace_size(ctypes.byref(desc), ctypes.byref(need)))
    if ws is None:
        ws = _scratch(x.device, stream, need.value)
    elif ws.numel() < need.value:
        raise ValueError(f"ws: {need.value} bytes needed, {ws.numel()} given")
    _check(load().lsh_attn_dense_forward(ctypes.byref(desc), _ptr(x), _ptr(v), _ptr(out),
                                         _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def lsh_attn_backward(x, v, buckets, out, lse, dout, *, n_buckets: int, chunk: int,
                      causal: bool, dlse=None, dx=None, dv=None, ws=None, stream=None):
    """Gradients (dx, dv) [B, H, n, d] of lsh_attn_forward(x, v, buckets=...)
    for upstream dout [B, H, n, d] (and dlse [B, H, rounds, n], or None),
    given that forward's out and lse."""
    _on_current_device(stream, x=x, v=v, buckets=buckets, out=out, lse=lse, dout=dout, dlse=dlse,
                       dx=dx, dv=dv, ws=ws)
    B, H, n, d = x.shape
    rounds = buckets.shape[2]
    _require(x, "x", None, None)
    for name, t in (("v", v), ("out", out), ("dout", dout)):
        _require(t, name, x.dtype, tuple(x.shape))
    _require(buckets, "buckets", torch.int32, (B, H, rounds, n))
    _require(lse, "lse", torch.float32, (B, H, rounds, n))
    if dlse is not None:
        _require(dlse, "dlse", torch.float32, (B, H, rounds, n))
    desc = make_desc(B, H, n, d, n_buckets, chunk, rounds, causal, x.dtype)
    if dx is None:
        dx = torch.empty_like(x)
    if dv is None:
        dv = torch.empty_like(x)
    _require(dx, "dx", x.dtype, tuple(x.shape))
    _require(dv, "dv", x.dtype, tuple(x.shape))
    need = ctypes.c_size_t(0)
    _check(load().lsh_attn_backward_workspace_size(ctypes.byref(desc), ctypes.byref(need)))
    if ws is None:
        ws = _scratch(x.device, stream, need.value)
    elif ws.numel() < need.value:
        raise ValueError(f"ws: {need.value} bytes needed, {ws.numel()} given")
    _check(load().lsh_attn_backward(ctypes.byref(desc), _ptr(x), _ptr(v), _ptr(buckets),
                                    _ptr(out), _ptr(lse), _ptr(dout), _ptr(dlse), _ptr(dx),
                                    _ptr(dv), _ptr(ws), ws.numel(), _stream(stream)))
    return dx, dv


def lsh_rev_block(in1, in2, weights: dict, *, heads: int, n_buckets: int, rounds: int,
                  causal: bool, ffn_chunk: int, R=None, buckets=None, inverse: bool = False,
                  out1=None, out2=None, ws=None, stream=None, chunk: int = 64):
    """Reversible layer: forward (x1, x2) -> (y1, y2), or inverse (y1, y2) ->
    (x1, x2), [B, n, d_model] bf16. weights: w_qk, w_v, w_o [d_model][d_model],
    w1 [d_ff][d_model], b1 [d_ff], w2 [d_model][d_ff], b2 [d_model] (bf16
    weights, fp32 biases). Forward without `buckets` hashes them (R needed)
    and returns them. Returns (out1, out2, buckets)."""
    W = weights
    _on_current_device(stream, in1=in1, in2=in2, R=R, buckets=buckets, out1=out1, out2=out2,
                       ws=ws, **W)
    B, n, dm = in1.shape
    dh = dm // heads
    d_ff = W["w1"].shape[0]
    for name, t in (("in1", in1), ("in2", in2)):
        _require(t, name, torch.bfloat16, (B, n, dm))
    for name, shape in (("w_qk", (dm, dm)), ("w_v", (dm, dm)), ("w_o", (dm, dm)),
                        ("w1", (d_ff, dm)), ("w2", (dm, d_ff))):
        _require(W[name], name, torch.bfloat16, shape)
    for name, shape in (("b1", (d_ff,)), ("b2", (dm,))):
        if W.get(name) is not None:
            _require(W[name], name, torch.float32, shape)
    hash_buckets = not inverse and buckets is None
    if buckets is None:
        if inverse:
            raise ValueError("the inverse needs the forward's bucket ids")
        if R is None:
            raise ValueError("either R or buckets is required")
        buckets = torch.empty((B, heads, rounds, n), dtype=torch.int32, device=in1.device)
    _require(buckets, "buckets", torch.int32, (B, heads, rounds, n))
    if R is not None:
        _require(R, "R", torch.bfloat16, (rounds, dh, n_buckets // 2))
    desc = LshRevDesc(B, n, dm, heads, dh, d_ff, ffn_chunk, n_buckets, chunk, rounds,
                      int(bool(causal)), int(hash_buckets))
    wts = LshRevWeights(*[ctypes.c_void_p(0 if W.get(k) is None else W[k].data_ptr())
                          for k in ("w_qk", "w_v", "w_o", "w1", "b1", "w2", "b2")])
    out1 = torch.empty_like(in1) if out1 is None else out1
    out2 = torch.empty_like(in2) if out2 is None else out2
    _require(out1, "out1", torch.bfloat16, (B, n, dm))
    _require(out2, "out2", torch.bfloat16, (B, n, dm))
    need = ctypes.c_size_t(0)
    _check(load().lsh_rev_workspace_size(ctypes.byref(desc), ctypes.byref(need)))
    if ws is None:
        ws = _scratch(in1.device, stream, need.value)
    elif ws.numel() < need.value:
        raise ValueError(f"ws: {need.value} bytes needed, {ws.numel()} given")
    _check(load().lsh_rev_block(ctypes.byref(desc), int(bool(inverse)), _ptr(in1), _ptr(in2),
                                ctypes.byref(wts), _ptr(R), _ptr(buckets), _ptr(out1), _ptr(out2),
                                _ptr(ws), ws.numel(), _stream(stream)))
    return out1, out2, buckets


def lsh_topk_forward(x, v, proj, *, n_buckets: int, top_k: int, causal: bool,
                     return_candidates: bool = False, out=None, lse=None, ws=None, stream=None):
    """The in-bucket top-k variant: x, v [B, H, n, d] bf16, proj [rounds, d,
    n_bits] bf16. Returns (out, lse [B, H, n]) and, if asked, the candidates
    [B, H, rounds, n, top_k] int32 (-1 past the kept ones)."""
    _on_current_device(stream, x=x, v=v, proj=proj, out=out, lse=lse, ws=ws)
    B, H, n, d = x.shape
    L, _, m = proj.shape
    _require(x, "x", torch.bfloat16, None)
    _require(v, "v", torch.bfloat16, tuple(x.shape))
    _require(proj, "proj", torch.bfloat16, (L, d, m))
    desc = LshTopkDesc(B, H, n, d, n_buckets, m, top_k, L, int(bool(causal)))
    out = torch.empty_like(x) if out is None else out
    lse = torch.empty((B, H, n), dtype=torch.float32, device=x.device) if lse is None else lse
    _require(out, "out", torch.bfloat16, tuple(x.shape))
    _require(lse, "lse", torch.float32, (B, H, n))
    cand = (torch.empty((B, H, L, n, top_k), dtype=torch.int32, device=x.device)
            if return_candidates else None)
    need = ctypes.c_size_t(0)
    _check(load().lsh_topk_workspace_size(ctypes.byref(desc), ctypes.byref(need)))
    if ws is None:
        ws = _scratch(x.device, stream, need.value)
    elif ws.numel() < need.value:
        raise ValueError(f"ws: {need.value} bytes needed, {ws.numel()} given")
    _check(load().lsh_topk_forward(ctypes.byref(desc), _ptr(x), _ptr(v), _ptr(proj), _ptr(out),
                                   _ptr(lse), _ptr(cand), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, lse, cand) if return_candidates else (out, lse)


def _scratch(device, stream, need: int) -> torch.Tensor:
    """The cached workspace of (device, stream), grown to `need` bytes."""
    dev = torch.device(device)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index, s.cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        _ws_cache.pop(key, None)
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def lsh_attn_sort_noalloc(buckets, n_buckets: int, perm=None, stream=None):
    """perm [B, H, rounds, n] of the stable bucket sort without any workspace:
    the library's fixed device scratch is used (see lsh_attn.h)."""
    _on_current_device(stream, buckets=buckets, perm=perm)
    B, H, rounds, n = buckets.shape
    _require(buckets, "buckets", torch.int32, None)
    desc = make_desc(B, H, n, 64, n_buckets, 1, rounds, False, torch.bfloat16)
    if perm is None:
        perm = torch.empty((B, H, rounds, n), dtype=torch.int32, device=buckets.device)
    _require(perm, "perm", torch.int32, (B, H, rounds, n))
    _check(load().lsh_attn_sort_noalloc(ctypes.byref(desc), _ptr(buckets), _ptr(perm),
                                        _stream(stream)))
    return perm


def lsh_attn_get_diag(ws, stream=None) -> dict:
    _on_current_device(stream, ws=ws)
    d = LshAttnDiag()
    _check(load().lsh_attn_get_diag(_ptr(ws), _stream(stream), ctypes.byref(d)))
    return {"status": d.status, "hash_refined": d.hash_refined,
            "bad_bucket_ids": d.bad_bucket_ids}


def lsh_attn_get_device_status(ws, stream=None) -> int:
    _on_current_device(stream, ws=ws)
    return load().lsh_attn_get_device_status(_ptr(ws), _stream(stream))


def lsh_attn_selftest_wait_timeout(ws, limit_us: int, stream=None) -> None:
    """Launch the bounded-wait self-test on `ws` (a uint8 CUDA tensor of at
    least 256 bytes): a wait that nothing completes gives up after
    `limit_us` and records LSH_ERR_TIMEOUT (read it with
    lsh_attn_get_device_status)."""
    _on_current_device(stream, ws=ws)
    _check(load().lsh_attn_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(),
                                                 int(limit_us), _stream(stream)))
