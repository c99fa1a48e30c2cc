"""CPU oracle for the Reformer shared-QK LSH-attention forward pass.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg may import this package; the library and its Python binding
never do. It shares no code with the CUDA path.

The arithmetic lives in ``lsh_oracle.c`` (plain C99, fp64, OpenMP over
independent (batch, head, round) units). This module builds it with gcc if the
shared object is missing and marshals numpy / torch arrays into fp64.
``backward.py`` restates the forward in float64 torch operations and gives its
gradients with respect to x and v (for a backward pass to be checked against).

Every input is widened to fp64 exactly (fp32 and bf16 values are fp64 values),
so the oracle evaluates the definition on the very numbers the GPU consumes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsh_oracle.c")
_LIB = os.path.join(_HERE, "liblsh_oracle.so")
# A test may point the wrapper at another build of the oracle (a copy with a
# planted mistake) to check that the pins catch it.
_LIB_OVERRIDE = os.environ.get("LSH_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
                        "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            lib.lsho_hash_rows.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int, _f64p, ctypes.c_int,
                                           _i32p, _f64p]
            lib.lsho_hash_rows.restype = None
            lib.lsho_hash_all.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _f64p,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _f64p]
            lib.lsho_hash_all.restype = None
            lib.lsho_sort.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, _i32p, _i32p]
            lib.lsho_sort.restype = ctypes.c_int
            lib.lsho_attend_slots.argtypes = [_f64p, _f64p, _i32p, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                              ctypes.c_int64, _f64p, _f64p]
            lib.lsho_attend_slots.restype = ctypes.c_int
            lib.lsho_merge.argtypes = [_f64p, _f64p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                       _f64p, _f64p]
            lib.lsho_merge.restype = None
            lib.lsho_forward.argtypes = [_f64p, _f64p, _f64p, ctypes.c_void_p] + \
                [ctypes.c_int] * 9 + [_f64p, _f64p, _i32p]
            lib.lsho_forward.restype = ctypes.c_int
            lib.lsho_forward_sampled.argtypes = [_f64p, _f64p, _i32p] + [ctypes.c_int] * 8 + \
                [_i32p, ctypes.c_int, ctypes.c_int, _f64p, _f64p]
            lib.lsho_forward_sampled.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (any dtype, incl. bf16): exact widening
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def hash_rows(x, R):
    """Buckets of rows x [N, d] under one rotation R [d, nb/2].
    Returns (bucket int32 [N], margin fp64 [N])."""
    x = _f64(x)
    R = _f64(R)
    N, d = x.shape
    nb = 2 * R.shape[1]
    b = np.empty(N, np.int32)
    mg = np.empty(N, np.float64)
    _load().lsho_hash_rows(x, N, d, R, nb, b, mg)
    return b, mg


def hash_all(x, R, nthreads: int = 0):
    """Buckets of x [B, H, n, d] under every round of R [rounds, d, nb/2].
    Returns (bucket int32 [B, H, rounds, n], margin fp64 [B, H, rounds, n])."""
    x = _f64(x)
    R = _f64(R)
    B, H, n, d = x.shape
    rounds, _, half = R.shape
    b = np.empty((B, H, rounds, n), np.int32)
    mg = np.empty((B, H, rounds, n), np.float64)
    _load().lsho_hash_all(x, B * H, n, d, R, rounds, 2 * half, nthreads, b, mg)
    return b, mg


def sort(bucket, nb: int):
    """Stable sort of positions by bucket for one sequence. Returns (perm, inv)."""
    b = _i32(bucket)
    n = b.shape[0]
    perm = np.empty(n, np.int32)
    inv = np.empty(n, np.int32)
    if _load().lsho_sort(b, n, nb, perm, inv) != 0:
        raise ValueError("bucket id out of range")
    return perm, inv


def attend_slots(x, v, perm, m: int, causal: bool, qslots=None):
    """Chunked attention of one (batch, head, round): x, v [n, d] in position
    order, perm [n]. Returns (out [nq, d], lse [nq]) in slot order (of qslots,
    or of all slots)."""
    x = _f64(x)
    v = _f64(v)
    perm = _i32(perm)
    n, d = x.shape
    if v.shape != x.shape or perm.shape != (n,):
        raise ValueError("x and v must both be [n, d]; perm must be [n]")
    if qslots is None:
        qp, nq = None, n
    else:
        qs = _i32(qslots)
        qp, nq = qs.ctypes.data_as(ctypes.c_void_p), qs.shape[0]
    out = np.empty((nq, d), np.float64)
    lse = np.empty(nq, np.float64)
    rc = _load().lsho_attend_slots(x, v, perm, n, d, m, int(causal), qp, nq, out, lse)
    if rc != 0:
        raise ValueError("n is not a multiple of the chunk size")
    return out, lse


def merge(o, lse):
    """Round merge: o [rounds, npos, d], lse [rounds, npos] -> (out [npos, d], L [npos])."""
    o = _f64(o)
    lse = _f64(lse)
    rounds, npos, d = o.shape
    out = np.empty((npos, d), np.float64)
    L = np.empty(npos, np.float64)
    _load().lsho_merge(o, lse, rounds, npos, d, out, L)
    return out, L


def forward(x, v, R, chunk: int, causal: bool, buckets=None, nthreads: int = 0):
    """Whole forward pass. x, v [B, H, n, d]; R [rounds, d, nb/2]; buckets
    [B, H, rounds, n] or None (hash here). Returns (out [B,H,n,d], lse
    [B,H,rounds,n], buckets [B,H,rounds,n]), all in position order."""
    x = _f64(x)
    v = _f64(v)
    R = _f64(R)
    B, H, n, d = x.shape
    rounds, _, half = R.shape
    nb = 2 * half
    out = np.empty((B, H, n, d), np.float64)
    lse = np.empty((B, H, rounds, n), np.float64)
    bk = np.empty((B, H, rounds, n), np.int32)
    if buckets is None:
        bp = None
    else:
        bi = _i32(buckets)
        assert bi.shape == (B, H, rounds, n)
        bp = bi.ctypes.data_as(ctypes.c_void_p)
    rc = _load().lsho_forward(x, v, R, bp, B, H, n, d, nb, chunk, rounds, int(causal), nthreads,
                              out, lse, bk)
    if rc != 0:
        raise ValueError(f"oracle forward failed ({rc})")
    return out, lse, bk


def forward_sampled(x, v, buckets, n_buckets: int, chunk: int, causal: bool, pos,
                    nthreads: int = 0):
    """Forward pass at sampled positions only, with given buckets.
    Returns (out [B, H, npos, d], lse [B, H, rounds, npos])."""
    x = _f64(x)
    v = _f64(v)
    bk = _i32(buckets)
    pos = _i32(pos)
    B, H, n, d = x.shape
    rounds = bk.shape[2]
    npos = pos.shape[0]
    out = np.empty((B, H, npos, d), np.float64)
    lse = np.empty((B, H, rounds, npos), np.float64)
    rc = _load().lsho_forward_sampled(x, v, bk, B, H, n, d, n_buckets, chunk, rounds, int(causal),
                                      pos, npos, nthreads, out, lse)
    if rc != 0:
        raise ValueError(f"oracle sampled forward failed ({rc})")
    return out, lse


def dense_sampled(x, v, causal: bool, pos, nthreads: int = 0):
    """Dense shared-QK attention at sampled positions: the forward pass with
    one round and one chunk spanning the sequence (every key is in the
    query's window whatever the bucket ids). Returns (out [B, H, npos, d],
    lse [B, H, npos])."""
    x = _f64(x)
    B, H, n, d = x.shape
    zeros = np.zeros((B, H, 1, n), np.int32)
    out, lse = forward_sampled(x, v, zeros, 2, n, causal, pos, nthreads)
    return out, lse[:, :, 0]
