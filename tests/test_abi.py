"""The C-ABI library builds, loads and exports every symbol include/*.h
declares; host-side argument checks return their status codes before any
launch. CPU only: no call here reaches the GPU."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from lsh_attention_b200 import binding as lb
from lsh_attention_b200 import build as lbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"^(?:lsh_status|const char \*)\s*(\w+)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    lbuild.build()
    return lb.load()


def test_header_declares_the_boundary():
    names = header_functions()
    for f in ("lsh_attn_hash", "lsh_attn_sort", "lsh_attn_forward", "lsh_attn_workspace_size"):
        assert f in names
    assert set(names) == set(lb.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lb.library_path()], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, re.M))
    for f in header_functions():
        assert f in exported, f
        assert getattr(lib, f) is not None


def test_library_targets_sm100a_only(lib):
    # the build passes exactly one -gencode: compute_100a -> sm_100a
    assert lbuild.FLAGS[lbuild.FLAGS.index("-gencode") + 1] == "arch=compute_100a,code=sm_100a"
    assert lbuild.FLAGS.count("-gencode") == 1


def desc(**kw):
    base = dict(batch=1, heads=8, n=4096, d=64, n_buckets=64, chunk=64, rounds=2, causal=1,
                dtype=lb.LSH_BF16)
    base.update(kw)
    return lb.LshAttnDesc(*[base[k] for k, _ in lb.LshAttnDesc._fields_])


def ws_size(lib, d):
    out = ctypes.c_size_t(0)
    return lib.lsh_attn_workspace_size(ctypes.byref(d), ctypes.byref(out)), out.value


@pytest.mark.parametrize("kw,status", [
    ({}, 0),
    ({"batch": 0}, 1), ({"n": -4}, 1), ({"causal": 2}, 1), ({"dtype": 5}, 1), ({"rounds": 0}, 1),
    ({"d": 96}, 2), ({"n_buckets": 7}, 2), ({"n_buckets": 8192}, 2), ({"rounds": 17}, 2),
    ({"chunk": 48}, 2), ({"chunk": 256}, 2), ({"n": 1 << 20, "n_buckets": 4096}, 2),
    ({"chunk": 8192}, 2),  # m >= n is one chunk of 4096: longer than 128
    ({"n": 100, "chunk": 128}, 0),  # one chunk of 100
])
def test_descriptor_validation(lib, kw, status):
    s, nbytes = ws_size(lib, desc(**kw))
    assert s == status, lib.lsh_attn_status_string(s)
    if status == 0:
        assert nbytes > 0 and nbytes % 256 == 0


def test_workspace_size_grows_with_problem(lib):
    _, a = ws_size(lib, desc())
    _, b = ws_size(lib, desc(rounds=4))
    _, c = ws_size(lib, desc(dtype=lb.LSH_F32))
    assert a < b and a < c


def test_calls_reject_bad_arguments_before_launch(lib):
    d = desc()
    p = ctypes.c_void_p(4096)  # never dereferenced: every check below fails first
    z = ctypes.c_void_p(0)
    # null inputs
    assert lib.lsh_attn_forward(ctypes.byref(d), z, p, p, z, p, p, p, 1 << 40, z) == 1
    assert lib.lsh_attn_hash(ctypes.byref(d), p, z, p, p, 1 << 40, z) == 1
    assert lib.lsh_attn_sort(ctypes.byref(d), z, z, z, p, z, z, p, 1 << 40, z) == 1
    # gather needs all four row pointers
    assert lib.lsh_attn_sort(ctypes.byref(d), p, p, z, p, p, p, p, 1 << 40, z) == 1
    # misaligned row pointer
    q = ctypes.c_void_p(4096 + 8)
    assert lib.lsh_attn_forward(ctypes.byref(d), q, p, p, z, p, p, p, 1 << 40, z) == 1
    # workspace: missing, misaligned, too small
    assert lib.lsh_attn_forward(ctypes.byref(d), p, p, p, z, p, p, z, 1 << 40, z) == 3
    assert lib.lsh_attn_forward(ctypes.byref(d), p, p, p, z, p, p, ctypes.c_void_p(4096 + 64),
                                1 << 40, z) == 3
    assert lib.lsh_attn_forward(ctypes.byref(d), p, p, p, z, p, p, p, 1024, z) == 3
    # unsupported problem
    d2 = desc(chunk=48)
    assert lib.lsh_attn_forward(ctypes.byref(d2), p, p, p, z, p, p, p, 1 << 40, z) == 2
    # a desc pointer of NULL
    assert lib.lsh_attn_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == 1


def test_wait_selftest_rejects_bad_arguments_before_launch(lib):
    f = lib.lsh_attn_selftest_wait_timeout
    p, z = ctypes.c_void_p(4096), None
    assert f(z, 4096, 1000, z) == 1          # no workspace
    assert f(p, 16, 1000, z) == 1            # smaller than the status header
    assert f(p, 4096, 0, z) == 1             # limit out of range
    assert f(p, 4096, 2000001, z) == 1


def test_status_strings(lib):
    for s in range(7):
        assert lib.lsh_attn_status_string(s).startswith(b"LSH_")
    assert b"unknown" in lib.lsh_attn_status_string(99)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(lb, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(lb, "_lib", None)
    with pytest.raises(ImportError):
        lb.load()


def test_dense_host_checks(lib):
    sz = ctypes.c_size_t(0)
    assert lib.lsh_attn_dense_workspace_size(ctypes.byref(desc(n=1000)), ctypes.byref(sz)) == 0
    # header, key scales [B*H][roundup(n, 128)], fixup queue [B*H*n]
    assert sz.value >= 256 + 8 * 1024 * 4 + 8 * 1000 * 4
    assert lib.lsh_attn_dense_workspace_size(ctypes.byref(desc(dtype=lb.LSH_F32)),
                                             ctypes.byref(sz)) == 2
    assert lib.lsh_attn_dense_workspace_size(ctypes.byref(desc(d=96)), ctypes.byref(sz)) == 2
    assert lib.lsh_attn_dense_workspace_size(ctypes.byref(desc(n=0)), ctypes.byref(sz)) == 1
    # null pointers and a missing workspace are refused before any launch
    p = ctypes.c_void_p(256)
    assert lib.lsh_attn_dense_forward(ctypes.byref(desc()), None, p, p, p, p, 1 << 30, None) == 1
    assert lib.lsh_attn_dense_forward(ctypes.byref(desc()), p, p, p, p, None, 0, None) == 3
