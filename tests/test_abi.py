"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before touching a GPU (CPU-only tests)."""
import ctypes
import os
import re

import pytest

import block_sparse_long_qsa_b200 as qsa
from block_sparse_long_qsa_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return qsa.load()


def header_functions(name="qsa.h"):
    src = open(os.path.join(ROOT, "include", name)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(qsa.EXPORTED)


def test_debug_build_exports_the_hooks():
    """The debug build (libqsa_debug.so) exports every symbol of qsa.h and
    the test hooks of qsa_debug.h; the release library has no hook."""
    path = _build.build(debug=True)
    D = ctypes.CDLL(path)
    for n in header_functions() + header_functions("qsa_debug.h"):
        assert hasattr(D, n), n
    R = ctypes.CDLL(_build.build())
    for n in header_functions("qsa_debug.h"):
        assert not hasattr(R, n), n


def test_status_strings(lib):
    for s in range(9):
        assert qsa.qsa_status_string(s)
    assert qsa.qsa_status_string(0) == "ok"


def test_default_params_match_pages(lib):
    p = qsa.params()
    assert (p.n_q_heads, p.n_kv_heads, p.head_dim, p.rope_dim) == (24, 2, 256, 64)
    assert (p.idx_heads, p.idx_dim, p.block_size, p.budget_blocks) == (4, 128, 4, 512)
    assert p.rope_theta == 1e7


def _call_prefill(p, T=64, align=0, null=None, ws_bytes=1 << 30):
    fake = 1 << 20
    ptrs = [fake + i * 4096 for i in range(12)]
    ptrs = [x + align for x in ptrs]
    if null is not None:
        ptrs[null] = None
    L = qsa.load()
    return L.qsa_prefill(ctypes.byref(p), T, 0, *ptrs[:6], ptrs[6], None, None, None, None, ptrs[11], ws_bytes,
                         None)


def test_host_validation_without_gpu(lib):
    p = qsa.params()
    bad = qsa.params(n_q_heads=32)
    assert _call_prefill(bad) == 2                         # unsupported shape
    assert _call_prefill(qsa.params(budget=1)) == 2        # budget < 2
    assert _call_prefill(p, null=0) == 1                   # null q
    assert _call_prefill(p, align=8) == 3                  # misaligned
    assert _call_prefill(p, T=0) == 1
    assert _call_prefill(p, ws_bytes=100) == 4             # workspace too small


def test_workspace_sizes(lib):
    p = qsa.params()
    mn, pref = qsa.qsa_prefill_workspace_size(p, 32768)
    assert 0 < mn <= pref
    mn1, pref1 = qsa.qsa_prefill_workspace_size(p, 1 << 20)
    assert pref1 <= (16 << 30) + (2 << 30)
    assert qsa.qsa_decode_workspace_size(p, 64, 262144 + 32) > 64 * 65537 * 4
    assert qsa.qsa_select_workspace_size(p) >= 4
    with pytest.raises(qsa.QSAError):
        qsa.qsa_prefill_workspace_size(p, 0)


def test_decode_validation(lib):
    p = qsa.params()
    L = qsa.load()
    lens = (ctypes.c_int64 * 2)(10, 20)
    fake = [(1 << 20) + 4096 * i for i in range(16)]
    # cache_len >= max_len is rejected before any launch
    rc = L.qsa_decode(ctypes.byref(p), 2, 16, lens, *fake[:11], fake[11], None, None, fake[12], 1 << 30, None)
    assert rc == 1
    rc = L.qsa_decode(ctypes.byref(p), 2, 64, lens, *fake[:11], fake[11], None, None, fake[12], 16, None)
    assert rc == 4


def header_arg_counts():
    """Number of parameters of every function prototype in the header."""
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for name, args in re.findall(r"\b(qsa_[a-z_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        args = args.strip()
        out[name] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_signatures_match_header(lib):
    """Every ctypes signature the binding declares has the header's
    parameter count (a wrong count would shift pointer arguments)."""
    counts = header_arg_counts()
    assert len(counts) >= 10
    for name, n in counts.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
