"""Python binding of libqsa.so, the C-ABI QSA hot path for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind ``include/qsa.h``.  PyTorch supplies device memory and the
current stream.  The entry points keep the C names (``qsa_prefill`` ...)
and take torch tensors; bf16 data may be ``torch.bfloat16`` or ``torch.uint16``
(bit patterns).  If libqsa.so is missing this module raises on first use:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")
LIB_DEBUG_PATH = os.path.join(_PKG, "libqsa_debug.so")   # the debug build (tests of the failure handling)

QSA_OK = 0
_STATUS = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_UNSUPPORTED", 3: "QSA_ERR_MISALIGNED",
           4: "QSA_ERR_WORKSPACE_TOO_SMALL", 5: "QSA_ERR_CUDA", 6: "QSA_ERR_DEVICE_TIMEOUT",
           7: "QSA_ERR_DEVICE_BOUNDS", 8: "QSA_ERR_ARCH"}

EXPORTED = ["qsa_default_params", "qsa_status_string", "qsa_last_error", "qsa_index_scores", "qsa_select_blocks",
            "qsa_select_workspace_size", "qsa_prefill", "qsa_prefill_workspace_size", "qsa_decode",
            "qsa_decode_workspace_size", "qsa_check_device_error", "qsa_trace_begin", "qsa_trace_end",
            "qsa_decode_noalloc", "qsa_prefill_cached", "qsa_prefill_cached_workspace_size",
            "qsa_index_workspace_size", "qsa_decode_mean_pool", "qsa_mean_pool_keys",
            "qsa_decode_reuse", "qsa_verify", "qsa_verify_workspace_size", "qsa_set_decode_splits",
            "qsa_decode_noalloc_check_error"]

KERNEL_NAMES = {1: "rope_table", 2: "rope_k", 3: "indexer", 4: "select", 5: "attention", 6: "decode_append",
                7: "decode_indexer", 8: "decode_attention", 9: "decode_combine",
                10: "mean_pool_keys", 11: "verify_expand", 12: "idx_rope"}


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class qsa_params(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("rope_theta", ctypes.c_double), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("budget_blocks", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("aggregation", ctypes.c_int32),
                ("yarn_factor", ctypes.c_double), ("yarn_original_max", ctypes.c_double),
                ("yarn_beta_fast", ctypes.c_double), ("yarn_beta_slow", ctypes.c_double),
                ("idx_rope", ctypes.c_int32)]


# block-score aggregation (qsa_params.aggregation)
AGG_TOKEN_MAX = 0
AGG_MEAN_POOL = 1

_lib = None


_libs: dict = {}
_lib_path = None


def load(path: str = LIB_PATH):
    """Load libqsa.so and declare its signatures (raises if it is not built).
    The first library loaded serves every call of this module (see
    use_library)."""
    global _lib, _lib_path
    if _lib is not None:
        return _lib
    _lib = _open(path)
    _lib_path = path
    return _lib


def use_library(path: str) -> str | None:
    """Route this module's calls to the library at ``path`` (e.g. the debug
    build, libqsa_debug.so); returns the path that served them before."""
    global _lib, _lib_path
    prev = _lib_path
    _lib = _open(path)
    _lib_path = path
    return prev


def _open(path: str):
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m block_sparse_long_qsa_b200._build` "
                          "(the QSA path has no non-CUDA fallback)")
    L = ctypes.CDLL(path)
    P, vp, i64, i32, sz = ctypes.POINTER(qsa_params), ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    psz = ctypes.POINTER(ctypes.c_size_t)
    L.qsa_default_params.argtypes = [P]
    L.qsa_default_params.restype = None
    L.qsa_status_string.argtypes = [ctypes.c_int]
    L.qsa_status_string.restype = ctypes.c_char_p
    L.qsa_last_error.argtypes = []
    L.qsa_last_error.restype = ctypes.c_char_p
    L.qsa_index_scores.argtypes = [P, i64, vp, vp, vp, i64, i64, vp, i64, vp, sz, vp]
    L.qsa_select_blocks.argtypes = [P, vp, i64, i64, i64, vp, vp, vp, sz, vp]
    L.qsa_select_workspace_size.argtypes = [P, psz]
    L.qsa_index_workspace_size.argtypes = [P, i64, psz]
    L.qsa_prefill.argtypes = [P, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.qsa_prefill_workspace_size.argtypes = [P, i64, psz, psz]
    L.qsa_prefill_cached.argtypes = [P, i64, i64] + [vp] * 16 + [sz, vp]
    L.qsa_prefill_cached_workspace_size.argtypes = [P, i64, i64, psz, psz]
    L.qsa_decode.argtypes = [P, i32, i64, ctypes.POINTER(ctypes.c_int64), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                             vp, vp, vp, vp, sz, vp]
    L.qsa_decode_workspace_size.argtypes = [P, i32, i64, psz]
    L.qsa_decode_mean_pool.argtypes = [P, i32, i64, ctypes.POINTER(ctypes.c_int64)] + [vp] * 15 + [vp, sz, vp]
    L.qsa_mean_pool_keys.argtypes = [P, i64, vp, vp, vp]
    L.qsa_verify.argtypes = [P, i32, i32, i64, ctypes.POINTER(ctypes.c_int64)] + [vp] * 15 + [vp, sz, vp]
    L.qsa_verify_workspace_size.argtypes = [P, i32, i32, i64, psz]
    L.qsa_decode_reuse.argtypes = [P, i32, i64, ctypes.POINTER(ctypes.c_int64)] + [vp] * 16 + [vp, sz, vp]
    L.qsa_decode_noalloc.argtypes = [P, i32, i64, ctypes.POINTER(ctypes.c_int64), vp, vp, vp, vp, vp, vp, vp, vp,
                                     vp, vp, vp, vp, vp, vp, vp]
    L.qsa_check_device_error.argtypes = [vp, vp]
    L.qsa_decode_noalloc_check_error.argtypes = [vp]
    L.qsa_set_decode_splits.argtypes = [i32]
    L.qsa_trace_begin.argtypes = [i32]
    L.qsa_trace_end.argtypes = [vp, vp, i32, ctypes.POINTER(ctypes.c_int32)]
    for f in EXPORTED:
        if f not in ("qsa_default_params", "qsa_status_string", "qsa_last_error"):
            getattr(L, f).restype = ctypes.c_int
    if hasattr(L, "qsa_debug_inject"):        # the debug build only
        L.qsa_debug_inject.argtypes = [i32]
        L.qsa_debug_inject.restype = ctypes.c_int
    _libs[path] = L
    return L


def params(budget: int = 512, **kw) -> qsa_params:
    p = qsa_params()
    load().qsa_default_params(ctypes.byref(p))
    p.budget_blocks = budget
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("QSA tensors must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != QSA_OK:
        detail = load().qsa_last_error().decode(errors="replace") if rc in (5, 8) else ""
        raise QSAError(rc, where, detail)


# ------------------------------------------------------------ raw entry points
def qsa_status_string(status: int) -> str:
    return load().qsa_status_string(status).decode()


def qsa_index_workspace_size(p: qsa_params, T: int) -> int:
    n = ctypes.c_size_t()
    _check(load().qsa_index_workspace_size(ctypes.byref(p), T, ctypes.byref(n)), "qsa_index_workspace_size")
    return n.value


def qsa_index_scores(p: qsa_params, T: int, q_idx, w, k_idx, qb_begin: int, qb_end: int, scores, ld: int,
                     ws=None, stream=None):
    _check(load().qsa_index_scores(ctypes.byref(p), T, _ptr(q_idx), _ptr(w), _ptr(k_idx), qb_begin, qb_end,
                                   _ptr(scores), ld, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream)), "qsa_index_scores")


def qsa_select_workspace_size(p: qsa_params) -> int:
    n = ctypes.c_size_t()
    _check(load().qsa_select_workspace_size(ctypes.byref(p), ctypes.byref(n)), "qsa_select_workspace_size")
    return n.value


def qsa_select_blocks(p: qsa_params, scores, ld: int, qb_begin: int, qb_end: int, sel, cnt, ws, stream=None):
    _check(load().qsa_select_blocks(ctypes.byref(p), _ptr(scores), ld, qb_begin, qb_end, _ptr(sel), _ptr(cnt),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "qsa_select_blocks")


def qsa_prefill_workspace_size(p: qsa_params, T: int) -> tuple[int, int]:
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().qsa_prefill_workspace_size(ctypes.byref(p), T, ctypes.byref(a), ctypes.byref(b)),
           "qsa_prefill_workspace_size")
    return a.value, b.value


def qsa_prefill(p: qsa_params, T: int, pos0: int, q, k, v, q_idx, w, k_idx, out, lse=None, sel_out=None,
                cnt_out=None, k_rot_out=None, ws=None, stream=None):
    _check(load().qsa_prefill(ctypes.byref(p), T, pos0, _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx), _ptr(w), _ptr(k_idx),
                              _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(cnt_out), _ptr(k_rot_out), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)), "qsa_prefill")


def qsa_prefill_cached_workspace_size(p: qsa_params, L_old: int, T_new: int) -> tuple[int, int]:
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().qsa_prefill_cached_workspace_size(ctypes.byref(p), L_old, T_new, ctypes.byref(a), ctypes.byref(b)),
           "qsa_prefill_cached_workspace_size")
    return a.value, b.value


def qsa_prefill_cached(p: qsa_params, L_old: int, T_new: int, k_cache, v_cache, kidx_cache, qidx_prev, w_prev, q, k,
                       v, q_idx, w, k_idx, out, lse=None, sel_out=None, cnt_out=None, ws=None, stream=None):
    _check(load().qsa_prefill_cached(ctypes.byref(p), L_old, T_new, _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache),
                                     _ptr(qidx_prev), _ptr(w_prev), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx), _ptr(w),
                                     _ptr(k_idx), _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(cnt_out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "qsa_prefill_cached")


def qsa_decode_workspace_size(p: qsa_params, B: int, max_len: int) -> int:
    n = ctypes.c_size_t()
    _check(load().qsa_decode_workspace_size(ctypes.byref(p), B, max_len, ctypes.byref(n)), "qsa_decode_workspace_size")
    return n.value


def qsa_decode(p: qsa_params, B: int, max_len: int, cache_len, k_cache, v_cache, kidx_cache, qidx_ring, w_ring,
               q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, out, sel_out=None, lse_out=None, ws=None,
               stream=None):
    """``cache_len``: host sequence of B ints (lengths before this token)."""
    lens = (ctypes.c_int64 * B)(*[int(x) for x in cache_len])
    _check(load().qsa_decode(ctypes.byref(p), B, max_len, lens, _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache),
                             _ptr(qidx_ring), _ptr(w_ring), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(q_idx_new),
                             _ptr(k_idx_new), _ptr(w_new), _ptr(out), _ptr(sel_out), _ptr(lse_out), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "qsa_decode")


def qsa_decode_mean_pool(p: qsa_params, B: int, max_len: int, cache_len, k_cache, v_cache, kidx_cache, kbar_cache,
                         qidx_ring, w_ring, q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, out, sel_out=None,
                         lse_out=None, ws=None, stream=None):
    lens = (ctypes.c_int64 * B)(*[int(x) for x in cache_len])
    _check(load().qsa_decode_mean_pool(ctypes.byref(p), B, max_len, lens, _ptr(k_cache), _ptr(v_cache),
                                       _ptr(kidx_cache), _ptr(kbar_cache), _ptr(qidx_ring), _ptr(w_ring),
                                       _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(q_idx_new), _ptr(k_idx_new),
                                       _ptr(w_new), _ptr(out), _ptr(sel_out), _ptr(lse_out), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)), "qsa_decode_mean_pool")


def qsa_decode_reuse(p: qsa_params, B: int, max_len: int, cache_len, k_cache, v_cache, kidx_cache, kbar_cache,
                     qidx_ring, w_ring, q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, sel_in, cnt_in, out,
                     lse_out=None, ws=None, stream=None):
    """Draft decode step over a reused selection (``kbar_cache`` None unless
    the parameters select mean pooling)."""
    lens = (ctypes.c_int64 * B)(*[int(x) for x in cache_len])
    _check(load().qsa_decode_reuse(ctypes.byref(p), B, max_len, lens, _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache),
                                   _ptr(kbar_cache), _ptr(qidx_ring), _ptr(w_ring), _ptr(q_new), _ptr(k_new),
                                   _ptr(v_new), _ptr(q_idx_new), _ptr(k_idx_new), _ptr(w_new), _ptr(sel_in),
                                   _ptr(cnt_in), _ptr(out), _ptr(lse_out), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "qsa_decode_reuse")


def qsa_verify_workspace_size(p: qsa_params, B: int, m: int, max_len: int) -> int:
    n = ctypes.c_size_t()
    _check(load().qsa_verify_workspace_size(ctypes.byref(p), B, m, max_len, ctypes.byref(n)),
           "qsa_verify_workspace_size")
    return n.value


def qsa_verify(p: qsa_params, B: int, m: int, max_len: int, cache_len, k_cache, v_cache, kidx_cache, qidx_prev,
               w_prev, q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, out, sel_out=None, lse_out=None, ws=None,
               stream=None, kbar_cache=None):
    """Verify m new tokens per sequence (``cache_len``: host sequence of B
    ints; ``kbar_cache`` only with mean-pooled parameters)."""
    lens = (ctypes.c_int64 * B)(*[int(x) for x in cache_len])
    _check(load().qsa_verify(ctypes.byref(p), B, m, max_len, lens, _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache),
                             _ptr(kbar_cache), _ptr(qidx_prev), _ptr(w_prev), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(q_idx_new),
                             _ptr(k_idx_new), _ptr(w_new), _ptr(out), _ptr(sel_out), _ptr(lse_out), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "qsa_verify")


def qsa_mean_pool_keys(p: qsa_params, T: int, k_idx, kbar, stream=None):
    _check(load().qsa_mean_pool_keys(ctypes.byref(p), T, _ptr(k_idx), _ptr(kbar), _stream(stream)),
           "qsa_mean_pool_keys")


def qsa_decode_noalloc(p: qsa_params, B: int, max_len: int, cache_len, k_cache, v_cache, kidx_cache, qidx_ring,
                       w_ring, q_new, k_new, v_new, q_idx_new, k_idx_new, w_new, out, sel_out=None, lse_out=None,
                       stream=None):
    """qsa_decode on the library's fixed scratch array (no workspace, no allocation)."""
    lens = (ctypes.c_int64 * B)(*[int(x) for x in cache_len])
    _check(load().qsa_decode_noalloc(ctypes.byref(p), B, max_len, lens, _ptr(k_cache), _ptr(v_cache),
                                     _ptr(kidx_cache), _ptr(qidx_ring), _ptr(w_ring), _ptr(q_new), _ptr(k_new),
                                     _ptr(v_new), _ptr(q_idx_new), _ptr(k_idx_new), _ptr(w_new), _ptr(out),
                                     _ptr(sel_out), _ptr(lse_out), _stream(stream)), "qsa_decode_noalloc")


def qsa_check_device_error(ws, stream=None) -> int:
    return load().qsa_check_device_error(_ptr(ws), _stream(stream))


def qsa_decode_noalloc_check_error(stream=None) -> int:
    """Device error word of qsa_decode_noalloc's fixed array (synchronises)."""
    return load().qsa_decode_noalloc_check_error(_stream(stream))


# fault-injection codes of the debug build (include/qsa_debug.h)
INJECT_INDEXER_STALL = 1
INJECT_ATTENTION_STALL = 2
INJECT_ATTENTION_BAD_BLOCK = 3
INJECT_ATTENTION_RESCALE_ALL = 4


def qsa_debug_inject(code: int):
    """Arm a test fault for the next launch of the kernel it names (the debug
    build, libqsa_debug.so, only)."""
    L = load()
    if not hasattr(L, "qsa_debug_inject"):
        raise RuntimeError("qsa_debug_inject exists only in the debug build (use_library(LIB_DEBUG_PATH))")
    _check(L.qsa_debug_inject(int(code)), "qsa_debug_inject")


def qsa_set_decode_splits(n: int):
    """Fix the number of split-KV decode ranges (1..16) for this process; 0 = automatic."""
    _check(load().qsa_set_decode_splits(int(n)), "qsa_set_decode_splits")


class trace:
    """Context manager: per-launch device times of this library's kernels,
    from CUDA events recorded on each launching stream.  ``.records`` is a
    list of (kernel name, milliseconds) in launch order."""

    def __init__(self, capacity: int = 4096):
        self.capacity = capacity
        self.records = []

    def __enter__(self):
        _check(load().qsa_trace_begin(self.capacity), "qsa_trace_begin")
        return self

    def __exit__(self, *exc):
        ids = (ctypes.c_int32 * self.capacity)()
        ms = (ctypes.c_float * self.capacity)()
        n = ctypes.c_int32()
        _check(load().qsa_trace_end(ids, ms, self.capacity, ctypes.byref(n)), "qsa_trace_end")
        self.records = [(KERNEL_NAMES.get(ids[i], str(ids[i])), ms[i]) for i in range(n.value)]
        return False

    def by_kernel(self) -> dict:
        out = {}
        for name, t in self.records:
            c, tot = out.get(name, (0, 0.0))
            out[name] = (c + 1, tot + t)
        return out


# ----------------------------------------------------- allocating conveniences
def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def prefill(q, k, v, q_idx, w, k_idx, budget: int = 512, pos0: int = 0, want_lse=True, want_sel=True,
            want_krot=False, ws_bytes: int | None = None, stream=None, aggregation: int = AGG_TOKEN_MAX,
            idx_rope: int = 0):
    """Allocate outputs and a workspace, run qsa_prefill; returns a dict."""
    T = q.shape[0]
    dev = q.device
    p = params(budget, aggregation=aggregation, idx_rope=idx_rope)
    mn, pref = qsa_prefill_workspace_size(p, T)
    ws = workspace(pref if ws_bytes is None else max(ws_bytes, mn), dev)
    nqb = (T + 3) // 4
    res = dict(out=torch.empty((T, 24, 256), dtype=torch.uint16, device=dev))
    res["lse"] = torch.empty((T, 24), dtype=torch.float32, device=dev) if want_lse else None
    res["sel"] = torch.empty((nqb, budget), dtype=torch.int32, device=dev) if want_sel else None
    res["cnt"] = torch.empty((nqb,), dtype=torch.int32, device=dev) if want_sel else None
    res["k_rot"] = torch.empty((T, 2, 256), dtype=torch.uint16, device=dev) if want_krot else None
    qsa_prefill(p, T, pos0, q, k, v, q_idx, w, k_idx, res["out"], res["lse"], res["sel"], res["cnt"], res["k_rot"],
                ws, stream)
    res["ws"] = ws
    return res
