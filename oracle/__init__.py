"""CPU oracle of the QSA hot path (fp64, plain definitions).

TEST INFRASTRUCTURE, NOT PRODUCT.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA library; ``oracle.c`` holds the definitions (with their
citations) and this module only marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


class Params(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("rope_theta", ctypes.c_double), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("budget", ctypes.c_int32),
                ("softmax_scale", ctypes.c_double), ("aggregation", ctypes.c_int32),
                ("yarn_factor", ctypes.c_double), ("yarn_original_max", ctypes.c_double),
                ("yarn_beta_fast", ctypes.c_double), ("yarn_beta_slow", ctypes.c_double),
                ("idx_rope", ctypes.c_int32), ("idx_exact", ctypes.c_int32), ("idx_pos0", ctypes.c_int64)]


# block-score aggregation: max over causal token pairs, or mean-pooled block keys
AGG_TOKEN_MAX = 0
AGG_MEAN_POOL = 1


def params(budget=512, block=4, n_q_heads=24, n_kv_heads=2, head_dim=256, rope_dim=64, rope_theta=1e7,
           idx_heads=4, idx_dim=128, softmax_scale=0.0, aggregation=AGG_TOKEN_MAX, yarn_factor=0.0,
           yarn_original_max=262144.0, yarn_beta_fast=32.0, yarn_beta_slow=1.0, idx_rope=0, idx_exact=0,
           idx_pos0=0) -> Params:
    return Params(n_q_heads, n_kv_heads, head_dim, rope_dim, rope_theta, idx_heads, idx_dim, block, budget,
                  softmax_scale, aggregation, yarn_factor, yarn_original_max, yarn_beta_fast, yarn_beta_slow,
                  idx_rope, idx_exact, idx_pos0)


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src)):
        return _LIB_PATH
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", src, "-o", _LIB_PATH, "-lm"],
                   check=True)
    return _LIB_PATH


def load_variant(path: str):
    """Load a separately compiled copy of oracle.c (used by the mutation tests)."""
    return _bind(ctypes.CDLL(path))


_lib = None


def _bind(L):
    P, vp, i64, i32 = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    L.oracle_rope.argtypes = [P, vp, i64, vp]
    L.oracle_token_score.argtypes = [P, vp, vp, vp]
    L.oracle_token_score.restype = ctypes.c_double
    L.oracle_block_scores.argtypes = [P, i64, ctypes.c_int, vp, vp, vp, vp]
    L.oracle_select.argtypes = [P, i64, vp, vp, vp]
    L.oracle_attend.argtypes = [P, vp, i64, vp, vp, vp, vp]
    L.oracle_index_scores.argtypes = [P, i64, vp, vp, vp, i64, i64, vp, i64]
    L.oracle_select_rows.argtypes = [P, vp, i64, i64, i64, vp, vp]
    L.oracle_attend_blocks.argtypes = [P, i64, i64, vp, vp, vp, i64, vp, vp, vp, vp, vp]
    L.oracle_prefill_blocks.argtypes = [P, i64, i64, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp]
    L.oracle_reuse_selection.argtypes = [i64, vp, ctypes.c_int32, vp]
    L.oracle_reuse_selection.restype = ctypes.c_int32
    L.oracle_select_blocks_list.argtypes = [P, i64, vp, vp, vp, i64, vp, vp, vp]
    L.oracle_attend_gathered.argtypes = [P, i64, vp, i64, vp, vp, vp, vp, vp]
    L.oracle_decode.argtypes = [P, i64, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
    L.oracle_decode.restype = i32
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


class Oracle:
    """numpy-facing wrapper; ``L`` may be a mutated variant for self-tests."""

    def __init__(self, P: Params | None = None, L=None):
        self.P = P if P is not None else params()
        self.L = L if L is not None else lib()

    @property
    def budget(self):
        return self.P.budget

    def rope(self, x: np.ndarray, pos: int) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty_like(x)
        self.L.oracle_rope(ctypes.byref(self.P), _p(x), pos, _p(y))
        return y

    def token_score(self, q_t, w_t, k_j) -> float:
        return self.L.oracle_token_score(ctypes.byref(self.P), _p(_u16(q_t)), _p(_u16(w_t)), _p(_u16(k_j)))

    def index_scores(self, T, q_idx, w, k_idx, qb_begin=0, qb_end=None, ld=None) -> np.ndarray:
        """S[(qb - qb_begin), kb] for kb <= qb; other entries NaN."""
        r = self.P.block
        nqb = (T + r - 1) // r
        qb_end = nqb if qb_end is None else qb_end
        ld = qb_end if ld is None else ld
        S = np.full((qb_end - qb_begin, ld), np.nan)
        q_idx, w, k_idx = _u16(q_idx), _u16(w), _u16(k_idx)
        self.L.oracle_index_scores(ctypes.byref(self.P), T, _p(q_idx), _p(w), _p(k_idx), qb_begin, qb_end, _p(S), ld)
        return S

    def block_scores(self, qb, q_blk, w_blk, k_idx) -> np.ndarray:
        q_blk, w_blk, k_idx = _u16(q_blk), _u16(w_blk), _u16(k_idx)
        S = np.empty(qb + 1)
        self.L.oracle_block_scores(ctypes.byref(self.P), qb, q_blk.shape[0], _p(q_blk), _p(w_blk), _p(k_idx), _p(S))
        return S

    def select(self, qb, S_row) -> tuple[np.ndarray, int]:
        S_row = np.ascontiguousarray(S_row, dtype=np.float64)
        sel = np.empty(self.P.budget, dtype=np.int32)
        cnt = np.zeros(1, dtype=np.int32)
        self.L.oracle_select(ctypes.byref(self.P), qb, _p(S_row), _p(sel), _p(cnt))
        return sel, int(cnt[0])

    def select_rows(self, S, qb_begin=0) -> tuple[np.ndarray, np.ndarray]:
        S = np.ascontiguousarray(S, dtype=np.float64)
        n = S.shape[0]
        sel = np.empty((n, self.P.budget), dtype=np.int32)
        cnt = np.empty(n, dtype=np.int32)
        self.L.oracle_select_rows(ctypes.byref(self.P), _p(S), S.shape[1], qb_begin, qb_begin + n, _p(sel), _p(cnt))
        return sel, cnt

    def attend(self, q_rot, k_rot, v) -> tuple[np.ndarray, np.ndarray]:
        q_rot = np.ascontiguousarray(q_rot, dtype=np.float64)
        k_rot = np.ascontiguousarray(k_rot, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        H, d = self.P.n_q_heads, self.P.head_dim
        out = np.empty((H, d))
        lse = np.empty(H)
        self.L.oracle_attend(ctypes.byref(self.P), _p(q_rot), k_rot.shape[0], _p(k_rot), _p(v), _p(out), _p(lse))
        return out, lse

    def attend_blocks(self, T, q, k, v, qb_list, sel, cnt, pos0=0):
        qb_list = np.ascontiguousarray(qb_list, dtype=np.int64)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        cnt = np.ascontiguousarray(cnt, dtype=np.int32)
        n, r = len(qb_list), self.P.block
        H, d = self.P.n_q_heads, self.P.head_dim
        out = np.empty((n * r, H, d))
        lse = np.empty((n * r, H))
        q, k, v = _u16(q), _u16(k), _u16(v)
        self.L.oracle_attend_blocks(ctypes.byref(self.P), T, pos0, _p(q), _p(k), _p(v), n, _p(qb_list), _p(sel),
                                    _p(cnt), _p(out), _p(lse))
        return out, lse

    def attend_gathered(self, pos_t, q_t, pos_j, k_rows, v_rows):
        """One token at position pos_t (unrotated q_t [24][256]) over the
        candidate keys at positions pos_j (unrotated k_rows, v_rows
        [n][2][256]); keys after pos_t are skipped.  -> (out [24][256], lse [24])."""
        H, d = self.P.n_q_heads, self.P.head_dim
        pos_j = np.ascontiguousarray(pos_j, dtype=np.int64)
        q_t, k_rows, v_rows = _u16(q_t), _u16(k_rows), _u16(v_rows)
        assert k_rows.shape[0] == v_rows.shape[0] == pos_j.shape[0]
        out = np.empty((H, d))
        lse = np.empty(H)
        self.L.oracle_attend_gathered(ctypes.byref(self.P), int(pos_t), _p(q_t), len(pos_j), _p(pos_j), _p(k_rows),
                                      _p(v_rows), _p(out), _p(lse))
        return out, lse

    def select_blocks_list(self, T, q_idx, w, k_idx, qb_list):
        """(sel [n][budget], cnt [n]) of the listed query blocks (scores + selection)."""
        qb_list = np.ascontiguousarray(qb_list, dtype=np.int64)
        n = len(qb_list)
        sel = np.empty((n, self.P.budget), dtype=np.int32)
        cnt = np.empty(n, dtype=np.int32)
        q_idx, w, k_idx = _u16(q_idx), _u16(w), _u16(k_idx)
        self.L.oracle_select_blocks_list(ctypes.byref(self.P), T, _p(q_idx), _p(w), _p(k_idx), n, _p(qb_list),
                                         _p(sel), _p(cnt))
        return sel, cnt

    def prefill_blocks(self, T, q, k, v, q_idx, w, k_idx, qb_list=None, pos0=0):
        """(sel [n][budget], cnt [n], out [n*r][H][d], lse [n*r][H]) for the listed query blocks."""
        r = self.P.block
        if qb_list is None:
            qb_list = np.arange((T + r - 1) // r)
        qb_list = np.ascontiguousarray(qb_list, dtype=np.int64)
        n = len(qb_list)
        H, d = self.P.n_q_heads, self.P.head_dim
        sel = np.empty((n, self.P.budget), dtype=np.int32)
        cnt = np.empty(n, dtype=np.int32)
        out = np.empty((n * r, H, d))
        lse = np.empty((n * r, H))
        q, k, v, q_idx, w, k_idx = map(_u16, (q, k, v, q_idx, w, k_idx))
        self.L.oracle_prefill_blocks(ctypes.byref(self.P), T, pos0, _p(q), _p(k), _p(v), _p(q_idx), _p(w), _p(k_idx),
                                     n, _p(qb_list), _p(sel), _p(cnt), _p(out), _p(lse))
        return sel, cnt, out, lse

    def decode(self, L, k_cache, v_cache, kidx_cache, ring_q_idx, ring_w, q_new, k_new, v_new, q_idx_new, k_idx_new,
               w_new, sel_in=None, cnt_in=0):
        """One decode token at position L; caches hold rows [0, L).  ring_q_idx
        [n][4][128] / ring_w [n][4] are the block-mates 4*(L//4) .. L-1, in
        order (n = L % 4 rows exactly; anything else raises)."""
        H, d = self.P.n_q_heads, self.P.head_dim
        out = np.empty((H, d))
        lse = np.empty(H)
        sel = np.empty(self.P.budget, dtype=np.int32)
        cnt = np.zeros(1, dtype=np.int32)
        args = [_u16(a) for a in (k_cache, v_cache, kidx_cache, ring_q_idx, ring_w, q_new, k_new, v_new, q_idx_new,
                                  k_idx_new, w_new)]
        n_ring = args[3].shape[0]
        if args[4].shape[0] != n_ring:
            raise ValueError("ring_q_idx and ring_w hold different numbers of block-mates")
        si = None if sel_in is None else np.ascontiguousarray(sel_in, dtype=np.int32)
        ptrs = [_p(a) for a in args]
        rc = self.L.oracle_decode(ctypes.byref(self.P), L, *ptrs[:5], int(n_ring), *ptrs[5:], _p(si), int(cnt_in),
                                  _p(sel), _p(cnt), _p(out), _p(lse))
        if rc != 0:
            raise ValueError(f"oracle_decode: {n_ring} ring rows given, token {L} has {L % self.P.block} block-mates")
        return sel, int(cnt[0]), out, lse

    def reuse_selection(self, qb, sel_in, cnt_in):
        """Blocks a draft token of query block qb attends with a reused top-k
        row (the row's first cnt_in entries joined with qb - 1 and qb)."""
        si = np.ascontiguousarray(np.asarray(sel_in, dtype=np.int32)[:cnt_in])
        out = np.empty(int(cnt_in) + 2, dtype=np.int32)
        n = self.L.oracle_reuse_selection(int(qb), _p(si) if cnt_in else None, int(cnt_in), _p(out))
        if n < 0:
            raise ValueError("reused selection is not causal")
        return out[:n], int(n)

    def decode_reuse(self, L, k_cache, v_cache, kidx_cache, ring_q_idx, ring_w, q_new, k_new, v_new, q_idx_new,
                     k_idx_new, w_new, sel_in, cnt_in):
        """Draft decode token at position L over a reused top-k row."""
        sel, n = self.reuse_selection(L // self.P.block, sel_in, cnt_in)
        _, _, out, lse = self.decode(L, k_cache, v_cache, kidx_cache, ring_q_idx, ring_w, q_new, k_new, v_new,
                                     q_idx_new, k_idx_new, w_new, sel_in=sel, cnt_in=n)
        return sel, n, out, lse
