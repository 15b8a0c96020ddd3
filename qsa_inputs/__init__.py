"""Seeded synthetic inputs for the QSA hot path.

Test and benchmark infrastructure: this module is the one place both the
CPU oracle and the CUDA library get their inputs from.  It holds none of the
attention method's arithmetic.  Every value is a pure function of
(seed, stream, element index) computed by ``gen.cu``, which is compiled for
the host (OpenMP) and for the GPU from one source and gives bit-identical
values on both, so a sampled element of a full-size device tensor can be
regenerated on the host for the oracle.

Workload recipe (synthetic stand-ins for the 32K-1M token contexts on which
the pages quote their kernel speedups; no dataset is involved):

* q ``[T][24][256]``, k, v ``[T][2][256]``, q_idx ``[T][4][128]``,
  k_idx ``[T][128]``: bf16 of N(0, 1).
* w ``[T][4]``: bf16 of the softmax of four N(0, 1) draws per token.
* planted blocks: every query block qb picks ``n_plant`` distinct earlier key
  blocks (uniform on [0, qb-1], or distance d = qb - kb from Zipf(1.1) on
  [1, qb] by exact inverse CDF); a key block picked by several query blocks
  belongs to the largest one; its 4 key rows of k_idx become
  bf16(mean of the planter's (token, head) q_idx vectors + 0.3 N(0,1)).
  Query blocks with qb <= n_plant plant all their earlier blocks.
* decode: sequence b draws from seed ``seq_seed(seed, b)``; its L cached
  tokens hold already-rotated keys (stream S_KROT), values and indexer keys;
  ``n_plant`` uniform key blocks are planted against the block-mates of the
  first decode token; decode token t uses the same per-token streams as a
  prefill of that sequence would.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libqsagen.so")

# stream ids, one per tensor
S_Q, S_K, S_V, S_QIDX, S_W, S_KIDX, S_PNOISE, S_PCHOICE, S_KROT = 1, 2, 3, 4, 5, 6, 7, 8, 9

N_Q_HEADS, N_KV_HEADS, HEAD_DIM = 24, 2, 256
IDX_HEADS, IDX_DIM, BLOCK = 4, 128, 4
MASK64 = (1 << 64) - 1
MAX_ATTEMPTS = 4096


def build(force: bool = False) -> str:
    """Compile gen.cu into libqsagen.so (host + sm_100a device code)."""
    src = os.path.join(_HERE, "gen.cu")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src)):
        return _LIB_PATH
    cmd = ["nvcc", "-O2", "--fmad=false", "-shared", "-Xcompiler", "-fPIC,-fopenmp,-ffp-contract=off",
           "-gencode", "arch=compute_100a,code=sm_100a", src, "-o", _LIB_PATH, "-lgomp"]
    subprocess.run(cmd, check=True)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, u32, i64, vp, ci = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        L.qsagen_normal_bf16.argtypes = [u64, u32, u64, u64, vp]
        L.qsagen_normal_f64.argtypes = [u64, u32, u64, u64, vp]
        L.qsagen_uniform.argtypes = [u64, u32, u64, u64, vp]
        L.qsagen_softmax4_bf16.argtypes = [u64, u32, u64, u64, vp]
        L.qsagen_plant.argtypes = [i64, ci, i64, i64, ci, ci, vp, vp, vp, vp, u64, u32]
        L.qsagen_normal_bf16_dev.argtypes = [u64, u32, u64, u64, vp, vp]
        L.qsagen_softmax4_bf16_dev.argtypes = [u64, u32, u64, u64, vp, vp]
        L.qsagen_plant_dev.argtypes = [i64, ci, i64, i64, ci, ci, vp, vp, vp, vp, u64, u32, vp]
        for f in ("qsagen_normal_bf16_dev", "qsagen_softmax4_bf16_dev", "qsagen_plant_dev"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def seq_seed(seed: int, b: int) -> int:
    """Seed of decode sequence b."""
    return (seed * 0x100000001B3 + (b + 1) * 0x9E3779B97F4A7C15) & MASK64


# ------------------------------------------------------------------ host side
def normal_bf16(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    if n:
        lib().qsagen_normal_bf16(seed & MASK64, stream, offset, n, _ptr(out))
    return out


def normal_f64(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        lib().qsagen_normal_f64(seed & MASK64, stream, offset, n, _ptr(out))
    return out


def uniform(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        lib().qsagen_uniform(seed & MASK64, stream, offset, n, _ptr(out))
    return out


def softmax4_bf16(seed: int, stream: int, tok0: int, ntok: int) -> np.ndarray:
    out = np.empty((ntok, 4), dtype=np.uint16)
    if ntok:
        lib().qsagen_softmax4_bf16(seed & MASK64, stream, tok0, ntok, _ptr(out))
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a).astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    return bf16_to_f32(a).astype(np.float64)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bits (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def uniform_at(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """Uniforms in [0, 1) at arbitrary counter indices: the same definition as
    ``gen_u64`` / ``gen_u01`` in gen.cu, evaluated in numpy uint64 arithmetic."""
    idx = np.asarray(idx, dtype=np.int64)
    with np.errstate(over="ignore"):
        key0 = (seed * 0xD1B54A32D192ED03 + stream * 0x9E3779B97F4A7C15 + 0x632BE59BD9B4E019) & MASK64
        key = _mix64_np(np.array([key0], dtype=np.uint64))[0]
        z = key + (idx.astype(np.uint64) + np.uint64(1)) * np.uint64(0x9E3779B97F4A7C15)
        r = _mix64_np(z)
    return (r >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


# ------------------------------------------------------------- planted blocks
_ZIPF_H: dict = {}


def _zipf_cum(n: int, s: float = 1.1) -> np.ndarray:
    """H[d] = sum_{i<=d} i^-s for d = 0..n (H[0] = 0)."""
    H = _ZIPF_H.get(s)
    if H is None or len(H) <= n:
        m = max(n + 1, 1024)
        H = np.concatenate([[0.0], np.cumsum(np.arange(1, m, dtype=np.float64) ** (-s))])
        _ZIPF_H[s] = H
    return H


def plant_choices(seed: int, qb_list, n_plant: int, dist: str):
    """Key blocks planted by each query block in ``qb_list``.

    Returns parallel int64 arrays (qbs, kbs).  Draw ``a`` of query block qb
    uses the uniform at counter index qb * MAX_ATTEMPTS + a of stream
    S_PCHOICE; a draw equal to an earlier pick of the same query block is
    skipped.
    """
    qb_list = np.asarray(qb_list, dtype=np.int64)
    out_q, out_k = [], []
    if n_plant <= 0 or len(qb_list) == 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    small = qb_list[(qb_list >= 1) & (qb_list <= n_plant)]
    for qb in small:
        out_q.append(np.full(qb, qb, dtype=np.int64))
        out_k.append(np.arange(qb, dtype=np.int64))
    big = qb_list[qb_list > n_plant]
    if len(big):
        chosen = np.full((len(big), n_plant), -1, dtype=np.int64)
        nch = np.zeros(len(big), dtype=np.int64)
        H = _zipf_cum(int(big.max())) if dist == "zipf" else None
        active = np.arange(len(big))
        for a in range(MAX_ATTEMPTS):
            if len(active) == 0:
                break
            qb = big[active]
            u = uniform_at(seed, S_PCHOICE, qb * MAX_ATTEMPTS + a)
            if dist == "uniform":
                kb = np.minimum((u * qb).astype(np.int64), qb - 1)
            elif dist == "zipf":
                d = np.searchsorted(H, u * H[qb], side="left")
                kb = qb - np.clip(d, 1, qb)
            else:
                raise ValueError(dist)
            ok = ~(chosen[active] == kb[:, None]).any(axis=1)
            rows = active[ok]
            chosen[rows, nch[rows]] = kb[ok]
            nch[rows] += 1
            active = active[nch[active] < n_plant]
        for i in active:  # attempts exhausted: nearest unchosen earlier blocks
            qb = int(big[i])
            for d in range(1, qb + 1):
                if nch[i] >= n_plant:
                    break
                if (qb - d) not in chosen[i, :nch[i]]:
                    chosen[i, nch[i]] = qb - d
                    nch[i] += 1
        out_q.append(np.repeat(big, n_plant))
        out_k.append(chosen.reshape(-1))
    if not out_q:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    return np.concatenate(out_q), np.concatenate(out_k)


def planter_map(seed: int, nqb: int, n_plant: int, dist: str) -> np.ndarray:
    """planter[kb] = largest query block that planted kb, or -1."""
    planter = np.full(nqb, -1, dtype=np.int64)
    qbs, kbs = plant_choices(seed, np.arange(nqb), n_plant, dist)
    if len(qbs):
        np.maximum.at(planter, kbs, qbs)
    return planter


def stratified_query_blocks(nqb: int, n: int = 256, budget: int = 512, seed: int = 0) -> np.ndarray:
    """A stratified sample of min(n, nqb) query-block indices of a prefill
    with nqb blocks (a sampling recipe for the checks and the CPU baseline,
    not part of the method): the first three, the last three, the six around
    the budget boundary (budget - 3 .. budget + 2, where selection starts to
    drop blocks), four seeded random ones, and the rest evenly spaced over
    [0, nqb); sorted and distinct."""
    n = min(n, nqb)
    fixed = [0, 1, 2, nqb - 3, nqb - 2, nqb - 1] + list(range(budget - 3, budget + 3))
    rng = np.random.default_rng(seed)
    fixed += rng.integers(0, max(nqb, 1), size=4).tolist()
    picked = sorted({int(q) for q in fixed if 0 <= q < nqb})[:n]
    chosen = set(picked)
    # evenly spaced fill: walk a fine grid and take every point not yet chosen
    need = n - len(chosen)
    if need > 0:
        free = np.setdiff1d(np.arange(nqb, dtype=np.int64), np.fromiter(chosen, np.int64, len(chosen)))
        idx = np.linspace(0, len(free) - 1, need).round().astype(np.int64)
        chosen.update(int(q) for q in free[np.unique(idx)])
        extra = need - len(np.unique(idx))
        if extra > 0:
            rest = np.setdiff1d(free, np.fromiter(chosen, np.int64, len(chosen)))
            chosen.update(int(q) for q in rest[:extra])
    return np.array(sorted(chosen), dtype=np.int64)


# ------------------------------------------------------------------ prefill
@dataclass
class PrefillProblem:
    """One prefill sequence of T tokens (see the module docstring)."""
    T: int
    seed: int = 0
    n_plant: int = 0
    dist: str = "uniform"

    @property
    def nqb(self) -> int:
        return (self.T + BLOCK - 1) // BLOCK

    def planter(self) -> np.ndarray:
        if not hasattr(self, "_planter"):
            self._planter = planter_map(self.seed, self.nqb, self.n_plant, self.dist)
        return self._planter

    # host rows [t0, t1)
    def q(self, t0=0, t1=None):
        t1 = self.T if t1 is None else t1
        n = N_Q_HEADS * HEAD_DIM
        return normal_bf16(self.seed, S_Q, t0 * n, (t1 - t0) * n).reshape(t1 - t0, N_Q_HEADS, HEAD_DIM)

    def k(self, t0=0, t1=None):
        t1 = self.T if t1 is None else t1
        n = N_KV_HEADS * HEAD_DIM
        return normal_bf16(self.seed, S_K, t0 * n, (t1 - t0) * n).reshape(t1 - t0, N_KV_HEADS, HEAD_DIM)

    def v(self, t0=0, t1=None):
        t1 = self.T if t1 is None else t1
        n = N_KV_HEADS * HEAD_DIM
        return normal_bf16(self.seed, S_V, t0 * n, (t1 - t0) * n).reshape(t1 - t0, N_KV_HEADS, HEAD_DIM)

    def q_idx(self, t0=0, t1=None):
        t1 = self.T if t1 is None else t1
        n = IDX_HEADS * IDX_DIM
        return normal_bf16(self.seed, S_QIDX, t0 * n, (t1 - t0) * n).reshape(t1 - t0, IDX_HEADS, IDX_DIM)

    def w(self, t0=0, t1=None):
        t1 = self.T if t1 is None else t1
        return softmax4_bf16(self.seed, S_W, t0, t1 - t0)

    def k_idx(self, t0=0, t1=None):
        """Indexer keys of tokens [t0, t1), planted blocks applied."""
        t1 = self.T if t1 is None else t1
        out = normal_bf16(self.seed, S_KIDX, t0 * IDX_DIM, (t1 - t0) * IDX_DIM).reshape(t1 - t0, IDX_DIM)
        if self.n_plant <= 0 or t1 <= t0:
            return out
        kb0, kb1 = t0 // BLOCK, (t1 - 1) // BLOCK + 1
        pl = self.planter()[kb0:kb1]
        if (pl < 0).all():
            return out
        # compact buffer of the planters' q_idx rows
        uniq = np.unique(pl[pl >= 0])
        slot = {int(p): i for i, p in enumerate(uniq)}
        q_src = np.zeros((len(uniq) * BLOCK, IDX_HEADS, IDX_DIM), dtype=np.uint16)
        n_src = np.zeros(kb1 - kb0, dtype=np.int64)
        src_tok = np.full(kb1 - kb0, -1, dtype=np.int64)
        for p, i in slot.items():
            tp0, tp1 = p * BLOCK, min(p * BLOCK + BLOCK, self.T)
            q_src[i * BLOCK: i * BLOCK + (tp1 - tp0)] = self.q_idx(tp0, tp1)
        for b, p in enumerate(pl):
            if p >= 0:
                src_tok[b] = slot[int(p)] * BLOCK
                n_src[b] = min(BLOCK, self.T - p * BLOCK)
        # keys buffer aligned to block kb0 (rows before t0 are scratch)
        r0 = kb0 * BLOCK
        buf = np.zeros((min(kb1 * BLOCK, self.T) - r0, IDX_DIM), dtype=np.uint16)
        buf[t0 - r0: t1 - r0] = out
        lib().qsagen_plant(kb1 - kb0, BLOCK, buf.shape[0], r0, IDX_HEADS, IDX_DIM, _ptr(src_tok), _ptr(n_src),
                           _ptr(q_src), _ptr(buf), self.seed & MASK64, S_PNOISE)
        return np.ascontiguousarray(buf[t0 - r0: t1 - r0])

    def host(self) -> dict:
        return dict(q=self.q(), k=self.k(), v=self.v(), q_idx=self.q_idx(), w=self.w(), k_idx=self.k_idx())

    def device_rows(self, name: str, t0: int, t1: int, device="cuda"):
        """Rows [t0, t1) of one input generated on the GPU, bit-identical to the
        host generator's rows -- except k_idx, whose planted blocks are not
        applied here (use ``device()`` or ``k_idx()`` for those)."""
        import torch
        shapes = dict(q=(N_Q_HEADS, HEAD_DIM, S_Q), k=(N_KV_HEADS, HEAD_DIM, S_K), v=(N_KV_HEADS, HEAD_DIM, S_V),
                      q_idx=(IDX_HEADS, IDX_DIM, S_QIDX), k_idx=(IDX_DIM, S_KIDX))
        cs = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
        L = lib()
        n = t1 - t0
        if name == "w":
            t = torch.empty((n, IDX_HEADS), dtype=torch.uint16, device=device)
            _chk(L.qsagen_softmax4_bf16_dev(self.seed & MASK64, S_W, t0, n, t.data_ptr(), cs))
            return t
        *dims, st = shapes[name]
        per = int(np.prod(dims))
        t = torch.empty((n, *dims), dtype=torch.uint16, device=device)
        _chk(L.qsagen_normal_bf16_dev(self.seed & MASK64, st, t0 * per, n * per, t.data_ptr(), cs))
        return t

    def device(self, device="cuda", stream=None) -> dict:
        """Full tensors generated on the GPU (bit-identical to ``host()``)."""
        import torch
        T = self.T
        cs = ctypes.c_void_p(stream.cuda_stream if stream is not None
                             else torch.cuda.current_stream(device).cuda_stream)
        L = lib()
        t = dict(q=torch.empty((T, N_Q_HEADS, HEAD_DIM), dtype=torch.uint16, device=device),
                 k=torch.empty((T, N_KV_HEADS, HEAD_DIM), dtype=torch.uint16, device=device),
                 v=torch.empty((T, N_KV_HEADS, HEAD_DIM), dtype=torch.uint16, device=device),
                 q_idx=torch.empty((T, IDX_HEADS, IDX_DIM), dtype=torch.uint16, device=device),
                 w=torch.empty((T, IDX_HEADS), dtype=torch.uint16, device=device),
                 k_idx=torch.empty((T, IDX_DIM), dtype=torch.uint16, device=device))
        for name, st in (("q", S_Q), ("k", S_K), ("v", S_V), ("q_idx", S_QIDX), ("k_idx", S_KIDX)):
            _chk(L.qsagen_normal_bf16_dev(self.seed & MASK64, st, 0, t[name].numel(), t[name].data_ptr(), cs))
        _chk(L.qsagen_softmax4_bf16_dev(self.seed & MASK64, S_W, 0, T, t["w"].data_ptr(), cs))
        if self.n_plant > 0:
            pl = self.planter()
            src_tok = np.where(pl >= 0, pl * BLOCK, -1).astype(np.int64)
            n_src = np.where(pl >= 0, np.minimum(BLOCK, T - pl * BLOCK), 0).astype(np.int64)
            d_src = torch.from_numpy(src_tok).to(device)
            d_n = torch.from_numpy(n_src).to(device)
            _chk(L.qsagen_plant_dev(self.nqb, BLOCK, T, 0, IDX_HEADS, IDX_DIM, d_src.data_ptr(), d_n.data_ptr(),
                                    t["q_idx"].data_ptr(), t["k_idx"].data_ptr(), self.seed & MASK64, S_PNOISE,
                                    cs))
            torch.cuda.current_stream(device).synchronize() if stream is None else stream.synchronize()
            del d_src, d_n
        return t


def _chk(rc: int):
    if rc != 0:
        raise RuntimeError(f"qsa_inputs device generator failed: cuda error {rc}")


# ------------------------------------------------------------------- decode
@dataclass
class DecodeProblem:
    """B sequences with L cached tokens each, then ``steps`` decode tokens."""
    B: int
    L: int
    steps: int
    seed: int = 0
    n_plant: int = 0

    def sseed(self, b: int) -> int:
        return seq_seed(self.seed, b)

    def tokens(self, b: int) -> PrefillProblem:
        """Per-token streams of sequence b (used for the decode tokens)."""
        return PrefillProblem(T=self.L + self.steps, seed=self.sseed(b), n_plant=0)

    def planted_blocks(self, b: int) -> np.ndarray:
        qb0 = self.L // BLOCK
        _, kbs = plant_choices(self.sseed(b), [qb0], self.n_plant, "uniform")
        return np.unique(kbs)

    def _plant_src(self, b: int):
        """q_idx vectors (tokens [4*qb0, L]) the planted keys are built from."""
        qb0 = self.L // BLOCK
        return self.tokens(b).q_idx(qb0 * BLOCK, self.L + 1)

    def cache_k(self, b: int, j0=0, j1=None):
        j1 = self.L if j1 is None else j1
        n = N_KV_HEADS * HEAD_DIM
        return normal_bf16(self.sseed(b), S_KROT, j0 * n, (j1 - j0) * n).reshape(j1 - j0, N_KV_HEADS, HEAD_DIM)

    def cache_v(self, b: int, j0=0, j1=None):
        j1 = self.L if j1 is None else j1
        return self.tokens(b).v(j0, j1)

    def cache_kidx(self, b: int, j0=0, j1=None):
        j1 = self.L if j1 is None else j1
        out = normal_bf16(self.sseed(b), S_KIDX, j0 * IDX_DIM, (j1 - j0) * IDX_DIM).reshape(j1 - j0, IDX_DIM)
        kbs = self.planted_blocks(b)
        kbs = kbs[(kbs * BLOCK < j1) & (kbs * BLOCK + BLOCK > j0)]
        if len(kbs) == 0:
            return out
        src = self._plant_src(b)
        for kb in kbs:
            buf = np.zeros((BLOCK, IDX_DIM), dtype=np.uint16)
            src_tok = np.zeros(1, np.int64)
            n_src = np.array([src.shape[0]], np.int64)
            lib().qsagen_plant(1, BLOCK, BLOCK, int(kb) * BLOCK, IDX_HEADS, IDX_DIM, _ptr(src_tok), _ptr(n_src),
                               _ptr(np.ascontiguousarray(src)), _ptr(buf), self.sseed(b) & MASK64, S_PNOISE)
            lo, hi = max(j0, kb * BLOCK), min(j1, kb * BLOCK + BLOCK)
            out[lo - j0: hi - j0] = buf[lo - kb * BLOCK: hi - kb * BLOCK]
        return out

    def fill_device_caches(self, k_cache, v_cache, kidx_cache, stream=None):
        """Fill rows [0, L) of caches shaped [B][max_len][...] on the GPU."""
        import torch
        dev = k_cache.device
        cs = ctypes.c_void_p(stream.cuda_stream if stream is not None
                             else torch.cuda.current_stream(dev).cuda_stream)
        L = lib()
        nk = N_KV_HEADS * HEAD_DIM
        for b in range(self.B):
            s = self.sseed(b) & MASK64
            _chk(L.qsagen_normal_bf16_dev(s, S_KROT, 0, self.L * nk, k_cache[b].data_ptr(), cs))
            _chk(L.qsagen_normal_bf16_dev(s, S_V, 0, self.L * nk, v_cache[b].data_ptr(), cs))
            _chk(L.qsagen_normal_bf16_dev(s, S_KIDX, 0, self.L * IDX_DIM, kidx_cache[b].data_ptr(), cs))
            kbs = self.planted_blocks(b)
            if len(kbs):
                src = torch.from_numpy(np.ascontiguousarray(self._plant_src(b))).to(dev)
                nb = int(kbs.max()) + 1
                src_tok = np.full(nb, -1, np.int64)
                src_tok[kbs] = 0
                n_src = np.full(nb, src.shape[0], np.int64)
                d_tok = torch.from_numpy(src_tok).to(dev)
                d_n = torch.from_numpy(n_src).to(dev)
                _chk(L.qsagen_plant_dev(nb, BLOCK, min(nb * BLOCK, self.L), 0, IDX_HEADS, IDX_DIM, d_tok.data_ptr(),
                                        d_n.data_ptr(), src.data_ptr(), kidx_cache[b].data_ptr(), s, S_PNOISE, cs))
                torch.cuda.synchronize(dev)
                del src, d_tok, d_n

    def step_inputs(self, s: int) -> dict:
        """Host inputs of decode step s for all sequences (token L + s)."""
        t = self.L + s
        out = dict(q=[], k=[], v=[], q_idx=[], w=[])
        for b in range(self.B):
            P = self.tokens(b)
            out["q"].append(P.q(t, t + 1)[0])
            out["k"].append(P.k(t, t + 1)[0])
            out["v"].append(P.v(t, t + 1)[0])
            out["q_idx"].append(P.q_idx(t, t + 1)[0])
            out["w"].append(P.w(t, t + 1)[0])
        return {k: np.ascontiguousarray(np.stack(v)) for k, v in out.items()}


# the five workloads (sizes, budgets, planting), by name
WORKLOADS = {
    "prefill_256": dict(kind="prefill", T=256, n_plant=3, dist="uniform", budgets=(16, 64)),
    "prefill_32k": dict(kind="prefill", T=32768, n_plant=8, dist="uniform", budgets=(512,)),
    "prefill_128k": dict(kind="prefill", T=131072, n_plant=8, dist="zipf", budgets=(512,)),
    "decode_64x256k": dict(kind="decode", B=64, L=262144, steps=32, n_plant=8, budgets=(512,)),
    "prefill_1m": dict(kind="prefill", T=1048576, n_plant=8, dist="zipf", budgets=(512,)),
}
