"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare with the oracle by the acceptance criteria."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_long_qsa_b200 as qsa
import qsa_inputs as Q

# tolerances of the acceptance criteria (bf16 outputs vs the fp64 oracle run
# on the GPU's own selection), and of the fp32 indexer scores vs fp64.
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
SEL_NEAR_TIE = 1e-3
# fp32 tensor-core dot products of 128 bf16 pairs: rounding error ~1e-6
# relative to the score; 1e-4 leaves two orders of margin.
SCORE_RTOL = 1e-4


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_out_to_f64(t: torch.Tensor) -> np.ndarray:
    return Q.bf16_to_f64(t.cpu().numpy())


def check_outputs(got_bf16: np.ndarray, want: np.ndarray, what=""):
    """got: bf16 bits; want: fp64.  max-abs and relative-L2 bounds."""
    g = Q.bf16_to_f64(got_bf16)
    diff = g - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-30))
    assert max_abs <= OUT_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {OUT_MAX_ABS}"
    assert rel <= OUT_REL_L2, f"{what}: rel-L2 {rel:.3e} > {OUT_REL_L2}"
    return max_abs, rel


def kth_candidate_score(S_row: np.ndarray, qb: int, budget: int) -> float:
    """Oracle score of the (budget-2)-th best candidate of [0, qb-2]."""
    cand = np.sort(S_row[:qb - 1])[::-1]
    return float(cand[budget - 3])


def check_selection(gpu_sel: np.ndarray, gpu_cnt: int, oracle_sel: np.ndarray, oracle_cnt: int,
                    S_row: np.ndarray, qb: int, budget: int, what=""):
    """GPU and oracle selections agree except for blocks whose oracle score is
    within SEL_NEAR_TIE (relative) of the oracle's k-th score; forced blocks
    always match; the GPU list is ascending, distinct, -1 padded."""
    assert gpu_cnt == oracle_cnt, f"{what}: cnt {gpu_cnt} vs {oracle_cnt}"
    g = gpu_sel[:gpu_cnt]
    assert np.all(np.diff(g) > 0), f"{what}: not ascending/distinct"
    assert np.all(gpu_sel[gpu_cnt:] == -1), f"{what}: bad padding"
    assert g.min() >= 0 and g.max() <= qb
    o = oracle_sel[:oracle_cnt]
    if qb + 1 <= budget:
        assert np.array_equal(g, o), what
        return 0
    assert qb in g and (qb - 1) in g, f"{what}: forced block missing"
    diff = np.setxor1d(g, o)
    if len(diff):
        kth = kth_candidate_score(S_row, qb, budget)
        for b in diff:
            assert abs(S_row[b] - kth) <= SEL_NEAR_TIE * abs(kth), \
                f"{what}: block {b} score {S_row[b]} vs k-th {kth}"
    return len(diff)


def gpu_prefill(P: Q.PrefillProblem, budget: int, host=None, ws_bytes=None, on_device=False):
    """Run qsa_prefill; returns (inputs on host or None, result dict of CPU numpy)."""
    if on_device:
        t = P.device()
    else:
        host = host or P.host()
        t = {k: dev(v) for k, v in host.items()}
    r = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, want_krot=True,
                    ws_bytes=ws_bytes)
    torch.cuda.synchronize()
    rc = qsa.qsa_check_device_error(r["ws"])
    assert rc == 0, f"device error {rc}"
    out = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) and k != "ws" else v) for k, v in r.items()}
    del r, t
    return host, out


def pmap(fn, items):
    """fn over items on a thread pool (the oracle's C calls release the GIL),
    results in order; exceptions re-raised in the caller."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    items = list(items)
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 4
    with ThreadPoolExecutor(max_workers=max(1, min(n, len(items)))) as ex:
        return list(ex.map(fn, items))


def gather_rows(blocks, T, k_fn, v_fn):
    """Positions and unrotated K / V rows of the listed key blocks (tokens
    4b .. min(4b + 4, T) - 1), from row generators k_fn(j0, j1), v_fn(j0, j1)."""
    pos, ks, vs = [], [], []
    for b in blocks:
        j0, j1 = 4 * int(b), min(4 * int(b) + 4, T)
        if j1 <= j0:
            continue
        pos.extend(range(j0, j1))
        ks.append(k_fn(j0, j1))
        vs.append(v_fn(j0, j1))
    return np.asarray(pos, np.int64), np.concatenate(ks), np.concatenate(vs)
