"""Index work at full size is bit-exact.  At 131,072 tokens (config 2, as the
benchmark runs it: preferred workspace, segment maxima and candidate lists in
the select) every one of the 32,768 selection rows that qsa_prefill makes must
equal an exact top-k computed on the CPU from the fp32 scores that
qsa_index_scores writes for the same inputs: forced blocks qb and qb - 1, the
budget - 2 highest of [0, qb - 2] by (score descending, index ascending, -0.0
equal to +0.0), ascending, -1 padded."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import qsa_inputs as Q

BUDGET = 512


@pytest.fixture(scope="module")
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def exact_selection_rows(S: np.ndarray, qb0: int, budget: int) -> list[np.ndarray]:
    """Exact stage-2 selection of rows qb0 .. qb0 + len(S) - 1 of fp32 scores
    (numpy: a k-th value by partition, then ties resolved by index)."""
    n, ld = S.shape
    qbs = qb0 + np.arange(n)
    out = [None] * n
    K = budget - 2
    short = qbs + 1 <= budget
    for i in np.nonzero(short)[0]:
        out[i] = np.arange(qbs[i] + 1)
    long_rows = np.nonzero(~short)[0]
    if len(long_rows):
        vals = S[long_rows].astype(np.float64) + 0.0          # -0.0 -> +0.0
        col = np.arange(ld)[None, :]
        vals[col >= (qbs[long_rows] - 1)[:, None]] = -np.inf   # candidates are [0, qb - 2]
        kth = -np.partition(-vals, K - 1, axis=1)[:, K - 1]
        greater = vals > kth[:, None]
        need = K - greater.sum(axis=1)
        eq = vals == kth[:, None]
        take = greater | (eq & (np.cumsum(eq, axis=1) <= need[:, None]))
        for j, i in enumerate(long_rows):
            qb = qbs[i]
            out[i] = np.concatenate([np.nonzero(take[j])[0], [qb - 1, qb]])
    return out


def test_exact_selection_rows_helper():
    """The CPU reference itself against a per-row lexsort on small rows with ties."""
    rng = np.random.default_rng(0)
    budget = 8
    S = np.round(rng.gamma(2.0, 1.0, size=(40, 44)).astype(np.float32) * 4) / 4
    S[::3, ::5] = -0.0
    got = exact_selection_rows(S, 0, budget)
    for qb in range(40):
        if qb + 1 <= budget:
            want = np.arange(qb + 1)
        else:
            v = S[qb, :qb - 1].astype(np.float64) + 0.0
            c = np.arange(qb - 1)
            o = np.lexsort((c, -v))
            want = np.sort(np.concatenate([c[o[:budget - 2]], [qb - 1, qb]]))
        assert np.array_equal(np.sort(got[qb]), want), qb


@pytest.mark.gpu
@pytest.mark.timeout(1800)
def test_prefill_selection_bit_exact_128k(_lib):
    T = 131072
    P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="zipf")
    d = P.device()
    p = qsa.params(BUDGET)
    nqb = P.nqb
    _, pref = qsa.qsa_prefill_workspace_size(p, T)
    ws = qsa.workspace(pref)
    out = torch.empty((T, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((nqb, BUDGET), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nqb,), dtype=torch.int32, device="cuda")
    qsa.qsa_prefill(p, T, 0, d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], out, None, sel, cnt, None, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    del ws, out
    sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
    torch.cuda.empty_cache()
    # stage 1 alone: the fp32 block scores of every row (4.3 GB)
    ld = (nqb + 3) // 4 * 4
    S = torch.empty((nqb, ld), dtype=torch.float32, device="cuda")
    wsi = qsa.workspace(qsa.qsa_index_workspace_size(p, T))
    qsa.qsa_index_scores(p, T, d["q_idx"], d["w"], d["k_idx"], 0, nqb, S, ld, wsi)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(wsi) == 0
    del d
    CH = 1024
    bad = []
    for r0 in range(0, nqb, CH):
        r1 = min(r0 + CH, nqb)
        want = exact_selection_rows(S[r0:r1].cpu().numpy(), r0, BUDGET)
        for i, w in enumerate(want):
            qb = r0 + i
            c = int(cnt_h[qb])
            if c != len(w) or not np.array_equal(sel_h[qb, :c], np.sort(w)) or not np.all(sel_h[qb, c:] == -1):
                bad.append(qb)
    assert not bad, f"{len(bad)} rows differ from the exact top-k, first {bad[:8]}"
