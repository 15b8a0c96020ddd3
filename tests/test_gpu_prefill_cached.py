"""GPU parity of the prefix-cached prefill (C ABI): L_old tokens in a cache,
T_new new tokens prefilled.  The result must be the last T_new rows of a
whole prefill of L_old + T_new tokens (bit for bit: the same kernels score
and attend the same blocks in the same order), the caches must receive the
new rows, and the oracle must agree on its own terms."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, check_selection, dev, gpu_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def run_cached(h, L_old, T_new, budget, k_rot_full, ws_bytes=None, aggregation=qsa.AGG_TOKEN_MAX):
    """Seed caches with the first L_old tokens, prefill the rest."""
    T = L_old + T_new
    p = qsa.params(budget, aggregation=aggregation)
    kc = torch.zeros((T, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.zeros_like(kc)
    ic = torch.zeros((T, 128), dtype=torch.uint16, device="cuda")
    if L_old:
        kc[:L_old] = dev(k_rot_full[:L_old])
        vc[:L_old] = dev(h["v"][:L_old])
        ic[:L_old] = dev(h["k_idx"][:L_old])
    t0 = 4 * (L_old // 4)
    r = L_old - t0
    qprev = dev(h["q_idx"][t0:L_old]) if r else None
    wprev = dev(h["w"][t0:L_old]) if r else None
    new = {k: dev(h[k][L_old:T]) for k in ("q", "k", "v", "q_idx", "w", "k_idx")}
    nq = (T + 3) // 4 - L_old // 4
    out = torch.empty((T_new, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((T_new, 24), dtype=torch.float32, device="cuda")
    sel = torch.empty((nq, budget), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nq,), dtype=torch.int32, device="cuda")
    mn, pref = qsa.qsa_prefill_cached_workspace_size(p, L_old, T_new)
    ws = qsa.workspace(ws_bytes if ws_bytes is not None else pref)
    qsa.qsa_prefill_cached(p, L_old, T_new, kc, vc, ic, qprev, wprev, new["q"], new["k"], new["v"], new["q_idx"],
                           new["w"], new["k_idx"], out, lse, sel, cnt, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    return dict(out=out.cpu().numpy(), lse=lse.cpu().numpy(), sel=sel.cpu().numpy(), cnt=cnt.cpu().numpy(),
                k_cache=kc.cpu().numpy(), v_cache=vc.cpu().numpy(), kidx_cache=ic.cpu().numpy(), min_ws=mn)


@pytest.mark.parametrize("L_old,T_new,budget", [(0, 301, 16), (256, 77, 16), (1001, 130, 64), (2047, 3, 16),
                                                (4096, 1, 512), (2050, 2049, 512), (6001, 999, 512)])
def test_cached_equals_whole_prefill(L_old, T_new, budget):
    T = L_old + T_new
    P = Q.PrefillProblem(T=T, seed=90 + T_new, n_plant=8)
    h, full = gpu_prefill(P, budget)
    c = run_cached(h, L_old, T_new, budget, full["k_rot"])
    qbA = L_old // 4
    assert np.array_equal(c["sel"], full["sel"][qbA:]), "selections"
    assert np.array_equal(c["cnt"], full["cnt"][qbA:]), "counts"
    assert np.array_equal(c["out"], full["out"][L_old:]), "outputs"
    assert np.array_equal(c["lse"], full["lse"][L_old:]), "lse"
    assert np.array_equal(c["k_cache"], full["k_rot"]), "rotated keys appended"
    assert np.array_equal(c["v_cache"], h["v"]) and np.array_equal(c["kidx_cache"], h["k_idx"]), "cache append"


def test_cached_chunked_workspace():
    """The smallest workspace (many query-block chunks, the first starting
    mid-sequence) gives the same result as one pass."""
    L_old, T_new, budget = 1999, 1201, 64
    T = L_old + T_new
    P = Q.PrefillProblem(T=T, seed=7, n_plant=8)
    h, full = gpu_prefill(P, budget)
    one = run_cached(h, L_old, T_new, budget, full["k_rot"])
    small = run_cached(h, L_old, T_new, budget, full["k_rot"], ws_bytes=one["min_ws"])
    for k in ("sel", "cnt", "out", "lse"):
        assert np.array_equal(one[k], small[k]), k


def test_cached_vs_oracle():
    """Direct oracle check: selections by the acceptance criterion, outputs on
    the GPU's own selection."""
    L_old, T_new, budget = 1030, 250, 64
    T = L_old + T_new
    P = Q.PrefillProblem(T=T, seed=11, n_plant=8)
    h = P.host()
    _, full = gpu_prefill(P, budget, host=h)
    c = run_cached(h, L_old, T_new, budget, full["k_rot"])
    O = oracle.Oracle(oracle.params(budget=budget))
    qbA = L_old // 4
    qbs = np.arange(qbA, (T + 3) // 4)
    S = O.index_scores(T, h["q_idx"], h["w"], h["k_idx"], qb_begin=qbA, qb_end=(T + 3) // 4)
    osel, ocnt = O.select_rows(S, qb_begin=qbA)
    for i, qb in enumerate(qbs):
        check_selection(c["sel"][i], int(c["cnt"][i]), osel[i], int(ocnt[i]), S[i], int(qb), budget, f"qb={qb}")
    oo, ol = O.attend_blocks(T, h["q"], h["k"], h["v"], qbs, c["sel"], c["cnt"])
    oo = oo.reshape(len(qbs) * 4, 24, 256)[L_old - 4 * qbA: L_old - 4 * qbA + T_new]
    check_outputs(c["out"], oo, "cached prefill vs oracle")
