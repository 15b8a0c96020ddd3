"""GPU parity of the mean-pooled indexer (qsa_params.aggregation =
AGG_MEAN_POOL): scores, selections and outputs against the oracle's mean-pool
definition; prefix-cached prefill bit-identical to the whole prefill; decode
refuses the mode."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import SCORE_RTOL, check_outputs, check_selection, dev, gpu_prefill
from test_gpu_prefill_cached import run_cached

pytestmark = pytest.mark.gpu
MEAN = qsa.AGG_MEAN_POOL


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def _oracle(budget=512):
    return oracle.Oracle(oracle.params(budget=budget, aggregation=oracle.AGG_MEAN_POOL))


def _scores_gpu_mean(T, host, qb_begin=0, qb_end=None, ld=None):
    nqb = (T + 3) // 4
    qb_end = nqb if qb_end is None else qb_end
    ld = ld or ((qb_end + 3) // 4 * 4)
    p = qsa.params(aggregation=MEAN)
    S = torch.full((qb_end - qb_begin, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = qsa.workspace(qsa.qsa_index_workspace_size(p, T))
    qsa.qsa_index_scores(p, T, dev(host["q_idx"]), dev(host["w"]), dev(host["k_idx"]), qb_begin, qb_end, S, ld, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    return S.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T", [1, 3, 5, 64, 333, 1000, 2049, 4099, 9001])
def test_mean_pool_scores_vs_oracle(T):
    """Every causal entry within the score tolerance; kb > qb never written.
    T = 2049 .. 9001 span several 128-block key tiles and ragged tails."""
    P = Q.PrefillProblem(T=T, seed=300 + T, n_plant=3)
    host = P.host()
    got = _scores_gpu_mean(T, host)
    want = _oracle().index_scores(T, host["q_idx"], host["w"], host["k_idx"], ld=got.shape[1])
    causal = ~np.isnan(want)
    assert np.isnan(got[~causal]).all(), "entries with kb > qb must not be written"
    err = np.abs(got[causal] - want[causal]) / np.maximum(np.abs(want[causal]), 1e-3)
    assert err.max() <= SCORE_RTOL, f"T={T}: max rel err {err.max():.3e}"


def test_mean_pool_scores_subrange():
    T = 5000
    P = Q.PrefillProblem(T=T, seed=8, n_plant=4)
    host = P.host()
    got = _scores_gpu_mean(T, host, 333, 1111, ld=1200)
    want = _oracle().index_scores(T, host["q_idx"], host["w"], host["k_idx"], 333, 1111, ld=1200)
    m = ~np.isnan(want)
    assert np.isnan(got[~m]).all()
    err = np.abs(got[m] - want[m]) / np.maximum(np.abs(want[m]), 1e-3)
    assert err.max() <= SCORE_RTOL


@pytest.mark.parametrize("T,budget", [(301, 16), (2053, 64), (9001, 512)])
def test_mean_pool_prefill_vs_oracle(T, budget):
    P = Q.PrefillProblem(T=T, seed=400 + T, n_plant=3)
    host = P.host()
    t = {k: dev(v) for k, v in host.items()}
    r = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, aggregation=MEAN)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(r["ws"]) == 0
    sel, cnt = r["sel"].cpu().numpy(), r["cnt"].cpu().numpy()
    O = _oracle(budget)
    nqb = P.nqb
    S = O.index_scores(T, host["q_idx"], host["w"], host["k_idx"])
    osel, ocnt = O.select_rows(np.nan_to_num(S, nan=-1.0))
    for qb in range(nqb):
        check_selection(sel[qb], int(cnt[qb]), osel[qb], int(ocnt[qb]), S[qb], qb, budget, f"qb={qb}")
    out, lse = O.attend_blocks(T, host["q"], host["k"], host["v"], np.arange(nqb), sel, cnt)
    check_outputs(r["out"].cpu().numpy(), out[:T], f"T={T} budget={budget}")
    assert np.allclose(r["lse"].cpu().numpy(), lse[:T], atol=1e-2, rtol=1e-3)


def test_mean_pool_cached_equals_whole_prefill():
    L_old, T_new, budget = 3001, 1500, 512
    T = L_old + T_new
    P = Q.PrefillProblem(T=T, seed=12, n_plant=8)
    host = P.host()
    t = {k: dev(v) for k, v in host.items()}
    full = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, want_krot=True,
                       aggregation=MEAN)
    torch.cuda.synchronize()
    full = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) and k != "ws" else v) for k, v in full.items()}
    c = run_cached(host, L_old, T_new, budget, full["k_rot"], aggregation=MEAN)
    qbA = L_old // 4
    assert np.array_equal(c["sel"], full["sel"][qbA:])
    assert np.array_equal(c["out"], full["out"][L_old:])
    assert np.array_equal(c["lse"], full["lse"][L_old:])


def test_mean_pool_decode_unsupported():
    p = qsa.params(aggregation=MEAN)
    B, max_len = 1, 64
    z = lambda *s: torch.zeros(s, dtype=torch.uint16, device="cuda")
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(qsa.params(), B, max_len))
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_decode(p, B, max_len, [5], z(B, max_len, 2, 256), z(B, max_len, 2, 256), z(B, max_len, 128),
                       z(B, 4, 4, 128), z(B, 4, 4), z(B, 24, 256), z(B, 2, 256), z(B, 2, 256), z(B, 4, 128),
                       z(B, 128), z(B, 4), z(B, 24, 256), ws=ws)
    assert "UNSUPPORTED" in str(e.value)
