"""GPU parity of the mean-pooled indexer (qsa_params.aggregation =
AGG_MEAN_POOL): scores, selections and outputs against the oracle's mean-pool
definition; prefix-cached prefill bit-identical to the whole prefill; the
compressed-key cache builder exact; qsa_decode_mean_pool equal to the
prefill's last token; qsa_decode refuses the mode (it has no key-block cache)."""
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


def test_mean_pool_keys_exact():
    """qsa_mean_pool_keys equals the oracle-side definition (exact fp64 mean,
    one rounding to bf16) bit for bit, ragged tail included."""
    T = 1001
    P = Q.PrefillProblem(T=T, seed=21, n_plant=2)
    k_idx = P.k_idx()
    kbar = torch.empty(((T + 3) // 4, 128), dtype=torch.uint16, device="cuda")
    qsa.qsa_mean_pool_keys(qsa.params(aggregation=MEAN), T, dev(k_idx), kbar)
    torch.cuda.synchronize()
    got = kbar.cpu().numpy()
    from oracle_pins import _bf16_rne_exact
    from fractions import Fraction
    kf = Q.bf16_to_f64(k_idx)
    for b in list(range(0, 20)) + [(T + 3) // 4 - 1]:
        rows = kf[4 * b: min(4 * b + 4, T)]
        for c in range(0, 128, 7):
            want = _bf16_rne_exact(float(sum(Fraction(float(v)) for v in rows[:, c])) / rows.shape[0])
            assert Q.bf16_to_f64(got[b, c]) == want, (b, c)


@pytest.mark.parametrize("budget", [16, 512])
def test_mean_pool_decode_equals_prefill(budget):
    """Decode with the compressed-key cache (seeded by qsa_mean_pool_keys from
    the prompt's k_idx) equals the mean-pool prefill's last token at every
    step, block-aligned and mid-block starts, and the oracle's mean-pool
    decode on the GPU's selection."""
    L_list = [2048 + 4 * budget, 2301, 4097] if budget == 512 else [64, 129, 301]
    steps = 5
    B = len(L_list)
    p = qsa.params(budget, aggregation=MEAN)
    probs = [Q.PrefillProblem(T=L + steps, seed=140 + b, n_plant=8) for b, L in enumerate(L_list)]
    max_len = max(L_list) + steps + 8
    kc = torch.zeros((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.zeros_like(kc)
    ic = torch.zeros((B, max_len, 128), dtype=torch.uint16, device="cuda")
    kbar = torch.zeros((B, (max_len + 3) // 4, 128), dtype=torch.uint16, device="cuda")
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    hosts = []
    for b, (P, L) in enumerate(zip(probs, L_list)):
        h = P.host()
        hosts.append(h)
        t = {k: dev(v[:L]) for k, v in h.items()}
        r = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, want_krot=True,
                        aggregation=MEAN)
        torch.cuda.synchronize()
        kc[b, :L] = r["k_rot"]
        vc[b, :L] = t["v"]
        ic[b, :L] = t["k_idx"]
        qsa.qsa_mean_pool_keys(p, L, ic[b], kbar[b])
        for tt in range((L // 4) * 4, L):
            ring[b, tt % 4] = t["q_idx"][tt]
            wring[b, tt % 4] = t["w"][tt]
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
    O = _oracle(budget)
    lens = list(L_list)
    for s in range(steps):
        new = {k: np.stack([hosts[b][k][lens[b]] for b in range(B)]) for k in ("q", "k", "v", "q_idx", "k_idx", "w")}
        out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
        sel = torch.empty((B, budget), dtype=torch.int32, device="cuda")
        qsa.qsa_decode_mean_pool(p, B, max_len, lens, kc, vc, ic, kbar, ring, wring, dev(new["q"]), dev(new["k"]),
                                 dev(new["v"]), dev(new["q_idx"]), dev(new["k_idx"]), dev(new["w"]), out, sel, ws=ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(ws) == 0
        for b in range(B):
            L = lens[b]
            h = hosts[b]
            t = {k: dev(v[:L + 1]) for k, v in h.items()}
            r = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, aggregation=MEAN)
            torch.cuda.synchronize()
            qb = L // 4
            assert np.array_equal(sel[b].cpu().numpy(), r["sel"][qb].cpu().numpy()), f"b={b} s={s} selection"
            check_outputs(out[b].cpu().numpy(), Q.bf16_to_f64(r["out"][L].cpu().numpy()), f"b={b} s={s}")
            g = sel[b].cpu().numpy()
            gc = int((g >= 0).sum())
            kcache = kc[b, :L].cpu().numpy()
            t0 = 4 * qb
            _, _, oo, _ = O.decode(L, kcache, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L],
                                   h["k"][L], h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L], sel_in=g, cnt_in=gc)
            check_outputs(out[b].cpu().numpy(), oo, f"b={b} s={s} vs oracle")
        lens = [L + 1 for L in lens]


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
