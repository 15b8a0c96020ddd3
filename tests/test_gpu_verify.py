"""GPU parity of the batched verify (qsa_verify): m new tokens per sequence
give what a prefill of the whole sequence gives for those tokens (selection
up to near-ties of the fp64 scores, outputs within the bf16 tolerance), the
oracle agrees on the verify's own selection, m = 1 is bit-identical to a
decode step, the caches receive the new rows and the ring is left alone."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, check_selection, dev, gpu_prefill
from test_gpu_decode import DecodeState

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def run_verify(st, m, ws=None, kbar=None):
    """qsa_verify of the next m tokens of every sequence of a DecodeState."""
    B = st.B
    new = {k: np.stack([st.hosts[b][k][st.lens[b]:st.lens[b] + m] for b in range(B)]) for k in
           ("q", "k", "v", "q_idx", "k_idx", "w")}
    out = torch.empty((B, m, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((B, m, 24), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, m, st.budget), dtype=torch.int32, device="cuda")
    if ws is None:
        ws = qsa.workspace(qsa.qsa_verify_workspace_size(st.p, B, m, st.max_len))
    qsa.qsa_verify(st.p, B, m, st.max_len, st.lens, st.k_cache, st.v_cache, st.kidx_cache, st.qidx_ring, st.w_ring,
                   dev(new["q"]), dev(new["k"]), dev(new["v"]), dev(new["q_idx"]), dev(new["k_idx"]), dev(new["w"]),
                   out, sel, lse, ws, kbar_cache=kbar)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    return out.cpu().numpy(), sel.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("budget,m", [(16, 5), (16, 3), (512, 5), (512, 9)])
def test_verify_equals_prefill(budget, m):
    L_list = [2048 + 4 * budget, 2301, 4099, 4094] if budget == 512 else [64, 129, 303, 301]
    probs = [Q.PrefillProblem(T=L + m, seed=600 + b + m, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + m + 8, budget=budget)
    ring_before = (st.qidx_ring.clone(), st.w_ring.clone())
    out, sel, lse = run_verify(st, m)
    assert torch.equal(st.qidx_ring, ring_before[0]) and torch.equal(st.w_ring, ring_before[1]), "ring is read-only"
    O = oracle.Oracle(oracle.params(budget=budget))
    for b, L in enumerate(L_list):
        h = st.hosts[b]
        T = L + m
        full_h, full = gpu_prefill(Q.PrefillProblem(T=T, seed=probs[b].seed), budget,
                                   host={k: v[:T] for k, v in h.items()})
        assert np.array_equal(st.v_cache[b, L:T].cpu().numpy(), h["v"][L:T])
        assert np.array_equal(st.kidx_cache[b, L:T].cpu().numpy(), h["k_idx"][L:T])
        for i in range(m):
            t = L + i
            qb = t // 4
            g = sel[b, i]
            gc = int((g >= 0).sum())
            S = O.block_scores(qb, h["q_idx"][4 * qb:min(4 * qb + 4, T)], h["w"][4 * qb:min(4 * qb + 4, T)],
                               h["k_idx"][:T])
            check_selection(g, gc, full["sel"][qb], int(full["cnt"][qb]), S, qb, budget, f"b={b} t={t}")
            check_outputs(out[b, i], Q.bf16_to_f64(full["out"][t]), f"verify vs prefill b={b} t={t}")
        # the oracle on the verify's own selection, block by block
        for qb in sorted({(L + i) // 4 for i in range(m)}):
            i0 = max(4 * qb, L) - L
            g = sel[b, i0]
            oo, ol = O.attend_blocks(T, h["q"], h["k"], h["v"], [qb], g[None], np.array([int((g >= 0).sum())]))
            for t in range(max(4 * qb, L), min(4 * qb + 4, T)):
                assert np.array_equal(sel[b, t - L], g), "tokens of one block share its selection"
                check_outputs(out[b, t - L], oo[t - 4 * qb], f"verify vs oracle b={b} t={t}")
                assert np.allclose(lse[b, t - L], ol[t - 4 * qb], atol=1e-2)


def test_verify_one_token_equals_decode():
    """m = 1: the same kernels on the same data as a decode step -- bit for
    bit (block-aligned and mid-block positions)."""
    budget = 64
    L_list = [1001, 2048, 4093, 302]
    probs = [Q.PrefillProblem(T=L + 1, seed=650 + b, n_plant=4) for b, L in enumerate(L_list)]
    a = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    b_ = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    vout, vsel, vlse = run_verify(a, 1)
    _, dout, dsel, dlse = b_.step()
    assert np.array_equal(vsel[:, 0], dsel)
    assert np.array_equal(vout[:, 0], dout) and np.array_equal(vlse[:, 0], dlse)
    assert torch.equal(a.k_cache, b_.k_cache) and torch.equal(a.v_cache, b_.v_cache)


def test_verify_checks():
    budget = 16
    st = DecodeState([Q.PrefillProblem(T=60, seed=660)], [33], max_len=40, budget=budget)
    with pytest.raises(qsa.QSAError) as e:          # 33 + 9 > max_len
        run_verify(st, 9)
    assert "INVALID_ARG" in str(e.value)
    with pytest.raises(qsa.QSAError) as e:          # m above 16
        qsa.qsa_verify_workspace_size(st.p, 1, 17, 40)
    assert "UNSUPPORTED" in str(e.value)
    st.p = qsa.params(budget, aggregation=qsa.AGG_MEAN_POOL)
    with pytest.raises(qsa.QSAError) as e:          # mean pool needs the compressed-key cache
        run_verify(st, 2, ws=qsa.workspace(1 << 20))
    assert "INVALID_ARG" in str(e.value)


@pytest.mark.parametrize("budget,m", [(16, 5), (512, 5), (512, 9)])
def test_verify_mean_pool_equals_prefill(budget, m):
    """Mean-pooled verify: the compressed keys of the touched blocks are
    rewritten (equal to qsa_mean_pool_keys over the extended cache) and every
    token matches the mean-pool prefill of the whole sequence."""
    L_list = [2048 + 4 * budget, 2302, 4099] if budget == 512 else [64, 129, 303]
    probs = [Q.PrefillProblem(T=L + m, seed=700 + b + m, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + m + 8, budget=budget)
    st.p = qsa.params(budget, aggregation=qsa.AGG_MEAN_POOL)
    kbar = torch.zeros((st.B, (st.max_len + 3) // 4, 128), dtype=torch.uint16, device="cuda")
    for b, L in enumerate(L_list):
        qsa.qsa_mean_pool_keys(st.p, L, st.kidx_cache[b], kbar[b])
    out, sel, lse = run_verify(st, m, kbar=kbar)
    O = oracle.Oracle(oracle.params(budget=budget, aggregation=oracle.AGG_MEAN_POOL))
    for b, L in enumerate(L_list):
        T = L + m
        want = torch.zeros_like(kbar[b])
        qsa.qsa_mean_pool_keys(st.p, T, st.kidx_cache[b], want)
        torch.cuda.synchronize()
        nb = (T + 3) // 4
        assert torch.equal(kbar[b, :nb], want[:nb]), f"b={b} compressed keys"
        h = st.hosts[b]
        t_in = {k: dev(v[:T]) for k, v in h.items()}
        full = qsa.prefill(t_in["q"], t_in["k"], t_in["v"], t_in["q_idx"], t_in["w"], t_in["k_idx"], budget=budget,
                           aggregation=qsa.AGG_MEAN_POOL)
        torch.cuda.synchronize()
        fsel, fcnt, fout = full["sel"].cpu().numpy(), full["cnt"].cpu().numpy(), full["out"].cpu().numpy()
        for i in range(m):
            t = L + i
            qb = t // 4
            g = sel[b, i]
            S = O.block_scores(qb, h["q_idx"][4 * qb:min(4 * qb + 4, T)], h["w"][4 * qb:min(4 * qb + 4, T)],
                               h["k_idx"][:T])
            check_selection(g, int((g >= 0).sum()), fsel[qb], int(fcnt[qb]), S, qb, budget, f"b={b} t={t}")
            check_outputs(out[b, i], Q.bf16_to_f64(fout[t]), f"mean-pool verify vs prefill b={b} t={t}")
