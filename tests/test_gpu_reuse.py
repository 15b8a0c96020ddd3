"""GPU parity of the draft decode step over a reused top-k row
(qsa_decode_reuse): one speculative round is a plain decode step followed by
draft steps that reuse its selection; every draft output is checked against
the oracle's reuse rule (the row joined with the forced blocks qb - 1, qb),
rows that are not causal or not ascending are reported on the device, and the
mean-pool variant keeps the compressed-key cache current."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, dev
from test_gpu_decode import DecodeState

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


@pytest.fixture
def automatic_splits_after():
    """Back to the automatic split-KV choice once the test is done."""
    yield
    qsa.qsa_set_decode_splits(0)


def _new(st):
    return {k: np.stack([st.hosts[b][k][st.lens[b]] for b in range(st.B)]) for k in
            ("q", "k", "v", "q_idx", "k_idx", "w")}


def reuse_step(st, sel_in, cnt_in, kbar=None):
    """One qsa_decode_reuse step on a DecodeState; returns positions, outputs, lse."""
    B = st.B
    new = _new(st)
    out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((B, 24), dtype=torch.float32, device="cuda")
    qsa.qsa_decode_reuse(st.p, B, st.max_len, st.lens, st.k_cache, st.v_cache, st.kidx_cache, kbar, st.qidx_ring,
                         st.w_ring, dev(new["q"]), dev(new["k"]), dev(new["v"]), dev(new["q_idx"]),
                         dev(new["k_idx"]), dev(new["w"]), sel_in, cnt_in, out, lse, st.ws)
    torch.cuda.synchronize()
    pos = list(st.lens)
    st.lens = [L + 1 for L in st.lens]
    return pos, out.cpu().numpy(), lse.cpu().numpy()


def _oracle_reuse(O, st, b, L, row, cnt):
    h = st.hosts[b]
    qb = L // 4
    t0 = 4 * qb
    kc = st.k_cache[b, :L].cpu().numpy()
    return O.decode_reuse(L, kc, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L], h["k"][L],
                          h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L], sel_in=row, cnt_in=cnt)


@pytest.mark.parametrize("budget", [16, 512])
def test_speculative_round_vs_oracle(budget):
    """Step 1 selects (qsa_decode); draft steps 2..5 reuse its rows, crossing
    into the next query block for every start position (aligned, mid-block,
    last token of a block) and, for the budget-16 rows, growing past the
    budget by the forced blocks."""
    L_list = [2048 + 4 * budget, 2301, 4099, 4096] if budget == 512 else [64, 129, 303, 301]
    steps = 5
    probs = [Q.PrefillProblem(T=L + steps, seed=500 + b, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + steps + 8, budget=budget)
    O = oracle.Oracle(oracle.params(budget=budget))
    pos, out, sel, lse = st.step()
    sel_d = torch.from_numpy(sel).cuda()
    cnt_h = (sel >= 0).sum(1).astype(np.int32)
    cnt_d = torch.from_numpy(cnt_h).cuda()
    for s in range(1, steps):
        # steps 1, 2 pass the counts; steps 3, 4 none (rows end at the -1 padding)
        pos, out, lse = reuse_step(st, sel_d, cnt_d if s <= 2 else None)
        assert qsa.qsa_check_device_error(st.ws) == 0
        for b in range(st.B):
            L = pos[b]
            rsel, n, oo, ol = _oracle_reuse(O, st, b, L, sel[b], int(cnt_h[b]))
            qb = L // 4
            assert rsel[-1] == qb and (qb == 0 or rsel[-2] == qb - 1)
            check_outputs(out[b], oo, f"reuse b={b} step={s} L={L} ({n} blocks)")
            assert np.allclose(lse[b], ol, atol=1e-2), f"b={b} step={s} lse"


def test_reuse_at_same_token_equals_decode(automatic_splits_after):
    """Reusing the row a decode step selected, at that same token, attends the
    same blocks in the same order: bit-identical output and lse (one KV range,
    so both take the same summation order)."""
    qsa.qsa_set_decode_splits(1)
    budget = 64
    L_list = [1001, 2048, 4093]
    probs = [Q.PrefillProblem(T=L + 1, seed=520 + b, n_plant=4) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    _, out, sel, lse = st.step()
    st.lens = list(L_list)   # the same token again (the caches get the same rows)
    sel_d = torch.from_numpy(sel).cuda()
    cnt_d = torch.from_numpy((sel >= 0).sum(1).astype(np.int32)).cuda()
    _, rout, rlse = reuse_step(st, sel_d, cnt_d)
    assert qsa.qsa_check_device_error(st.ws) == 0
    assert np.array_equal(rout, out) and np.array_equal(rlse, lse)


@pytest.mark.parametrize("bad", ["future_block", "descending", "duplicate", "count_over_budget", "negative"])
def test_reuse_rejects_invalid_rows(bad):
    """Rows that are not ascending, distinct and causal are reported
    (QSA_ERR_DEVICE_BOUNDS) by the append kernel's check; the other sequences
    of the batch are unaffected."""
    budget = 16
    L_list = [201, 301]
    probs = [Q.PrefillProblem(T=L + 2, seed=540 + b, n_plant=2) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    _, _, sel, _ = st.step()
    O = oracle.Oracle(oracle.params(budget=budget))
    cnt = (sel >= 0).sum(1).astype(np.int32)
    good = sel.copy()
    qb1 = st.lens[1] // 4
    if bad == "future_block":
        sel[1, 3] = qb1 + 1
        sel[1, :cnt[1]] = np.sort(sel[1, :cnt[1]])
    elif bad == "descending":
        sel[1, [2, 3]] = sel[1, [3, 2]]
    elif bad == "duplicate":
        sel[1, 3] = sel[1, 2]
    elif bad == "count_over_budget":
        cnt[1] = budget + 1
    else:
        sel[1, 0] = -1
    pos, out, _ = reuse_step(st, torch.from_numpy(sel).cuda(), torch.from_numpy(cnt).cuda())
    assert qsa.qsa_check_device_error(st.ws) == 7
    _, _, oo, _ = _oracle_reuse(O, st, 0, pos[0], good[0], int(cnt[0]))
    check_outputs(out[0], oo, "valid row of the batch")


def test_reuse_mean_pool_keeps_compressed_keys():
    """Draft steps with mean-pooled parameters rewrite the compressed key of
    their block, so a later full decode step sees the same cache as after
    plain mean-pool decode steps."""
    budget = 16
    L_list = [129, 302]
    steps = 4
    probs = [Q.PrefillProblem(T=L + steps, seed=560 + b, n_plant=2) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + steps + 8, budget=budget)
    p = qsa.params(budget, aggregation=qsa.AGG_MEAN_POOL)
    st.p = p
    kbar = torch.zeros((st.B, (st.max_len + 3) // 4, 128), dtype=torch.uint16, device="cuda")
    for b, L in enumerate(L_list):
        qsa.qsa_mean_pool_keys(p, L, st.kidx_cache[b], kbar[b])
    sel = torch.zeros((st.B, budget), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((st.B,), dtype=torch.int32, device="cuda")   # empty rows: forced blocks only
    for _ in range(steps):
        reuse_step(st, sel, cnt, kbar=kbar)
        assert qsa.qsa_check_device_error(st.ws) == 0
    want = torch.zeros_like(kbar)
    for b in range(st.B):
        qsa.qsa_mean_pool_keys(p, st.lens[b], st.kidx_cache[b], want[b])
    torch.cuda.synchronize()
    for b in range(st.B):
        nb = (st.lens[b] + 3) // 4
        assert torch.equal(kbar[b, :nb], want[b, :nb]), b


def test_reuse_argument_checks():
    budget = 16
    st = DecodeState([Q.PrefillProblem(T=40, seed=570)], [33], max_len=48, budget=budget)
    sel = torch.zeros((1, budget), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    kbar = torch.zeros((1, 12, 128), dtype=torch.uint16, device="cuda")
    with pytest.raises(qsa.QSAError) as e:      # kbar_cache given without mean pooling
        reuse_step(st, sel, cnt, kbar=kbar)
    assert "INVALID_ARG" in str(e.value)
    st.lens = [33]
    with pytest.raises(qsa.QSAError) as e:      # no selection
        reuse_step(st, None, cnt)
    assert "INVALID_ARG" in str(e.value)
