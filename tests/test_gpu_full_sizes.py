"""GPU parity at the full workload sizes (32K, 128K and 1M prefill; decode of
64 sequences x 256K), run as the benchmark runs them (same workspace, so the
same chunking), checked on sampled query blocks / sequences that the fp64
oracle computes one by one, plus structural checks of every selection row."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, check_selection

pytestmark = pytest.mark.gpu

BUDGET = 512


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def _sample_blocks(nqb: int, seed: int) -> list[int]:
    fixed = [0, 1, 2, 509, 510, 511, 512, 513, 2047, nqb // 3, nqb // 2, (2 * nqb) // 3, nqb - 2, nqb - 1]
    rng = np.random.default_rng(seed)
    extra = rng.integers(0, nqb, size=4).tolist()
    return sorted({int(q) for q in fixed + extra if 0 <= q < nqb})


def _check_selection_structure(sel: torch.Tensor, cnt: torch.Tensor):
    """Every row: cnt = min(qb+1, budget), ascending distinct, own and previous
    block present, -1 padding (on the device, all rows)."""
    nqb = sel.shape[0]
    qb = torch.arange(nqb, device=sel.device, dtype=torch.int64)
    want = torch.clamp(qb + 1, max=BUDGET).to(torch.int32)
    assert torch.equal(cnt, want), "selection counts"
    col = torch.arange(BUDGET, device=sel.device)
    valid = col[None, :] < cnt[:, None]
    assert bool(((sel >= 0) == valid).all()), "padding"
    s64 = sel.to(torch.int64)
    inc = (s64[:, 1:] > s64[:, :-1]) | ~valid[:, 1:]
    assert bool(inc.all()), "ascending"
    last = s64.gather(1, (cnt.to(torch.int64) - 1)[:, None])[:, 0]
    assert torch.equal(last, qb), "own block last"
    prev = s64.gather(1, torch.clamp(cnt.to(torch.int64) - 2, min=0)[:, None])[:, 0]
    assert bool(((prev == qb - 1) | (qb == 0)).all()), "previous block forced"
    assert bool((s64 <= qb[:, None]).all()), "causal"


def _oracle_block_outputs(O, P, qb, sel_row, cnt):
    """fp64 attention of the tokens of block qb over the given selection."""
    T = P.T
    t0, t1 = 4 * qb, min(4 * qb + 4, T)
    blocks = sel_row[:cnt]
    ks, vs, js = [], [], []
    for b in blocks:
        j0, j1 = 4 * int(b), min(4 * int(b) + 4, T)
        k = Q.bf16_to_f64(P.k(j0, j1))
        v = Q.bf16_to_f64(P.v(j0, j1))
        for j in range(j0, j1):
            ks.append(np.stack([O.rope(k[j - j0, g], j) for g in range(2)]))
            vs.append(v[j - j0])
            js.append(j)
    ks, vs, js = np.stack(ks), np.stack(vs), np.asarray(js)
    q = Q.bf16_to_f64(P.q(t0, t1))
    res = []
    for t in range(t0, t1):
        q_rot = np.stack([O.rope(q[t - t0, h], t) for h in range(24)])
        m = js <= t
        res.append(O.attend(q_rot, ks[m], vs[m]))
    return res


@pytest.mark.timeout(1800)
@pytest.mark.parametrize("T,dist", [(32768, "uniform"), (131072, "zipf"), (1048576, "zipf")])
def test_prefill_full_size_sampled(T, dist):
    P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist=dist)
    d = P.device()
    p = qsa.params(BUDGET)
    _, pref = qsa.qsa_prefill_workspace_size(p, T)
    ws = qsa.workspace(pref)
    nqb = P.nqb
    out = torch.empty((T, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((T, 24), dtype=torch.float32, device="cuda")
    sel = torch.empty((nqb, BUDGET), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nqb,), dtype=torch.int32, device="cuda")
    qsa.qsa_prefill(p, T, 0, d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], out, lse, sel, cnt, None, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    del d, ws
    _check_selection_structure(sel, cnt)

    O = oracle.Oracle(oracle.params(budget=BUDGET))
    k_idx = P.k_idx()
    n_diff = 0
    for qb in _sample_blocks(nqb, seed=T):
        t0, t1 = 4 * qb, min(4 * qb + 4, T)
        S = O.block_scores(qb, P.q_idx(t0, t1), P.w(t0, t1), k_idx[:t1])
        osel, ocnt = O.select(qb, S)
        g = sel[qb].cpu().numpy()
        gc = int(cnt[qb])
        n_diff += check_selection(g, gc, osel, ocnt, S, qb, BUDGET, f"T={T} qb={qb}")
        want = _oracle_block_outputs(O, P, qb, g, gc)
        got = out[t0:t1].cpu().numpy()
        got_lse = lse[t0:t1].cpu().numpy()
        for i, (o, l) in enumerate(want):
            check_outputs(got[i], o, f"T={T} t={t0 + i}")
            assert np.allclose(got_lse[i], l, atol=1e-2), f"T={T} t={t0 + i} lse"
    print(f"T={T}: sampled rows differ from the oracle selection in {n_diff} near-tie blocks")


@pytest.mark.timeout(1800)
def test_decode_full_size_sampled():
    B, L = 64, 262144
    D = Q.DecodeProblem(B=B, L=L, steps=1, seed=0, n_plant=8)
    max_len = L + 8
    kc = torch.empty((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.empty_like(kc)
    ic = torch.empty((B, max_len, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    p = qsa.params(BUDGET)
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
    x = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in D.step_inputs(0).items()}
    kin = np.stack([D.tokens(b).k_idx(L, L + 1)[0] for b in range(B)])
    out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((B, BUDGET), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, 24), dtype=torch.float32, device="cuda")
    qsa.qsa_decode(p, B, max_len, [L] * B, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"], x["q_idx"],
                   torch.from_numpy(kin).cuda(), x["w"], out, sel, lse, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    del kc, vc, ic
    O = oracle.Oracle(oracle.params(budget=BUDGET))
    inp = D.step_inputs(0)
    qb = L // 4
    for b in (0, 1, 31, 63):
        kcache, vcache, icache = D.cache_k(b), D.cache_v(b), D.cache_kidx(b)
        ring_q = np.zeros((0, 4, 128), np.uint16)
        ring_w = np.zeros((0, 4), np.uint16)
        S = O.block_scores(qb, inp["q_idx"][b][None], inp["w"][b][None], np.concatenate([icache, kin[b][None]]))
        osel, ocnt, _, _ = O.decode(L, kcache, vcache, icache, ring_q, ring_w, inp["q"][b], inp["k"][b], inp["v"][b],
                                    inp["q_idx"][b], kin[b], inp["w"][b])
        g = sel[b].cpu().numpy()
        gc = int((g >= 0).sum())
        check_selection(g, gc, osel, ocnt, S, qb, BUDGET, f"decode b={b}")
        _, _, oo, ol = O.decode(L, kcache, vcache, icache, ring_q, ring_w, inp["q"][b], inp["k"][b], inp["v"][b],
                                inp["q_idx"][b], kin[b], inp["w"][b], sel_in=g, cnt_in=gc)
        check_outputs(out[b].cpu().numpy(), oo, f"decode b={b}")
        assert np.allclose(lse[b].cpu().numpy(), ol, atol=1e-2), f"decode b={b} lse"


@pytest.mark.timeout(600)
def test_prefill_all_scores_tied_32k():
    """All indexer scores 0 (zero indexer queries): every long row falls back
    from the segment-maxima filter to the exact path and keeps the lowest
    indices, as the tie rule demands."""
    T = 32768
    P = Q.PrefillProblem(T=T, seed=3, n_plant=0)
    d = P.device()
    d["q_idx"].zero_()
    r = qsa.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], budget=BUDGET, want_lse=False)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(r["ws"]) == 0
    sel, cnt = r["sel"], r["cnt"]
    _check_selection_structure(sel, cnt)
    nqb = P.nqb
    qb = torch.arange(nqb, device=sel.device)
    long = qb >= BUDGET
    want_low = torch.arange(BUDGET - 2, device=sel.device, dtype=torch.int32)
    assert bool((sel[long][:, :BUDGET - 2] == want_low[None, :]).all()), "ties must keep the lowest blocks"


@pytest.mark.timeout(1800)
def test_prefill_mean_pool_1m_sampled():
    """The mean-pooled indexer at 1M tokens, run as the benchmark runs it."""
    T = 1048576
    P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="zipf")
    d = P.device()
    p = qsa.params(BUDGET, aggregation=qsa.AGG_MEAN_POOL)
    _, pref = qsa.qsa_prefill_workspace_size(p, T)
    ws = qsa.workspace(pref)
    nqb = P.nqb
    out = torch.empty((T, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((T, 24), dtype=torch.float32, device="cuda")
    sel = torch.empty((nqb, BUDGET), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nqb,), dtype=torch.int32, device="cuda")
    qsa.qsa_prefill(p, T, 0, d["q"], d["k"], d["v"], d["q_idx"], d["w"], d["k_idx"], out, lse, sel, cnt, None, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    del d, ws
    _check_selection_structure(sel, cnt)
    O = oracle.Oracle(oracle.params(budget=BUDGET, aggregation=oracle.AGG_MEAN_POOL))
    k_idx = P.k_idx()
    n_diff = 0
    for qb in _sample_blocks(nqb, seed=7)[::2]:
        t0, t1 = 4 * qb, min(4 * qb + 4, T)
        S = O.block_scores(qb, P.q_idx(t0, t1), P.w(t0, t1), k_idx[:t1])
        osel, ocnt = O.select(qb, S)
        g = sel[qb].cpu().numpy()
        gc = int(cnt[qb])
        n_diff += check_selection(g, gc, osel, ocnt, S, qb, BUDGET, f"mean pool qb={qb}")
        want = _oracle_block_outputs(O, P, qb, g, gc)
        got = out[t0:t1].cpu().numpy()
        for i, (o, l) in enumerate(want):
            check_outputs(got[i], o, f"mean pool t={t0 + i}")
    print(f"mean pool 1M: sampled rows differ from the oracle selection in {n_diff} near-tie blocks")


def _decode_full_setup(B, L, aggregation=0):
    D = Q.DecodeProblem(B=B, L=L, steps=2, seed=0, n_plant=8)
    max_len = L + 8
    kc = torch.empty((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.empty_like(kc)
    ic = torch.empty((B, max_len, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    p = qsa.params(BUDGET, aggregation=aggregation)
    kbar = None
    if aggregation:
        kbar = torch.zeros((B, (max_len + 3) // 4, 128), dtype=torch.uint16, device="cuda")
        for b in range(B):
            qsa.qsa_mean_pool_keys(p, L, ic[b], kbar[b])
    st = dict(D=D, max_len=max_len, kc=kc, vc=vc, ic=ic, kbar=kbar, p=p,
              ring=torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda"),
              wring=torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda"),
              ws=qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len)))
    return st


def _step_tensors(D, s):
    x = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in D.step_inputs(s).items()}
    x["k_idx"] = torch.from_numpy(np.stack([D.tokens(b).k_idx(D.L + s, D.L + s + 1)[0] for b in range(D.B)])).cuda()
    return x


@pytest.mark.timeout(1800)
def test_decode_mean_pool_and_reuse_full_size_sampled():
    """64 sequences x 256K: a mean-pool decode step (compressed-key cache),
    then a draft step at the next token reusing its selection; sampled
    sequences against the oracle's mean-pool decode and reuse rule."""
    B, L = 64, 262144
    st = _decode_full_setup(B, L, aggregation=qsa.AGG_MEAN_POOL)
    D, p = st["D"], st["p"]
    outs, sels = [], None
    for s in range(2):
        x = _step_tensors(D, s)
        out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
        if s == 0:
            sels = torch.empty((B, BUDGET), dtype=torch.int32, device="cuda")
            qsa.qsa_decode_mean_pool(p, B, st["max_len"], [L] * B, st["kc"], st["vc"], st["ic"], st["kbar"],
                                     st["ring"], st["wring"], x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["w"],
                                     out, sels, None, st["ws"])
        else:
            qsa.qsa_decode_reuse(p, B, st["max_len"], [L + 1] * B, st["kc"], st["vc"], st["ic"], st["kbar"],
                                 st["ring"], st["wring"], x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["w"],
                                 sels, None, out, None, st["ws"])
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(st["ws"]) == 0
        outs.append(out.cpu().numpy())
    sel_h = sels.cpu().numpy()
    del st
    O = oracle.Oracle(oracle.params(budget=BUDGET, aggregation=oracle.AGG_MEAN_POOL))
    in0, in1 = D.step_inputs(0), D.step_inputs(1)
    qb = L // 4
    for b in (0, 17, 63):
        P = D.tokens(b)
        kin0 = P.k_idx(L, L + 1)[0]
        kin1 = P.k_idx(L + 1, L + 2)[0]
        kcache, vcache, icache = D.cache_k(b), D.cache_v(b), D.cache_kidx(b)
        ring_q = np.zeros((0, 4, 128), np.uint16)
        ring_w = np.zeros((0, 4), np.uint16)
        S = O.block_scores(qb, in0["q_idx"][b][None], in0["w"][b][None], np.concatenate([icache, kin0[None]]))
        osel, ocnt, _, _ = O.decode(L, kcache, vcache, icache, ring_q, ring_w, in0["q"][b], in0["k"][b], in0["v"][b],
                                    in0["q_idx"][b], kin0, in0["w"][b])
        g = sel_h[b]
        gc = int((g >= 0).sum())
        check_selection(g, gc, osel, ocnt, S, qb, BUDGET, f"mean-pool decode b={b}")
        _, _, oo, _ = O.decode(L, kcache, vcache, icache, ring_q, ring_w, in0["q"][b], in0["k"][b], in0["v"][b],
                               in0["q_idx"][b], kin0, in0["w"][b], sel_in=g, cnt_in=gc)
        check_outputs(outs[0][b], oo, f"mean-pool decode b={b}")
        # draft step at L + 1 over the reused row; the cache now holds token L,
        # rotated by the GPU append (compared against the oracle's fp64 rotation
        # through the output tolerance)
        k_new_rot = np.stack([O.rope(Q.bf16_to_f64(in0["k"][b][g]), L) for g in range(2)])
        kc1 = np.concatenate([kcache, Q.f32_to_bf16(k_new_rot.astype(np.float32))[None]])
        vc1 = np.concatenate([vcache, in0["v"][b][None]])
        ic1 = np.concatenate([icache, kin0[None]])
        _, _, oo1, _ = O.decode_reuse(L + 1, kc1, vc1, ic1, in0["q_idx"][b][None], in0["w"][b][None], in1["q"][b],
                                      in1["k"][b], in1["v"][b], in1["q_idx"][b], kin1, in1["w"][b], sel_in=g,
                                      cnt_in=gc)
        check_outputs(outs[1][b], oo1, f"reuse draft step b={b}")


@pytest.mark.timeout(1800)
def test_verify_full_size_sampled():
    """64 sequences x 256K cached tokens, 5 new tokens each (as the benchmark's
    verify calls): sampled sequences against the oracle -- selection of both
    touched query blocks, and every new token's output on its selection."""
    B, L, m = 64, 262144, 5
    st = _decode_full_setup(B, L)
    D, p = st["D"], st["p"]
    new = {k: [] for k in ("q", "k", "v", "q_idx", "k_idx", "w")}
    for b in range(B):
        P = D.tokens(b)
        for k in new:
            new[k].append(getattr(P, k)(L, L + m))
    x = {k: torch.from_numpy(np.ascontiguousarray(np.stack(v))).cuda() for k, v in new.items()}
    ws = qsa.workspace(qsa.qsa_verify_workspace_size(p, B, m, st["max_len"]))
    out = torch.empty((B, m, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((B, m, BUDGET), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, m, 24), dtype=torch.float32, device="cuda")
    qsa.qsa_verify(p, B, m, st["max_len"], [L] * B, st["kc"], st["vc"], st["ic"], st["ring"], st["wring"], x["q"],
                   x["k"], x["v"], x["q_idx"], x["k_idx"], x["w"], out, sel, lse, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    out, sel, lse = out.cpu().numpy(), sel.cpu().numpy(), lse.cpu().numpy()
    new_krot = st["kc"][:, L:L + m].cpu().numpy()
    del st, ws
    O = oracle.Oracle(oracle.params(budget=BUDGET))
    ring_q, ring_w = np.zeros((0, 4, 128), np.uint16), np.zeros((0, 4), np.uint16)
    for b in (0, 33, 63):
        nb = {k: v[b] for k, v in new.items()}
        kid = np.concatenate([D.cache_kidx(b), nb["k_idx"]])
        kc_full, vc_full = D.cache_k(b), D.cache_v(b)
        for qb in sorted({(L + i) // 4 for i in range(m)}):
            t0, t1 = max(4 * qb, L), min(4 * qb + 4, L + m)
            S = O.block_scores(qb, nb["q_idx"][t0 - L:t1 - L], nb["w"][t0 - L:t1 - L], kid[:t1])
            osel, ocnt = O.select(qb, S)
            g = sel[b, t0 - L]
            gc = int((g >= 0).sum())
            check_selection(g, gc, osel, ocnt, S, qb, BUDGET, f"verify b={b} qb={qb}")
            for t in range(t0, t1):
                i = t - L
                assert np.array_equal(sel[b, i], g)
                kc = np.concatenate([kc_full, new_krot[b, :i]])
                vc = np.concatenate([vc_full, nb["v"][:i]])
                _, _, oo, ol = O.decode(t, kc, vc, kid[:t], ring_q, ring_w, nb["q"][i], nb["k"][i], nb["v"][i],
                                        nb["q_idx"][i], kid[t], nb["w"][i], sel_in=g, cnt_in=gc)
                check_outputs(out[b, i], oo, f"verify b={b} t={t}")
                assert np.allclose(lse[b, i], ol, atol=1e-2), f"verify b={b} t={t} lse"
