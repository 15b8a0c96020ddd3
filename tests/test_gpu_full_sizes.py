"""GPU parity at the full workload sizes (32K, 128K and 1M prefill; the
mean-pool, reuse and verify paths at 64 sequences x 256K), run as the
benchmark runs them (same workspace, so the same chunking), checked on
stratified query blocks / sampled sequences that the fp64 oracle computes one
by one, plus structural checks of every selection row.  The plain decode of
config 3 (all 32 appending steps) is in test_gpu_decode_config3.py."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, check_selection, gather_rows, pmap

pytestmark = pytest.mark.gpu

BUDGET = 512


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def _sample_blocks(nqb: int, seed: int, n: int = 18) -> list[int]:
    """n stratified query blocks: the first and last, those around the budget
    boundary, seeded random ones and evenly spaced ones."""
    return [int(q) for q in Q.stratified_query_blocks(nqb, n=n, budget=BUDGET, seed=seed)]


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
    pos, ks, vs = gather_rows(sel_row[:cnt], T, P.k, P.v)
    t0, t1 = 4 * qb, min(4 * qb + 4, T)
    q = P.q(t0, t1)
    return [O.attend_gathered(t, q[t - t0], pos, ks, vs) for t in range(t0, t1)]


def _check_sampled_blocks(O, P, qbs, sel, cnt, out, lse, what, k_idx=None):
    """Oracle scores, selection and attention of the sampled query blocks (a
    thread pool over blocks), compared by the acceptance criteria; returns the
    number of near-tie selection differences."""
    T = P.T
    k_idx = P.k_idx() if k_idx is None else k_idx
    sel_h = sel[torch.tensor(qbs, device=sel.device)].cpu().numpy()
    cnt_h = cnt[torch.tensor(qbs, device=cnt.device)].cpu().numpy()
    rows = torch.cat([torch.arange(4 * q, min(4 * q + 4, T)) for q in qbs]).to(out.device)
    out_h = out.view(torch.int16)[rows].cpu().numpy().view(np.uint16)   # no uint16 gather on CUDA
    lse_h = lse[rows].cpu().numpy() if lse is not None else None
    first = {}
    n = 0
    for q in qbs:
        first[q] = n
        n += min(4 * q + 4, T) - 4 * q

    def one(i):
        qb = qbs[i]
        t0, t1 = 4 * qb, min(4 * qb + 4, T)
        S = O.block_scores(qb, P.q_idx(t0, t1), P.w(t0, t1), k_idx[:t1])
        osel, ocnt = O.select(qb, S)
        return S, osel, ocnt, _oracle_block_outputs(O, P, qb, sel_h[i], int(cnt_h[i]))

    n_diff = 0
    for i, (S, osel, ocnt, want) in enumerate(pmap(one, range(len(qbs)))):
        qb = qbs[i]
        n_diff += check_selection(sel_h[i], int(cnt_h[i]), osel, ocnt, S, qb, BUDGET, f"{what} qb={qb}")
        for k, (o, l) in enumerate(want):
            r = first[qb] + k
            check_outputs(out_h[r], o, f"{what} t={4 * qb + k}")
            if lse_h is not None:
                assert np.allclose(lse_h[r], l, atol=1e-2), f"{what} t={4 * qb + k} lse"
    return n_diff


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
    # 256 stratified query blocks at 1M (the stratified sample the CPU baseline times too), 64 below
    qbs = _sample_blocks(nqb, seed=T, n=256 if T >= 1 << 20 else 64)
    n_diff = _check_sampled_blocks(O, P, qbs, sel, cnt, out, lse, f"T={T}")
    print(f"T={T}: {len(qbs)} sampled query blocks, {n_diff} near-tie selection differences")


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
@pytest.mark.parametrize("rope", [0, 1])
def test_prefill_mean_pool_1m_sampled(rope):
    """The mean-pooled indexer at 1M tokens, run as the benchmark runs it;
    rope = 1: with the indexer's RoPE (queries at their token, each compressed
    key at its block's first token)."""
    T = 1048576
    P = Q.PrefillProblem(T=T, seed=0, n_plant=8, dist="zipf")
    d = P.device()
    p = qsa.params(BUDGET, aggregation=qsa.AGG_MEAN_POOL, idx_rope=rope)
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
    O = oracle.Oracle(oracle.params(budget=BUDGET, aggregation=oracle.AGG_MEAN_POOL, idx_rope=rope))
    qbs = _sample_blocks(nqb, seed=7, n=64)
    what = "mean pool 1M" + (" with RoPE" if rope else "")
    n_diff = _check_sampled_blocks(O, P, qbs, sel, cnt, out, None, what)
    print(f"{what}: {len(qbs)} sampled query blocks, {n_diff} near-tie selection differences")


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
    assert L % 4 == 0
    O = oracle.Oracle(oracle.params(budget=BUDGET))
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
                # block-mates 4 qb .. t - 1 (new tokens, as L % 4 == 0)
                m0 = 4 * qb - L
                _, _, oo, ol = O.decode(t, kc, vc, kid[:t], nb["q_idx"][m0:i], nb["w"][m0:i], nb["q"][i], nb["k"][i],
                                        nb["v"][i], nb["q_idx"][i], kid[t], nb["w"][i], sel_in=g, cnt_in=gc)
                check_outputs(out[b, i], oo, f"verify b={b} t={t}")
                assert np.allclose(lse[b, i], ol, atol=1e-2), f"verify b={b} t={t} lse"
