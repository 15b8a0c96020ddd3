"""Config 3 as specified, at its full size: 64 sequences with 262,144 cached
tokens each and 32 consecutive decode steps appending to the cache, run as
the benchmark runs them.  Sampled sequences at steps 0, 1, 2, 3 and 31 are
checked against the fp64 oracle: the selection by the near-tie rule and the
outputs and lse on the GPU's own selection.  The ring carries the block-mates
the earlier steps appended, so at steps 1-3 the query block holds 2-4 tokens.
A second test checks decode against prefill's last token at 256K: two
sequences decode 32 tokens from a cache seeded by a prefill of their first
262,144 tokens, and each step must match qsa_prefill over the first
262,145 .. 262,176 tokens."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, check_selection, gather_rows, pmap

pytestmark = pytest.mark.gpu

BUDGET = 512
B, L, STEPS = 64, 262144, 32
CHECK_STEPS = (0, 1, 2, 3, 31)
SAMPLED = (0, 1, 31, 63)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def _decode_inputs(D, s):
    """Device inputs of decode step s (token L + s of every sequence)."""
    x = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in D.step_inputs(s).items()}
    x["k_idx"] = torch.from_numpy(np.stack([D.tokens(b).k_idx(D.L + s, D.L + s + 1)[0]
                                            for b in range(D.B)])).cuda()
    return x


@pytest.mark.timeout(2400)
def test_decode_32_appending_steps_64x256k():
    D = Q.DecodeProblem(B=B, L=L, steps=STEPS, seed=0, n_plant=8)
    max_len = L + STEPS + 4
    kc = torch.empty((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.empty_like(kc)
    ic = torch.empty((B, max_len, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    p = qsa.params(BUDGET)
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
    out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((B, BUDGET), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, 24), dtype=torch.float32, device="cuda")
    got = {}
    idx = torch.tensor(SAMPLED, device="cuda")
    for s in range(STEPS):
        x = _decode_inputs(D, s)
        qsa.qsa_decode(p, B, max_len, [L + s] * B, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"], x["q_idx"],
                       x["k_idx"], x["w"], out, sel, lse, ws)
        if s in CHECK_STEPS:
            got[s] = (out.view(torch.int16)[idx].cpu().numpy().view(np.uint16), sel[idx].cpu().numpy(),
                      lse[idx].cpu().numpy())
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    # every sequence appended all 32 tokens: the last appended indexer key
    last_kidx = ic[:, L + STEPS - 1].cpu().numpy()
    del kc, vc, ic, ws
    torch.cuda.empty_cache()
    for i, b in enumerate(range(B)):
        assert np.array_equal(last_kidx[b], D.tokens(b).k_idx(L + STEPS - 1, L + STEPS)[0]), b

    O = oracle.Oracle(oracle.params(budget=BUDGET))

    def one(case):
        i, b, s = case
        P = D.tokens(b)
        t = L + s
        qb = t // 4
        t0 = 4 * qb
        kid = np.concatenate([D.cache_kidx(b), P.k_idx(L, t + 1)])          # keys 0 .. t
        # block-mates t0 .. t-1 (all appended by earlier steps, since L % 4 == 0)
        ring_q, ring_w = P.q_idx(t0, t), P.w(t0, t)
        q_blk = np.concatenate([ring_q, P.q_idx(t, t + 1)])
        w_blk = np.concatenate([ring_w, P.w(t, t + 1)])
        S = O.block_scores(qb, q_blk, w_blk, kid)
        osel, ocnt = O.select(qb, S)
        g_out, g_sel, g_lse = got[s][0][i], got[s][1][i], got[s][2][i]
        gc = int((g_sel >= 0).sum())
        # the oracle's decode on the GPU's selection; cache rows the selection
        # needs: the synthetic prompt rows, and the decode tokens L .. t-1
        # rotated by the oracle's RoPE and stored as bf16 (the cache's type)
        kc_h = np.zeros((t, 2, 256), np.uint16)
        vc_h = np.zeros((t, 2, 256), np.uint16)
        for blk in g_sel[:gc]:
            a0, a1 = 4 * int(blk), min(4 * int(blk) + 4, L)
            if a1 > a0:
                kc_h[a0:a1] = D.cache_k(b, a0, a1)
                vc_h[a0:a1] = D.cache_v(b, a0, a1)
        for j in range(L, t):
            kj = P.k(j, j + 1)[0]
            kc_h[j] = Q.f32_to_bf16(np.stack([O.rope(Q.bf16_to_f64(kj[g]), j) for g in range(2)]).astype(np.float32))
            vc_h[j] = P.v(j, j + 1)[0]
        x = {k: getattr(P, k)(t, t + 1)[0] for k in ("q", "k", "v", "q_idx", "w")}
        # the oracle's own decode selection (its ring path) must equal the
        # selection from the block scores above
        dsel, dcnt, _, _ = O.decode(t, kc_h, vc_h, kid[:t], ring_q, ring_w, x["q"], x["k"], x["v"], x["q_idx"],
                                    kid[t], x["w"])
        _, _, oo, ol = O.decode(t, kc_h, vc_h, kid[:t], ring_q, ring_w, x["q"], x["k"], x["v"], x["q_idx"], kid[t],
                                x["w"], sel_in=g_sel, cnt_in=gc)
        return b, s, qb, S, osel, ocnt, dsel, dcnt, g_out, g_sel, gc, g_lse, oo, ol

    cases = [(i, b, s) for s in CHECK_STEPS for i, b in enumerate(SAMPLED)]
    n_diff = 0
    for b, s, qb, S, osel, ocnt, dsel, dcnt, g_out, g_sel, gc, g_lse, oo, ol in pmap(one, cases):
        what = f"decode step {s} b={b}"
        assert dcnt == ocnt and np.array_equal(dsel, osel), f"{what}: oracle decode vs its block scores"
        n_diff += check_selection(g_sel, gc, osel, ocnt, S, qb, BUDGET, what)
        check_outputs(g_out, oo, what)
        assert np.allclose(g_lse, ol, atol=1e-2), f"{what}: lse"
    print(f"config 3: {len(cases)} (step, sequence) pairs checked, {n_diff} near-tie selection differences")


@pytest.mark.timeout(2400)
def test_decode_equals_prefill_last_token_256k():
    """North-star check 3 at 256K: decode step s (token L + s) equals the last
    token of qsa_prefill over the first L + s + 1 tokens, s = 0 .. 31."""
    NB = 2
    T_full = L + STEPS
    seqs = [Q.PrefillProblem(T=T_full, seed=Q.seq_seed(5, b), n_plant=8, dist="uniform") for b in range(NB)]
    p = qsa.params(BUDGET)
    max_len = L + STEPS + 4
    kc = torch.zeros((NB, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.zeros_like(kc)
    ic = torch.zeros((NB, max_len, 128), dtype=torch.uint16, device="cuda")
    ring = torch.zeros((NB, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((NB, 4, 4), dtype=torch.uint16, device="cuda")
    pre_out = np.zeros((NB, STEPS, 24, 256), np.uint16)
    pre_lse = np.zeros((NB, STEPS, 24), np.float32)
    pre_sel = np.zeros((NB, STEPS, BUDGET), np.int32)
    inputs = []
    for b, P in enumerate(seqs):
        d = P.device()
        # the cache of the first L tokens, from a prefill of them (rotated keys)
        r = qsa.prefill(d["q"][:L], d["k"][:L], d["v"][:L], d["q_idx"][:L], d["w"][:L], d["k_idx"][:L],
                        budget=BUDGET, want_krot=True, want_lse=False)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(r["ws"]) == 0
        kc[b, :L] = r["k_rot"]
        vc[b, :L] = d["v"][:L]
        ic[b, :L] = d["k_idx"][:L]
        del r
        for s in range(STEPS):
            T = L + s + 1
            r = qsa.prefill(d["q"][:T], d["k"][:T], d["v"][:T], d["q_idx"][:T], d["w"][:T], d["k_idx"][:T],
                            budget=BUDGET)
            torch.cuda.synchronize()
            assert qsa.qsa_check_device_error(r["ws"]) == 0
            pre_out[b, s] = r["out"][T - 1].cpu().numpy()
            pre_lse[b, s] = r["lse"][T - 1].cpu().numpy()
            pre_sel[b, s] = r["sel"][(T - 1) // 4].cpu().numpy()
            del r
        inputs.append({k: d[k][L:L + STEPS].clone() for k in ("q", "k", "v", "q_idx", "w", "k_idx")})
        del d
        torch.cuda.empty_cache()
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, NB, max_len))
    out = torch.empty((NB, 24, 256), dtype=torch.uint16, device="cuda")
    sel = torch.empty((NB, BUDGET), dtype=torch.int32, device="cuda")
    lse = torch.empty((NB, 24), dtype=torch.float32, device="cuda")
    dec_out = np.zeros_like(pre_out)
    dec_lse = np.zeros_like(pre_lse)
    dec_sel = np.zeros_like(pre_sel)
    for s in range(STEPS):
        x = {k: torch.stack([inputs[b][k][s] for b in range(NB)]).contiguous() for k in inputs[0]}
        qsa.qsa_decode(p, NB, max_len, [L + s] * NB, kc, vc, ic, ring, wring, x["q"], x["k"], x["v"], x["q_idx"],
                       x["k_idx"], x["w"], out, sel, lse, ws)
        dec_out[:, s] = out.cpu().numpy()
        dec_lse[:, s] = lse.cpu().numpy()
        dec_sel[:, s] = sel.cpu().numpy()
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    del kc, vc, ic, ws
    torch.cuda.empty_cache()

    O = oracle.Oracle(oracle.params(budget=BUDGET))
    n_sel_diff = 0
    for b, P in enumerate(seqs):
        kid = None
        for s in range(STEPS):
            t = L + s
            what = f"decode vs prefill b={b} t={t}"
            ds, ps = dec_sel[b, s], pre_sel[b, s]
            if not np.array_equal(ds, ps):
                # the two paths score with different tensor-core kernels (fp32
                # sums in different orders): a difference must be a near tie
                # of the oracle's scores
                if kid is None:
                    kid = P.k_idx(0, L + STEPS)
                qb = t // 4
                S = O.block_scores(qb, P.q_idx(4 * qb, t + 1), P.w(4 * qb, t + 1), kid[:t + 1])
                osel, ocnt = O.select(qb, S)
                n_sel_diff += check_selection(ds, int((ds >= 0).sum()), osel, ocnt, S, qb, BUDGET, what + " (decode)")
                check_selection(ps, int((ps >= 0).sum()), osel, ocnt, S, qb, BUDGET, what + " (prefill)")
            check_outputs(dec_out[b, s], Q.bf16_to_f64(pre_out[b, s]), what)
            assert np.allclose(dec_lse[b, s], pre_lse[b, s], atol=1e-2), what + " lse"
    print(f"decode == prefill at 256K: {NB * STEPS} tokens, {n_sel_diff} near-tie selection differences")
