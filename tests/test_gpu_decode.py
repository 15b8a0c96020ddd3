"""GPU parity of the decode path (C ABI): decode equals prefill's last token,
and matches the oracle on its own selection."""
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


@pytest.fixture
def automatic_splits_after():
    """Back to the automatic split-KV choice once the test is done."""
    yield
    qsa.qsa_set_decode_splits(0)


class DecodeState:
    """Caches [B][max_len] seeded from a prefill of each sequence's first L tokens."""

    def __init__(self, probs, L_list, max_len, budget, transform=None):
        self.B = len(probs)
        self.max_len = max_len
        self.budget = budget
        self.p = qsa.params(budget)
        B = self.B
        self.k_cache = torch.zeros((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
        self.v_cache = torch.zeros_like(self.k_cache)
        self.kidx_cache = torch.zeros((B, max_len, 128), dtype=torch.uint16, device="cuda")
        self.qidx_ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
        self.w_ring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
        self.hosts = []
        self.lens = list(L_list)
        for b, (P, L) in enumerate(zip(probs, L_list)):
            h = P.host()
            if transform is not None:
                h = transform(h)
            self.hosts.append(h)
            pre = Q.PrefillProblem(T=L, seed=P.seed, n_plant=P.n_plant, dist=P.dist)
            # the first L tokens of P are a prefix of P's token streams except k_idx planting,
            # so the prefill runs on P's own tensors truncated to L
            sub = {k: v[:L] for k, v in h.items()}
            _, r = gpu_prefill(pre, budget, host=sub)
            self.k_cache[b, :L] = dev(r["k_rot"])
            self.v_cache[b, :L] = dev(sub["v"])
            self.kidx_cache[b, :L] = dev(sub["k_idx"])
            t0 = (L // 4) * 4
            for t in range(t0, L):
                self.qidx_ring[b, t % 4] = dev(h["q_idx"][t])
                self.w_ring[b, t % 4] = dev(h["w"][t])
        self.ws = qsa.workspace(qsa.qsa_decode_workspace_size(self.p, B, max_len))

    def step(self):
        B = self.B
        new = {k: np.stack([self.hosts[b][k][self.lens[b]] for b in range(B)]) for k in
               ("q", "k", "v", "q_idx", "k_idx", "w")}
        out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
        sel = torch.empty((B, self.budget), dtype=torch.int32, device="cuda")
        lse = torch.empty((B, 24), dtype=torch.float32, device="cuda")
        qsa.qsa_decode(self.p, B, self.max_len, self.lens, self.k_cache, self.v_cache, self.kidx_cache,
                       self.qidx_ring, self.w_ring, dev(new["q"]), dev(new["k"]), dev(new["v"]), dev(new["q_idx"]),
                       dev(new["k_idx"]), dev(new["w"]), out, sel, lse, self.ws)
        torch.cuda.synchronize()
        assert qsa.qsa_check_device_error(self.ws) == 0
        pos = list(self.lens)
        self.lens = [L + 1 for L in self.lens]
        return pos, out.cpu().numpy(), sel.cpu().numpy(), lse.cpu().numpy()


def _large_logits(h):
    """Queries x 8 and keys x 1 / 2 / 4 over the first half, third quarter and
    last quarter of the tokens (exact bf16 exponent shifts): the running
    maximum of a row rises across its tiles and the online softmax rescales."""
    def times_pow2(a, e):
        a = a.copy()
        nz = ((a >> 7) & 0xFF) != 0
        a[nz] += np.uint16(e << 7)
        return a
    h = dict(h)
    T = h["k"].shape[0]
    h["q"] = times_pow2(h["q"], 3)
    k = h["k"].copy()
    k[T // 2:3 * T // 4] = times_pow2(k[T // 2:3 * T // 4], 1)
    k[3 * T // 4:] = times_pow2(k[3 * T // 4:], 2)
    h["k"] = k
    return h


@pytest.mark.parametrize("budget,large", [(16, False), (512, False), (512, True)])
def test_decode_matches_prefill_last_token(budget, large):
    """Prefill L+s+1 tokens; decode token L+s from a cache seeded with the
    first L rotated keys; compare at every step s.  Covers a block-aligned
    start, mid-block starts (ring seeded from the prompt) and budget-limited
    selection; large: attention logits far from unit scale (~80 nats), so
    both kernels' online softmax rescales along a row.  There decode is held
    to prefill only: the bf16 rounding of the rotated queries and keys, which
    the fp64 oracle does not share, moves such logits by ~0.1 and the outputs
    beyond the acceptance bounds that assume unit-scale logits."""
    L_list = [2048 + 4 * budget, 2301, 4097] if budget == 512 else [64, 129, 301]
    steps = 5
    probs = [Q.PrefillProblem(T=L + steps, seed=40 + b, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + steps + 8, budget=budget,
                     transform=_large_logits if large else None)
    O = oracle.Oracle(oracle.params(budget=budget))
    for s in range(steps):
        pos, out, sel, lse = st.step()
        for b, P in enumerate(probs):
            L = pos[b]
            h = st.hosts[b]
            T = L + 1
            sub = {k: v[:T] for k, v in h.items()}
            _, r = gpu_prefill(Q.PrefillProblem(T=T, seed=P.seed), budget, host=sub)
            qb = L // 4
            # same selection up to near-ties of the fp64 scores
            S = O.block_scores(qb, h["q_idx"][4 * qb:T], h["w"][4 * qb:T], h["k_idx"][:T])
            check_selection(sel[b], int((sel[b] >= 0).sum()), r["sel"][qb], int(r["cnt"][qb]), S, qb, budget,
                            f"b={b} s={s}")
            # decode vs prefill's last token
            check_outputs(out[b], Q.bf16_to_f64(r["out"][L]), f"decode vs prefill b={b} s={s}")
            if large:
                continue
            # decode vs the oracle on the GPU's own selection (cache = bf16 rotated keys)
            kc = st.k_cache[b, :L].cpu().numpy()
            t0 = 4 * qb
            cnt = int((sel[b] >= 0).sum())
            _, _, oo, ol = O.decode(L, kc, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L],
                                    h["k"][L], h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L], sel_in=sel[b],
                                    cnt_in=cnt)
            check_outputs(out[b], oo, f"decode vs oracle b={b} s={s}")
            assert np.allclose(lse[b], ol, atol=1e-2)


def test_decode_append_writes_caches():
    L_list = [10, 13]
    probs = [Q.PrefillProblem(T=L + 2, seed=60 + b) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=32, budget=16)
    st.step()
    O = oracle.Oracle(oracle.params(budget=16))
    for b, L in enumerate(L_list):
        h = st.hosts[b]
        assert np.array_equal(st.v_cache[b, L].cpu().numpy(), h["v"][L])
        assert np.array_equal(st.kidx_cache[b, L].cpu().numpy(), h["k_idx"][L])
        assert np.array_equal(st.qidx_ring[b, L % 4].cpu().numpy(), h["q_idx"][L])
        assert np.array_equal(st.w_ring[b, L % 4].cpu().numpy(), h["w"][L])
        kr = np.stack([O.rope(Q.bf16_to_f64(h["k"][L, g]), L) for g in range(2)])
        assert np.abs(Q.bf16_to_f64(st.k_cache[b, L].cpu().numpy()) - kr).max() < 0.05


@pytest.mark.parametrize("splits", [1, 2, 5, 16])
def test_decode_split_kv_ranges(splits, automatic_splits_after):
    """Split-KV decode with a fixed number of ranges, including ranges left
    empty by a short sequence (1 tile) next to full-budget ones (32 tiles):
    output and lse match the oracle on the kernel's own selection."""
    qsa.qsa_set_decode_splits(splits)
    budget = 512
    L_list = [3001, 37, 9000]
    probs = [Q.PrefillProblem(T=L + 1, seed=70 + b, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    O = oracle.Oracle(oracle.params(budget=budget))
    pos, out, sel, lse = st.step()
    for b in range(len(L_list)):
        L = pos[b]
        h = st.hosts[b]
        qb = L // 4
        t0 = 4 * qb
        cnt = int((sel[b] >= 0).sum())
        assert cnt == min(qb + 1, budget)
        kc = st.k_cache[b, :L].cpu().numpy()
        _, _, oo, ol = O.decode(L, kc, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L],
                                h["k"][L], h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L], sel_in=sel[b],
                                cnt_in=cnt)
        check_outputs(out[b], oo, f"splits={splits} b={b}")
        assert np.allclose(lse[b], ol, atol=1e-2), f"splits={splits} b={b}"


def test_decode_largest_budget():
    """Budget 4096 (the largest accepted): the selection binds only past
    16K keys; decode against the prefill's last token and the oracle."""
    budget = 4096
    L_list = [20001, 16390]
    probs = [Q.PrefillProblem(T=L + 1, seed=90 + b, n_plant=8) for b, L in enumerate(L_list)]
    st = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
    pos, out, sel, lse = st.step()
    O = oracle.Oracle(oracle.params(budget=budget))
    for b, L in enumerate(pos):
        h = st.hosts[b]
        T = L + 1
        _, r = gpu_prefill(Q.PrefillProblem(T=T, seed=probs[b].seed), budget, host={k: v[:T] for k, v in h.items()})
        qb = L // 4
        cnt = int((sel[b] >= 0).sum())
        assert cnt == min(qb + 1, budget)
        S = O.block_scores(qb, h["q_idx"][4 * qb:T], h["w"][4 * qb:T], h["k_idx"][:T])
        check_selection(sel[b], cnt, r["sel"][qb], int(r["cnt"][qb]), S, qb, budget, f"b={b}")
        check_outputs(out[b], Q.bf16_to_f64(r["out"][L]), f"budget 4096 decode b={b}")
        kc = st.k_cache[b, :L].cpu().numpy()
        t0 = 4 * qb
        _, _, oo, _ = O.decode(L, kc, h["v"][:L], h["k_idx"][:L], h["q_idx"][t0:L], h["w"][t0:L], h["q"][L], h["k"][L],
                               h["v"][L], h["q_idx"][L], h["k_idx"][L], h["w"][L], sel_in=sel[b], cnt_in=cnt)
        check_outputs(out[b], oo, f"budget 4096 decode vs oracle b={b}")
