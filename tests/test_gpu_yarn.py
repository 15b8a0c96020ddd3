"""GPU parity with static YaRN (qsa_params.yarn_factor = 4, original length
262144): prefill outputs against the oracle's YaRN attention on the GPU's own
selection, decode equal to prefill's last token, and the rotated keys."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import oracle
import qsa_inputs as Q
from gpu_util import check_outputs, dev

pytestmark = pytest.mark.gpu
YARN = dict(yarn_factor=4.0, yarn_original_max=262144.0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()


def _prefill(h, T, budget, pos0=0):
    p = qsa.params(budget, **YARN)
    t = {k: dev(v) for k, v in h.items()}
    mn, pref = qsa.qsa_prefill_workspace_size(p, T)
    ws = qsa.workspace(pref)
    nqb = (T + 3) // 4
    out = torch.empty((T, 24, 256), dtype=torch.uint16, device="cuda")
    lse = torch.empty((T, 24), dtype=torch.float32, device="cuda")
    sel = torch.empty((nqb, budget), dtype=torch.int32, device="cuda")
    cnt = torch.empty((nqb,), dtype=torch.int32, device="cuda")
    krot = torch.empty((T, 2, 256), dtype=torch.uint16, device="cuda")
    qsa.qsa_prefill(p, T, pos0, t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], out, lse, sel, cnt, krot, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    return {k: v.cpu().numpy() for k, v in dict(out=out, lse=lse, sel=sel, cnt=cnt, k_rot=krot).items()}


@pytest.mark.parametrize("T,budget,pos0", [(301, 16, 0), (2053, 64, 0), (777, 16, 300000)])
def test_yarn_prefill_vs_oracle(T, budget, pos0):
    P = Q.PrefillProblem(T=T, seed=500 + T, n_plant=3)
    h = P.host()
    r = _prefill(h, T, budget, pos0)
    O = oracle.Oracle(oracle.params(budget=budget, **YARN))
    nqb = P.nqb
    out, lse = O.attend_blocks(T, h["q"], h["k"], h["v"], np.arange(nqb), r["sel"], r["cnt"], pos0=pos0)
    check_outputs(r["out"], out[:T], f"yarn T={T} pos0={pos0}")
    assert np.allclose(r["lse"], lse[:T], atol=1e-2, rtol=1e-3)
    kr = np.stack([[O.rope(Q.bf16_to_f64(h["k"][t, g]), pos0 + t) for g in range(2)] for t in range(0, T, 37)])
    assert np.abs(Q.bf16_to_f64(r["k_rot"][::37]) - kr).max() < 0.05


def test_yarn_decode_equals_prefill_last_token():
    budget = 64
    L = 1301
    T = L + 1
    P = Q.PrefillProblem(T=T, seed=77, n_plant=4)
    h = P.host()
    full = _prefill(h, T, budget)
    pre = _prefill({k: v[:L] for k, v in h.items()}, L, budget)
    p = qsa.params(budget, **YARN)
    B, max_len = 1, L + 8
    kc = torch.zeros((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.zeros_like(kc)
    ic = torch.zeros((B, max_len, 128), dtype=torch.uint16, device="cuda")
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    kc[0, :L] = dev(pre["k_rot"])
    vc[0, :L] = dev(h["v"][:L])
    ic[0, :L] = dev(h["k_idx"][:L])
    for t in range((L // 4) * 4, L):
        ring[0, t % 4] = dev(h["q_idx"][t])
        wring[0, t % 4] = dev(h["w"][t])
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
    out = torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda")
    one = lambda k: dev(h[k][L:L + 1])
    qsa.qsa_decode(p, B, max_len, [L], kc, vc, ic, ring, wring, one("q"), one("k"), one("v"), one("q_idx"),
                   one("k_idx"), one("w"), out, ws=ws)
    torch.cuda.synchronize()
    assert qsa.qsa_check_device_error(ws) == 0
    check_outputs(out[0].cpu().numpy(), Q.bf16_to_f64(full["out"][L]), "yarn decode vs prefill")
    assert np.array_equal(kc[0, L].cpu().numpy(), full["k_rot"][L]), "appended key rotated like prefill's"
