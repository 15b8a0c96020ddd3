"""qsa_decode_noalloc (decode with the library's fixed scratch array, for
callers that cannot allocate device memory on their decode path) against
qsa_decode with a caller-provided workspace, through the C ABI, on two
consecutive decode calls.  Collected last on purpose; self-contained so it
also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import qsa_inputs as Q
from gpu_util import OUT_MAX_ABS, OUT_REL_L2

pytestmark = pytest.mark.gpu


def _caches(B, max_len, D):
    kc = torch.zeros((B, max_len, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.zeros_like(kc)
    ic = torch.zeros((B, max_len, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    ring = torch.zeros((B, 4, 4, 128), dtype=torch.uint16, device="cuda")
    wring = torch.zeros((B, 4, 4), dtype=torch.uint16, device="cuda")
    return [kc, vc, ic, ring, wring]


def test_decode_noalloc_matches_workspace_decode():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    qsa.load()
    B, L, budget = 3, 2401, 512
    max_len = L + 8
    D = Q.DecodeProblem(B=B, L=L, steps=2, seed=77, n_plant=8)
    p = qsa.params(budget)
    a = _caches(B, max_len, D)                 # caches of the workspace path
    b = [t.clone() for t in a]                 # identical caches for the no-alloc path
    ws = qsa.workspace(qsa.qsa_decode_workspace_size(p, B, max_len))
    seqs = [D.tokens(i) for i in range(B)]
    # every tensor of both calls exists before the first no-alloc call, so
    # nothing in between can allocate device memory
    xs, outs = [], []
    for s in range(2):
        t = L + s
        xs.append({k: torch.from_numpy(np.ascontiguousarray(np.stack([getattr(seqs[i], k)(t, t + 1)[0]
                                                                       for i in range(B)]))).cuda()
                   for k in ("q", "k", "v", "q_idx", "k_idx", "w")})
        outs.append(dict(out_ws=torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda"),
                         out_na=torch.empty((B, 24, 256), dtype=torch.uint16, device="cuda"),
                         sel_ws=torch.empty((B, budget), dtype=torch.int32, device="cuda"),
                         sel_na=torch.empty((B, budget), dtype=torch.int32, device="cuda"),
                         lse_ws=torch.empty((B, 24), dtype=torch.float32, device="cuda"),
                         lse_na=torch.empty((B, 24), dtype=torch.float32, device="cuda")))
    torch.cuda.synchronize()
    free_after_first = None
    for s in range(2):                         # two calls in a row
        t = L + s
        x, o = xs[s], outs[s]
        qsa.qsa_decode(p, B, max_len, [t] * B, *a, x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["w"],
                       o["out_ws"], o["sel_ws"], o["lse_ws"], ws)
        qsa.qsa_decode_noalloc(p, B, max_len, [t] * B, *b, x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["w"],
                               o["out_na"], o["sel_na"], o["lse_na"])
        torch.cuda.synchronize()
        free_now, _ = torch.cuda.mem_get_info()
        if s == 0:
            free_after_first = free_now          # the first call may map the fixed array
        else:
            assert free_now == free_after_first, "the second no-alloc call changed free device memory"
        assert qsa.qsa_check_device_error(ws) == 0
        assert qsa.qsa_decode_noalloc_check_error() == 0
        # the same kernels with the same split on the same inputs: identical
        assert torch.equal(o["sel_ws"], o["sel_na"])
        assert torch.equal(o["out_ws"], o["out_na"])
        assert torch.equal(o["lse_ws"], o["lse_na"])
        # and within the tolerance the other tests use (a non-empty output)
        g = Q.bf16_to_f64(o["out_na"].cpu().numpy())
        w = Q.bf16_to_f64(o["out_ws"].cpu().numpy())
        assert np.abs(g - w).max() <= OUT_MAX_ABS
        assert np.linalg.norm(g - w) <= OUT_REL_L2 * np.linalg.norm(w)
        assert np.linalg.norm(w) > 0
    for ta, tb in zip(a, b):                   # both paths appended the same tokens
        assert torch.equal(ta, tb)


def test_decode_noalloc_rejects_oversize():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    p = qsa.params(512)
    dummy = torch.zeros(16, dtype=torch.uint16, device="cuda")
    with pytest.raises(qsa.QSAError) as e:
        # 4096 sequences at 1M context need far more than the fixed scratch
        qsa.qsa_decode_noalloc(p, 4096, 1 << 20, [0] * 4096, *([dummy] * 11), dummy)
    assert e.value.status == 4
