"""Failure handling of the device side, on the debug build (libqsa_debug.so:
bounds checks, a 20 ms limit on every bounded wait, and the test hooks of
include/qsa_debug.h).  No GPU fault is involved: a stall withholds one
completion signal inside a kernel, so a waiting role's bounded wait runs out,
the kernel records QSA_ERR_DEVICE_TIMEOUT, drains what it issued and exits; a
bad block index is reported by the bounds check before any access (and would
be masked by the causal test anyway).  After each, a normal call in the same
process must be correct: bit-identical to the release library's result."""
import numpy as np
import pytest
import torch

import block_sparse_long_qsa_b200 as qsa
import qsa_inputs as Q
from gpu_util import dev

pytestmark = pytest.mark.gpu

TIMEOUT, BOUNDS = 6, 7


@pytest.fixture(scope="module")
def libs():
    from block_sparse_long_qsa_b200 import _build
    _build.build()
    _build.build(debug=True)
    qsa.load()
    yield
    qsa.use_library(qsa.LIB_PATH)


def _with(path, fn):
    prev = qsa.use_library(path)
    try:
        return fn()
    finally:
        qsa.use_library(prev or qsa.LIB_PATH)


def _prefill(t, budget=64):
    r = qsa.prefill(t["q"], t["k"], t["v"], t["q_idx"], t["w"], t["k_idx"], budget=budget, want_krot=True)
    torch.cuda.synchronize()
    rc = qsa.qsa_check_device_error(r["ws"])
    return rc, {k: v.cpu() for k, v in r.items() if isinstance(v, torch.Tensor) and k != "ws"}


def _scores(T, t):
    nqb = (T + 3) // 4
    ld = (nqb + 3) // 4 * 4
    S = torch.zeros((nqb, ld), dtype=torch.float32, device="cuda")
    p = qsa.params()
    ws = qsa.workspace(qsa.qsa_index_workspace_size(p, T))
    qsa.qsa_index_scores(p, T, t["q_idx"], t["w"], t["k_idx"], 0, nqb, S, ld, ws)
    torch.cuda.synchronize()
    return qsa.qsa_check_device_error(ws), S.cpu()


@pytest.fixture(scope="module")
def problem():
    T = 2053
    P = Q.PrefillProblem(T=T, seed=91, n_plant=8)
    return T, {k: dev(v) for k, v in P.host().items()}


def test_debug_build_equals_release(libs, problem):
    """All bounds checks pass on a normal prefill and the debug build computes
    exactly what the release build does."""
    T, t = problem
    rc_r, rel = _prefill(t)
    rc_d, dbg = _with(qsa.LIB_DEBUG_PATH, lambda: _prefill(t))
    assert rc_r == 0 and rc_d == 0
    for k in rel:
        assert torch.equal(rel[k], dbg[k]), k


def test_indexer_wait_times_out_and_next_call_is_correct(libs, problem):
    T, t = problem
    _, want = _scores(T, t)

    def run():
        qsa.qsa_debug_inject(qsa.INJECT_INDEXER_STALL)
        rc1, _ = _scores(T, t)
        rc2, S2 = _scores(T, t)
        return rc1, rc2, S2
    rc1, rc2, S2 = _with(qsa.LIB_DEBUG_PATH, run)
    assert rc1 == TIMEOUT, f"stalled indexer: device status {rc1}, expected QSA_ERR_DEVICE_TIMEOUT"
    assert rc2 == 0
    causal = torch.tril(torch.ones(S2.shape[0], S2.shape[0], dtype=torch.bool))
    assert torch.equal(S2[:, :S2.shape[0]][causal], want[:, :want.shape[0]][causal])


def test_attention_wait_times_out_and_next_call_is_correct(libs, problem):
    T, t = problem
    _, want = _prefill(t)

    def run():
        qsa.qsa_debug_inject(qsa.INJECT_ATTENTION_STALL)
        rc1, _ = _prefill(t)
        rc2, got = _prefill(t)
        return rc1, rc2, got
    rc1, rc2, got = _with(qsa.LIB_DEBUG_PATH, run)
    assert rc1 == TIMEOUT, f"stalled attention: device status {rc1}, expected QSA_ERR_DEVICE_TIMEOUT"
    assert rc2 == 0
    for k in want:
        assert torch.equal(got[k], want[k]), k


def test_bounds_check_reports_non_causal_block(libs, problem):
    T, t = problem
    _, want = _prefill(t)

    def run():
        qsa.qsa_debug_inject(qsa.INJECT_ATTENTION_BAD_BLOCK)
        rc1, _ = _prefill(t)
        rc2, got = _prefill(t)
        return rc1, rc2, got
    rc1, rc2, got = _with(qsa.LIB_DEBUG_PATH, run)
    assert rc1 == BOUNDS, f"bad block: device status {rc1}, expected QSA_ERR_DEVICE_BOUNDS"
    assert rc2 == 0
    assert torch.equal(got["out"], want["out"])


def test_attention_rescale_on_every_tile(libs):
    """The online softmax's rescale of the accumulated output (taken only when
    a tile's maximum exceeds the running one by more than 2^8, which unit-scale
    inputs almost never reach) forced on every tile by the debug hook, in a
    prefill with 32-tile rows and in a decode step: the outputs stay within the
    acceptance bounds of the oracle (prefill, on the GPU's own selection) and
    of the normal run (decode)."""
    import oracle
    from gpu_util import check_outputs
    from test_gpu_decode import DecodeState
    T, budget = 4096, 512
    P = Q.PrefillProblem(T=T, seed=93, n_plant=8)
    host = P.host()
    t = {k: dev(v) for k, v in host.items()}

    def run():
        qsa.qsa_debug_inject(qsa.INJECT_ATTENTION_RESCALE_ALL)
        return _prefill(t, budget)
    rc, got = _with(qsa.LIB_DEBUG_PATH, run)
    assert rc == 0
    out, sel, cnt = got["out"].numpy(), got["sel"].numpy(), got["cnt"].numpy()
    nqb = P.nqb
    qbs = np.array(sorted({0, 1, budget - 1, budget, nqb - 1} | set(range(530, nqb, 41))), dtype=np.int64)
    O = oracle.Oracle(oracle.params(budget=budget))
    want, _ = O.attend_blocks(T, host["q"], host["k"], host["v"], qbs, sel[qbs], cnt[qbs])
    rows = np.concatenate([np.arange(4 * q, min(4 * q + 4, T)) for q in qbs])
    check_outputs(out[rows], want[:len(rows)], "prefill, rescale on every tile")

    L_list = [2301, 4097]
    probs = [Q.PrefillProblem(T=L + 1, seed=95 + b, n_plant=8) for b, L in enumerate(L_list)]

    def step(inject):
        st = DecodeState(probs, L_list, max_len=max(L_list) + 8, budget=budget)
        if inject:
            qsa.qsa_debug_inject(qsa.INJECT_ATTENTION_RESCALE_ALL)
        return st.step()
    _, o_ref, s_ref, _ = step(False)
    _, o_dbg, s_dbg, _ = _with(qsa.LIB_DEBUG_PATH, lambda: step(True))
    assert np.array_equal(s_ref, s_dbg)
    for b in range(len(L_list)):
        check_outputs(o_dbg[b], Q.bf16_to_f64(o_ref[b]), f"decode b={b}, rescale on every tile")


def test_release_library_has_no_hooks(libs):
    with pytest.raises(RuntimeError):
        qsa.qsa_debug_inject(qsa.INJECT_INDEXER_STALL)
