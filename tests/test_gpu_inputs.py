"""The device fill of the input generator is bit-identical to the host fill
(so sampled full-size checks can regenerate any element on the host)."""
import numpy as np
import pytest
import torch

import qsa_inputs as Q

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,dist", [(4099, "uniform"), (8192, "zipf")])
def test_prefill_inputs_device_equals_host(T, dist):
    P = Q.PrefillProblem(T=T, seed=5, n_plant=8, dist=dist)
    d = P.device()
    h = P.host()
    for k in h:
        assert np.array_equal(d[k].cpu().numpy(), h[k]), k
    # row slices regenerate the same values
    assert np.array_equal(P.k_idx(1000, 1010), h["k_idx"][1000:1010])


def test_decode_caches_device_equals_host():
    D = Q.DecodeProblem(B=3, L=1000, steps=2, seed=9, n_plant=8)
    kc = torch.empty((3, 1010, 2, 256), dtype=torch.uint16, device="cuda")
    vc = torch.empty_like(kc)
    ic = torch.empty((3, 1010, 128), dtype=torch.uint16, device="cuda")
    D.fill_device_caches(kc, vc, ic)
    for b in range(3):
        assert np.array_equal(kc[b, :1000].cpu().numpy(), D.cache_k(b))
        assert np.array_equal(vc[b, :1000].cpu().numpy(), D.cache_v(b))
        assert np.array_equal(ic[b, :1000].cpu().numpy(), D.cache_kidx(b))


def test_device_rows_equal_host_rows():
    """Row ranges generated on the device (the profiling cases that never
    build the whole query tensor) equal the host generator's rows; the
    indexer keys there are the unplanted ones."""
    P = Q.PrefillProblem(T=9000, seed=6, n_plant=0)
    for name, (t0, t1) in (("q", (8000, 9000)), ("k", (0, 9000)), ("v", (123, 4567)), ("q_idx", (8192, 9000)),
                           ("w", (7, 8999)), ("k_idx", (0, 9000))):
        got = P.device_rows(name, t0, t1).cpu().numpy()
        want = getattr(P, name)(t0, t1)
        assert np.array_equal(got, want), name
