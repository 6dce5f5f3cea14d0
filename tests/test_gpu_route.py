"""moe_route on the GPU against the oracle: indices bit-exact, weights to a few
fp32 ulps."""
import numpy as np
import pytest
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _route_both(L_np, k):
    Ld = torch.from_numpy(L_np).cuda()
    idx, w = moe.route(Ld, k)
    torch.cuda.synchronize()
    ridx, rw, _ = O.route(L_np, k)
    return idx.cpu().numpy(), w.cpu().numpy(), ridx, rw


@pytest.mark.parametrize("name", G.WORKLOAD_ORDER)
def test_route_workloads(name):
    wl = G.WORKLOADS[name]
    _, L = G.make_activations(wl, G.default_seed(wl))
    idx, w, ridx, rw = _route_both(L.numpy(), wl.k)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=0)
    np.testing.assert_allclose(w.astype(np.float64).sum(1), 1.0, atol=2e-6)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (37, 3, 2), (200, 32, 32), (129, 33, 5), (64, 256, 8),
                                   (50, 1024, 16), (300, 1000, 1), (5, 1024, 1024)])
def test_route_shapes_with_ties(T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    L = rng.integers(-2, 3, size=(T, E)).astype(np.float32)  # heavy ties
    L[0, :] = 0.0  # a fully tied row
    idx, w, ridx, rw = _route_both(L, k)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=0)


def test_route_empty_is_noop():
    L = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    idx, w = moe.route(L, 2)
    assert idx.shape == (0, 2)
