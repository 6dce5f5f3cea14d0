"""moe_router (router GEMM + routing in one kernel) on the GPU: the fp32 logits
against the oracle's float64 x W_r^T within the fp32 accumulation bound, and
the routing taken on the kernel's own fp32 logits (the precision the decision
is made in): indices bit-exact against the oracle's route() and bit-identical
to moe_route on the same logits, weights within 2e-6."""
import numpy as np
import pytest
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    # (T, H, E, k): the configs' router shapes, ragged token counts, E not a multiple of 16, E = 256, k = E
    (64, 128, 8, 2),
    (16, 2048, 60, 4),
    (8192, 2048, 128, 8),
    (4096, 7168, 256, 8),
    (300, 1024, 200, 6),
    (129, 64, 1, 1),
    (5, 256, 16, 16),
]


def _run(T, H, E, k, seed):
    wl = G.Workload("router", T, H, 128, E, k)
    x, _ = G.make_activations(wl, seed)
    w_r = G.make_router_weights(wl, seed, device="cuda")
    idx, w, lg = moe.router(x.cuda(), w_r, k, logits=True)
    torch.cuda.synchronize()
    return x, w_r, idx.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("T,H,E,k", CASES)
def test_router_matches_oracle(T, H, E, k):
    x, w_r, idx, w, lg = _run(T, H, E, k, seed=T + E)
    xf = x.float().numpy().astype(np.float64)
    wf = w_r.float().cpu().numpy().astype(np.float64)
    ref = O.router_logits(xf, wf)
    # fp32 accumulation over H products: error well under 1e-5 of sum |x w|
    bound = 1e-5 * (np.abs(xf) @ np.abs(wf).T) + 1e-6
    assert (np.abs(lg - ref) <= bound).all(), float(np.max(np.abs(lg - ref) / bound))
    ridx, rw, _ = O.route(lg, k)
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=0)
    # the same selection code as moe_route: identical bits on the same logits
    i2, w2 = moe.route(torch.from_numpy(lg).cuda(), k)
    torch.cuda.synchronize()
    assert np.array_equal(i2.cpu().numpy(), idx) and np.array_equal(w2.cpu().numpy(), w)


def test_router_without_logits_output():
    T, H, E, k = 256, 512, 64, 4
    x, w_r, idx, w, lg = _run(T, H, E, k, seed=3)
    idx2, w2 = moe.router(x.cuda(), w_r, k)
    torch.cuda.synchronize()
    assert np.array_equal(idx2.cpu().numpy(), idx) and np.array_equal(w2.cpu().numpy(), w)


def test_router_feeds_the_layer():
    """Router -> forward equals oracle router -> oracle forward (tiny layer)."""
    wl = G.WORKLOADS["tiny"]
    x, _ = G.make_activations(wl, 9)
    W = G.make_weights(wl, 9, device="cuda")
    w_r = G.make_router_weights(wl, 9, device="cuda")
    idx, w, lg = moe.router(x.cuda(), w_r, wl.k, logits=True)
    out, _ = moe.forward(x.cuda(), idx, w, W["w_gate_up"], W["w_down"])
    torch.cuda.synchronize()
    ridx, rw, _ = O.route(lg.cpu().numpy(), wl.k)
    from parity import ExpertView, assert_bf16_close
    ref = O.moe_forward(x.float().numpy(), ridx, rw, ExpertView(W["w_gate_up"]), ExpertView(W["w_down"]))
    assert_bf16_close(out.float().cpu().numpy(), ref, "router+forward")


def test_router_in_a_cuda_graph():
    """moe_router captured in a CUDA graph replays to the eager result."""
    T, H, E, k = 512, 1024, 64, 4
    wl = G.Workload("routergraph", T, H, 128, E, k)
    w_r = G.make_router_weights(wl, 2, device="cuda")
    x_static = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    moe.router(x_static, w_r, k)  # eager warm-up (one-time set-up outside the capture)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        idx_g, w_g = moe.router(x_static, w_r, k)
    for seed in (5, 6):
        x, _ = G.make_activations(wl, seed)
        x_static.copy_(x.cuda())
        g.replay()
        idx_e, w_e = moe.router(x.cuda(), w_r, k)
        torch.cuda.synchronize()
        assert torch.equal(idx_g, idx_e) and torch.equal(w_g, w_e)
