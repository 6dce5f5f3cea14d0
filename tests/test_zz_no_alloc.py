"""moe_forward_noalloc, the entry point for callers that cannot allocate device
memory (a plugin handed only its input and output buffers, or a serving path
that must not call cudaMalloc because it can synchronise the device). It runs
the forward with the library's own fixed scratch array; these tests call it
through the C ABI and compare it with moe_forward on a caller workspace.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

from parity import assert_bf16_close


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # host-side check, nothing is enqueued: the prefill-shaped layer needs far more than 8 MiB
    wl = G.WORKLOADS["prefill"]
    s = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k)
    assert moe.workspace_size(s) > 8 << 20
    fake = 1 << 20
    r = moe.lib().moe_forward_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, None, None, fake, None)
    assert r == -8 and "scratch" in moe.status_string(r)


def _inputs(wl, seed):
    x, L = G.make_activations(wl, seed)
    idx, w, _ = O.route(L.numpy(), wl.k)
    return x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("name,path", [("decode", "decode"), ("tiny", "prefill")])
def test_noalloc_matches_forward_on_two_calls(name, path):
    wl = G.WORKLOADS[name]
    W = G.make_weights(wl, G.default_seed(wl), device="cuda")
    for call, seed in enumerate((11, 12)):  # two calls in a row, different inputs
        x, idx, w = _inputs(wl, seed)
        got = moe.forward_noalloc(x, idx, w, W["w_gate_up"], W["w_down"], path=path)
        ref, _ = moe.forward(x, idx, w, W["w_gate_up"], W["w_down"], path=path)
        torch.cuda.synchronize()
        assert_bf16_close(got.float().cpu().numpy(), ref.float().cpu().numpy(), f"{name} call {call}")
        # same kernels on the same inputs: the results are in fact identical
        assert torch.equal(got, ref)
