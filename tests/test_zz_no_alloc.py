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


@pytest.mark.gpu
@pytest.mark.parametrize("wl,path", [
    (G.Workload("na_fp8_dec", 16, 512, 256, 8, 2, wdtype="e4m3"), "decode"),
    (G.Workload("na_fp8_pre", 64, 256, 256, 8, 2, wdtype="e4m3"), "prefill"),
])
def test_noalloc_fp8_matches_forward_on_two_calls(wl, path):
    """The e4m3 workspace layouts (x codes and scales, h codes and scales, the
    fp32 h of the DECODE path) inside the fixed scratch: identical results to
    moe_forward on a caller workspace, two calls in a row."""
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e4m3", path)
    assert moe.workspace_size(shape) <= 8 << 20
    W = G.make_weights(wl, 9, device="cuda")
    for call, seed in enumerate((13, 14)):
        x, idx, w = _inputs(wl, seed)
        got = moe.forward_noalloc(x, idx, w, W["w_gate_up"], W["w_down"], W["sw_gate_up"], W["sw_down"], path=path)
        ref, _ = moe.forward(x, idx, w, W["w_gate_up"], W["w_down"], W["sw_gate_up"], W["sw_down"], path=path)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"{wl.name} call {call}"
        assert moe.noalloc_device_status() == 0


@pytest.mark.gpu
def test_noalloc_reports_device_errors():
    """A routing index out of range reaches the caller through the status
    word in the scratch; the next good call clears it."""
    wl = G.Workload("na_bad", 40, 128, 128, 4, 2)
    W = G.make_weights(wl, 1, device="cuda")
    x, idx, w = _inputs(wl, 3)
    bad = idx.clone()
    bad[3, 1] = 4  # out of range: the permute rejects it without touching memory for it
    moe.forward_noalloc(x, bad, w, W["w_gate_up"], W["w_down"], path="decode")
    assert moe.noalloc_device_status() == -7
    moe.forward_noalloc(x, idx, w, W["w_gate_up"], W["w_down"], path="decode")
    assert moe.noalloc_device_status() == 0
