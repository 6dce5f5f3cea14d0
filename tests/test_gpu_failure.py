"""Failure detection on the GPU without a fault: the gate/up GEMM's producer is
told to issue no loads, so the MMA issuer's bounded wait on its first stage
runs out. The call must come back within the short limit, the workspace's
status word must read MOE_ERR_DEVICE_TIMEOUT, and the next call on the same
context and workspace must run normally and match the oracle."""
import time

import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

import pytest
from parity import assert_bf16_close, device_inputs, oracle_forward_bf16

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms


def test_bounded_wait_gives_up_and_context_survives():
    wl = G.Workload("stall", 300, 256, 384, 8, 2)
    x, L, W = device_inputs(wl, 4)
    idx, w, _ = O.route(L.numpy(), wl.k)
    xd, idxd, wd = x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda()
    ref, ws = moe.forward(xd, idxd, wd, W["w_gate_up"], W["w_down"], path="prefill")  # also loads the kernels
    assert moe.read_device_status(ws) == 0
    assert_bf16_close(ref.float().cpu().numpy(), oracle_forward_bf16(x, idx, w, W), "before timeout")
    moe.set_test_hooks(stall_gate_up_loads=True, wait_limit_ns=LIMIT_NS)
    try:
        t0 = time.perf_counter()
        moe.forward(xd, idxd, wd, W["w_gate_up"], W["w_down"], path="prefill", workspace=ws)
        status = moe.read_device_status(ws)
        elapsed = time.perf_counter() - t0
    finally:
        moe.set_test_hooks(False, 0)
    assert status == -6, moe.status_string(status)
    assert elapsed < 1.0  # the 20 ms limit, not the 2 s default, ended the wait
    # the context and the workspace are still good: the next call gives the
    # same bits as the one before the timeout
    out, _ = moe.forward(xd, idxd, wd, W["w_gate_up"], W["w_down"], path="prefill", workspace=ws)
    assert moe.read_device_status(ws) == 0
    assert torch.equal(out, ref)
