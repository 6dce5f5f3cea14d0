"""FP8 (e4m3 experts, UE8M0 128x128 weight scales, 1x128 fp32 activation
scales) on the GPU against the oracle: the quantised activations bit-exact,
h and the outputs within the FP8 tolerance, including edge counts and the
full-size layer on sampled tokens."""
import numpy as np
import pytest
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

from parity import (ExpertView, assert_fp8_close, check_permutation, device_inputs, oracle_forward_fp8, rel_fro)

pytestmark = pytest.mark.gpu


def _run(wl, seed, idx=None, w=None, path="auto"):
    x, L, W = device_inputs(wl, seed)
    if idx is None:
        idx, w, _ = O.route(L.numpy(), wl.k)
    out, ws = moe.forward(x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(), W["w_gate_up"],
                          W["w_down"], W["sw_gate_up"], W["sw_down"], path=path)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    return x, idx, w, W, out, ws


def _ws_bytes(ws, off, n):
    return ws[off:off + n].cpu().numpy()


def _ws_f32(ws, off, n):
    return ws[off:off + 4 * n].view(torch.float32).cpu().numpy()


@pytest.mark.parametrize("path", ["prefill", "decode"])
def test_small_fp8_layer_full_parity(path):
    wl = G.Workload("fp8small", 96, 512, 384, 8, 2, wdtype="e4m3")
    x, idx, w, W, out, ws = _run(wl, 4, path=path)
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e4m3", path)
    assert moe.workspace_layout(shape).path == moe.PATH[path]
    lay, perm = check_permutation(ws, shape, idx)
    rows = np.nonzero(perm["row_src"] >= 0)[0]
    a = perm["row_src"][rows]
    # quantised activations: codes and fp32 scales bit-exact; PREFILL stores
    # them per permuted row, DECODE once per token
    codes, scales, xdq = O.quantize_1x128(x.float().numpy()[a // wl.k])
    if path == "prefill":
        xq = _ws_bytes(ws, lay.xa, lay.m_rows * wl.H).reshape(lay.m_rows, wl.H)[rows]
        xs = _ws_f32(ws, lay.xs, lay.m_rows * wl.H // 128).reshape(lay.m_rows, -1)[rows]
    else:
        xq = _ws_bytes(ws, lay.xa, wl.T * wl.H).reshape(wl.T, wl.H)[a // wl.k]
        xs = _ws_f32(ws, lay.xs, wl.T * wl.H // 128).reshape(wl.T, -1)[a // wl.k]
    assert np.array_equal(xq, codes)
    assert np.array_equal(xs, scales)
    # h (dequantised) against the oracle's FP8 expert pieces
    hq = _ws_bytes(ws, lay.h, lay.m_rows * wl.I).reshape(lay.m_rows, wl.I)[rows]
    hs = _ws_f32(ws, lay.hs, lay.m_rows * wl.I // 128).reshape(lay.m_rows, -1)[rows]
    h_gpu = (O.e4m3_decode(hq).reshape(len(rows), -1, 128) * hs[:, :, None]).reshape(len(rows), -1)
    Vq, Vs = ExpertView(W["w_gate_up"], True), ExpertView(W["sw_gate_up"], True)
    e_of = idx.ravel()[a]
    h_ref = np.zeros_like(h_gpu)
    for e in np.unique(e_of):
        sel = e_of == e
        Wgu = O.dequantize_blocks(Vq[e], Vs[e])
        hh = (O.silu(xdq[sel] @ Wgu[:wl.I].T) * (xdq[sel] @ Wgu[wl.I:].T)).astype(np.float32)
        h_ref[sel] = O.quantize_1x128(hh)[2]
    assert rel_fro(h_gpu, h_ref) < 1e-2
    ref = oracle_forward_fp8(x, idx, w, W)
    r = assert_fp8_close(out.float().cpu().numpy(), ref, "fp8 small")
    assert r < 1e-2  # far inside the stated bound: both sides quantise the same way


DECODE_EDGE = [
    # (T, H, I, E, k, counts): empty experts, token groups of 1..4 and beyond, H not a multiple of 256
    (24, 384, 256, 8, 1, [0, 1, 4, 5, 9, 0, 3, 2]),
    (8, 256, 384, 4, 4, [8, 8, 8, 8]),  # k = E: every expert sees every token
    (1, 512, 128, 16, 3, [1, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 1]),
]


@pytest.mark.parametrize("T,H,I,E,k,counts", DECODE_EDGE)
def test_fp8_decode_edge_counts(T, H, I, E, k, counts):
    wl = G.Workload("fp8dec", T, H, I, E, k, wdtype="e4m3")
    idx, w = G.routed_inputs_with_counts(wl, counts, seed=T + 1)
    x, idx_np, w_np, W, out, ws = _run(wl, 7, idx.numpy(), w.numpy(), path="decode")
    check_permutation(ws, moe.make_shape(T, H, I, E, k, "e4m3", "decode"), idx_np)
    r = assert_fp8_close(out.float().cpu().numpy(), oracle_forward_fp8(x, idx_np, w_np, W), f"fp8 decode {counts}")
    assert r < 1e-2


def test_fp8_decode_full_size_sampled():
    """The FP8 decode-shaped layer (T=16, H=7168, I=2048, E=256, k=8) in the
    launch configuration the benchmark times (AUTO picks DECODE); the oracle
    computes a sample of tokens, the permutation is checked in full."""
    wl = G.WORKLOADS["fp8_decode"]
    seed = G.default_seed(wl)
    x, L, W = device_inputs(wl, seed)
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    out = layer(x.cuda(), L.cuda())
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, x.cuda().device)
    assert moe.read_device_status(ws) == 0
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e4m3")
    assert moe.workspace_layout(shape).path == moe.PATH["decode"]
    idx, w, _ = O.route(L.numpy(), wl.k)
    check_permutation(ws, shape, idx)
    toks = np.array([0, 7, 15])
    ref = oracle_forward_fp8(x, idx, w, W, tokens=toks)
    assert assert_fp8_close(out.float().cpu().numpy()[toks], ref, "fp8 decode full") < 1e-2
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("counts", [[0, 1, 127, 128, 129, 255, 256, 0], [300, 0, 0, 0, 0, 0, 0, 0]])
def test_fp8_edge_counts(counts):
    T = sum(counts)
    wl = G.Workload("fp8edge", T, 256, 256, 8, 1, wdtype="e4m3")
    idx, w = G.routed_inputs_with_counts(wl, counts, seed=1)
    x, idx_np, w_np, W, out, ws = _run(wl, 2, idx.numpy(), w.numpy())
    check_permutation(ws, moe.make_shape(T, 256, 256, 8, 1, "e4m3"), idx_np)
    assert_fp8_close(out.float().cpu().numpy(), oracle_forward_fp8(x, idx_np, w_np, W), f"fp8 {counts}")


def test_fp8_rejections():
    s = moe.make_shape(4, 128, 256, 4, 1, "e4m3", "prefill")  # H not a multiple of 256
    fake = 1 << 20
    import ctypes
    r = moe.lib().moe_forward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, fake, 1 << 40, None)
    assert r == -2


def test_fp8_full_size_sampled():
    wl = G.WORKLOADS["fp8"]
    seed = G.default_seed(wl)
    x, L, W = device_inputs(wl, seed)
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    out = layer(x.cuda(), L.cuda())
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, x.cuda().device)
    assert moe.read_device_status(ws) == 0
    idx, w, _ = O.route(L.numpy(), wl.k)
    check_permutation(ws, moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e4m3"), idx)
    toks = np.array([0, 1023, 2048, 4095])
    ref = oracle_forward_fp8(x, idx, w, W, tokens=toks)
    assert_fp8_close(out.float().cpu().numpy()[toks], ref, "fp8 full")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("path", ["prefill", "decode"])
@pytest.mark.parametrize("act", ["gelu", "relu"])
def test_fp8_gated_activations(act, path):
    wl = G.Workload("fp8act", 64, 256, 256, 8, 2, wdtype="e4m3")
    x, L, W = device_inputs(wl, 6)
    idx, w, _ = O.route(L.numpy(), wl.k)
    out, ws = moe.forward(x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(), W["w_gate_up"],
                          W["w_down"], W["sw_gate_up"], W["sw_down"], act=act, path=path)
    torch.cuda.synchronize()
    ref = O.moe_forward_fp8(x.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True),
                            ExpertView(W["sw_gate_up"], True), ExpertView(W["w_down"], True),
                            ExpertView(W["sw_down"], True), act=act)
    assert assert_fp8_close(out.float().cpu().numpy(), ref, f"fp8 {act}") < 1e-2


@pytest.mark.parametrize("T", [16, 300])
def test_fp8_graph_replay_matches_eager(T):
    """MoEGraph (route + forward in one CUDA graph) on FP8 experts, on the
    DECODE (T=16) and PREFILL (T=300) paths: bit-identical to eager calls."""
    wl = G.Workload("fp8graph", T, 512, 256, 16, 4, wdtype="e4m3")
    W = G.make_weights(wl, 0, device="cuda")
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    g = moe.MoEGraph(layer, wl.T)
    for seed in (31, 32):
        x, L = G.make_activations(wl, seed)
        got = g(x.cuda(), L.cuda()).clone()
        ref = layer(x.cuda(), L.cuda())
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
