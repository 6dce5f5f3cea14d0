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

from parity import (ExpertView, assert_fp8_close, assert_tokens_close, check_combine_bit_exact, check_permutation, device_topk_w,
                    device_inputs, oracle_forward_fp8, rel_fro)

# Per-token bound for FP8 layers: the layer's stated bound (3e-2 relative
# Frobenius) applied to every token on its own, so a localised error cannot
# hide in the norm over thousands of tokens.
FP8_TOKEN_REL_FRO = 3e-2

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


def test_fp8_decode_full_size_every_token():
    """The FP8 decode-shaped layer (T=16, H=7168, I=2048, E=256, k=8) in the
    launch configuration the benchmark times (AUTO picks DECODE): every token
    against the oracle, the permutation and the combine bit-exact."""
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
    check_combine_bit_exact(ws, shape, device_topk_w(L, wl.k, idx), out)
    ref = oracle_forward_fp8(x, idx, w, W, cache=False)
    got = out.float().cpu().numpy()
    assert assert_fp8_close(got, ref, "fp8 decode full") < 1e-2
    assert_tokens_close(got, ref, FP8_TOKEN_REL_FRO, "fp8 decode full")


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


def test_fp8_full_size_every_token():
    """The large FP8 layer (T=4096, H=7168, I=2048, E=256, k=8) in the launch
    configuration the benchmark times: every token against the oracle, as a
    whole and token by token; the permutation, the x codes and scales of every
    permuted row, and the combine bit-exact; the dequantised h of a block of
    experts against the oracle's FP8 expert pieces."""
    wl = G.WORKLOADS["fp8"]
    seed = G.default_seed(wl)
    x, L, W = device_inputs(wl, seed)
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    out = layer(x.cuda(), L.cuda())
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, x.cuda().device)
    assert moe.read_device_status(ws) == 0
    idx, w, _ = O.route(L.numpy(), wl.k)
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e4m3")
    lay, perm = check_permutation(ws, shape, idx)
    check_combine_bit_exact(ws, shape, device_topk_w(L, wl.k, idx), out)
    # x codes and scales: quantised once per token by the oracle, compared on every permuted row
    codes, scales, xdq = O.quantize_1x128(x.float().numpy())
    rows = np.nonzero(perm["row_src"] >= 0)[0]
    tok = perm["row_src"][rows] // wl.k
    G128 = wl.H // 128
    for r0 in range(0, rows.size, 4096):
        rr = torch.from_numpy(rows[r0:r0 + 4096].astype(np.int64)).cuda()
        xq = ws[lay.xa:lay.xa + lay.m_rows * wl.H].reshape(lay.m_rows, wl.H).index_select(0, rr).cpu().numpy()
        xs = ws[lay.xs:lay.xs + 4 * lay.m_rows * G128].view(torch.float32).reshape(lay.m_rows, G128)
        xs = xs.index_select(0, rr).cpu().numpy()
        assert np.array_equal(xq, codes[tok[r0:r0 + 4096]])
        assert np.array_equal(xs, scales[tok[r0:r0 + 4096]])
    # h of the first, a middle and the last expert
    Vq, Vs = ExpertView(W["w_gate_up"], True, False), ExpertView(W["sw_gate_up"], True, False)
    for e in (0, wl.E // 2, wl.E - 1):
        r0, c = int(perm["off"][e]), int(perm["cnt"][e])
        a = perm["row_src"][r0:r0 + c]
        hq = _ws_bytes(ws, lay.h + r0 * wl.I, c * wl.I).reshape(c, wl.I)
        hs = _ws_f32(ws, lay.hs + 4 * r0 * (wl.I // 128), c * (wl.I // 128)).reshape(c, -1)
        h_gpu = (O.e4m3_decode(hq).reshape(c, -1, 128) * hs[:, :, None]).reshape(c, -1)
        Wgu = O.dequantize_blocks(Vq[e], Vs[e])
        xe = xdq[a // wl.k]
        hh = (O.silu(xe @ Wgu[:wl.I].T) * (xe @ Wgu[wl.I:].T)).astype(np.float32)
        assert rel_fro(h_gpu, O.quantize_1x128(hh)[2]) < 1e-2, f"h of expert {e}"
    ref = oracle_forward_fp8(x, idx, w, W, cache=False)
    got = out.float().cpu().numpy()
    assert assert_fp8_close(got, ref, "fp8 full") < 1e-2
    assert_tokens_close(got, ref, FP8_TOKEN_REL_FRO, "fp8 full")


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
