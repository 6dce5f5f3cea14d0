"""FP4 (e2m1) experts on the GPU against the oracle: packed e2m1 weights with
one UE8M0 scale per row and 32 elements, bf16 activations. The layer is the
bf16 layer on the dequantised weights, so the bf16 tolerances apply; the
permutation and the combine are bit-exact."""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

from parity import (ExpertView, assert_bf16_close, assert_tokens_close, check_combine_bit_exact, check_permutation, device_topk_w,
                    device_inputs, ws_bf16)

pytestmark = pytest.mark.gpu

TOKEN_REL_FRO = 2e-2  # per-token bound, as for the bf16 layers


def oracle_fp4(x, idx, w, W, tokens=None, cache=True):
    return O.moe_forward_fp4(x.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True, cache),
                             ExpertView(W["sw_gate_up"], True, cache), ExpertView(W["w_down"], True, cache),
                             ExpertView(W["sw_down"], True, cache), tokens=tokens)


def _run(wl, seed, idx=None, w=None, path="auto", act="silu"):
    x, L, W = device_inputs(wl, seed)
    if idx is None:
        idx, w, _ = O.route(L.numpy(), wl.k)
    out, ws = moe.forward(x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(), W["w_gate_up"],
                          W["w_down"], W["sw_gate_up"], W["sw_down"], path=path, act=act)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    return x, idx, w, W, out, ws


@pytest.mark.parametrize("act", ["silu", "gelu", "relu"])
def test_small_fp4_decode_layer(act):
    wl = G.Workload("fp4small", 24, 512, 384, 8, 2, wdtype="e2m1")
    x, idx, w, W, out, ws = _run(wl, 4, path="decode", act=act)
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1", "decode")
    check_permutation(ws, shape, idx)
    check_combine_bit_exact(ws, shape, w, out)
    ref = O.moe_forward_fp4(x.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True),
                            ExpertView(W["sw_gate_up"], True), ExpertView(W["w_down"], True),
                            ExpertView(W["sw_down"], True), act=act)
    assert_bf16_close(out.float().cpu().numpy(), ref, f"fp4 {act}")


FP4_DECODE_EDGE = [
    # (T, H, I, E, k, counts): empty experts, 1, 2 and 3 tokens per expert (token pairs and a tail), k = E
    (12, 256, 128, 8, 1, [0, 1, 2, 3, 0, 5, 1, 0]),
    (6, 128, 256, 4, 4, [6, 6, 6, 6]),
    (1, 384, 128, 16, 3, [1, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 1]),
]


@pytest.mark.parametrize("T,H,I,E,k,counts", FP4_DECODE_EDGE)
def test_fp4_decode_edge_counts(T, H, I, E, k, counts):
    wl = G.Workload("fp4edge", T, H, I, E, k, wdtype="e2m1")
    idx, w = G.routed_inputs_with_counts(wl, counts, seed=T + 3)
    x, idx_np, w_np, W, out, ws = _run(wl, 8, idx.numpy(), w.numpy(), path="decode")
    shape = moe.make_shape(T, H, I, E, k, "e2m1", "decode")
    check_permutation(ws, shape, idx_np)
    check_combine_bit_exact(ws, shape, w_np, out)
    assert_bf16_close(out.float().cpu().numpy(), oracle_fp4(x, idx_np, w_np, W), f"fp4 decode {counts}")


def test_fp4_decode_full_size_every_token():
    """The large layer's shape with FP4 experts at decode size (T=16, H=7168,
    I=2048, E=256, k=8), in the launch configuration the benchmark times:
    every token against the oracle, the permutation and combine bit-exact."""
    wl = G.WORKLOADS["fp4_decode"]
    x, L, W = device_inputs(wl, G.default_seed(wl))
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    out = layer(x.cuda(), L.cuda())
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, x.cuda().device)
    assert moe.read_device_status(ws) == 0
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1")
    assert moe.workspace_layout(shape).path == moe.PATH["decode"]
    idx, w, _ = O.route(L.numpy(), wl.k)
    check_permutation(ws, shape, idx)
    check_combine_bit_exact(ws, shape, device_topk_w(L, wl.k, idx), out)
    ref = oracle_fp4(x, idx, w, W, cache=False)
    got = out.float().cpu().numpy()
    assert_bf16_close(got, ref, "fp4 decode full")
    assert_tokens_close(got, ref, TOKEN_REL_FRO, "fp4 decode full")


@pytest.mark.parametrize("act", ["silu", "gelu", "relu"])
def test_small_fp4_prefill_layer(act):
    """The PREFILL path (codes widened to bf16 in shared memory, tcgen05 bf16
    MMAs): several row blocks per expert and a ragged last block; h and y of
    every row against the oracle's expert MLP on the dequantised weights."""
    wl = G.Workload("fp4pre", 300, 512, 384, 8, 2, wdtype="e2m1")
    x, idx, w, W, out, ws = _run(wl, 5, path="prefill", act=act)
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1", "prefill")
    lay, perm = check_permutation(ws, shape, idx)
    check_combine_bit_exact(ws, shape, w, out)
    ref = O.moe_forward_fp4(x.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True),
                            ExpertView(W["sw_gate_up"], True), ExpertView(W["w_down"], True),
                            ExpertView(W["sw_down"], True), act=act)
    assert_bf16_close(out.float().cpu().numpy(), ref, f"fp4 prefill {act}")
    if act == "silu":
        check_h_y(ws, lay, perm, x, idx, W, wl, "fp4 prefill")


def check_h_y(ws, lay, perm, x, idx, W, wl, what, act="silu"):
    """h and y of every permuted row against the oracle's expert MLP on the
    dequantised weights."""
    rows = np.nonzero(perm["row_src"] >= 0)[0]
    h = ws_bf16(ws, lay.h, lay.m_rows, wl.I)[rows]
    y = ws_bf16(ws, lay.y, lay.m_rows, wl.H)[rows]
    a = perm["row_src"][rows]
    xr = x.float().numpy()[a // wl.k]
    e_of = idx.ravel()[a]
    href, yref = np.zeros_like(h, dtype=np.float64), np.zeros_like(y, dtype=np.float64)
    for e in np.unique(e_of):
        sel = e_of == e
        Wgu = O.dequantize_fp4(W["w_gate_up"][e].cpu().numpy(), W["sw_gate_up"][e].cpu().numpy())
        Wd = O.dequantize_fp4(W["w_down"][e].cpu().numpy(), W["sw_down"][e].cpu().numpy())
        href[sel], yref[sel] = O.expert_mlp(xr[sel].astype(np.float64), Wgu, Wd, "bf16", act=act)
    assert_bf16_close(h, href, f"{what} h")
    assert_bf16_close(y, yref, f"{what} y")


@pytest.mark.parametrize("counts", [[0, 1, 127, 128, 129, 255, 256, 257, 300, 15], [16, 0, 130, 0]])
def test_fp4_decode_path_many_tokens(counts):
    """The DECODE path with many tokens per expert (its kernels take an
    expert's tokens four at a time, so every tail length shows up): 0, 1,
    127..129, 255..257 and 300 tokens; h and y of every row against the oracle."""
    T = sum(counts)
    wl = G.Workload("fp4many", T, 256, 384, len(counts), 1, wdtype="e2m1")
    idx, w = G.routed_inputs_with_counts(wl, counts, seed=11)
    x, idx_np, w_np, W, out, ws = _run(wl, 9, idx.numpy(), w.numpy(), path="decode")
    shape = moe.make_shape(T, wl.H, wl.I, wl.E, 1, "e2m1", "decode")
    lay, perm = check_permutation(ws, shape, idx_np)
    check_combine_bit_exact(ws, shape, w_np, out)
    assert_bf16_close(out.float().cpu().numpy(), oracle_fp4(x, idx_np, w_np, W), f"fp4 decode {counts}")
    check_h_y(ws, lay, perm, x, idx_np, W, wl, f"fp4 decode {counts}")


@pytest.mark.parametrize("path", ["decode", "prefill"])
@pytest.mark.parametrize("which,shift,bvals", [("sw_gate_up", 100, (2, 3, 4)),
                                               ("sw_gate_up", -18, (140, 141, 142, 143, 144, 145)),
                                               ("sw_down", 0, (140, 141, 142, 143, 144, 145))])
def test_fp4_scale_bytes_at_the_widening_edges(path, which, shift, bvals):
    """Scale bytes far from those of N(0, 0.02) weights, small (2..4) and large
    (140..145), on both paths: every weight must act as e2m1 * 2^(b-127)
    exactly. x is scaled by 2^shift (exact in bf16) so every product and sum
    stays a normal fp32 number; h and y of every row against the oracle."""
    wl = G.Workload("fp4edge_scales", 40, 256, 256, 4, 2, wdtype="e2m1")
    x, L, W = device_inputs(wl, 6)
    x = (x.float() * 2.0 ** shift).to(torch.bfloat16)
    rng = np.random.default_rng(abs(shift) + len(bvals))
    W[which] = torch.from_numpy(rng.choice(np.array(bvals, dtype=np.uint8), size=tuple(W[which].shape))).to(
        W[which].device)
    idx, w, _ = O.route(L.numpy(), wl.k)
    out, ws = moe.forward(x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda(), W["w_gate_up"],
                          W["w_down"], W["sw_gate_up"], W["sw_down"], path=path)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1", path)
    lay, perm = check_permutation(ws, shape, idx)
    assert_bf16_close(out.float().cpu().numpy(), oracle_fp4(x, idx, w, W), f"fp4 scales {which} {bvals}")
    check_h_y(ws, lay, perm, x, idx, W, wl, f"fp4 scales {which} {bvals}")


@pytest.mark.parametrize("counts", [[0, 1, 127, 128, 129, 255, 256, 0], [300, 0, 0, 0, 0, 0, 0, 0]])
def test_fp4_prefill_edge_counts(counts):
    T = sum(counts)
    wl = G.Workload("fp4edge", T, 256, 256, 8, 1, wdtype="e2m1")
    idx, w = G.routed_inputs_with_counts(wl, counts, seed=2)
    x, idx_np, w_np, W, out, ws = _run(wl, 3, idx.numpy(), w.numpy(), path="prefill")
    shape = moe.make_shape(T, 256, 256, 8, 1, "e2m1", "prefill")
    check_permutation(ws, shape, idx_np)
    check_combine_bit_exact(ws, shape, w_np, out)
    assert_bf16_close(out.float().cpu().numpy(), oracle_fp4(x, idx_np, w_np, W), f"fp4 prefill {counts}")


def test_fp4_full_size_every_token():
    """The large layer's shape with FP4 experts (T=4096, H=7168, I=2048, E=256,
    k=8) in the launch configuration the benchmark times (the AUTO path), and
    the same routing through the other path: every token against the oracle,
    as a whole and token by token; permutation and combine bit-exact."""
    wl = G.WORKLOADS["fp4"]
    x, L, W = device_inputs(wl, G.default_seed(wl))
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    out = layer(x.cuda(), L.cuda())
    torch.cuda.synchronize()
    ws = layer._workspace(wl.T, x.cuda().device)
    assert moe.read_device_status(ws) == 0
    shape = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1")
    auto = moe.workspace_layout(shape).path
    idx, w, _ = O.route(L.numpy(), wl.k)
    check_permutation(ws, shape, idx)
    w_dev = device_topk_w(L, wl.k, idx)
    check_combine_bit_exact(ws, shape, w_dev, out)
    ref = oracle_fp4(x, idx, w, W, cache=False)
    got = out.float().cpu().numpy()
    assert_bf16_close(got, ref, "fp4 full")
    assert_tokens_close(got, ref, TOKEN_REL_FRO, "fp4 full")
    other = "prefill" if auto == moe.PATH["decode"] else "decode"
    out2, ws2 = moe.forward(x.cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(w_dev).cuda(), W["w_gate_up"],
                            W["w_down"], W["sw_gate_up"], W["sw_down"], path=other)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws2) == 0
    shape2 = moe.make_shape(wl.T, wl.H, wl.I, wl.E, wl.k, "e2m1", other)
    check_permutation(ws2, shape2, idx)
    check_combine_bit_exact(ws2, shape2, w_dev, out2)
    got2 = out2.float().cpu().numpy()
    assert_bf16_close(got2, ref, f"fp4 full {other}")
    assert_tokens_close(got2, ref, TOKEN_REL_FRO, f"fp4 full {other}")


@pytest.mark.parametrize("T", [16, 300])
def test_fp4_graph_replay_matches_eager(T):
    wl = G.Workload("fp4graph", T, 512, 256, 16, 4, wdtype="e2m1")
    W = G.make_weights(wl, 0, device="cuda")
    layer = moe.MoELayer(W["w_gate_up"], W["w_down"], wl.k, W["sw_gate_up"], W["sw_down"])
    g = moe.MoEGraph(layer, wl.T)
    for seed in (51, 52):
        x, L = G.make_activations(wl, seed)
        got = g(x.cuda(), L.cuda()).clone()
        ref = layer(x.cuda(), L.cuda())
        torch.cuda.synchronize()
        assert torch.equal(got, ref)


def test_fp4_host_errors():
    s = moe.make_shape(4, 128, 128, 4, 1, "e2m1", "decode")
    fake = 1 << 20
    # FP4 experts without their UE8M0 scales are refused
    assert moe.lib().moe_forward(ctypes.byref(s), fake, fake, fake, fake, fake, None, None, fake, fake, 1 << 40,
                                 None) == -3
    # PREFILL with H not a multiple of 256: refused before any launch
    s = moe.make_shape(300, 384, 128, 4, 1, "e2m1", "prefill")
    assert moe.lib().moe_forward(ctypes.byref(s), fake, fake, fake, fake, fake, fake, fake, fake, fake, 1 << 40,
                                 None) == -2
