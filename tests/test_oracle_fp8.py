"""Pins of the oracle's FP8 pieces: e4m3 encoding against hand-worked codes and
torch's float8_e4m3fn conversion, UE8M0 scales, block dequantisation against a
torch restatement, exact 1x128 quantisation on the e4m3 grid, and the FP8
forward against the unquantised forward (no GPU)."""
import numpy as np
import pytest
import torch

from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O


def test_e4m3_golden(golden):
    g = golden("e4m3_codes.json")
    for v, code in g["encode"]:
        assert int(O.e4m3_encode(np.array([v]))[0]) == code, v
    for b, s in g["ue8m0"]:
        assert O.ue8m0_scale(np.array([b]))[0] == s


def test_e4m3_matches_torch_cast():
    rng = np.random.default_rng(0)
    mags = np.concatenate([
        rng.uniform(0, 464, 100000), rng.uniform(0, 2.0 ** -6, 50000),
        np.exp2(rng.uniform(-12, 8.85, 100000)),
        O.e4m3_decode(np.arange(0, 127, dtype=np.uint8)),  # every finite code
    ])
    # every midpoint between neighbouring finite codes (ties)
    grid = O.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    mags = np.concatenate([mags, (grid[:-1] + grid[1:]) / 2])
    v = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    v = v[np.abs(v) <= 464]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn)
    assert np.array_equal(O.e4m3_encode(v.astype(np.float64)), ref.view(torch.uint8).numpy())
    assert np.array_equal(O.e4m3_round(v), ref.float().numpy().astype(np.float64))


def test_e4m3_saturates():
    v = np.array([448.0, 464.0, 470.0, 1e4, -500.0, -3e38])
    assert O.e4m3_round(v).tolist() == [448.0, 448.0, 448.0, 448.0, -448.0, -448.0]


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_block_dequantisation_matches_torch():
    wl = G.Workload("q", 4, 256, 384, 2, 1, wdtype="e4m3")
    W = G.make_weights(wl, 7)
    for name, sname in (("w_gate_up", "sw_gate_up"), ("w_down", "sw_down")):
        q, s = W[name], W[sname]
        ref = q.float().double() * torch.exp2(s.double() - 127).repeat_interleave(128, 1).repeat_interleave(128, 2)
        for e in range(wl.E):
            got = O.dequantize_blocks(q[e].view(torch.uint8).numpy(), s[e].numpy())
            assert np.array_equal(got, ref[e].numpy())


def test_quantize_1x128_exact_on_grid():
    rng = np.random.default_rng(1)
    R, C = 6, 512
    grid = O.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    q = rng.choice(grid, size=(R, C)) * rng.choice([-1, 1], size=(R, C))
    q.reshape(R, C // 128, 128)[:, :, 5] = 448.0  # every group reaches amax = 448 * 2^j
    j = rng.integers(-8, 8, size=(R, C // 128))
    a = (q.reshape(R, C // 128, 128) * np.exp2(j)[:, :, None]).reshape(R, C).astype(np.float32)
    a[2, 128:256] = 0.0  # an all-zero group
    codes, s, deq = O.quantize_1x128(a)
    expect_s = np.exp2(j).astype(np.float32)
    expect_s[2, 1] = 1.0
    assert np.array_equal(s, expect_s)
    assert np.array_equal(deq, a.astype(np.float64))
    assert (codes[2, 128:256] == 0).all()


def test_fp8_forward_without_activation_quant_equals_dequantised_bf16_forward():
    wl = G.Workload("q", 16, 256, 256, 4, 2, wdtype="e4m3")
    x, L = G.make_activations(wl, 3)
    W = G.make_weights(wl, 3)
    xn = x.float().numpy()
    idx, w, _ = O.route(L.numpy(), wl.k)
    u8 = lambda t: t.view(torch.uint8).numpy()
    deq = lambda q, s: (q.float().double() * torch.exp2(s.double() - 127)
                        .repeat_interleave(128, 1).repeat_interleave(128, 2)).numpy()
    wgu, wd = deq(W["w_gate_up"], W["sw_gate_up"]), deq(W["w_down"], W["sw_down"])
    a = O.moe_forward_fp8(xn, idx, w, u8(W["w_gate_up"]), W["sw_gate_up"].numpy(), u8(W["w_down"]),
                          W["sw_down"].numpy(), quantize_acts=False)
    b = O.moe_forward(xn, idx, w, wgu, wd, intermediate="exact")
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel < 4e-3  # only the fp32 h and bf16 y roundings differ
    # activation quantisation (x and h, each at most 2^-4 relative per code) is
    # present and stays inside twice the per-code bound
    c = O.moe_forward_fp8(xn, idx, w, u8(W["w_gate_up"]), W["sw_gate_up"].numpy(), u8(W["w_down"]),
                          W["sw_down"].numpy(), quantize_acts=True)
    rel_q = np.linalg.norm(c - b) / np.linalg.norm(b)
    assert 1e-2 < rel_q < 2 * 2.0 ** -4


def test_fp8_h_quantised_from_fp32_hand_worked(golden):
    """h is quantised 1x128 from its fp32 value (reading R7), not from a bf16
    copy: a hand-worked ReLU case where h = 1.064453125 rounds to e4m3 1.125,
    while its bf16 value 1.0625 is an exact e4m3 midpoint that rounds to 1.0."""
    c = golden("rounding_points.json")["fp8_h_from_fp32"]
    H, I = c["H"], c["I"]
    x = np.zeros((1, H))
    for col, v in c["x_nonzero"]:
        x[0, col] = v
    wgu = np.zeros((2 * I, H), dtype=np.uint8)
    for r, col, code in c["w_gate_up_codes"]:
        wgu[r, col] = code
    wd = np.zeros((H, I), dtype=np.uint8)
    for r, col, code in c["w_down_codes"]:
        wd[r, col] = code
    sgu = np.full((2 * I // 128, H // 128), c["scale_byte"], dtype=np.uint8)
    sd = np.full((H // 128, I // 128), c["scale_byte"], dtype=np.uint8)
    y = O.expert_mlp_fp8(x, wgu, sgu, wd, sd, act=c["act"])
    want = np.zeros((1, H))
    for col, v in c["y_nonzero"]:
        want[0, col] = v
    assert np.array_equal(y, want)
    assert y[0, 0] != c["y0_if_h_quantised_from_bf16"]
    # the h codes the hand derivation names, from the activation quantiser itself
    h = np.zeros((1, I), dtype=np.float32)
    h[0, 0], h[0, 1] = 448.0, 1.064453125
    codes, scales, _ = O.quantize_1x128(h)
    assert scales[0, 0] == 1.0
    assert [(int(i), int(codes[0, i])) for i in np.nonzero(codes[0])[0]] == [tuple(v) for v in c["h_codes_nonzero"]]
