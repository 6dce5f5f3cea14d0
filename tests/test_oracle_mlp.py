"""Pins of the oracle's expert MLP and eager forward: a hand-worked closed form,
a dense single-expert MLP computed with torch's own silu, an independent
per-assignment batched formulation, invariances, and bf16 rounding against
torch's conversion (no GPU)."""
import numpy as np
import pytest
import torch

from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([(rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000)).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, 1e-40], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = O.bf16_round(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_closed_form_single_expert(golden):
    g = golden("mlp_closed_form.json")
    H, I = g["H"], g["I"]
    wgu = np.zeros((1, 2 * I, H))
    wgu[0, :I, 0] = g["gate_col0"]
    wgu[0, I:, 0] = g["up_col0"]
    wd = np.array(g["w_down"])[None]
    x = np.array([g["x"]])
    h, y = O.expert_mlp(x, wgu[0], wd[0], intermediate="none")
    np.testing.assert_allclose(h[0], g["h"], rtol=1e-14, atol=1e-14)
    out = O.moe_forward(x, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32), wgu, wd,
                        intermediate="none")
    np.testing.assert_allclose(out[0], g["out"], rtol=1e-14, atol=1e-14)


def _torch_dense_swiglu(x, wg, wu, wd):
    X = torch.from_numpy(x)
    return (torch.nn.functional.silu(X @ torch.from_numpy(wg).T) * (X @ torch.from_numpy(wu).T)) \
        @ torch.from_numpy(wd).T


def test_single_expert_reduces_to_dense_mlp():
    rng = np.random.default_rng(3)
    T, H, I = 17, 64, 96
    x = rng.standard_normal((T, H))
    wgu = rng.standard_normal((1, 2 * I, H)) * 0.1
    wd = rng.standard_normal((1, H, I)) * 0.1
    out = O.moe_forward(x, np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32), wgu, wd,
                        intermediate="none")
    ref = _torch_dense_swiglu(x, wgu[0, :I], wgu[0, I:], wd[0]).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def _batched_formulation(x, idx, w, wgu, wd):
    """Per-assignment form of the page's batched_mm backend: gather each
    assignment's expert parameters, run all assignments in one batched matmul."""
    T, k = idx.shape
    I = wgu.shape[1] // 2
    xi = torch.from_numpy(np.repeat(x, k, axis=0))[:, None, :]  # [A,1,H]
    W = torch.from_numpy(wgu)[torch.from_numpy(idx.ravel().astype(np.int64))]  # [A,2I,H]
    gu = torch.bmm(xi, W.transpose(1, 2))[:, 0]  # [A,2I]
    h = torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]
    D = torch.from_numpy(wd)[torch.from_numpy(idx.ravel().astype(np.int64))]  # [A,H,I]
    y = torch.bmm(h[:, None, :], D.transpose(1, 2))[:, 0].reshape(T, k, -1)
    return (torch.from_numpy(w.astype(np.float64))[:, :, None] * y).sum(1).numpy()


@pytest.mark.parametrize("T,H,I,E,k", [(9, 32, 48, 5, 2), (33, 64, 32, 8, 3), (20, 16, 16, 4, 4)])
def test_eager_loop_matches_batched_formulation(T, H, I, E, k):
    rng = np.random.default_rng(T)
    x = rng.standard_normal((T, H))
    L = rng.standard_normal((T, E), dtype=np.float32)
    idx, w, _ = O.route(L, k)
    wgu = rng.standard_normal((E, 2 * I, H)) * 0.1
    wd = rng.standard_normal((E, H, I)) * 0.1
    out = O.moe_forward(x, idx, w, wgu, wd, intermediate="none")
    ref = _batched_formulation(x, idx, w, wgu, wd)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_output_invariant_under_token_permutation():
    wl = G.Workload("t", 48, 128, 128, 6, 2)
    x, L = G.make_activations(wl, 5)
    W = G.make_weights(wl, 5)
    xn = x.float().numpy()
    wgu, wd = W["w_gate_up"].float().numpy(), W["w_down"].float().numpy()
    idx, w, _ = O.route(L.numpy(), wl.k)
    out = O.moe_forward(xn, idx, w, wgu, wd)
    perm = np.random.default_rng(0).permutation(wl.T)
    idx2, w2, _ = O.route(L.numpy()[perm], wl.k)
    out2 = O.moe_forward(xn[perm], idx2, w2, wgu, wd)
    assert np.array_equal(out[perm], out2)
    # a token subset gives the same rows as the full computation
    sub = np.array([3, 17, 40])
    assert np.array_equal(O.moe_forward(xn, idx, w, wgu, wd, tokens=sub), out[sub])


def test_bf16_intermediates_close_to_exact():
    wl = G.WORKLOADS["tiny"]
    x, L = G.make_activations(wl, 0)
    W = G.make_weights(wl, 0)
    xn = x.float().numpy()
    wgu, wd = W["w_gate_up"].float().numpy(), W["w_down"].float().numpy()
    idx, w, _ = O.route(L.numpy(), wl.k)
    a = O.moe_forward(xn, idx, w, wgu, wd, intermediate="bf16")
    b = O.moe_forward(xn, idx, w, wgu, wd, intermediate="none")
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-4 < rel < 5e-3  # rounding is present, and small


def test_planted_mistakes_are_caught(golden):
    """A swapped gate/up or a dropped up projection breaks the closed-form case
    (a transposed down matrix cannot even be applied, since H != I there)."""
    g = golden("mlp_closed_form.json")
    H, I = g["H"], g["I"]
    wg = np.zeros((I, H)); wg[:, 0] = g["gate_col0"]
    wu = np.zeros((I, H)); wu[:, 0] = g["up_col0"]
    wd = np.array(g["w_down"])
    x = np.array([g["x"]])
    right = (O.silu(x @ wg.T) * (x @ wu.T)) @ wd.T
    swapped = (O.silu(x @ wu.T) * (x @ wg.T)) @ wd.T
    dropped = O.silu(x @ wg.T) @ wd.T
    np.testing.assert_allclose(right[0], g["out"], rtol=1e-14, atol=1e-14)
    for bad in (swapped, dropped):
        assert not np.allclose(bad[0], g["out"])


def test_gated_activations_match_torch():
    z = np.linspace(-12, 12, 20001)
    t = torch.from_numpy(z)
    np.testing.assert_allclose(O.silu(z), torch.nn.functional.silu(t).numpy(), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(O.gelu(z), torch.nn.functional.gelu(t).numpy(), rtol=1e-13, atol=1e-15)
    assert np.array_equal(O.relu(z), torch.relu(t).numpy())
    # closed forms: gelu(0) = 0, gelu(x) -> x for large x, Phi(1) = (1 + erf(1/sqrt 2)) / 2
    assert O.gelu(0.0) == 0.0 and abs(O.gelu(40.0) - 40.0) < 1e-12
    assert abs(O.gelu(1.0) - 0.8413447460685429) < 1e-15
    assert O.relu(-1.0) == 0.0 and O.relu(2.5) == 2.5


@pytest.mark.parametrize("act", ["gelu", "relu"])
def test_gated_activation_forward_matches_batched(act):
    rng = np.random.default_rng(9)
    T, H, I, E, k = 12, 32, 48, 5, 2
    x = rng.standard_normal((T, H))
    L = rng.standard_normal((T, E), dtype=np.float32)
    idx, w, _ = O.route(L, k)
    wgu = rng.standard_normal((E, 2 * I, H)) * 0.2
    wd = rng.standard_normal((E, H, I)) * 0.2
    out = O.moe_forward(x, idx, w, wgu, wd, intermediate="none", act=act)
    f = torch.nn.functional.gelu if act == "gelu" else torch.relu
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            xt = torch.from_numpy(x[t])
            h = f(torch.from_numpy(wgu[e, :I]) @ xt) * (torch.from_numpy(wgu[e, I:]) @ xt)
            ref[t] += float(w[t, j]) * (torch.from_numpy(wd[e]) @ h).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_bf16_rounding_points_hand_worked(golden):
    """h is rounded to bf16 before the down projection and y is rounded to
    bf16 (reading R4): a hand-worked ReLU case whose exact values sit so that
    dropping either rounding, or moving it, changes y."""
    c = golden("rounding_points.json")["bf16_intermediates"]
    x = np.array(c["x"], dtype=np.float64)
    wgu = np.array(c["w_gate_up"], dtype=np.float64)
    wd = np.array(c["w_down"], dtype=np.float64)
    h, y = O.expert_mlp(x, wgu, wd, "bf16", act=c["act"])
    assert np.array_equal(h, np.array(c["h"]))
    assert np.array_equal(y, np.array(c["y"]))
    # the case separates the readings: each wrong rounding point gives another y
    assert not np.array_equal(np.array(c["y"]), np.array(c["y_if_h_not_rounded"]))
    assert not np.array_equal(np.array(c["y"]), np.array(c["y_if_y_not_rounded"]))
    # "exact" mode (no intermediate rounding) lands on neither rounded value
    _, y_exact = O.expert_mlp(x, wgu, wd, "exact", act=c["act"])
    assert y_exact[0, 0] != c["y"][0][0]
    # through the whole layer (E=1, k=1, w=1): the output is bf16(y) = y
    out = O.moe_forward(x, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32), wgu[None], wd[None],
                        act=c["act"])
    assert np.array_equal(out, np.array(c["y"]))
