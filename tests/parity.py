"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare them at the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_routed_moe_b200 as moe
from mixture_experts_routed_moe_b200 import inputs as G
from oracle import moe_oracle as O

# Output tolerances for bf16 experts: relative Frobenius error and max-abs
# error relative to the largest reference magnitude; FP8 experts: relative
# Frobenius error.
BF16_REL_FRO = 5e-3
BF16_MAX_ABS = 2e-2
FP8_REL_FRO = 3e-2


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_bf16_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    r = rel_fro(got, ref)
    m = float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300))
    assert r <= BF16_REL_FRO and m <= BF16_MAX_ABS, f"{what}: rel_fro={r:.3e} max_abs/max|ref|={m:.3e}"
    return r, m


def assert_fp8_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    r = rel_fro(got, ref)
    assert r <= FP8_REL_FRO, f"{what}: rel_fro={r:.3e}"
    return r


class ExpertView:
    """Per-expert host copies of device expert weights, made on first use, so
    the oracle can index w[e] without copying experts nobody selected."""

    def __init__(self, t: torch.Tensor, as_codes: bool = False):
        self.t = t
        self.shape = tuple(t.shape)
        self.as_codes = as_codes
        self._cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self._cache:
            v = self.t[e].cpu()
            self._cache[e] = v.view(torch.uint8).numpy() if self.as_codes else v.float().numpy()
        return self._cache[e]


def ws_i32(ws: torch.Tensor, off: int, n: int) -> np.ndarray:
    return ws[off:off + 4 * n].view(torch.int32).cpu().numpy()


def ws_bf16(ws: torch.Tensor, off: int, rows: int, cols: int) -> np.ndarray:
    return ws[off:off + 2 * rows * cols].view(torch.bfloat16).reshape(rows, cols).float().cpu().numpy()


def check_permutation(ws, shape, idx_np):
    """Bit-exact comparison of the device permutation with the oracle's."""
    lay = moe.workspace_layout(shape)
    E, k, T = shape.E, shape.k, shape.T
    ref = O.permute(idx_np, E, lay.bm)
    cnt = ws_i32(ws, lay.cnt, E)
    mt = ws_i32(ws, lay.mt_base, E + 1)
    assert np.array_equal(cnt, ref["cnt"])
    assert np.array_equal(mt.astype(np.int64) * lay.bm, ref["off"])
    rows = int(ref["off"][-1])
    assert np.array_equal(ws_i32(ws, lay.row_src, rows), ref["row_src"])
    assert np.array_equal(ws_i32(ws, lay.slot_row, T * k), ref["slot_row"])
    return lay, ref


def device_inputs(wl: G.Workload, seed: int, weights_device="cuda"):
    x, logits = G.make_activations(wl, seed)
    W = G.make_weights(wl, seed, device=weights_device)
    return x, logits, W


def oracle_forward_bf16(x_cpu, idx, w, W, tokens=None, intermediate="bf16"):
    return O.moe_forward(x_cpu.float().numpy(), idx, w, ExpertView(W["w_gate_up"]), ExpertView(W["w_down"]),
                         intermediate=intermediate, tokens=tokens)


def oracle_forward_fp8(x_cpu, idx, w, W, tokens=None):
    return O.moe_forward_fp8(x_cpu.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True),
                             ExpertView(W["sw_gate_up"], True), ExpertView(W["w_down"], True),
                             ExpertView(W["sw_down"], True), tokens=tokens)
