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
    the oracle can index w[e] without copying experts nobody selected. With
    cache=False each access copies again and nothing is kept (the full-size
    layers' weights would not fit in host memory twice over)."""

    def __init__(self, t: torch.Tensor, as_codes: bool = False, cache: bool = True):
        self.t = t
        self.shape = tuple(t.shape)
        self.as_codes = as_codes
        self.cache = cache
        self._cache = {}

    def _copy(self, e):
        v = self.t[e].cpu()
        return v.view(torch.uint8).numpy() if self.as_codes else v.float().numpy()

    def __getitem__(self, e):
        e = int(e)
        if not self.cache:
            return self._copy(e)
        if e not in self._cache:
            self._cache[e] = self._copy(e)
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


def oracle_forward_bf16(x_cpu, idx, w, W, tokens=None, intermediate="bf16", cache=True):
    return O.moe_forward(x_cpu.float().numpy(), idx, w, ExpertView(W["w_gate_up"], cache=cache),
                         ExpertView(W["w_down"], cache=cache), intermediate=intermediate, tokens=tokens)


def oracle_forward_fp8(x_cpu, idx, w, W, tokens=None, cache=True):
    return O.moe_forward_fp8(x_cpu.float().numpy(), idx, w, ExpertView(W["w_gate_up"], True, cache),
                             ExpertView(W["sw_gate_up"], True, cache), ExpertView(W["w_down"], True, cache),
                             ExpertView(W["sw_down"], True, cache), tokens=tokens)


def device_topk_w(logits_cpu, k, idx_ref):
    """The routing weights the device itself uses for these logits (moe_route
    is deterministic, so a layer that routed the same logits got these bits),
    after checking that its indices equal the oracle's. The combine pin takes
    these: the device's weights differ from the oracle's by exp/division
    rounding, which a bit-exact comparison must not see."""
    idx_d, w_d = moe.route(logits_cpu.cuda(), k)
    assert np.array_equal(idx_d.cpu().numpy(), idx_ref)
    return w_d.cpu().numpy()


def check_combine_bit_exact(ws, shape, topk_w_np, out, chunk=1024):
    """The device combine against the oracle's fixed-order fp32 combine on the
    expert outputs y the device itself produced (read from the workspace):
    every output bit must agree."""
    lay = moe.workspace_layout(shape)
    T, k, H = shape.T, shape.k, shape.H
    slot = ws_i32(ws, lay.slot_row, T * k).reshape(T, k)
    y_all = ws[lay.y:lay.y + 2 * lay.m_rows * H].view(torch.bfloat16).reshape(lay.m_rows, H)
    got = out.float().cpu().numpy()
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        rows = torch.from_numpy(slot[t0:t1].reshape(-1).astype(np.int64)).to(y_all.device)
        Y = y_all.index_select(0, rows).float().cpu().numpy().reshape(t1 - t0, k, H)
        ref = O.combine_fp32_fma(Y, topk_w_np[t0:t1])
        bad = np.nonzero(got[t0:t1] != ref)
        assert bad[0].size == 0, f"combine differs at {bad[0].size} elements, first token {t0 + bad[0][0]}"


def assert_tokens_close(got, ref, bound, what=""):
    """Per-token relative error (Frobenius over the token's H outputs) at most
    `bound`: a check that no single token is wrong, which the whole-layer norm
    could hide among thousands of good ones."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.linalg.norm(got - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    worst = int(np.argmax(num / den))
    assert (num / den).max() <= bound, f"{what}: token {worst} rel_fro={num[worst] / den[worst]:.3e}"
