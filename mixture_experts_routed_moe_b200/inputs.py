"""Seeded synthetic inputs for the routed MoE expert forward.

This module only draws numbers. It holds none of the method's arithmetic
(no routing, no permutation, no expert MLP, no activation quantisation), so
both the CUDA path and the CPU oracle can be fed from it without sharing any
of the computation they are compared on.

Workloads (names and sizes):

    tiny     T=64    H=128  I=256    E=8    k=2  bf16
    decode   T=16    H=2048 I=1408   E=60   k=4  bf16
    prefill  T=8192  H=2048 I=768    E=128  k=8  bf16
    fp8      T=4096  H=7168 I=2048   E=256  k=8  e4m3 weights, 128x128 UE8M0 scales
    skewed   T=4096  H=4096 I=14336  E=8    k=2  bf16, router bias 2.0*(1 - e/7)

Distributions: hidden states N(0,1) rounded to bf16; expert weights
N(0, 0.02) rounded to bf16 (or quantised to e4m3, see below); router logits
N(0,1) in fp32.

FP4 weights (e2m1, the FP4-packed experts of the same section) are prepared
the same way per row and block of 32 consecutive columns: the smallest s
with 6 * 2^s >= amax, UE8M0 byte s + 127, codes = w / 2^s rounded to the
nearest e2m1 value (ties to the even code), two codes per byte with the even
column in the low nibble. torch has no e2m1 cast, so the rounding is done
here with plain tensor arithmetic on the e2m1 grid.

Hidden states and logits come from numpy's PCG64 seeded with ``seed`` and do
not depend on the device. Expert weights are drawn per expert from a torch
generator on the device that will hold them (seed ``seed * 100003 + e``), so a
full-size layer never has to pass through host memory; tests that need the
weights on the CPU copy them back.

FP8 weights are pre-quantised checkpoints in the "Experts backends" page's
sense (section "FP8 and FP4 quantized experts"): the quantisation is part of
producing the checkpoint, not of the forward pass. Per 128x128 block of an
expert matrix, with amax the block's largest magnitude, the scale exponent is
the smallest integer s with 2^s >= amax/448 (so nothing overflows), stored
biased as a UE8M0 byte s + 127 (byte 127, scale 1, for an all-zero block); the
codes are w / 2^s cast to float8_e4m3fn by torch (round to nearest even).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

WEIGHT_STD = 0.02
E4M3_MAX = 448.0
QBLOCK = 128  # weight scale block (rows and columns)
E2M1_MAX = 6.0
FP4_BLOCK = 32  # FP4 weight scale block (columns of one row)
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    wdtype: str = "bf16"  # "bf16", "e4m3" or "e2m1"
    router_bias: bool = False

    @property
    def A(self) -> int:
        """Number of (token, slot) assignments."""
        return self.T * self.k

    def flops(self) -> int:
        """Algorithmic FLOPs of the expert MLPs: 3 GEMMs of 2*A*H*I each."""
        return 6 * self.A * self.H * self.I

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 128, 256, 8, 2),
    "decode": Workload("decode", 16, 2048, 1408, 60, 4),
    "prefill": Workload("prefill", 8192, 2048, 768, 128, 8),
    "fp8": Workload("fp8", 4096, 7168, 2048, 256, 8, wdtype="e4m3"),
    "skewed": Workload("skewed", 4096, 4096, 14336, 8, 2, router_bias=True),
    # the FP8 layer's experts at decode size: 16 tokens, weight-streaming path
    "fp8_decode": Workload("fp8_decode", 16, 7168, 2048, 256, 8, wdtype="e4m3"),
    # the large layer's shape with FP4 (e2m1) experts, at prefill and decode size
    "fp4": Workload("fp4", 4096, 7168, 2048, 256, 8, wdtype="e2m1"),
    "fp4_decode": Workload("fp4_decode", 16, 7168, 2048, 256, 8, wdtype="e2m1"),
}
# the seed of each named workload is its position in this list
WORKLOAD_ORDER = ["tiny", "decode", "prefill", "fp8", "skewed", "fp8_decode", "fp4", "fp4_decode"]


def default_seed(wl: Workload) -> int:
    return WORKLOAD_ORDER.index(wl.name) if wl.name in WORKLOAD_ORDER else 0


def router_bias(E: int) -> np.ndarray:
    """Per-expert logit bias 2.0*(1 - e/7) of the skewed workload, fp32."""
    return np.array([2.0 * (1.0 - e / 7.0) for e in range(E)], dtype=np.float32)


def make_activations(wl: Workload, seed: int):
    """x: bf16 [T,H] (torch, CPU); logits: fp32 [T,E] (torch, CPU)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((wl.T, wl.H), dtype=np.float32)
    logits = rng.standard_normal((wl.T, wl.E), dtype=np.float32)
    if wl.router_bias:
        logits = logits + router_bias(wl.E)[None, :]
    return torch.from_numpy(x).to(torch.bfloat16), torch.from_numpy(np.ascontiguousarray(logits))


def _expert_generator(seed: int, e: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 100003 + e)
    return g


def _draw(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * WEIGHT_STD


def quantize_weight_blocks(w: torch.Tensor):
    """Checkpoint-style e4m3 quantisation of one [R, C] fp32 matrix
    (R, C multiples of 128). Returns (codes float8_e4m3fn [R,C], ue8m0 uint8 [R/128, C/128])."""
    R, C = w.shape
    blk = w.reshape(R // QBLOCK, QBLOCK, C // QBLOCK, QBLOCK)
    amax = blk.abs().amax(dim=(1, 3))
    ratio = amax / E4M3_MAX
    m, ex = torch.frexp(ratio)  # ratio = m * 2^ex, m in [0.5, 1)
    s = ex - (m == 0.5).to(ex.dtype)  # smallest s with 2^s >= ratio
    s = torch.where(amax > 0, s, torch.zeros_like(s))
    scale = torch.ldexp(torch.ones_like(ratio), s)
    q = blk / scale[:, None, :, None]
    q = q.clamp(-E4M3_MAX, E4M3_MAX).reshape(R, C).to(torch.float8_e4m3fn)
    return q, (s + 127).to(torch.uint8)


def quantize_fp4_rows(w: torch.Tensor):
    """Checkpoint-style FP4 quantisation of one [R, C] fp32 matrix (C a
    multiple of 32). Returns (packed uint8 [R, C/2], ue8m0 uint8 [R, C/32])."""
    R, C = w.shape
    blk = w.reshape(R, C // FP4_BLOCK, FP4_BLOCK)
    amax = blk.abs().amax(dim=2)
    ratio = amax / E2M1_MAX
    m, ex = torch.frexp(ratio)
    s = ex - (m == 0.5).to(ex.dtype)  # smallest s with 2^s >= amax / 6
    s = torch.where(amax > 0, s, torch.zeros_like(s))
    q = blk / torch.ldexp(torch.ones_like(ratio), s)[:, :, None]
    mag = q.abs().clamp(max=E2M1_MAX)
    step = torch.where(mag < 2.0, 0.5, torch.where(mag < 4.0, 1.0, 2.0))
    r = torch.minimum(torch.round(mag / step) * step, torch.full_like(mag, E2M1_MAX))  # round: ties to even
    grid = torch.tensor(_E2M1_GRID, device=w.device)
    code = torch.searchsorted(grid, r.contiguous()).to(torch.uint8) | (torch.signbit(q).to(torch.uint8) << 3)
    code = code.reshape(R, C)
    return (code[:, 0::2] | (code[:, 1::2] << 4)).contiguous(), (s + 127).to(torch.uint8)


def make_weights(wl: Workload, seed: int, device="cpu"):
    """Expert weights on ``device``.

    bf16: dict(w_gate_up=[E,2I,H] bf16 (rows 0..I-1 gate, I..2I-1 up), w_down=[E,H,I] bf16)
    e4m3: the same shapes as float8_e4m3fn plus sw_gate_up uint8 [E,2I/128,H/128] and
          sw_down uint8 [E,H/128,I/128].
    """
    E, H, I = wl.E, wl.H, wl.I
    if wl.wdtype == "bf16":
        wgu = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=device)
        wd = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
        for e in range(E):
            g = _expert_generator(seed, e, device)
            wgu[e] = _draw((2 * I, H), g, device).to(torch.bfloat16)
            wd[e] = _draw((H, I), g, device).to(torch.bfloat16)
        return dict(w_gate_up=wgu, w_down=wd)
    if wl.wdtype == "e4m3":
        wgu = torch.empty((E, 2 * I, H), dtype=torch.float8_e4m3fn, device=device)
        wd = torch.empty((E, H, I), dtype=torch.float8_e4m3fn, device=device)
        sgu = torch.empty((E, 2 * I // QBLOCK, H // QBLOCK), dtype=torch.uint8, device=device)
        sd = torch.empty((E, H // QBLOCK, I // QBLOCK), dtype=torch.uint8, device=device)
        for e in range(E):
            g = _expert_generator(seed, e, device)
            wgu[e], sgu[e] = quantize_weight_blocks(_draw((2 * I, H), g, device))
            wd[e], sd[e] = quantize_weight_blocks(_draw((H, I), g, device))
        return dict(w_gate_up=wgu, w_down=wd, sw_gate_up=sgu, sw_down=sd)
    if wl.wdtype == "e2m1":
        wgu = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=device)
        wd = torch.empty((E, H, I // 2), dtype=torch.uint8, device=device)
        sgu = torch.empty((E, 2 * I, H // FP4_BLOCK), dtype=torch.uint8, device=device)
        sd = torch.empty((E, H, I // FP4_BLOCK), dtype=torch.uint8, device=device)
        for e in range(E):
            g = _expert_generator(seed, e, device)
            wgu[e], sgu[e] = quantize_fp4_rows(_draw((2 * I, H), g, device))
            wd[e], sd[e] = quantize_fp4_rows(_draw((H, I), g, device))
        return dict(w_gate_up=wgu, w_down=wd, sw_gate_up=sgu, sw_down=sd)
    raise ValueError(f"unknown weight dtype {wl.wdtype!r}")


def make_expert_weights(wl: Workload, seed: int, e: int, device="cpu"):
    """One expert's weights, identical to slice e of :func:`make_weights` on the same device."""
    g = _expert_generator(seed, e, device)
    a = _draw((2 * wl.I, wl.H), g, device)
    b = _draw((wl.H, wl.I), g, device)
    if wl.wdtype == "bf16":
        return dict(w_gate_up=a.to(torch.bfloat16), w_down=b.to(torch.bfloat16))
    if wl.wdtype == "e2m1":
        qa, sa = quantize_fp4_rows(a)
        qb, sb = quantize_fp4_rows(b)
        return dict(w_gate_up=qa, w_down=qb, sw_gate_up=sa, sw_down=sb)
    qa, sa = quantize_weight_blocks(a)
    qb, sb = quantize_weight_blocks(b)
    return dict(w_gate_up=qa, w_down=qb, sw_gate_up=sa, sw_down=sb)


def make_router_weights(wl: Workload, seed: int, device="cpu") -> torch.Tensor:
    """Router weights W_r [E, H] ~ N(0, 0.02) as bf16, from a torch generator
    on `device` (seed * 100003 + 99991, apart from every expert's stream)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed * 100003 + 99991)
    w = torch.randn((wl.E, wl.H), generator=g, device=device, dtype=torch.float32) * 0.02
    return w.to(torch.bfloat16)


def routed_inputs_with_counts(wl: Workload, counts, seed: int = 0):
    """Hand-placed routing for edge cases: a [T,k] int32 choice in which expert e
    is picked by exactly counts[e] tokens (sum(counts) == T*k, max(counts) <= T),
    every token picking k distinct experts, plus fp32 weights in (0,1) that sum
    to 1 per token. Experts are placed in order of decreasing count, each on the
    tokens with the fewest slots filled so far (lowest token index first), which
    realises every feasible count vector."""
    T, k, E = wl.T, wl.k, wl.E
    counts = [int(c) for c in counts]
    assert len(counts) == E and sum(counts) == T * k and max(counts) <= T
    idx = np.full((T, k), -1, dtype=np.int32)
    fill = np.zeros(T, dtype=np.int64)
    for e in sorted(range(E), key=lambda e: (-counts[e], e)):
        if counts[e] == 0:
            continue
        order = np.lexsort((np.arange(T), fill))  # fewest filled first, then lower token
        chosen = np.sort(order[: counts[e]])
        assert (fill[chosen] < k).all(), "count vector is not realisable"
        idx[chosen, fill[chosen]] = e
        fill[chosen] += 1
    assert (fill == k).all()
    rng = np.random.default_rng(seed)
    w = rng.random((T, k), dtype=np.float32) + np.float32(0.05)
    w = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    return torch.from_numpy(idx), torch.from_numpy(w)


def flops_and_bytes(wl: Workload, touched_experts: int | None = None):
    """Algorithmic FLOPs and minimum HBM bytes of one forward (route excluded):
    touched expert weights + x read + out written."""
    E_t = wl.E if touched_experts is None else touched_experts
    welem = {"e4m3": 1.0, "e2m1": 0.5}.get(wl.wdtype, 2.0)
    wbytes = int(E_t * 3 * wl.H * wl.I * welem)
    if wl.wdtype == "e4m3":
        wbytes += E_t * (2 * wl.I // QBLOCK * wl.H // QBLOCK + wl.H // QBLOCK * wl.I // QBLOCK)
    if wl.wdtype == "e2m1":
        wbytes += E_t * 3 * wl.H * wl.I // FP4_BLOCK
    act = wl.T * wl.H * 2 * 2
    return wl.flops(), wbytes + act


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "Workload", "WORKLOADS", "WORKLOAD_ORDER", "default_seed", "make_activations", "make_weights",
    "make_expert_weights", "make_router_weights", "quantize_weight_blocks", "quantize_fp4_rows",
    "routed_inputs_with_counts",
    "flops_and_bytes",
    "router_bias", "ceil_div",
]
