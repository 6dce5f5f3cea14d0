"""CPU oracle for the routed mixture-of-experts expert forward.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain, obviously-correct
statement of what the CUDA path computes. Only the tests, the smoke check and
the benchmark's CPU-baseline leg may import it; the product path never does.
It shares no code with the CUDA library (no kernels, headers, tables or
helpers) and imports nothing from it.

Source: Hugging Face Transformers docs page "Experts backends"
(experts_interface). Its introduction describes the one computation that all
backends share: a router chooses k experts per token, every chosen expert maps
the token's hidden state through its own weights, and the token's output is the
routing-weighted sum of those expert results; only the way the expert matmuls
are executed differs between backends. The "eager" row of the backend table is
the reference implementation: a loop over the selected experts that applies the
projections to their tokens. That eager loop is the algorithm written out here.
The expert is a gated MLP: a joint gate/up projection, the SwiGLU activation,
then the down projection (backend table, row "deepgemm_megamoe"; section "Fused
Mega MoE on Blackwell"), and the section "SonicMoE" maps the gated activations
SwiGLU/GeGLU/ReGLU to silu/gelu/relu; all three are supported (gelu in its
exact erf form).

Arithmetic is float64 throughout. The pages fix no precision; where they are
silent this module takes the readings below (each one is also listed in the
design notes):

  R1 selection key: the k experts are chosen on the fp32 logits, which orders
     them exactly as the exact softmax does (softmax is strictly increasing);
     equal logits go to the lower expert index; slot j holds the j-th largest.
  R2 weights: softmax over all E experts, then renormalised over the chosen k,
     returned as float32 (the boundary's routing-weight type).
  R3 expert weight layout: w_gate_up[e] is [2I, H] with rows 0..I-1 the gate
     projection and rows I..2I-1 the up projection; w_down[e] is [H, I]; both
     are row-major with the reduction dimension contiguous.
     h = silu(x Wg^T) * (x Wu^T), y = h Wd^T.
  R4 intermediate rounding ("bf16" mode): a bf16 layer stores h and y as bf16
     (round to nearest even) and the aggregated output as bf16; "exact" mode
     rounds only the output.
  R5 aggregation: out[t] = sum_j w[t,j] * y[t,j] with the given fp32 weights.
  R6 permutation: expert-major, tokens ascending within an expert, each expert's
     block padded up to a multiple of BM rows (pad rows carry source -1).
  R8 FP4 experts (section "FP8 and FP4 quantized experts": FP4-packed expert
     weights with UE8M0 scales on Blackwell): weights are OCP MX e2m1 codes
     (sign, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5,
     1, 1.5, 2, 3, 4, 6), two per byte with the even element in the low
     nibble, times 2^(byte-127) for each block of 32 consecutive elements
     along the reduction dimension (the OCP MX block). The page names no
     activation format for FP4 experts, so activations stay bf16 (weight-only
     quantisation); every e2m1 value times a power of two is exact in bf16,
     so the layer is the bf16 layer (R4) on the dequantised weights.
  R7 FP8 (section "FP8 and FP4 quantized experts", and its note on Blackwell
     UE8M0 scales): weights are e4m3 codes times 2^(byte-127) per 128x128
     block; activations are quantised per token, per 128-column group, with an
     fp32 scale s = amax/448 (s = 1 for an all-zero group) and codes
     e4m3(x / s) rounded to nearest even and saturated at +-448, the division
     done in fp32. x is quantised from its bf16 value, h from its fp32 value;
     y is stored as bf16.

Parity status: routing, permutation, the expert MLP and the FP8 encoding are
pinned by the CPU tests (brute force, closed forms, invariants and library
routines). The pages print no worked example, so end-to-end values on the
seeded workloads are pinned only through those pieces.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
QBLOCK = 128  # FP8 weight block and activation group size


# ---------------------------------------------------------------------------
# rounding helpers (reading R4, R7)
# ---------------------------------------------------------------------------

def bf16_round(a) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even); returns float64.

    bf16 keeps 8 significant bits; normal exponents reach down to 2^-126 and
    below that the spacing is fixed at 2^-133."""
    a = np.asarray(a, dtype=np.float64)
    _, ex = np.frexp(a)  # a = m * 2^ex, 0.5 <= |m| < 1
    ex = np.maximum(ex, -125)
    ulp = np.ldexp(1.0, ex - 8)
    with np.errstate(invalid="ignore", over="ignore"):
        r = np.rint(a / ulp) * ulp
    r = np.where(np.abs(r) > 3.3895313892515355e38, np.copysign(np.inf, a), r)
    return np.where(np.isfinite(a), r, a)


def e4m3_round(v) -> np.ndarray:
    """Nearest e4m3 (OCP FP8, bias 7, no infinities) value of float values v,
    ties to even, saturating to +-448; returns float64.

    Normal numbers run from 2^-6 to 448 with 3 mantissa bits, so the spacing at
    exponent ex is 2^(ex-3); below 2^-6 the spacing is the subnormal step 2^-9."""
    v = np.asarray(v, dtype=np.float64)
    mag = np.abs(v)
    _, ex = np.frexp(mag)  # mag = m * 2^ex, m in [0.5, 1) -> leading bit at 2^(ex-1)
    lead = np.maximum(ex - 1, -6)
    step = np.ldexp(1.0, lead - 3)
    r = np.rint(mag / step) * step
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_encode(v) -> np.ndarray:
    """e4m3 byte codes (sign bit 7, exponent bits 6..3, mantissa bits 2..0) of
    float values v after :func:`e4m3_round`."""
    r = e4m3_round(v)
    sign = (np.signbit(r)).astype(np.uint8) << 7
    mag = np.abs(r)
    code = np.zeros(mag.shape, dtype=np.int64)
    normal = mag >= 2.0 ** -6
    _, ex = np.frexp(np.where(normal, mag, 1.0))
    e_unb = ex - 1
    mant = np.where(normal, mag / np.ldexp(1.0, e_unb) - 1.0, 0.0) * 8.0
    code = np.where(normal, ((e_unb + 7) << 3) | np.rint(mant).astype(np.int64), code)
    sub = ~normal
    code = np.where(sub, np.rint(mag / 2.0 ** -9).astype(np.int64), code)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def _e4m3_value(c) -> np.ndarray:
    """Float64 value of each e4m3 byte code: sign bit 7, exponent field e (bits
    6..3, bias 7), mantissa m (bits 2..0); e = 0 is subnormal m * 2^-9,
    otherwise (1 + m/8) * 2^(e-7); 0x7F and 0xFF are NaN."""
    c = np.asarray(c, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


# the 256 values, one per code, so that decoding a large matrix is one lookup
_E4M3_VALUES = _e4m3_value(np.arange(256, dtype=np.uint8))


def e4m3_decode(codes) -> np.ndarray:
    """Float64 values of e4m3 byte codes (0x7F/0xFF are NaN): the value of
    each code, looked up in the table of all 256."""
    return _E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def ue8m0_scale(b) -> np.ndarray:
    """Power-of-two scale 2^(b-127) of UE8M0 bytes (byte 255 is NaN)."""
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


# ---------------------------------------------------------------------------
# routing (readings R1, R2)
# ---------------------------------------------------------------------------

def route(logits, k: int):
    """Top-k routing of fp32 router logits [T, E].

    Experts backends, introduction: the router picks k experts per token and
    their outputs are summed with the routing weights. Softmax over all
    experts, choose the k largest (R1), renormalise their probabilities over
    the k (R2).

    Returns (topk_idx int32 [T,k], topk_w float32 [T,k], topk_w64 float64 [T,k])."""
    L = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = L.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    # a stable sort on the negated logits keeps equal logits in index order
    order = np.argsort(-L, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    m = L.max(axis=1, keepdims=True)
    p = np.exp(L - m)
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    w64 = sel / sel.sum(axis=1, keepdims=True)
    return idx, w64.astype(np.float32), w64


def router_logits(x, w_router):
    """Router logits [T, E] = x W_r^T, float64, from the given (bf16-valued)
    x [T, H] and router weights W_r [E, H]: the router step ahead of the experts
    (backend table, row "sonicmoe", which fuses the router dispatch with the
    expert GEMMs; the introduction's router that picks k experts per token).
    The routing itself is route() on these logits."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T


# ---------------------------------------------------------------------------
# permutation (reading R6)
# ---------------------------------------------------------------------------

def permute(topk_idx, E: int, BM: int):
    """Expert-major layout of the T*k assignments.

    Backend table, rows "grouped_mm" and "deepgemm": tokens are sorted by their
    selected expert so that one grouped GEMM (tile-aligned, for the TMA-based
    kernel) covers every expert. Within an expert, tokens keep ascending order.
    Expert e owns rows [off[e], off[e+1]) with off[e+1]-off[e] =
    ceil(cnt[e]/BM)*BM; the first cnt[e] of them hold assignments, the rest are
    padding.

    Returns dict(cnt int32 [E], off int64 [E+1], row_src int32 [off[E]]
    (assignment t*k+j, or -1 for padding), slot_row int32 [T*k])."""
    ti = np.asarray(topk_idx, dtype=np.int64)
    T, k = ti.shape
    cnt = np.zeros(E, dtype=np.int64)
    for e in ti.ravel():
        cnt[e] += 1
    padded = -(-cnt // BM) * BM
    off = np.zeros(E + 1, dtype=np.int64)
    off[1:] = np.cumsum(padded)
    row_src = np.full(int(off[E]), -1, dtype=np.int64)
    slot_row = np.full(T * k, -1, dtype=np.int64)
    fill = off[:E].copy()
    for t in range(T):  # ascending token order
        for j in range(k):
            e = ti[t, j]
            row_src[fill[e]] = t * k + j
            slot_row[t * k + j] = fill[e]
            fill[e] += 1
    return dict(cnt=cnt.astype(np.int32), off=off, row_src=row_src.astype(np.int32),
                slot_row=slot_row.astype(np.int32))


# ---------------------------------------------------------------------------
# expert MLP and the eager forward (readings R3, R4, R5)
# ---------------------------------------------------------------------------

def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)) (section "SonicMoE": silu <-> SwiGLU)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gelu(z):
    """gelu(z) = z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)), the exact (erf) form
    (section "SonicMoE": gelu <-> GeGLU). erf from scipy."""
    import scipy.special

    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + scipy.special.erf(z / np.sqrt(2.0)))


def relu(z):
    """relu(z) = max(z, 0) (section "SonicMoE": relu <-> ReGLU)."""
    return np.maximum(np.asarray(z, dtype=np.float64), 0.0)


ACTIVATIONS = {"silu": silu, "gelu": gelu, "relu": relu}


def expert_mlp(X, w_gate_up_e, w_down_e, intermediate: str = "bf16", act: str = "silu"):
    """One expert's gated MLP on its tokens X [n, H] (float64):
    up projection (gate and up halves of w_gate_up_e), gated activation
    act(gate) * up (SwiGLU by default), down projection.
    Backend table, row "deepgemm_megamoe" (up projection, SwiGLU, down projection)."""
    I = w_gate_up_e.shape[0] // 2
    Wg = np.asarray(w_gate_up_e[:I], dtype=np.float64)
    Wu = np.asarray(w_gate_up_e[I:], dtype=np.float64)
    Wd = np.asarray(w_down_e, dtype=np.float64)
    G = X @ Wg.T
    U = X @ Wu.T
    h = ACTIVATIONS[act](G) * U
    if intermediate == "bf16":
        h = bf16_round(h)
    y = h @ Wd.T
    if intermediate == "bf16":
        y = bf16_round(y)
    return h, y


def _expert_loop(x, topk_idx, E, tokens, mlp):
    """Eager loop over the experts (backend table, row "eager"): for every expert
    that some token in ``tokens`` selected, run its MLP on those tokens.
    Returns Y [len(tokens), k, H] with Y[i, j] the output of slot j of tokens[i]."""
    ti = np.asarray(topk_idx, dtype=np.int64)[tokens]
    n, k = ti.shape
    Y = None
    for e in range(E):
        rows, slots = np.nonzero(ti == e)
        if rows.size == 0:
            continue
        X = np.asarray(x[tokens[rows]], dtype=np.float64)
        y = mlp(e, X)
        if Y is None:
            Y = np.zeros((n, k, y.shape[1]), dtype=np.float64)
        Y[rows, slots] = y
    return Y


def combine(Y, topk_w, intermediate: str = "bf16"):
    """out[t] = sum_j w[t,j] * Y[t,j] (introduction: the routing-weighted sum of the experts' results)."""
    w = np.asarray(topk_w, dtype=np.float32).astype(np.float64)
    out = np.zeros((Y.shape[0], Y.shape[2]), dtype=np.float64)
    for j in range(Y.shape[1]):
        out += w[:, j:j + 1] * Y[:, j]
    return bf16_round(out) if intermediate in ("bf16", "exact") else out


def fma_f32(a, b, c) -> np.ndarray:
    """Single-precision fused multiply-add, round(a*b + c) to the nearest
    float32 (ties to even), for float32-valued inputs; returns float64.

    The product of two float32 values has at most 48 significant bits, so a*b
    is exact in float64. The sum is split exactly into s + err (Knuth's
    TwoSum); s is then moved to its odd neighbour when err is nonzero and s is
    even (rounding to odd), after which one rounding to float32 is the correct
    one: float64 carries more than 24 + 1 extra bits, so no double rounding."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    p = a * b
    s = p + c
    bv = s - p
    err = (p - (s - bv)) + (c - bv)
    even = (s.view(np.int64) & 1) == 0
    toward = np.where(err > 0, np.inf, -np.inf)
    s = np.where((err != 0) & even, np.nextafter(s, toward), s)
    return s.astype(np.float32).astype(np.float64)


def combine_fp32_fma(Y, topk_w):
    """The aggregation of reading R5 in the precision the boundary states:
    acc = 0 in float32, then acc = fma(w[t,j], Y[t,j], acc) for j = 0..k-1 in
    ascending order, and the output rounded to bf16 once at the end
    (introduction: the routing-weighted sum of the experts' results). With the
    same Y this fixes every bit of the output."""
    w = np.asarray(topk_w, dtype=np.float32).astype(np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    acc = np.zeros((Y.shape[0], Y.shape[2]), dtype=np.float64)
    for j in range(Y.shape[1]):
        acc = fma_f32(w[:, j:j + 1], Y[:, j], acc)
    return bf16_round(acc)


def moe_forward(x, topk_idx, topk_w, w_gate_up, w_down, intermediate: str = "bf16",
                tokens=None, act: str = "silu"):
    """Routed MoE forward for bf16 experts.

    x [T,H]; topk_idx int [T,k]; topk_w fp32 [T,k]; w_gate_up [E,2I,H];
    w_down [E,H,I] (any float arrays holding the bf16 values). ``tokens``
    restricts the computation to a subset of tokens (each output row depends
    only on its own token). ``intermediate``: "bf16" (R4), "exact" (round the
    output only) or "none" (no rounding at all). ``act``: the gate activation
    ("silu", "gelu" or "relu"). Returns float64 [len(tokens), H]."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    E = w_gate_up.shape[0]
    mode = "bf16" if intermediate == "bf16" else "exact"

    def mlp(e, X):
        return expert_mlp(X, w_gate_up[e], w_down[e], mode, act)[1]

    Y = _expert_loop(x, topk_idx, E, tokens, mlp)
    w = np.asarray(topk_w)[tokens]
    if intermediate == "none":
        return combine(Y, w, "none")
    return combine(Y, w, "bf16")


# ---------------------------------------------------------------------------
# FP8 experts (reading R7)
# ---------------------------------------------------------------------------

def dequantize_blocks(codes, scale_bytes):
    """Weights of one expert matrix [R, C] from e4m3 codes and one UE8M0 byte per
    128x128 block (section "FP8 and FP4 quantized experts": power-of-two block
    scales on Blackwell)."""
    q = e4m3_decode(codes)
    s = ue8m0_scale(scale_bytes)
    R, C = q.shape
    # element (r, c) takes the scale of block (r // 128, c // 128)
    q4 = q.reshape(R // QBLOCK, QBLOCK, C // QBLOCK, QBLOCK)
    return (q4 * s[:, None, :, None]).reshape(R, C)


def quantize_1x128(a):
    """Dynamic per-row activation quantisation (section "FP8 and FP4 quantized
    experts": per-row dynamic activation scales): each row is split into groups
    of 128 columns; per group s = amax/448 in fp32 (1 if amax is 0) and codes
    e4m3(a/s), the division in fp32.

    a: float32-valued [R, C] (C multiple of 128). Returns (codes uint8 [R,C],
    scales float32 [R, C/128], dequantised float64 [R,C])."""
    a32 = np.asarray(a, dtype=np.float32)
    R, C = a32.shape
    g = a32.reshape(R, C // QBLOCK, QBLOCK)
    amax = np.abs(g).max(axis=2)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)
    v = (g / s[:, :, None]).astype(np.float32)  # fp32 division
    codes = e4m3_encode(v).reshape(R, C)
    deq = (e4m3_decode(codes).reshape(R, C // QBLOCK, QBLOCK) * s[:, :, None].astype(np.float64))
    return codes, s, deq.reshape(R, C)


def expert_mlp_fp8(X, wgu_codes, wgu_sb, wd_codes, wd_sb, quantize_acts: bool = True, act: str = "silu"):
    """One FP8 expert on its tokens X [n,H] (bf16 values): x quantised 1x128,
    gate/up projection, SwiGLU evaluated on the fp32 result, h quantised 1x128,
    down projection, y rounded to bf16."""
    Wgu = dequantize_blocks(wgu_codes, wgu_sb)
    Wd = dequantize_blocks(wd_codes, wd_sb)
    I = Wgu.shape[0] // 2
    Xq = quantize_1x128(X)[2] if quantize_acts else np.asarray(X, dtype=np.float64)
    G = Xq @ Wgu[:I].T
    U = Xq @ Wgu[I:].T
    h = (ACTIVATIONS[act](G) * U).astype(np.float32)
    hq = quantize_1x128(h)[2] if quantize_acts else h.astype(np.float64)
    return bf16_round(hq @ Wd.T)


def moe_forward_fp8(x, topk_idx, topk_w, wgu_codes, wgu_sb, wd_codes, wd_sb,
                    tokens=None, quantize_acts: bool = True, act: str = "silu"):
    """Routed MoE forward for FP8 experts (e4m3 codes + UE8M0 block bytes).
    Shapes: wgu_codes uint8 [E,2I,H], wgu_sb uint8 [E,2I/128,H/128],
    wd_codes uint8 [E,H,I], wd_sb uint8 [E,H/128,I/128]. Returns float64 [len(tokens),H]."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    E = wgu_codes.shape[0]

    def mlp(e, X):
        return expert_mlp_fp8(X, wgu_codes[e], wgu_sb[e], wd_codes[e], wd_sb[e], quantize_acts, act)

    Y = _expert_loop(x, topk_idx, E, tokens, mlp)
    return combine(Y, np.asarray(topk_w)[tokens], "bf16")


# ---------------------------------------------------------------------------
# FP4 experts (reading R8)
# ---------------------------------------------------------------------------

E2M1_MAX = 6.0
FP4_BLOCK = 32  # elements per UE8M0 scale, along the reduction dimension


def _e2m1_value(c) -> np.ndarray:
    """Float64 value of each 4-bit e2m1 code: sign bit 3, exponent field e
    (bits 2..1, bias 1), mantissa m (bit 0); e = 0 is subnormal m * 0.5,
    otherwise (1 + m/2) * 2^(e-1)."""
    c = np.asarray(c, dtype=np.int64) & 0xF
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    return s * np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.ldexp(1.0, e - 1))


_E2M1_VALUES = _e2m1_value(np.arange(16))


def e2m1_decode(codes) -> np.ndarray:
    """Float64 values of 4-bit e2m1 codes (the table of all 16)."""
    return _E2M1_VALUES[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_round(v) -> np.ndarray:
    """Nearest e2m1 value, ties to the even code (mantissa bit 0), magnitudes
    above 6 saturating to 6; returns float64. The spacing is 0.5 below 2, 1 on
    [2, 4) and 2 on [4, 6]."""
    v = np.asarray(v, dtype=np.float64)
    mag = np.minimum(np.abs(v), E2M1_MAX)
    step = np.where(mag < 2.0, 0.5, np.where(mag < 4.0, 1.0, 2.0))
    r = np.rint(mag / step) * step  # rint: ties to even multiples of the step
    return np.copysign(np.minimum(r, E2M1_MAX), v)


def e2m1_encode(v) -> np.ndarray:
    """4-bit e2m1 codes (uint8 0..15) of float values v after :func:`e2m1_round`."""
    r = e2m1_round(v)
    mag = np.abs(r)
    idx = np.searchsorted(_E2M1_VALUES[:8], mag)  # the 8 magnitudes are increasing
    return (idx.astype(np.uint8) | (np.signbit(r).astype(np.uint8) << 3)).astype(np.uint8)


def unpack_e2m1(packed) -> np.ndarray:
    """4-bit codes [..., 2n] from bytes [..., n]: element 2i in the low nibble of byte i."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def pack_e2m1(codes) -> np.ndarray:
    """Bytes [..., n] from 4-bit codes [..., 2n] (inverse of :func:`unpack_e2m1`)."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def dequantize_fp4(packed, scale_bytes):
    """Weights [R, C] of one FP4 expert matrix from packed e2m1 bytes [R, C/2]
    and one UE8M0 byte per row and block of 32 columns [R, C/32]."""
    q = e2m1_decode(unpack_e2m1(packed))
    s = ue8m0_scale(scale_bytes)
    R, C = q.shape
    return (q.reshape(R, C // FP4_BLOCK, FP4_BLOCK) * s[:, :, None]).reshape(R, C)


def moe_forward_fp4(x, topk_idx, topk_w, wgu_packed, wgu_sb, wd_packed, wd_sb, tokens=None, act: str = "silu"):
    """Routed MoE forward for FP4 experts (reading R8): the bf16 forward on the
    dequantised weights. Shapes: wgu_packed uint8 [E,2I,H/2], wgu_sb uint8
    [E,2I,H/32], wd_packed uint8 [E,H,I/2], wd_sb uint8 [E,H,I/32]."""
    E = len(wgu_packed) if not hasattr(wgu_packed, "shape") else wgu_packed.shape[0]

    class _Deq:
        def __init__(self, packed, sb):
            self.packed, self.sb = packed, sb
            self.shape = (E,)

        def __getitem__(self, e):
            return dequantize_fp4(self.packed[e], self.sb[e])

    return moe_forward(x, topk_idx, topk_w, _Deq(wgu_packed, wgu_sb), _Deq(wd_packed, wd_sb), tokens=tokens, act=act)
