"""Pins of the FP4 (e2m1) expert pieces of the oracle (reading R8): the code
table against the format's bit layout worked by hand, rounding against a
brute-force nearest-value search, nibble packing, the per-32-column block
scales, and the forward as the bf16 forward on the dequantised weights."""
import numpy as np
import pytest

from oracle import moe_oracle as O


def test_e2m1_table_golden(golden):
    g = golden("e2m1_codes.json")
    for code, v in g["values"].items():
        got = O.e2m1_decode(np.array([int(code)]))[0]
        assert got == v and np.signbit(got) == np.signbit(v), code
    for case in g["rounding"]:
        assert O.e2m1_encode(np.array([case["in"]]))[0] == case["code"], case
    for case in g["packing"]:
        assert O.pack_e2m1(np.array(case["codes"], dtype=np.uint8))[0] == case["byte"]
        assert list(O.unpack_e2m1(np.array([case["byte"]], dtype=np.uint8))) == case["codes"]


def test_e2m1_round_is_the_nearest_value_brute_force():
    """Against an exhaustive search over the 8 magnitudes: the nearest one,
    and of two equally near the one whose code has mantissa bit 0."""
    mags = O.e2m1_decode(np.arange(8))
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-8, 8, 20000), np.arange(-7, 7.01, 0.25)])  # every tie on the grid
    got = O.e2m1_round(v)
    for x, r in zip(v, got):
        a = min(abs(x), 6.0)
        d = np.abs(mags - a)
        best = np.nonzero(d == d.min())[0]
        pick = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        assert r == np.copysign(mags[pick], x), x
    # encode then decode is the rounding
    assert np.array_equal(O.e2m1_decode(O.e2m1_encode(v)), got)


def test_packing_round_trip():
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, (5, 64)).astype(np.uint8)
    assert np.array_equal(O.unpack_e2m1(O.pack_e2m1(codes)), codes)


def test_dequantize_fp4_block_placement():
    """Each UE8M0 byte scales its row's 32 consecutive columns: a matrix of
    ones (code 2) with scale bytes 127 + r + 2b yields 2^(r + 2b) on row r,
    columns 32b..32b+31; a transposed or 128-wide block reading fails."""
    R, C = 3, 128
    codes = np.full((R, C), 2, dtype=np.uint8)
    sb = np.array([[127 + r + 2 * b for b in range(C // 32)] for r in range(R)], dtype=np.uint8)
    w = O.dequantize_fp4(O.pack_e2m1(codes), sb)
    for r in range(R):
        for c in range(C):
            assert w[r, c] == 2.0 ** (r + 2 * (c // 32))


def test_fp4_forward_is_bf16_forward_on_dequantised_weights():
    """With e2m1 weights the expert arithmetic is the bf16 layer's (h, y
    rounded to bf16): the FP4 forward equals moe_forward on the dequantised
    matrices, and those matrices are exact in bf16."""
    rng = np.random.default_rng(2)
    T, H, I, E, k = 12, 64, 96, 3, 2
    x = O.bf16_round(rng.standard_normal((T, H)))
    idx, w, _ = O.route(rng.standard_normal((T, E)).astype(np.float32), k)
    gu = rng.integers(0, 16, (E, 2 * I, H)).astype(np.uint8)
    dn = rng.integers(0, 16, (E, H, I)).astype(np.uint8)
    sgu = rng.integers(118, 124, (E, 2 * I, H // 32)).astype(np.uint8)
    sdn = rng.integers(118, 124, (E, H, I // 32)).astype(np.uint8)
    pgu, pdn = O.pack_e2m1(gu), O.pack_e2m1(dn)
    got = O.moe_forward_fp4(x, idx, w, pgu, sgu, pdn, sdn)
    Wgu = np.stack([O.dequantize_fp4(pgu[e], sgu[e]) for e in range(E)])
    Wd = np.stack([O.dequantize_fp4(pdn[e], sdn[e]) for e in range(E)])
    assert np.array_equal(O.bf16_round(Wgu), Wgu) and np.array_equal(O.bf16_round(Wd), Wd)
    assert np.array_equal(got, O.moe_forward(x, idx, w, Wgu, Wd))


@pytest.mark.parametrize("planted", ["high_nibble_first", "scale_per_128"])
def test_planted_fp4_mistakes_are_caught(planted):
    """Plausible mistakes, planted in a copy on the CPU, fail the block test."""
    R, C = 2, 64
    codes = np.arange(R * C, dtype=np.uint8).reshape(R, C) % 16
    sb = np.array([[120, 125], [127, 130]], dtype=np.uint8)
    ref = O.dequantize_fp4(O.pack_e2m1(codes), sb)
    if planted == "high_nibble_first":
        b = O.pack_e2m1(codes)
        wrong_codes = np.empty_like(codes)
        wrong_codes[:, 0::2], wrong_codes[:, 1::2] = b >> 4, b & 0xF
        wrong = O.e2m1_decode(wrong_codes) * np.repeat(O.ue8m0_scale(sb), 32, axis=1)
    else:
        wrong = O.e2m1_decode(codes) * O.ue8m0_scale(sb)[:, :1]
    assert not np.array_equal(np.nan_to_num(ref), np.nan_to_num(wrong))
