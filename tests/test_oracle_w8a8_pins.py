"""Pins of the oracle's FP8-activation (W8A8) functions against things other
than themselves: torch's own E4M3 and bf16 conversions (independent
implementations of the same rounding), exact rational arithmetic for the
power-of-two row exponent, every code and every midpoint of the format, and
the W8A8 expert FFN recomposed from those library conversions.

The reading pinned here (the pages give no activation format): one scale
2^e per row, e the smallest integer with max|row| <= 448 * 2^e, then round
to nearest E4M3, ties to even; the SwiGLU output rounded to bf16 before its
own quantisation.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_oracle as F


def _torch_e4m3(v):
    """torch's fp32 -> float8_e4m3fn cast (round to nearest even) as codes;
    only called on magnitudes <= 448 (torch does not saturate)."""
    t = torch.from_numpy(np.asarray(v, dtype=np.float32).copy())
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _brute_exponent(row):
    """Smallest integer e with max|row| <= 448 * 2^e, by exact rationals."""
    amax = max((Fraction(float(abs(v))) for v in row), default=Fraction(0))
    if amax == 0:
        return 0
    e = -200
    while Fraction(448) * Fraction(2) ** e < amax:
        e += 1
    return e


def test_every_code_encodes_to_itself():
    codes = np.arange(256, dtype=np.uint8)
    vals = F.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    got = F.e4m3_encode(vals[finite])
    np.testing.assert_array_equal(got, codes[finite])


def test_encode_matches_torch_on_random_and_edge_values():
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.normal(size=200_000) * 40,
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 20_000),        # subnormal range
        [0.0, -0.0, 1e-9, -1e-9, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 448.0, -448.0],
    ]).astype(np.float32).astype(np.float64)
    v = np.clip(v, -448, 448)
    np.testing.assert_array_equal(F.e4m3_encode(v), _torch_e4m3(v))


def test_midpoints_round_to_the_even_code_and_neighbours_to_the_nearest():
    tab = F.e4m3_decode(np.arange(127, dtype=np.uint8))
    mid = (tab[:-1] + tab[1:]) / 2
    got = F.e4m3_encode(mid)
    assert np.all(got % 2 == 0)
    np.testing.assert_array_equal(got, _torch_e4m3(mid))
    below, above = np.nextafter(mid, -np.inf), np.nextafter(mid, np.inf)
    np.testing.assert_array_equal(F.e4m3_encode(below), np.arange(126))
    np.testing.assert_array_equal(F.e4m3_encode(above), np.arange(1, 127))


def test_saturation_and_sign():
    assert F.e4m3_encode(np.array([449.0, 1e30, -500.0])).tolist() == [0x7E, 0x7E, 0xFE]
    assert F.e4m3_encode(np.array([-0.0, -1e-30])).tolist() == [0x80, 0x80]


@pytest.mark.parametrize("seed", range(3))
def test_row_exponent_is_the_smallest_covering_power(seed):
    rng = np.random.default_rng(seed)
    rows = rng.normal(size=(40, 33)) * np.exp(rng.uniform(-30, 30, (40, 1)))
    rows[0] = 0.0
    rows[1, :] = 0.0
    rows[1, 5] = 448.0 * 2.0 ** 7            # exactly on a power: e = 7
    rows[2, :] = 0.0
    rows[2, 0] = np.nextafter(448.0 * 2.0 ** -3, np.inf)  # just above: e = -2
    got = F.pow2_row_exponent(rows)
    want = [_brute_exponent(r) for r in rows]
    assert got.tolist() == want
    assert got[1] == 7 and got[2] == -2 and got[0] == 0


def test_quantised_rows_stay_in_range_and_close():
    rng = np.random.default_rng(5)
    a = rng.normal(size=(64, 257)) * 3
    codes, scale = F.quantise_rows_pow2(a)
    vals = F.e4m3_decode(codes)
    assert np.all(np.abs(vals) <= 448)
    # the row maximum lands in (224, 448]: the scale is the smallest that fits
    amax = np.abs(a).max(axis=1) / scale
    assert np.all((amax > 224) & (amax <= 448))
    # normal-range elements: relative error at most half a unit (2^-4)
    deq = F.dequantise_rows(codes, scale)
    big = np.abs(a / scale[:, None]) >= 2.0 ** -6
    assert np.all(np.abs(deq - a)[big] <= 2.0 ** -4 * np.abs(a)[big])


def test_bf16_round_matches_torch_on_fp32_values_and_avoids_double_rounding():
    rng = np.random.default_rng(9)
    v = (rng.normal(size=100_000) * 10).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(F.bf16_round(v), want)
    # just above the midpoint between 1 and its bf16 successor 1 + 2^-7: the
    # nearest bf16 is 1 + 2^-7 (a detour through fp32 would land on the tie
    # and round to 1)
    assert F.bf16_round(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1 + 2.0 ** -7
    assert F.bf16_round(np.array([1 + 2.0 ** -8]))[0] == 1.0        # tie, even


def test_w8a8_ffn_equals_its_recomposition_from_library_casts():
    """The expert FFN with quantised inputs, recomposed from torch's fp8 and
    bf16 casts and exact exponents; an h element whose fp32 rounding lands on
    a bf16 tie would make torch's fp64 -> bf16 cast double-round, so the seed
    is checked to have none."""
    rng = np.random.default_rng(11)
    n, d, f = 9, 96, 64
    X = rng.normal(size=(n, d))
    w13 = rng.normal(size=(2 * f, d)) / np.sqrt(d)
    w2 = rng.normal(size=(d, f)) / np.sqrt(f)

    def q(rows):
        e = np.array([_brute_exponent(r) for r in rows])
        c = _torch_e4m3(np.ldexp(rows, -e[:, None]))
        return F.e4m3_decode(c) * np.ldexp(1.0, e)[:, None]

    Xq = q(X)
    g, u = Xq @ w13[:f].T, Xq @ w13[f:].T
    h = oracle.silu(g) * u
    h32 = h.astype(np.float32).astype(np.float64)
    hb = torch.from_numpy(h).to(torch.bfloat16).double().numpy()
    ulp = np.ldexp(1.0, np.frexp(hb)[1] - 8)
    assert not np.any(np.abs(np.abs(h32 - hb) - ulp / 2) == 0), "double-rounding tie in seed"
    want = q(hb) @ w2.T
    got = F.w8a8_ffn(X, w13, w2)
    np.testing.assert_array_equal(got, want)


def test_w8a8_layer_reduces_to_the_fp8_weight_layer_on_representable_inputs():
    """Tokens already of the form e4m3 * 2^e quantise to themselves, so the
    first GEMM sees exactly the tokens of the W8A16 layer; with one expert
    whose down projection is a multiple of a unit vector and SwiGLU outputs
    of one value per row, the two layers agree exactly."""
    rng = np.random.default_rng(2)
    T, d, f, E = 5, 32, 16, 1
    codes_x = rng.integers(0, 0x7E, size=(T, d)).astype(np.uint8)
    x = F.e4m3_decode(codes_x) * 2.0 ** -3
    w_g = rng.normal(size=(d, E))
    c13 = np.zeros((E, 2 * f, d), dtype=np.uint8)
    c13[0, :, 0] = 0x38                       # 1.0 in column 0: g = u = x[:, 0]
    s13 = np.ones((E, 2 * f))
    c2 = np.zeros((E, d, f), dtype=np.uint8)
    c2[0, 0, :] = 0x38
    s2 = np.ones((E, d))
    a = oracle.moe_forward_w8a8(x, w_g, None, c13, s13, c2, s2, k=1)
    b = oracle.moe_forward_fp8(x, w_g, None, c13, s13, c2, s2, k=1)
    # h = silu(x0) * x0, the same for every column of a row, so its row
    # quantisation is a single rounding: compare against that rounding
    x0 = x[:, 0]
    h = F.bf16_round(oracle.silu(x0) * x0)
    hq = F.e4m3_decode(F.e4m3_encode(np.ldexp(h, -F.pow2_row_exponent(h[:, None])))) * \
        np.ldexp(1.0, F.pow2_row_exponent(h[:, None]))
    np.testing.assert_array_equal(a["z"][:, 0], f * hq[a["perm"]])
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["y"], b["y"], rtol=0.07, atol=1e-12)
