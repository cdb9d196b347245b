"""Plain CPU oracle for the layer with FP8 expert weights.

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests and bench.py's CPU
legs may use it; it shares nothing with the CUDA library.

What the pages fix, and the reading taken where they are silent:

* "Serving MoE models with expert parallelism on 8xH200", section
  "Memory math for 8xH200": DeepSeek-V3 and the Qwen3 FP8 variants store
  their weights at one byte per parameter; section "Quantization choices":
  native FP8 checkpoints are the default choice.
* The pages name no FP8 encoding and no scale granularity.  Reading: OCP
  FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
  exponent field 0 holds the subnormals m/8 * 2^-6; S.1111.111 is NaN; there
  are no infinities), and one scale per output row of each expert matrix:
  W[e, r, c] = e4m3(code[e, r, c]) * scale[e, r].
* Given those weights the layer is exactly the bf16 layer's definition
  (moe_oracle.moe_forward) applied to the dequantised matrices, in fp64.
* FP8 activations (the W8A8 layer, both GEMM operands in E4M3 so the tensor
  cores multiply one-byte codes): the pages fix no activation format either.
  Reading: each activation row (a token's hidden state before GEMM1, an
  expert row's SwiGLU output before GEMM2) gets one power-of-two scale
  2^e, e the smallest integer with max|row| <= 448 * 2^e (e = 0 for an
  all-zero row), and every element becomes the E4M3 value nearest to
  value * 2^-e, ties to the even code.  A power of two makes value * 2^-e
  exact, so the codes are a function of the input alone.  The SwiGLU output
  is held in bf16 (round to nearest even) before it is quantised, as the
  layer stores it between the two GEMMs.
"""

from __future__ import annotations

import numpy as np

from . import moe_oracle as _m

__all__ = ["e4m3_decode", "dequantise_rows", "moe_forward_fp8", "LazyDequant",
           "e4m3_encode", "pow2_row_exponent", "quantise_rows_pow2", "bf16_round",
           "moe_forward_w8a8", "w8a8_ffn"]

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Value of every E4M3 code, in fp64 (exact): (-1)^s * 2^(e-7) * (1 + m/8)
    for exponent field e > 0, (-1)^s * 2^-6 * m/8 for e = 0, NaN for
    exponent 15 with mantissa 7."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e > 0, np.ldexp(1.0 + m / 8.0, e - 7), np.ldexp(m / 8.0, -6))
    v = sign * mag
    return np.where((e == 15) & (m == 7), np.nan, v)


def dequantise_rows(codes, scale):
    """W[..., r, c] = e4m3(codes[..., r, c]) * scale[..., r], fp64.  The
    codes are looked up in the decoded table of all 256 codes (the same
    values as decoding each element, much faster on large matrices)."""
    table = e4m3_decode(np.arange(256, dtype=np.uint8))
    return table[np.asarray(codes, dtype=np.uint8)] * np.asarray(scale, dtype=np.float64)[..., None]


class LazyDequant:
    """Indexable view that dequantises one expert at a time (keeps host memory
    to one expert's fp64 matrix)."""

    def __init__(self, codes, scale):
        self.codes, self.scale = codes, scale

    def __getitem__(self, e):
        return dequantise_rows(self.codes[int(e)], self.scale[int(e)])


def moe_forward_fp8(x, w_g, bias, w13_codes, w13_scale, w2_codes, w2_scale, k, R=0,
                    select_dtype=np.float32, idx=None):
    """The layer with FP8 expert weights: the bf16 layer's steps with every
    expert matrix dequantised first.  `w13_codes`/`w2_codes` may be arrays or
    anything indexable by expert (the scale arguments alike)."""
    return _m.moe_forward(x, w_g, bias, LazyDequant(w13_codes, w13_scale),
                          LazyDequant(w2_codes, w2_scale), k, R=R,
                          select_dtype=select_dtype, idx=idx)


# ------------------------------------------------------------ FP8 activations
def _e4m3_finite_table():
    """The non-negative finite E4M3 values in code order (codes 0..126): the
    order of the codes is the order of the values."""
    return e4m3_decode(np.arange(127, dtype=np.uint8))


def e4m3_encode(v):
    """E4M3 code of the value nearest to each fp64 v, ties to the even code
    (the even mantissa), magnitudes above 448 saturating to 448; the sign bit
    is v's sign bit, also when the magnitude rounds to zero (as an IEEE
    conversion keeps it).  Written as the definition: a search of the 127
    non-negative finite values."""
    v = np.asarray(v, dtype=np.float64)
    tab = _e4m3_finite_table()
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, 126)  # tab[hi] >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - tab[lo], tab[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.int64)
    code = np.where(a == tab[hi], hi, code)  # exact values
    sign = np.signbit(v).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def pow2_row_exponent(a):
    """Per row of a (..., n): the smallest integer e with max|a| <= 448 * 2^e,
    and 0 for a row of zeros.  Exact: the candidates are checked with fp64
    products by powers of two."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    amax = a.max(axis=-1) if a.shape[-1] else np.zeros(a.shape[:-1])
    e = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    # frexp: amax = m * 2^x with 0.5 <= m < 1, so 448 * 2^e >= amax near e = x - 9
    x = np.frexp(amax[nz])[1].astype(np.int64)
    cand = x - 10
    am = amax[nz]
    for _ in range(4):
        too_small = np.ldexp(E4M3_MAX, cand) < am
        cand = np.where(too_small, cand + 1, cand)
    # smallest: step back while the smaller exponent still covers amax
    for _ in range(4):
        ok_smaller = np.ldexp(E4M3_MAX, cand - 1) >= am
        cand = np.where(ok_smaller, cand - 1, cand)
    e[nz] = cand
    return e


def quantise_rows_pow2(a):
    """(codes uint8 (..., n), scales fp64 (...) = 2^e): the row quantisation
    of the W8A8 reading above."""
    a = np.asarray(a, dtype=np.float64)
    e = pow2_row_exponent(a)
    codes = e4m3_encode(np.ldexp(a, -e[..., None]))
    return codes, np.ldexp(1.0, e)


def bf16_round(a):
    """Nearest bf16 value of each fp64 element, ties to even, for the normal
    bf16 range: bf16 keeps 8 significant bits, so the significand is rounded
    to 8 bits directly (no detour through fp32, whose own rounding could
    create a false tie)."""
    a = np.asarray(a, dtype=np.float64)
    m, x = np.frexp(a)                    # a = m * 2^x, 0.5 <= |m| < 1
    q = np.round(np.ldexp(m, 8))          # an integer in [128, 256]; half to even
    return np.ldexp(q, x - 8)


def w8a8_ffn(X, w13_e, w2_e):
    """One expert's SwiGLU FFN with both GEMM inputs quantised per row
    (fp64 arithmetic on the dequantised codes)."""
    cx, sx = quantise_rows_pow2(X)
    Xq = dequantise_rows(cx, sx)
    w13_e = np.asarray(w13_e, dtype=np.float64)
    w2_e = np.asarray(w2_e, dtype=np.float64)
    f = w13_e.shape[0] // 2
    g = Xq @ w13_e[:f].T
    u = Xq @ w13_e[f:].T
    h = bf16_round(_m.silu(g) * u)
    ch, sh = quantise_rows_pow2(h)
    return dequantise_rows(ch, sh) @ w2_e.T


def moe_forward_w8a8(x, w_g, bias, w13_codes, w13_scale, w2_codes, w2_scale, k, R=0,
                     select_dtype=np.float32, idx=None):
    """The layer with FP8 expert weights and FP8 activations: routing, gates,
    dispatch and combine as in the bf16 layer; each expert row's FFN by
    w8a8_ffn on the dequantised weights."""
    return _m.moe_forward(x, w_g, bias, LazyDequant(w13_codes, w13_scale),
                          LazyDequant(w2_codes, w2_scale), k, R=R,
                          select_dtype=select_dtype, idx=idx, ffn=w8a8_ffn)
