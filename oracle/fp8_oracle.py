"""Plain CPU oracle for the layer with FP8 expert weights.

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests and bench.py's CPU
legs may use it; it shares nothing with the CUDA library.

What the pages fix, and the reading taken where they are silent:

* "Serving mixture-of-experts models: expert parallelism on H200", section
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
"""

from __future__ import annotations

import numpy as np

from . import moe_oracle as _m

__all__ = ["e4m3_decode", "dequantise_rows", "moe_forward_fp8", "LazyDequant"]


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
