"""Seeded synthetic inputs for the routed MoE layer.

This module only draws random tensors; it holds none of the layer's
arithmetic, and both the CUDA path and the oracle take its tensors as inputs.

Shapes follow the model families the expert-parallel serving pages discuss
(Qwen3-30B-A3B, Mixtral-8x7B, DeepSeek-V3 routed experts).  The pages serve
real checkpoints with unstated prompts; none of that exists here, so every
tensor is drawn from the distributions below:

* hidden states x ~ N(0, 1), rounded to bf16;
* router W_g ~ N(0, 1/d) in fp32 (d x E);
* expert weights ~ N(0, 1/fan_in) in bf16: w13 (E, 2f, d) with fan_in d,
  w2 (E, d, f) with fan_in f;
* optional skew bias b[e] = -s * ln(pi(e) + 1) with pi a seeded permutation of
  the experts, so the top-1 popularity of expert e falls off like a Zipf(s)
  law in its popularity rank pi(e).

Each tensor has its own stream: ``torch.Generator(device)`` seeded with
``1000 * seed + tensor_id`` (x=1, W_g=2, skew permutation=3, w13=4, w2=5).
Expert weights are drawn one expert at a time from their stream.  The values
depend on the device the generator runs on (CPU and CUDA streams differ), so a
test draws on one device and copies to the other.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

X_ID, WG_ID, PERM_ID, W13_ID, W2_ID = 1, 2, 3, 4, 5
W13Q_ID, W2Q_ID, W13S_ID, W2S_ID = 6, 7, 8, 9


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """One layer shape: T tokens, hidden d, E experts, top-k, intermediate f,
    R virtual expert-parallel ranks (0 = no virtual layout), and the Zipf
    exponent of the skew bias (None = no bias)."""

    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    R: int = 0
    zipf_s: Optional[float] = None

    def with_T(self, T: int) -> "MoEConfig":
        return dataclasses.replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")

    @property
    def P(self) -> int:
        return self.T * self.k

    def expert_bytes(self) -> int:
        """bf16 bytes of one expert's three matrices (3*d*f*2)."""
        return 3 * self.d * self.f * 2

    def as_dict(self) -> dict:
        return dataclasses.asdict(self)


# The workloads, named by what they are.
TINY = MoEConfig("tiny", T=64, d=256, E=8, k=2, f=512)
QWEN3_30B_A3B_DECODE = MoEConfig("qwen3-30b-a3b-decode", T=64, d=2048, E=128,
                                 k=8, f=768, zipf_s=1.0)
QWEN3_30B_A3B_PREFILL = MoEConfig("qwen3-30b-a3b-prefill", T=8192, d=2048,
                                  E=128, k=8, f=768)
MIXTRAL_8X7B = MoEConfig("mixtral-8x7b", T=4096, d=4096, E=8, k=2, f=14336)
DEEPSEEK_V3_ROUTED = MoEConfig("deepseek-v3-routed", T=64, d=7168, E=256, k=8,
                               f=2048, R=8, zipf_s=1.2)

QWEN_DECODE_SWEEP_T = (1, 8, 64, 256)
DEEPSEEK_SWEEP_T = (1, 64, 512, 16384)

CONFIGS = {
    c.name: c
    for c in (TINY, QWEN3_30B_A3B_DECODE, QWEN3_30B_A3B_PREFILL, MIXTRAL_8X7B,
              DEEPSEEK_V3_ROUTED)
}


def _gen(device, seed: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + tensor_id)
    return g


def make_hidden(cfg: MoEConfig, device="cpu", seed: int = 0) -> torch.Tensor:
    """x (T, d) bf16 ~ N(0, 1)."""
    g = _gen(device, seed, X_ID)
    x = torch.randn(cfg.T, cfg.d, generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_router(cfg: MoEConfig, device="cpu", seed: int = 0):
    """(W_g (d, E) fp32 ~ N(0, 1/d), bias (E,) fp32 or None)."""
    g = _gen(device, seed, WG_ID)
    w_g = torch.randn(cfg.d, cfg.E, generator=g, device=device,
                      dtype=torch.float32) * (1.0 / math.sqrt(cfg.d))
    bias = None
    if cfg.zipf_s is not None:
        gp = _gen(device, seed, PERM_ID)
        pi = torch.randperm(cfg.E, generator=gp, device=device)
        bias = (-cfg.zipf_s) * torch.log(pi.to(torch.float64) + 1.0)
        bias = bias.to(torch.float32)
    return w_g.contiguous(), bias


def make_experts(cfg: MoEConfig, device="cpu", seed: int = 0):
    """(w13 (E, 2f, d) bf16 ~ N(0, 1/d), w2 (E, d, f) bf16 ~ N(0, 1/f)).

    Drawn expert by expert so the fp32 staging buffer stays one expert big.
    """
    w13 = torch.empty(cfg.E, 2 * cfg.f, cfg.d, device=device, dtype=torch.bfloat16)
    w2 = torch.empty(cfg.E, cfg.d, cfg.f, device=device, dtype=torch.bfloat16)
    g13 = _gen(device, seed, W13_ID)
    g2 = _gen(device, seed, W2_ID)
    s13 = 1.0 / math.sqrt(cfg.d)
    s2 = 1.0 / math.sqrt(cfg.f)
    for e in range(cfg.E):
        w13[e] = (torch.randn(2 * cfg.f, cfg.d, generator=g13, device=device,
                              dtype=torch.float32) * s13).to(torch.bfloat16)
        w2[e] = (torch.randn(cfg.d, cfg.f, generator=g2, device=device,
                             dtype=torch.float32) * s2).to(torch.bfloat16)
    return w13, w2


# FP8 codes are drawn as N(0, FP8_CODE_STD^2), clamped to the largest E4M3
# magnitude and cast to the nearest code, so they use most of E4M3's range.
FP8_CODE_STD = 64.0
FP8_MAX = 448.0


def make_experts_fp8(cfg: MoEConfig, device="cpu", seed: int = 0):
    """FP8 expert weights: (w13 codes (E, 2f, d) uint8, w13 row scales (E, 2f)
    fp32, w2 codes (E, d, f) uint8, w2 row scales (E, d) fp32).

    Codes are E4M3 bit patterns; each row scale is sigma / FP8_CODE_STD times
    a U(0.5, 1.5) draw, sigma the bf16 weights' std (1/sqrt(d) for w13,
    1/sqrt(f) for w2), so the weights have the bf16 weights' size and every
    row a different scale.
    """
    def codes(rows, cols, g):
        v = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        v = (v * FP8_CODE_STD).clamp_(-FP8_MAX, FP8_MAX)
        return v.to(torch.float8_e4m3fn).view(torch.uint8)

    w13 = torch.empty(cfg.E, 2 * cfg.f, cfg.d, device=device, dtype=torch.uint8)
    w2 = torch.empty(cfg.E, cfg.d, cfg.f, device=device, dtype=torch.uint8)
    g13, g2 = _gen(device, seed, W13Q_ID), _gen(device, seed, W2Q_ID)
    for e in range(cfg.E):
        w13[e] = codes(2 * cfg.f, cfg.d, g13)
        w2[e] = codes(cfg.d, cfg.f, g2)
    u13 = torch.rand(cfg.E, 2 * cfg.f, generator=_gen(device, seed, W13S_ID), device=device)
    u2 = torch.rand(cfg.E, cfg.d, generator=_gen(device, seed, W2S_ID), device=device)
    s13 = (u13 + 0.5) * (1.0 / (math.sqrt(cfg.d) * FP8_CODE_STD))
    s2 = (u2 + 0.5) * (1.0 / (math.sqrt(cfg.f) * FP8_CODE_STD))
    return w13, s13.float().contiguous(), w2, s2.float().contiguous()


def make_layer(cfg: MoEConfig, device="cpu", seed: int = 0) -> dict:
    """Every input of one layer call."""
    w_g, bias = make_router(cfg, device, seed)
    w13, w2 = make_experts(cfg, device, seed)
    return dict(x=make_hidden(cfg, device, seed), w_g=w_g, bias=bias,
                w13=w13, w2=w2)


def make_logits(T: int, E: int, device="cpu", seed: int = 0, kind: str = "normal"):
    """Router-logit-shaped fp32 test inputs for the selection step alone.

    kind="normal": N(0, 1); kind="ties": small integers in [-2, 2] with signed
    zeros mixed in, so most tokens have ties at the selection boundary;
    kind="const": every logit of a token equal (the all-tie case).
    """
    g = _gen(device, seed, 100 + {"normal": 0, "ties": 1, "const": 2}[kind])
    if kind == "normal":
        return torch.randn(T, E, generator=g, device=device, dtype=torch.float32)
    if kind == "ties":
        v = torch.randint(-2, 3, (T, E), generator=g, device=device).to(torch.float32)
        neg = torch.randint(0, 2, (T, E), generator=g, device=device).bool()
        v = torch.where((v == 0) & neg, torch.full_like(v, -0.0), v)
        return v
    if kind == "const":
        c = torch.randn(T, 1, generator=g, device=device, dtype=torch.float32)
        return c.expand(T, E).contiguous()
    raise ValueError(kind)
