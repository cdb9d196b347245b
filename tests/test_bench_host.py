"""Host-side bookkeeping of bench.py: the algorithmic bytes / flops behind
the roofline fractions and the kernel-launch count behind gpu_launches.
No GPU is involved."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routing_dispatch_expert_softmax_b200 import workloads as wl  # noqa: E402


@pytest.mark.parametrize("cfg,touched", [(wl.QWEN3_30B_A3B_DECODE, 57),
                                         (wl.DEEPSEEK_V3_ROUTED.with_T(512), 84),
                                         (wl.TINY, 8)])
def test_algorithmic_bytes_and_flops(cfg, touched):
    T, d, E, k, f = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f
    router = d * E * 4 + (E * 4 if cfg.zipf_s is not None else 0)
    act = 2 * T * d * 2                                  # x read, y written
    bf16 = bench.algorithmic(cfg, touched)
    assert bf16["bytes"] == touched * 3 * d * f * 2 + router + act
    assert bf16["gemm1_bytes"] + bf16["gemm2_bytes"] == touched * 3 * d * f * 2
    assert bf16["flops"] == 6 * T * k * d * f + 2 * T * d * E
    assert bf16["gemm1_flops"] == 2 * bf16["gemm2_flops"] == 4 * T * k * d * f
    fp8 = bench.algorithmic(cfg, touched, fp8=True)      # 1-byte codes + a 4-byte scale per row
    assert fp8["bytes"] == touched * (3 * d * f + (2 * f + d) * 4) + router + act
    assert fp8["gemm1_bytes"] == touched * (2 * f * d + 2 * f * 4)
    assert fp8["flops"] == bf16["flops"]


def test_launch_counts_match_the_profiled_launch_lists():
    # profiles/launches_qwen3_decode_T64.md: 6 kernels per layer call;
    # profiles/launches_qwen3_prefill_T8192.md: 13 (split router with a
    # finish kernel, four routing kernels, gather, two pair GEMMs each with
    # its lone-tile kernel, combine); the FP8 layer runs its two 128-row-tile
    # GEMMs at every batch size (11 at prefill).
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE) == 6
    # up to 16 tokens GEMM1 reads x itself: no row gather
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE.with_T(8)) == 5
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE.with_T(16)) == 5
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE.with_T(17)) == 6
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE.with_T(8), w8a8=True) == 7
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE, fp8=True) == 6
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_PREFILL) == 13
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_PREFILL, fp8=True) == 11
    # FP8 activations: the SwiGLU output's quantisation between the GEMMs
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE, w8a8=True) == 7
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_PREFILL, w8a8=True) == 14
    # replicas: top-k, remap, histogram, scan, scatter instead of the fused kernel
    assert bench.launches_per_forward(wl.QWEN3_30B_A3B_DECODE, eplb_redundant=16) == 10
