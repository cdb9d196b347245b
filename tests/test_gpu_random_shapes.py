"""Seeded random layer shapes against the fp64 oracle: token counts across the
layer's kernel switches (no row gather up to 16 tokens, one work item per
touched expert up to 64, 128-row tiles up to 256, the large-batch kernels
above), hidden and expert sizes that are any multiple of 64, expert counts
that are not powers of two, k from 1 to 8.  Each case checks the routing and
the output the way the per-configuration tests do (the selection valid under
the logit error bound, the output within the layer tolerance), in bf16 and
with E4M3 weights and activations."""

import numpy as np
import pytest

from routing_dispatch_expert_softmax_b200 import workloads as wl

import test_gpu_parity as P
import test_gpu_w8a8 as W

pytestmark = pytest.mark.gpu

_T_CHOICES = [1, 2, 3, 5, 8, 13, 16, 17, 31, 33, 64, 65, 100, 200, 256, 257, 300, 700, 1500,
              2048]


def _shapes(seed, n, prefix):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T = int(rng.choice(_T_CHOICES))
        big = T > 300                          # keep the oracle's work small
        d = 64 * int(rng.integers(1, 9 if big else 17))   # 64 .. 512 (1024)
        E = int(rng.integers(1, 65))           # 1 .. 64
        k = int(rng.integers(1, min(E, 8) + 1))
        f = 64 * int(rng.integers(1, 5 if big else 9))    # 64 .. 256 (512)
        out.append(wl.MoEConfig(f"{prefix}{i}", T=T, d=d, E=E, k=k, f=f))
    return out


@pytest.mark.parametrize("cfg", _shapes(20240, 40, "rand-bf16-"),
                         ids=lambda c: f"{c.name}-T{c.T}-d{c.d}-E{c.E}-k{c.k}-f{c.f}")
def test_forward_random_shape(cfg):
    P._check_forward(cfg, seed=3)


@pytest.mark.parametrize("cfg", _shapes(20241, 24, "rand-w8a8-"),
                         ids=lambda c: f"{c.name}-T{c.T}-d{c.d}-E{c.E}-k{c.k}-f{c.f}")
def test_forward_w8a8_random_shape(cfg):
    W._forward_case(cfg, seed=3)
