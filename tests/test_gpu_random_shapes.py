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
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape
from parity_utils import LazyExperts, assert_layer_close

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


def _offsets(rng, P, E):
    """Per-expert row counts summing to P: skewed, with empty experts, and at
    times one expert holding more rows than the batch has tokens (moe_ffn's
    caller offsets allow it)."""
    w = rng.pareto(1.0, E) + 1e-3
    w[rng.random(E) < 0.3] = 0.0
    if w.sum() == 0:
        w[0] = 1.0
    counts = np.floor(w / w.sum() * P).astype(np.int64)
    counts[int(np.argmax(w))] += P - counts.sum()
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _ffn_shapes(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        cfg = _shapes(seed * 7 + i, 1, f"rand-ffn-{i}-")[0]
        out.append((cfg, _offsets(rng, cfg.T * cfg.k, cfg.E)))
    return out


@pytest.mark.parametrize("cfg,offsets", _ffn_shapes(20242, 16),
                         ids=lambda v: v.name if hasattr(v, "name") else "")
def test_ffn_random_offsets(cfg, offsets):
    P = int(offsets[-1])
    x_perm = wl.make_hidden(wl.MoEConfig("rows", T=P, d=cfg.d, E=1, k=1, f=64), "cuda", 5)
    w13, w2 = wl.make_experts(cfg, "cuda", 5)
    shape = MoEShape.from_config(cfg)
    z = torch.empty(P, cfg.d, dtype=torch.bfloat16, device="cuda")
    ws = moe.workspace(shape)
    moe.moe_ffn(x_perm, torch.from_numpy(offsets).cuda(), w13, w2, z, shape, ws)
    assert moe.moe_check(ws) == moe.MOE_OK
    ref = oracle.expert_outputs(x_perm.double().cpu().numpy(), np.arange(P), offsets,
                                LazyExperts(w13), LazyExperts(w2))
    assert_layer_close(z, ref, f"moe_ffn {cfg.name} T={cfg.T}")


@pytest.mark.parametrize("cfg,offsets", _ffn_shapes(20243, 10),
                         ids=lambda v: v.name if hasattr(v, "name") else "")
def test_ffn_w8a8_random_offsets(cfg, offsets):
    P = int(offsets[-1])
    x_perm = wl.make_hidden(wl.MoEConfig("rows", T=P, d=cfg.d, E=1, k=1, f=64), "cuda", 5)
    W._ffn_case(cfg, seed=5, offsets=offsets, x_perm=x_perm)


def _dispatch_cases(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        T = int(rng.choice([1, 7, 64, 255, 256, 257, 1000, 1025, 3000, 9000]))
        R = int(rng.choice([0, 2, 4, 8, 16, 64]))
        E = (R if R > 1 else 1) * int(rng.integers(1, 17))      # a multiple of R, <= 1024
        k = int(rng.integers(1, min(E, 32) + 1))
        d = 64 * int(rng.integers(1, 5))
        out.append((T, d, E, k, R))
    return out


@pytest.mark.parametrize("T,d,E,k,R", _dispatch_cases(20244, 20))
def test_dispatch_random_shape(T, d, E, k, R):
    """Counts, offsets, permutation, row map, gathered rows and the virtual
    EP layout bit for bit against the oracle (both routing-table kernels: the
    fused one up to 1024 tokens, the four-kernel form above)."""
    P.test_dispatch_bit_exact(T, d, E, k, R)
