"""GPU parity of the FP8-weight expert path (E4M3 codes, fp32 row scales)
against the fp64 oracle.

The oracle dequantises the same codes and scales exactly and runs the bf16
layer's definition on them, so the tolerance is the bf16 path's: relative L2
<= 5e-3 and per element |delta| <= 2e-2 (1 + |ref|).  Routing is unaffected by
the expert weights and is checked as in the bf16 tests.
"""

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape

from parity_utils import (assert_layer_close, logit_bound, logit_bound_tensor_cores, np64,
                          order_by_logit, selection_is_valid, token_sample, unique_selection)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()


def _check_clean(ws):
    st = moe.moe_check(ws)
    assert st == moe.MOE_OK, moe.moe_error_string(st)


class _Host:
    """Expert-indexed host copies of a device tensor, fetched on demand."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[int(e)].cpu().numpy()


def _ffn_fp8_case(cfg, seed=0):
    """Oracle-made dispatch, then moe_ffn_fp8 against the oracle per row."""
    x = wl.make_hidden(cfg, DEV, seed)
    w_g, bias = wl.make_router(cfg, DEV, seed)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, seed)
    L = oracle.router_logits(np64(x), np64(w_g), None if bias is None else np64(bias))
    idx = oracle.topk_select_sorted(L.astype(np.float32), cfg.k)
    counts = oracle.expert_counts(idx, cfg.E)
    offsets = oracle.expert_offsets(counts)
    perm, _ = oracle.dispatch_rows(idx, cfg.E)
    x_perm = x[torch.from_numpy(perm).long().to(DEV)].contiguous()
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    z = torch.empty(cfg.P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_fp8(x_perm, torch.from_numpy(offsets).to(DEV), c13, s13, c2, s2, z, shape, ws)
    _check_clean(ws)
    w13 = oracle.LazyDequant(_Host(c13), _Host(s13))
    w2 = oracle.LazyDequant(_Host(c2), _Host(s2))
    ref = oracle.expert_outputs(np64(x), perm, offsets, w13, w2)
    return assert_layer_close(z, ref, f"moe_ffn_fp8 {cfg.name} T={cfg.T}")


def test_ffn_fp8_tiny():
    _ffn_fp8_case(wl.TINY)


@pytest.mark.parametrize("T", wl.QWEN_DECODE_SWEEP_T)
def test_ffn_fp8_qwen_decode(T):
    # T <= 64: one work item per touched expert; T = 256: 128-row tiles
    _ffn_fp8_case(wl.QWEN3_30B_A3B_DECODE.with_T(T))


def test_ffn_fp8_ragged_shapes():
    # d = 320: the last 128-row W_down tile is partial; 37 tokens: ragged
    # 16-row token groups; one expert with all rows.
    _ffn_fp8_case(wl.MoEConfig("ragged", T=37, d=320, E=3, k=2, f=192))
    _ffn_fp8_case(wl.MoEConfig("one-expert", T=100, d=128, E=1, k=1, f=128))


def _forward_fp8_case(cfg, sample=None, seed=0):
    """moe_forward_fp8 against the oracle (routing validated as in the bf16
    tests: a near-tie selection must be one the fp32 error bound allows, and
    the output is compared for the library's selection)."""
    x = wl.make_hidden(cfg, DEV, seed)
    w_g, bias = wl.make_router(cfg, DEV, seed)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, seed)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    gw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    moe.moe_forward_fp8(x, w_g, bias, c13, s13, c2, s2, y, shape, ws, idx_out=idx, w_out=gw)
    _check_clean(ws)
    idx_h = idx.cpu().numpy()
    if sample is None:
        toks = np.arange(cfg.T)
    elif callable(sample):
        toks = sample(idx_h, oracle.expert_counts(idx_h, cfg.E))
    else:
        toks = sample
    x64 = np64(x[torch.from_numpy(toks).long().to(DEV)])
    wg64, b64 = np64(w_g), None if bias is None else np64(bias)
    L64 = oracle.router_logits(x64, wg64, b64)
    # above 256 tokens the router runs on the tensor cores
    bound = logit_bound_tensor_cores if cfg.T > 256 else logit_bound
    delta = bound(x64, wg64, b64)
    sel = []
    for i, t in enumerate(toks):
        g = idx_h[t].tolist()
        assert selection_is_valid(L64[i], delta[i], g), (t, g)
        u = unique_selection(L64[i], delta[i], cfg.k)
        if u is not None:
            assert set(g) == u, (t, g, u)
        sel.append(order_by_logit(L64[i], g))
    ref = oracle.moe_forward_fp8(x64, wg64, b64, _Host(c13), _Host(s13), _Host(c2), _Host(s2),
                                 cfg.k, idx=np.array(sel, dtype=np.int32))
    return assert_layer_close(y[torch.from_numpy(toks).long().to(DEV)], ref["y"],
                              f"moe_forward_fp8 {cfg.name} T={cfg.T}")


def test_forward_fp8_tiny():
    _forward_fp8_case(wl.TINY)


@pytest.mark.parametrize("T", [1, 64, 256])
def test_forward_fp8_qwen_decode(T):
    _forward_fp8_case(wl.QWEN3_30B_A3B_DECODE.with_T(T))


@pytest.mark.parametrize("T", [1, 64])
def test_forward_fp8_deepseek(T):
    # d = 7168, f = 2048, E = 256: 112 K-stages per GEMM1 item; sampled tokens
    sample = None if T == 1 else np.array([0, 1, 17, 40, 63])
    _forward_fp8_case(wl.DEEPSEEK_V3_ROUTED.with_T(T), sample=sample)


@pytest.mark.parametrize("cfg", [wl.QWEN3_30B_A3B_DECODE.with_T(257),
                                 wl.QWEN3_30B_A3B_PREFILL,
                                 wl.DEEPSEEK_V3_ROUTED.with_T(512)], ids=lambda c: c.name)
def test_forward_fp8_large_batches(cfg):
    # above 256 tokens: tensor-core router, plain 128-row token tiles (an
    # expert with more rows is several work items); a 256-token sample with
    # tokens of the hottest and coldest experts
    _forward_fp8_case(cfg, sample=None if cfg.T <= 257 else token_sample())


def test_ffn_fp8_large_batch_ragged_tiles():
    # caller offsets: experts of 0, 1, 127, 128, 129, 300 and 640 rows
    counts = np.array([0, 1, 127, 128, 129, 300, 640], dtype=np.int64)
    E, P = counts.size, int(counts.sum())
    cfg = wl.MoEConfig("fp8-tiles", T=P, d=256, E=E, k=1, f=384)
    x_perm = wl.make_hidden(cfg, DEV, 3)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, 3)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    z = torch.empty(P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_fp8(x_perm, torch.from_numpy(offsets).to(DEV), c13, s13, c2, s2, z, shape, ws)
    _check_clean(ws)
    xp = np64(x_perm)
    ref = np.zeros((P, cfg.d))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            w13 = oracle.dequantise_rows(c13[e].cpu().numpy(), s13[e].cpu().numpy())
            w2 = oracle.dequantise_rows(c2[e].cpu().numpy(), s2[e].cpu().numpy())
            ref[a:b] = oracle.swiglu_ffn(xp[a:b], w13, w2)
    assert_layer_close(z, ref, "moe_ffn_fp8 tiles")


def test_forward_fp8_graph_replay_is_deterministic():
    cfg = wl.QWEN3_30B_A3B_DECODE
    x = wl.make_hidden(cfg, DEV, 3)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, 0)
    layer = moe.MoELayer(w_g, bias, c13, c2, cfg.k, w13_scale=s13, w2_scale=s2)
    y_eager = layer(x).clone()
    assert layer.check() == moe.MOE_OK
    y1 = layer.forward_graphed(x).clone()
    y2 = layer.forward_graphed(x).clone()
    assert layer.check() == moe.MOE_OK
    assert torch.equal(y_eager, y1) and torch.equal(y1, y2)


def test_fp8_with_exact_bf16_weights_matches_the_bf16_path():
    # Power-of-two row scales make every dequantised weight an exact bf16
    # value; the FP8 path then multiplies the same fp32 accumulators by
    # powers of two, so it must give the bf16 path's output bit for bit.
    cfg = wl.QWEN3_30B_A3B_DECODE
    x = wl.make_hidden(cfg, DEV, 5)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    c13, _, c2, _ = wl.make_experts_fp8(cfg, DEV, 0)
    g = torch.Generator(device=DEV)
    g.manual_seed(77)
    s13 = torch.pow(2.0, -torch.randint(9, 12, (cfg.E, 2 * cfg.f), generator=g, device=DEV)
                    .float()).contiguous()
    s2 = torch.pow(2.0, -torch.randint(9, 12, (cfg.E, cfg.d), generator=g, device=DEV)
                   .float()).contiguous()
    w13 = (c13.view(torch.float8_e4m3fn).float() * s13[..., None]).to(torch.bfloat16)
    w2 = (c2.view(torch.float8_e4m3fn).float() * s2[..., None]).to(torch.bfloat16)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y8 = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    y16 = torch.empty_like(y8)
    moe.moe_forward_fp8(x, w_g, bias, c13, s13, c2, s2, y8, shape, ws)
    moe.moe_forward(x, w_g, bias, w13, w2, y16, shape, ws)
    _check_clean(ws)
    assert torch.equal(y8, y16)
