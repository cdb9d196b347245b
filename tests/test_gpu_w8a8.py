"""GPU parity of the FP8-activation (W8A8) expert path against the fp64 oracle.

The row quantiser's codes and scales are unique results of their bf16 input
(a power-of-two scale makes the scaling exact), so they must match the
oracle bit for bit.  The layer's tokens are quantised the same way on both
sides; the SwiGLU output is an fp32 (library) or fp64 (oracle) value rounded
to bf16 and then quantised, so a code can differ by one E4M3 unit where the
two roundings straddle a boundary (rare: about one element in 10^4).  The
outputs are compared with the bf16 layer's tolerance: relative L2 <= 5e-3
and per element |delta| <= 2e-2 (1 + |ref|).
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


# ------------------------------------------------------------ row quantiser
def _quant_case(a):
    rows, cols = a.shape
    codes = torch.full((rows, cols), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((rows,), -1.0, dtype=torch.float32, device=DEV)
    moe.moe_quantise_rows_e4m3(a, codes, scales)
    want_c, want_s = oracle.quantise_rows_pow2(np64(a))
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), want_s)


@pytest.mark.parametrize("rows,cols,seed", [(1, 16, 0), (37, 64, 1), (300, 2048, 2),
                                            (9, 7168, 3), (64, 768, 4)])
def test_quantiser_matches_the_oracle_bit_for_bit(rows, cols, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    a = torch.randn(rows, cols, generator=g) * torch.exp(torch.empty(rows, 1).uniform_(
        -20, 20, generator=g))
    _quant_case(a.to(torch.bfloat16).to(DEV))


def test_quantiser_edge_rows():
    cols = 32
    a = torch.zeros(8, cols, dtype=torch.float32)
    # row 0: all zeros (scale 1, codes 0; the -0.0 keeps its sign bit)
    a[0, 3] = -0.0
    # row 1: maximum exactly 448: scale 1, and E4M3 midpoints that tie to even
    a[1, :6] = torch.tensor([448.0, 1.0625, 1.1875, -1.0625, 3 * 2.0 ** -10, 2.0 ** -10])
    # row 2: maximum 448 * 2^5 exactly, and one just above 448 * 2^-3 in row 3
    a[2, 0] = 448.0 * 32
    a[2, 1:5] = torch.tensor([-3.0, 1e-3, -1e-30, 7.0])
    a[3, 0] = 58.0  # bf16 neighbours of 56 = 448 / 8: 58 needs e = -2
    # row 4: bf16 subnormals only (scale below 2^-126)
    a[4, :4] = torch.tensor([2.0 ** -133, -3 * 2.0 ** -133, 2.0 ** -130, 0.0])
    # row 5: huge values
    a[5, :3] = torch.tensor([3.0e38, -1.0e38, 1.0])
    # rows 6, 7: tiny normals and a single nonzero element
    a[6] = torch.linspace(-2.0 ** -120, 2.0 ** -120, cols)
    a[7, 31] = -5.0
    _quant_case(a.to(torch.bfloat16).to(DEV))


# ------------------------------------------------------------ expert FFNs
def _ffn_case(cfg, seed=0, offsets=None, x_perm=None):
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, seed)
    if offsets is None:
        x = wl.make_hidden(cfg, DEV, seed)
        w_g, bias = wl.make_router(cfg, DEV, seed)
        L = oracle.router_logits(np64(x), np64(w_g), None if bias is None else np64(bias))
        idx = oracle.topk_select_sorted(L.astype(np.float32), cfg.k)
        offsets = oracle.expert_offsets(oracle.expert_counts(idx, cfg.E))
        perm, _ = oracle.dispatch_rows(idx, cfg.E)
        x_perm = x[torch.from_numpy(perm).long().to(DEV)].contiguous()
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    P = int(offsets[-1])
    z = torch.empty(P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_w8a8(x_perm, torch.from_numpy(np.asarray(offsets, np.int32)).to(DEV), c13, s13,
                     c2, s2, z, shape, ws)
    _check_clean(ws)
    w13 = oracle.LazyDequant(_Host(c13), _Host(s13))
    w2 = oracle.LazyDequant(_Host(c2), _Host(s2))
    ref = oracle.expert_outputs(np64(x_perm), np.arange(P), offsets, w13, w2,
                                ffn=oracle.w8a8_ffn)
    return assert_layer_close(z, ref, f"moe_ffn_w8a8 {cfg.name} T={cfg.T}")


def test_ffn_w8a8_tiny():
    _ffn_case(wl.TINY)


@pytest.mark.parametrize("T", wl.QWEN_DECODE_SWEEP_T)
def test_ffn_w8a8_qwen_decode(T):
    # T <= 64: one work item per touched expert; T = 256: 128-row tiles
    _ffn_case(wl.QWEN3_30B_A3B_DECODE.with_T(T))


def test_ffn_w8a8_ragged_shapes():
    # d = 320: a partial last 128-column K block of GEMM1 and a partial last
    # 128-row W_down tile; f = 192: a partial K block of GEMM2; 37 tokens
    _ffn_case(wl.MoEConfig("ragged", T=37, d=320, E=3, k=2, f=192))
    _ffn_case(wl.MoEConfig("one-expert", T=100, d=128, E=1, k=1, f=128))
    # at most 64 (token, expert) rows: the per-entry quantiser beside GEMM1,
    # with the same partial K blocks and tiles
    _ffn_case(wl.MoEConfig("ragged-entries", T=7, d=320, E=5, k=3, f=192))
    _ffn_case(wl.MoEConfig("one-row", T=1, d=128, E=1, k=1, f=128))
    # 128-row tiles with the per-entry quantiser (at least 16 experts): ragged
    # widths, and experts of more than one tile (about 128 rows each)
    _ffn_case(wl.MoEConfig("ragged-tiles", T=300, d=320, E=20, k=2, f=192))
    _ffn_case(wl.MoEConfig("multi-tile-entries", T=256, d=256, E=16, k=8, f=384))
    # the per-entry quantiser's register rows end at 1024 columns; 1088 takes
    # the two-pass row quantisation
    _ffn_case(wl.MoEConfig("quant-regs-1024", T=40, d=256, E=20, k=2, f=1024))
    _ffn_case(wl.MoEConfig("quant-two-pass-1088", T=40, d=256, E=20, k=2, f=1088))


@pytest.mark.parametrize("T,counts", [
    (16, [100, 0, 20, 8, 0, 0, 0, 0]),           # an item of 100 rows: 2 passes of 64
    (200, [0, 1, 127, 128, 129, 300, 640, 275]),  # 128-row tiles, ragged
], ids=["T16", "T200"])
def test_ffn_w8a8_caller_offsets(T, counts):
    counts = np.array(counts, dtype=np.int64)
    E, P = counts.size, int(counts.sum())
    k = P // T
    assert T * k == P
    cfg = wl.MoEConfig("w8a8-offsets", T=T, d=256, E=E, k=k, f=384)
    x_perm = wl.make_hidden(cfg.with_T(P), DEV, 3)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    _ffn_case(cfg, 3, offsets=offsets, x_perm=x_perm)


@pytest.mark.parametrize("counts", [
    # CTA-pair regime (T*k >= 128*E): lone-tile experts (<= 128 rows) go to the
    # leftover list (swap-AB kernels), odd tile counts to padded pairs, empty
    # experts to nothing
    [600, 100, 300, 50, 0, 50, 0, 1],
    [0, 128, 1, 127, 64, 8, 9, 1024 + 129],
], ids=["mixed", "lone"])
def test_ffn_w8a8_pair_regime_tile_kinds(counts):
    counts = np.array(counts, dtype=np.int64)
    E, P = counts.size, int(counts.sum())
    cfg = wl.MoEConfig("w8a8-pairs", T=P, d=256, E=E, k=1, f=384)
    assert P > 256 and P >= 128 * E
    x_perm = wl.make_hidden(cfg, DEV, 7)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    _ffn_case(cfg, 7, offsets=offsets, x_perm=x_perm)


def test_ffn_w8a8_pair_regime_ragged_widths():
    # f = 192: a partial 128-column gate tile; d = 320: a partial 256-column
    # output tile and partial last K blocks on both GEMMs
    counts = np.array([300, 129, 0, 700], dtype=np.int64)
    E, P = counts.size, int(counts.sum())
    cfg = wl.MoEConfig("w8a8-pairs-ragged", T=P, d=320, E=E, k=1, f=192)
    x_perm = wl.make_hidden(cfg, DEV, 8)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    _ffn_case(cfg, 8, offsets=offsets, x_perm=x_perm)


# ------------------------------------------------------------ whole layer
def _forward_case(cfg, sample=None, seed=0):
    x = wl.make_hidden(cfg, DEV, seed)
    w_g, bias = wl.make_router(cfg, DEV, seed)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, seed)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    moe.moe_forward_w8a8(x, w_g, bias, c13, s13, c2, s2, y, shape, ws, idx_out=idx)
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
    ref = oracle.moe_forward_w8a8(x64, wg64, b64, _Host(c13), _Host(s13), _Host(c2),
                                  _Host(s2), cfg.k, idx=np.array(sel, dtype=np.int32))
    return assert_layer_close(y[torch.from_numpy(toks).long().to(DEV)], ref["y"],
                              f"moe_forward_w8a8 {cfg.name} T={cfg.T}")


def test_forward_w8a8_tiny():
    _forward_case(wl.TINY)


@pytest.mark.parametrize("T", [1, 8, 64, 256])
def test_forward_w8a8_qwen_decode(T):
    _forward_case(wl.QWEN3_30B_A3B_DECODE.with_T(T))


@pytest.mark.parametrize("T", [1, 64])
def test_forward_w8a8_deepseek(T):
    sample = None if T == 1 else np.array([0, 1, 17, 40, 63])
    _forward_case(wl.DEEPSEEK_V3_ROUTED.with_T(T), sample=sample)


@pytest.mark.parametrize("cfg", [wl.QWEN3_30B_A3B_DECODE.with_T(257),
                                 wl.QWEN3_30B_A3B_PREFILL,
                                 wl.DEEPSEEK_V3_ROUTED.with_T(512)], ids=lambda c: c.name)
def test_forward_w8a8_large_batches(cfg):
    # above 256 tokens: the CTA-pair kernels once experts average 128 rows (the
    # prefill), the swap-AB kernels on 128-row tiles below that (T = 257,
    # DeepSeek-V3 at T = 512)
    _forward_case(cfg, sample=None if cfg.T <= 257 else token_sample())


def test_forward_w8a8_layer_graph_replay_is_deterministic():
    cfg = wl.QWEN3_30B_A3B_DECODE
    x = wl.make_hidden(cfg, DEV, 3)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, 0)
    layer = moe.MoELayer(w_g, bias, c13, c2, cfg.k, w13_scale=s13, w2_scale=s2,
                         fp8_activations=True)
    y_eager = layer(x).clone()
    assert layer.check() == moe.MOE_OK
    y1 = layer.forward_graphed(x).clone()
    y2 = layer.forward_graphed(x).clone()
    assert layer.check() == moe.MOE_OK
    assert torch.equal(y_eager, y1) and torch.equal(y1, y2)


def test_forward_w8a8_ffn_equals_forward_on_the_same_rows():
    # the layer's expert outputs equal moe_ffn_w8a8 on the layer's own dispatch
    # (the gather-fused quantiser and the plain one give the same codes)
    cfg = wl.QWEN3_30B_A3B_DECODE
    x = wl.make_hidden(cfg, DEV, 4)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    c13, s13, c2, s2 = wl.make_experts_fp8(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    moe.moe_forward_w8a8(x, w_g, bias, c13, s13, c2, s2, y, shape, ws, idx_out=idx, w_out=w)
    _check_clean(ws)
    idx_h = idx.cpu().numpy()
    offsets = oracle.expert_offsets(oracle.expert_counts(idx_h, cfg.E))
    perm, row_of = oracle.dispatch_rows(idx_h, cfg.E)
    x_perm = x[torch.from_numpy(perm).long().to(DEV)].contiguous()
    ws2 = moe.workspace(shape)
    z = torch.empty(cfg.P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn_w8a8(x_perm, torch.from_numpy(offsets).to(DEV), c13, s13, c2, s2, z, shape, ws2)
    _check_clean(ws2)
    y2 = torch.empty_like(y)
    moe.moe_combine(z, torch.from_numpy(row_of).to(DEV), w, y2, shape)
    assert torch.equal(y, y2)
