"""GPU parity: every C-ABI entry point against the fp64 oracle.

Routing (expert ids, counts, offsets, permutation, virtual-EP send counts) is
compared bit-exactly on the same fp32 logits; outputs with bf16 inputs and
fp32 accumulation must meet relative L2 <= 5e-3 and per element
|delta| <= 2e-2 (1 + |ref|).  Inputs are seeded synthetic tensors from the
workload generator; the oracle never sees a value computed by the library
except where a full-layer test validates a near-tie selection (see
``_check_forward``).
"""

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape

from parity_utils import (LazyExperts, assert_layer_close, logit_bound,
                          logit_bound_tensor_cores, np64, order_by_logit,
                          selection_is_valid, token_sample, unique_selection)

ROUTER_TC_MIN_T = 257  # from this batch size the router runs on the tensor cores


def router_bound(T, x64, wg64, b64):
    if T >= ROUTER_TC_MIN_T:
        return logit_bound_tensor_cores(x64, wg64, b64)
    return logit_bound(x64, wg64, b64)

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


# ---------------------------------------------------------------- failure path
def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    moe.moe_selftest_bounded_wait(1_000_000, ws)  # 1 ms limit, nothing arrives
    assert moe.moe_check(ws) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_check(ws) == moe.MOE_OK  # cleared; the context is still usable
    torch.ones(4, device=DEV).sum().item()


# ---------------------------------------------------------------- top-k
TOPK_CASES = [  # (T, E, k)
    (300, 8, 2), (1000, 128, 8), (517, 256, 8), (64, 1024, 32), (33, 6, 6),
    (5, 1, 1), (1, 128, 8), (4097, 64, 4), (40, 16, 16),
]


@pytest.mark.parametrize("kind", ["normal", "ties", "const"])
@pytest.mark.parametrize("T,E,k", TOPK_CASES)
def test_topk_bit_exact(kind, T, E, k):
    L = wl.make_logits(T, E, device="cpu", seed=T * 7 + E, kind=kind)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    moe.moe_topk(L.to(DEV), idx, w, MoEShape.of(T, 64, E, k, 64))
    ref_idx = oracle.topk_select_sorted(L.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    if T * E <= 20000:
        np.testing.assert_array_equal(ref_idx, oracle.topk_select(L.numpy(), k))
    ref_w = oracle.gate_weights(L.numpy().astype(np.float64), ref_idx)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-7)


def test_topk_signed_zeros_tie():
    L = torch.tensor([[-0.0, 0.0, -1.0, -0.0, 0.0, 0.5]], dtype=torch.float32)
    idx = torch.empty(1, 4, dtype=torch.int32, device=DEV)
    w = torch.empty(1, 4, dtype=torch.float32, device=DEV)
    moe.moe_topk(L.to(DEV), idx, w, MoEShape.of(1, 64, 6, 4, 64))
    assert idx.cpu().tolist() == [[5, 0, 1, 3]]


@pytest.mark.parametrize("cfg", [wl.QWEN3_30B_A3B_DECODE.with_T(256),
                                 wl.DEEPSEEK_V3_ROUTED.with_T(512)], ids=lambda c: c.name)
def test_topk_on_router_logits_of_model_shapes(cfg):
    """Selection on the fp32 rounding of the oracle's router logits."""
    x = wl.make_hidden(cfg, "cpu", 0)
    w_g, bias = wl.make_router(cfg, "cpu", 0)
    L32 = oracle.router_logits(np64(x), np64(w_g), np64(bias)).astype(np.float32)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    moe.moe_topk(torch.from_numpy(L32).to(DEV), idx, w, MoEShape.from_config(cfg))
    np.testing.assert_array_equal(idx.cpu().numpy(), oracle.topk_select_sorted(L32, cfg.k))


# ---------------------------------------------------------------- router
@pytest.mark.parametrize("cfg", [wl.TINY, wl.QWEN3_30B_A3B_DECODE.with_T(256),
                                 wl.DEEPSEEK_V3_ROUTED.with_T(64),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(1),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(257),
                                 wl.QWEN3_30B_A3B_PREFILL.with_T(4096),
                                 wl.DEEPSEEK_V3_ROUTED.with_T(1000),
                                 wl.MIXTRAL_8X7B.with_T(700),
                                 # E not a multiple of 4: the tensor-core epilogue's scalar stores
                                 wl.MoEConfig("router-odd-E", T=300, d=256, E=6, k=2, f=64,
                                              zipf_s=1.0),
                                 # cluster router: one token in a 32-token tile (the warps
                                 # that multiply a single row), 448-deep K slices
                                 wl.DEEPSEEK_V3_ROUTED.with_T(1),
                                 # 64-expert tiles (the 32-expert grid would need 336 CTAs)
                                 # with a partial last expert tile and an 8-token last tile
                                 wl.MoEConfig("router-64-wide", T=200, d=1024, E=96, k=4, f=64,
                                              zipf_s=1.0),
                                 # 32-expert tiles, a partial expert tile, a 5-token last tile
                                 wl.MoEConfig("router-partial", T=37, d=512, E=40, k=2, f=64,
                                              zipf_s=1.0)],
                         ids=lambda c: f"{c.name}-T{c.T}")
def test_router_within_fp32_error_bound(cfg):
    x = wl.make_hidden(cfg, "cpu", 0)
    w_g, bias = wl.make_router(cfg, "cpu", 0)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=DEV)
    shape = MoEShape.from_config(cfg)
    moe.moe_router(x.to(DEV), w_g.to(DEV), None if bias is None else bias.to(DEV), logits,
                   shape, moe.workspace(shape))
    x64, wg64, b64 = np64(x), np64(w_g), (None if bias is None else np64(bias))
    ref = oracle.router_logits(x64, wg64, b64)
    err = np.abs(np64(logits) - ref)
    bound = router_bound(cfg.T, x64, wg64, b64)
    assert np.all(err <= bound), float((err / bound).max())
    # typical error is far inside the bound: fp32-level agreement
    assert np.median(err / (np.abs(x64) @ np.abs(wg64) + 1e-30)) < 1e-6


# ---------------------------------------------------------------- dispatch
DISPATCH_CASES = [  # (T, d, E, k, R)
    (64, 256, 8, 2, 0), (300, 128, 8, 2, 4), (1, 2048, 128, 8, 0), (517, 64, 256, 8, 8),
    (1000, 128, 128, 8, 0), (16384, 64, 256, 8, 8), (5, 64, 4, 4, 2), (2049, 64, 1024, 32, 64),
]


@pytest.mark.parametrize("T,d,E,k,R", DISPATCH_CASES)
def test_dispatch_bit_exact(T, d, E, k, R):
    L = wl.make_logits(T, E, device="cpu", seed=T + 11 * E)
    ref_idx = oracle.topk_select_sorted(L.numpy(), k)
    x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), "cpu", 1)
    shape = MoEShape.of(T, d, E, k, 64, R)
    ws = moe.workspace(shape)
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(P, dtype=torch.int32, device=DEV)
    row_of = torch.empty(T, k, dtype=torch.int32, device=DEV)
    x_perm = torch.empty(P, d, dtype=torch.bfloat16, device=DEV)
    send = torch.empty(R, R, dtype=torch.int32, device=DEV) if R > 1 else None
    roff = torch.empty(R + 1, dtype=torch.int32, device=DEV) if R > 1 else None
    xd = x.to(DEV)
    moe.moe_dispatch(torch.from_numpy(ref_idx).to(DEV), xd, counts, offsets, perm, row_of,
                     x_perm, shape, ws, send, roff)
    _check_clean(ws)
    ref_counts = oracle.expert_counts(ref_idx, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref_counts)
    np.testing.assert_array_equal(offsets.cpu().numpy(), oracle.expert_offsets(ref_counts))
    ref_perm, ref_row_of = oracle.dispatch_rows(ref_idx, E)
    np.testing.assert_array_equal(perm.cpu().numpy(), ref_perm)
    np.testing.assert_array_equal(row_of.cpu().numpy(), ref_row_of)
    assert torch.equal(x_perm.cpu(), x[torch.from_numpy(ref_perm).long()])
    if R > 1:
        S, ro = oracle.virtual_ep_layout(ref_idx, E, R)
        np.testing.assert_array_equal(send.cpu().numpy(), S)
        np.testing.assert_array_equal(roff.cpu().numpy(), ro)


def test_dispatch_records_bad_expert_ids():
    T, d, E, k = 40, 64, 8, 2
    idx = torch.tensor([[0, 1]] * T, dtype=torch.int32)
    idx[3, 1] = 9      # out of range
    idx[7, 0] = -1     # out of range
    idx[9] = torch.tensor([2, 2])  # repeated expert
    shape = MoEShape.of(T, d, E, k, 64)
    ws = moe.workspace(shape)
    x = torch.zeros(T, d, dtype=torch.bfloat16, device=DEV)
    outs = [torch.full((E,), -7, dtype=torch.int32, device=DEV),
            torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
            torch.full((T * k,), -7, dtype=torch.int32, device=DEV),
            torch.full((T, k), -7, dtype=torch.int32, device=DEV),
            torch.zeros(T * k, d, dtype=torch.bfloat16, device=DEV)]
    moe.moe_dispatch(idx.to(DEV), x, *outs, shape, ws)
    assert moe.moe_check(ws) == moe.MOE_ERR_DEVICE_CHECK
    torch.ones(2, device=DEV).sum().item()  # context still healthy


def test_empty_batch_dispatch_zeroes_tables():
    shape = MoEShape.of(0, 64, 8, 2, 64, 4)
    ws = moe.workspace(shape)
    counts = torch.full((8,), 5, dtype=torch.int32, device=DEV)
    offsets = torch.full((9,), 5, dtype=torch.int32, device=DEV)
    send = torch.full((4, 4), 5, dtype=torch.int32, device=DEV)
    roff = torch.full((5,), 5, dtype=torch.int32, device=DEV)
    e = torch.empty(0, dtype=torch.int32, device=DEV)
    moe.moe_dispatch(None, None, counts, offsets, None, None, None, shape, ws, send, roff)
    assert counts.sum().item() == 0 and offsets.sum().item() == 0
    assert send.sum().item() == 0 and roff.sum().item() == 0
    del e


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("T,d,E,k", [(64, 256, 8, 2), (333, 2048, 128, 8), (1, 7168, 256, 8),
                                     # large batches: 512 columns per warp, and d off that grid
                                     (2049, 2048, 64, 4), (2000, 2304, 32, 3)])
def test_combine_matches_oracle(T, d, E, k):
    L = wl.make_logits(T, E, device="cpu", seed=5 + T)
    idx = oracle.topk_select_sorted(L.numpy(), k)
    w = oracle.gate_weights(L.numpy().astype(np.float64), idx).astype(np.float32)
    perm, row_of = oracle.dispatch_rows(idx, E)
    z = wl.make_hidden(wl.MoEConfig("z", T=T * k, d=d, E=E, k=k, f=64), "cpu", 3)
    y = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(z.to(DEV), torch.from_numpy(row_of).to(DEV), torch.from_numpy(w).to(DEV),
                    y, MoEShape.of(T, d, E, k, 64))
    ref = oracle.combine(np64(z), row_of, w.astype(np.float64))
    assert_layer_close(y, ref, "combine")


def test_dispatch_then_combine_identity_k1():
    T, d, E, k = 200, 512, 16, 1
    L = wl.make_logits(T, E, device="cpu", seed=77)
    idx = torch.from_numpy(oracle.topk_select_sorted(L.numpy(), k)).to(DEV)
    x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), "cpu", 9).to(DEV)
    shape = MoEShape.of(T, d, E, k, 64)
    ws = moe.workspace(shape)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T, dtype=torch.int32, device=DEV)
    row_of = torch.empty(T, k, dtype=torch.int32, device=DEV)
    x_perm = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(idx, x, counts, offsets, perm, row_of, x_perm, shape, ws)
    y = torch.empty_like(x)
    moe.moe_combine(x_perm, row_of, torch.ones(T, k, device=DEV), y, shape)
    assert torch.equal(y, x)  # unit gates, identity experts: bit-exact


# ---------------------------------------------------------------- expert FFN
def _ffn_case(cfg, seed=0, sample_rows=None):
    """Oracle-made dispatch of the layer's tokens, then moe_ffn vs oracle z."""
    x = wl.make_hidden(cfg, DEV, seed)
    w_g, bias = wl.make_router(cfg, DEV, seed)
    w13, w2 = wl.make_experts(cfg, DEV, seed)
    L32 = oracle.router_logits(np64(x), np64(w_g), None if bias is None else np64(bias))
    idx = oracle.topk_select_sorted(L32.astype(np.float32), cfg.k)
    counts = oracle.expert_counts(idx, cfg.E)
    offsets = oracle.expert_offsets(counts)
    perm, _ = oracle.dispatch_rows(idx, cfg.E)
    x_perm = x[torch.from_numpy(perm).long().to(DEV)].contiguous()
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    z = torch.empty(cfg.P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn(x_perm, torch.from_numpy(offsets).to(DEV), w13, w2, z, shape, ws)
    _check_clean(ws)
    rows = np.arange(cfg.P) if sample_rows is None else sample_rows(offsets, counts)
    # expert of each sampled row
    exp_of = np.searchsorted(offsets, rows, side="right") - 1
    xp = np64(x_perm[torch.from_numpy(rows).long().to(DEV)])
    lazy13, lazy2 = LazyExperts(w13), LazyExperts(w2)
    ref = np.zeros((rows.size, cfg.d))
    for e in np.unique(exp_of):
        sel = exp_of == e
        ref[sel] = oracle.swiglu_ffn(xp[sel], lazy13[e], lazy2[e])
    got = z[torch.from_numpy(rows).long().to(DEV)]
    return assert_layer_close(got, ref, f"moe_ffn {cfg.name}")


def _sample_rows(n_random=256, seed=0):
    """Rows of the expert-major buffer to check: the first and last row of
    every touched expert, the rows on both sides of every 128-row tile
    boundary inside an expert (where a tile-indexing mistake would show),
    and a seeded random sample of n_random rows."""
    def pick(offsets, counts):
        rng = np.random.default_rng(seed)
        offsets = np.asarray(offsets, dtype=np.int64)
        touched = np.nonzero(counts)[0]
        rows = [offsets[touched], offsets[touched + 1] - 1]
        for e in touched:
            a, b = offsets[e], offsets[e + 1]
            edges = np.arange(a + 128, b, 128)
            rows += [edges - 1, edges]
        rows.append(rng.integers(0, offsets[-1], n_random))
        return np.unique(np.concatenate(rows))
    return pick


def test_ffn_tiny_full():
    _ffn_case(wl.TINY)


@pytest.mark.parametrize("T", wl.QWEN_DECODE_SWEEP_T)
def test_ffn_qwen_decode_full(T):
    _ffn_case(wl.QWEN3_30B_A3B_DECODE.with_T(T))


def test_ffn_ragged_rows_and_single_expert():
    _ffn_case(wl.MoEConfig("ragged", T=301, d=320, E=3, k=2, f=192))
    _ffn_case(wl.MoEConfig("one-expert", T=129, d=128, E=1, k=1, f=128))


@pytest.mark.parametrize("counts", [
    # CTA-pair regime (T*k >= 128*E): lone-tile experts (<= 128 rows) go to the
    # single-CTA list, odd tile counts (300 -> 3, 600 -> 5 tiles) to padded pairs,
    # empty experts to nothing
    [600, 100, 300, 50, 0, 50, 0, 1],
    # every expert a lone tile but one, the first empty
    [0, 128, 1, 127, 64, 8, 9, 1024 + 129],
], ids=["mixed", "lone"])
def test_ffn_pair_regime_tile_kinds(counts):
    """moe_ffn on caller offsets chosen to hit each kind of work item of the
    large-batch GEMMs, checked row by row against the oracle."""
    counts = np.array(counts, dtype=np.int64)
    E, P = counts.size, int(counts.sum())
    cfg = wl.MoEConfig("tile-kinds", T=P, d=256, E=E, k=1, f=384)
    x_perm = wl.make_hidden(cfg, DEV, 7)
    w13, w2 = wl.make_experts(cfg, DEV, 7)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    z = torch.empty(P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn(x_perm, torch.from_numpy(offsets).to(DEV), w13, w2, z, shape, ws)
    _check_clean(ws)
    xp = np64(x_perm)
    ref = np.zeros((P, cfg.d))
    lazy13, lazy2 = LazyExperts(w13), LazyExperts(w2)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            ref[a:b] = oracle.swiglu_ffn(xp[a:b], lazy13[e], lazy2[e])
    assert_layer_close(z, ref, "moe_ffn tile kinds")


@pytest.mark.parametrize("T,counts", [
    # T <= 64: one item per expert of at most 64 rows; 100 rows -> 2 passes
    (16, [100, 0, 20, 8, 0, 0, 0, 0]),
    # T <= 64: items of at most 64 rows; 300 rows -> 5 passes, 65 -> 2
    (64, [300, 1, 64, 65, 0, 82, 0, 0]),
    # 64 < T <= 256: 128-row tiles
    (200, [1000, 300, 0, 300, 0, 0, 0, 0]),
], ids=["T16", "T64", "T200"])
def test_ffn_small_batch_expert_with_more_rows_than_tokens(T, counts):
    """moe_ffn at decode batch sizes on caller offsets that give one expert
    more rows than the batch has tokens (the header allows any monotone
    offsets ending at T*k): every row still matches the oracle and no error
    is recorded."""
    counts = np.array(counts, dtype=np.int64)
    E, k = counts.size, 8
    P = int(counts.sum())
    assert P == T * k
    cfg = wl.MoEConfig("swap-passes", T=T, d=256, E=E, k=k, f=384)
    x_perm = wl.make_hidden(cfg.with_T(P), DEV, 11)
    w13, w2 = wl.make_experts(cfg, DEV, 11)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    z = torch.empty(P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn(x_perm, torch.from_numpy(offsets).to(DEV), w13, w2, z, shape, ws)
    _check_clean(ws)
    xp = np64(x_perm)
    ref = np.zeros((P, cfg.d))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            ref[a:b] = oracle.swiglu_ffn(xp[a:b], np64(w13[e]), np64(w2[e]))
    assert_layer_close(z, ref, f"moe_ffn T={T} oversized expert")


def test_ffn_qwen_prefill_sampled():
    _ffn_case(wl.QWEN3_30B_A3B_PREFILL, sample_rows=_sample_rows())


def test_ffn_mixtral_sampled():
    _ffn_case(wl.MIXTRAL_8X7B.with_T(1024), sample_rows=_sample_rows())


def test_ffn_deepseek_full():
    # every row of every touched expert (512 rows over the experts the
    # Zipf-skewed batch touches)
    _ffn_case(wl.DEEPSEEK_V3_ROUTED.with_T(64))


def test_ffn_deepseek_large_batch_sampled():
    # T = 512: single-CTA 128-row tiles over sparse, skewed experts
    _ffn_case(wl.DEEPSEEK_V3_ROUTED.with_T(512), sample_rows=_sample_rows())


# ---------------------------------------------------------------- whole layer
def _check_forward(cfg, sample=None, seed=0):
    """moe_forward vs the oracle.

    The library selects on its fp32 logits; the oracle's fp64 logits differ by
    at most the fp32 dot-product error bound.  Where that bound leaves one
    possible selection, it must be the library's.  Where two selections are
    both consistent with the bound (a near-tie at the k-th slot), the
    library's must be one of them, and its output is compared with the
    oracle's output for that (valid) selection.
    """
    x = wl.make_hidden(cfg, DEV, seed)
    w_g, bias = wl.make_router(cfg, DEV, seed)
    w13, w2 = wl.make_experts(cfg, DEV, seed)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    gw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    moe.moe_forward(x, w_g, bias, w13, w2, y, shape, ws, idx, gw, counts)
    _check_clean(ws)
    idx_h = idx.cpu().numpy()
    # routing totals hold for the whole batch
    np.testing.assert_array_equal(counts.cpu().numpy(), oracle.expert_counts(idx_h, cfg.E))
    toks = np.arange(cfg.T) if sample is None else sample(idx_h, counts.cpu().numpy())
    x64 = np64(x[torch.from_numpy(toks).long().to(DEV)])
    wg64 = np64(w_g)
    b64 = None if bias is None else np64(bias)
    L64 = oracle.router_logits(x64, wg64, b64)
    delta = router_bound(cfg.T, x64, wg64, b64)
    sel = []
    flips = 0
    for i, t in enumerate(toks):
        g = idx_h[t].tolist()
        assert selection_is_valid(L64[i], delta[i], g), (t, g)
        u = unique_selection(L64[i], delta[i], cfg.k)
        if u is not None:
            assert set(g) == u, (t, g, u)
        else:
            flips += int(set(g) != set(np.argsort(-L64[i], kind="stable")[:cfg.k].tolist()))
        sel.append(order_by_logit(L64[i], g))
    ref = oracle.moe_forward(x64, wg64, b64, LazyExperts(w13), LazyExperts(w2), cfg.k,
                             idx=np.array(sel, dtype=np.int32))
    got_w = gw.cpu().numpy()[toks]
    # gates: compare per expert (the slot order of near-equal logits may differ)
    for i, t in enumerate(toks):
        ref_w = dict(zip(ref["idx"][i].tolist(), ref["w"][i].tolist()))
        for j, e in enumerate(idx_h[t].tolist()):
            assert abs(got_w[i, j] - ref_w[e]) <= 4 * delta[i].max() + 2e-6
    rel = assert_layer_close(y[torch.from_numpy(toks).long().to(DEV)], ref["y"],
                             f"moe_forward {cfg.name}")
    return rel, flips


def test_forward_tiny():
    _check_forward(wl.TINY)


@pytest.mark.parametrize("T", wl.QWEN_DECODE_SWEEP_T)
def test_forward_qwen_decode(T):
    _check_forward(wl.QWEN3_30B_A3B_DECODE.with_T(T))


def test_forward_qwen_prefill_sampled():
    _check_forward(wl.QWEN3_30B_A3B_PREFILL, sample=token_sample())


def test_forward_mixtral_sampled():
    _check_forward(wl.MIXTRAL_8X7B, sample=token_sample())


@pytest.mark.parametrize("T", [1, 64, 512, 16384])
def test_forward_deepseek(T):
    # T <= 64: every token.  T = 512: single-CTA tiles over sparse experts;
    # T = 16384: multi-block routing tables and CTA-pair tiles with E = 256;
    # both on a 256-token sample that includes tokens routed to the hottest
    # and the coldest experts.
    _check_forward(wl.DEEPSEEK_V3_ROUTED.with_T(T), sample=None if T <= 64 else token_sample())


@pytest.mark.parametrize("cfg", [
    # 2-SM tile pairs, routing in one block (T <= 1024)
    wl.MoEConfig("pairs-fused", T=1000, d=256, E=8, k=2, f=512),
    # 2-SM tile pairs, multi-block routing; d and f not multiples of 256 / 128
    wl.MoEConfig("pairs-tables", T=1100, d=192, E=4, k=1, f=320),
    # sparse experts: single-CTA 128 x 128 tiles
    wl.MoEConfig("narrow", T=600, d=256, E=64, k=2, f=256),
    # single-CTA 128 x 256 tiles
    wl.MoEConfig("wide", T=700, d=256, E=16, k=2, f=256),
], ids=lambda c: c.name)
def test_forward_large_batch_gemm_regimes(cfg):
    _check_forward(cfg)


@pytest.mark.parametrize("cfg", [wl.QWEN3_30B_A3B_DECODE.with_T(1),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(16),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(17),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(64),
                                 wl.QWEN3_30B_A3B_DECODE.with_T(256),
                                 wl.MoEConfig("ragged-combine", T=37, d=320, E=6, k=3, f=128),
                                 wl.MoEConfig("ragged-direct", T=13, d=320, E=6, k=3, f=128)],
                         ids=["T1", "T16", "T17", "T64", "T256", "ragged", "ragged-direct"])
def test_forward_equals_ffn_then_combine(cfg):
    """moe_forward's y equals moe_combine over moe_ffn's z on the layer's own
    dispatch bit for bit (the layer's gather, GEMMs and combine against the
    caller-offset FFN and the standalone combine), including a partial last
    128-column tile (d = 320), and again on a second call on the same
    workspace.  Up to 16 tokens the layer's GEMM1 reads x itself (no gather)
    and maps rows in its epilogue (T = 1, 13, 16; T = 17 is the first size
    with the gather)."""
    x = wl.make_hidden(cfg, DEV, 4)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    w13, w2 = wl.make_experts(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    for _ in range(2):  # the second call runs on counters the first one used
        y.fill_(float("nan"))
        moe.moe_forward(x, w_g, bias, w13, w2, y, shape, ws, idx_out=idx, w_out=w)
        _check_clean(ws)
    idx_h = idx.cpu().numpy()
    offsets = oracle.expert_offsets(oracle.expert_counts(idx_h, cfg.E))
    perm, row_of = oracle.dispatch_rows(idx_h, cfg.E)
    x_perm = x[torch.from_numpy(perm).long().to(DEV)].contiguous()
    ws2 = moe.workspace(shape)
    z = torch.empty(cfg.P, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_ffn(x_perm, torch.from_numpy(offsets).to(DEV), w13, w2, z, shape, ws2)
    _check_clean(ws2)
    y2 = torch.empty_like(y)
    moe.moe_combine(z, torch.from_numpy(row_of).to(DEV), w, y2, shape)
    assert torch.equal(y, y2)


def test_forward_k_equals_E_and_single_expert():
    _check_forward(wl.MoEConfig("dense-k=E", T=70, d=128, E=4, k=4, f=128))
    _check_forward(wl.MoEConfig("E=1", T=33, d=256, E=1, k=1, f=192))


def test_forward_is_deterministic():
    cfg = wl.QWEN3_30B_A3B_DECODE.with_T(64)
    x = wl.make_hidden(cfg, DEV, 0)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    w13, w2 = wl.make_experts(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    ys = []
    for _ in range(3):
        y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
        moe.moe_forward(x, w_g, bias, w13, w2, y, shape, ws)
        ys.append(y)
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


@pytest.mark.parametrize("T", [512, 64, 1])
def test_forward_matches_router_then_topk(T):
    """moe_forward's routing equals moe_topk(moe_router(x)) bit for bit (the
    tensor-core router at T = 512; the cluster router with 64-expert tiles
    at T = 64 and with single-row warps at T = 1)."""
    cfg = wl.DEEPSEEK_V3_ROUTED.with_T(T)
    import dataclasses
    cfg = dataclasses.replace(cfg, f=64)
    x = wl.make_hidden(cfg, DEV, 0)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    w13, w2 = wl.make_experts(cfg, DEV, 0)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=DEV)
    moe.moe_router(x, w_g, bias, logits, shape, ws)
    i1 = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    g1 = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    moe.moe_topk(logits, i1, g1, shape)
    i2 = torch.empty_like(i1)
    g2 = torch.empty_like(g1)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(x, w_g, bias, w13, w2, y, shape, ws, i2, g2)
    assert torch.equal(i1, i2) and torch.equal(g1, g2)


def test_layer_graph_replay_matches_eager():
    """MoELayer's captured-graph path gives the eager call's bits."""
    cfg = wl.QWEN3_30B_A3B_DECODE.with_T(8)
    t = wl.make_layer(cfg, DEV, 0)
    layer = moe.MoELayer(t["w_g"], t["bias"], t["w13"], t["w2"], cfg.k)
    y_eager = layer(t["x"]).clone()
    y_graph = layer.forward_graphed(t["x"]).clone()
    x2 = wl.make_hidden(cfg, DEV, 5)
    y2_graph = layer.forward_graphed(x2).clone()  # replay with new contents
    y2_eager = layer(x2)
    x_host = t["x"].cpu().pin_memory()
    y_host = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()
    layer.forward_host(x_host, y_host)
    torch.cuda.synchronize()
    assert layer.check() == moe.MOE_OK
    assert torch.equal(y_eager, y_graph) and torch.equal(y2_eager, y2_graph)
    assert torch.equal(y_host, y_eager.cpu())
    # the host graph re-reads the pinned input on every replay
    x_host.copy_(x2.cpu())
    layer.forward_host(x_host, y_host)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y2_eager.cpu())
