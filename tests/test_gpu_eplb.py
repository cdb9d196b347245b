"""GPU parity of expert load balancing with replicated experts.

The plan itself is host code (checked against the oracle in
test_abi_host.py); here the device remap is compared with the oracle bit for
bit, and the replicated-expert layer with the plain layer: replicas carry the
same weights and every output row depends only on its own token, so the
outputs agree bit for bit whenever both pick the same GEMM kernels, and the
per-physical-expert rows must add up to the per-logical-expert rows."""

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape
from parity_utils import (LazyExperts, assert_layer_close, logit_bound, np64,
                          selection_is_valid, unique_selection)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_clean(ws):
    assert moe.moe_check(ws) == moe.MOE_OK


@pytest.mark.parametrize("T,E,k,R,rd", [(64, 16, 4, 4, 4), (1000, 128, 8, 8, 8),
                                       (7, 8, 8, 1, 3)])
def test_eplb_remap_matches_oracle(T, E, k, R, rd):
    rng = np.random.default_rng(T)
    logits = rng.normal(size=(T, E)) - np.log(np.arange(1, E + 1))
    idx = oracle.topk_select_sorted(logits.astype(np.float32), k).astype(np.int32)
    counts = oracle.expert_counts(idx, E)
    p2l, off, phys = oracle.eplb_plan(counts, rd, R)
    want = oracle.eplb_remap(idx, off, phys)
    shape = MoEShape.of(T, 64, E, k, 64)
    ws = moe.workspace(shape)
    got = torch.empty(T, k, dtype=torch.int32, device=DEV)
    moe.moe_eplb_remap(torch.from_numpy(idx).to(DEV),
                       torch.from_numpy(off.astype(np.int32)).to(DEV),
                       torch.from_numpy(phys.astype(np.int32)).to(DEV), E + rd, got, shape, ws)
    _check_clean(ws)
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_eplb_remap_flags_bad_ids():
    T, E, k = 5, 4, 2
    idx = torch.tensor([[0, 1], [2, 3], [4, 0], [1, -1], [3, 2]], dtype=torch.int32)
    off = torch.tensor([0, 1, 2, 3, 4], dtype=torch.int32)
    phys = torch.tensor([0, 1, 2, 3], dtype=torch.int32)
    shape = MoEShape.of(T, 64, E, k, 64)
    ws = moe.workspace(shape)
    got = torch.empty(T, k, dtype=torch.int32, device=DEV)
    moe.moe_eplb_remap(idx.to(DEV), off.to(DEV), phys.to(DEV), E, got, shape, ws)
    assert moe.moe_check(ws) == moe.MOE_ERR_DEVICE_CHECK
    g = got.cpu()
    assert g[2, 0] == -1 and g[3, 1] == -1
    assert g[0].tolist() == [0, 1] and g[4].tolist() == [3, 2]


def _layer(cfg):
    x = wl.make_hidden(cfg, DEV, 0)
    w_g, bias = wl.make_router(cfg, DEV, 0)
    w13, w2 = wl.make_experts(cfg, DEV, 0)
    return x, w_g, bias, w13, w2


def _forward_pair(cfg, rd):
    """moe_forward, then a plan from its counts (the load window) and
    moe_forward_eplb with the replicated weights."""
    x, w_g, bias, w13, w2 = _layer(cfg)
    shape = MoEShape.from_config(cfg)
    ws = moe.workspace(shape)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=DEV)
    gw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=DEV)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    moe.moe_forward(x, w_g, bias, w13, w2, y, shape, ws, idx, gw, counts)
    _check_clean(ws)
    R = max(cfg.R, 1)
    p2l, off, phys = moe.moe_eplb_plan(counts.cpu().long(), cfg.E, R, rd)
    E_phys = cfg.E + rd
    sel = p2l.long().to(DEV)
    w13_p = w13.index_select(0, sel).contiguous()
    w2_p = w2.index_select(0, sel).contiguous()
    ws_e = moe.workspace_eplb(shape, E_phys)
    y_e = torch.empty_like(y)
    idx_e = torch.empty_like(idx)
    gw_e = torch.empty_like(gw)
    counts_p = torch.empty(E_phys, dtype=torch.int32, device=DEV)
    moe.moe_forward_eplb(x, w_g, bias, w13_p, w2_p, y_e, shape, off.to(DEV), phys.to(DEV),
                         E_phys, ws_e, idx_e, gw_e, counts_p)
    _check_clean(ws_e)
    return dict(x=x, w_g=w_g, bias=bias, w13=w13, w2=w2, y=y, idx=idx, gw=gw, counts=counts,
                y_e=y_e, idx_e=idx_e, gw_e=gw_e, counts_p=counts_p, p2l=p2l, off=off,
                phys=phys, R=R)


@pytest.mark.parametrize("cfg,rd", [
    (wl.TINY, 2),
    (wl.QWEN3_30B_A3B_DECODE.with_T(64), 8),
    (wl.QWEN3_30B_A3B_DECODE.with_T(256), 16),
    (wl.DEEPSEEK_V3_ROUTED.with_T(64), 8),
], ids=lambda v: getattr(v, "name", str(v)))
def test_forward_eplb_equals_forward(cfg, rd):
    r = _forward_pair(cfg, rd)
    assert torch.equal(r["idx_e"], r["idx"]) and torch.equal(r["gw_e"], r["gw"])
    assert torch.equal(r["y_e"], r["y"])           # bit for bit (T <= 256: same kernels)
    cl = r["counts"].cpu().numpy()
    cp = r["counts_p"].cpu().numpy()
    off, phys = r["off"].numpy(), r["phys"].numpy()
    for e in range(cfg.E):
        assert cp[phys[off[e]:off[e + 1]]].sum() == cl[e]
    # physical counts are the oracle's remap of the same selection
    want = oracle.expert_counts(oracle.eplb_remap(r["idx"].cpu().numpy(), off, phys),
                                cfg.E + rd)
    np.testing.assert_array_equal(cp, want)


def test_forward_eplb_large_batch_and_balance():
    """A large DeepSeek-shaped batch (multi-block routing, CTA-pair GEMMs):
    outputs within the layer tolerance of the plain layer on sampled tokens,
    counts conserved, and the busiest virtual rank lighter with replicas."""
    cfg = wl.DEEPSEEK_V3_ROUTED.with_T(4096)
    r = _forward_pair(cfg, 16)
    assert torch.equal(r["idx_e"], r["idx"])
    toks = torch.arange(0, cfg.T, 61, device=DEV)
    assert_layer_close(r["y_e"][toks], np64(r["y"][toks]), "forward_eplb vs forward")
    cl = r["counts"].cpu().numpy()
    cp = r["counts_p"].cpu().numpy()
    assert cp.sum() == cl.sum()
    assert oracle.rank_loads(cp, r["R"]).max() < oracle.rank_loads(cl, r["R"]).max()


def test_forward_eplb_against_oracle():
    """Against the oracle's own selection: every token's selected set must be
    the unique one the fp32 logit error bound allows (true for this seed), and
    then y matches the oracle's layer within the layer tolerance."""
    cfg = wl.MoEConfig("eplb-oracle", T=96, d=256, E=8, k=2, f=256, R=4, zipf_s=1.2)
    r = _forward_pair(cfg, 4)
    x64, wg64 = np64(r["x"]), np64(r["w_g"])
    b64 = None if r["bias"] is None else np64(r["bias"])
    ref = oracle.moe_forward(x64, wg64, b64, LazyExperts(r["w13"]), LazyExperts(r["w2"]), cfg.k)
    L64 = oracle.router_logits(x64, wg64, b64)
    delta = logit_bound(x64, wg64, b64)
    got = r["idx_e"].cpu().numpy()
    sure = []
    for t in range(cfg.T):
        u = unique_selection(L64[t], delta[t], cfg.k)
        if u is None:  # an fp32 near-tie: either choice is right
            assert selection_is_valid(L64[t], delta[t], got[t].tolist())
        else:
            assert set(got[t].tolist()) == u
            sure.append(t)
    assert len(sure) >= cfg.T // 2
    sure = np.array(sure)
    assert_layer_close(r["y_e"][torch.from_numpy(sure).to(DEV)], ref["y"][sure],
                       "forward_eplb vs oracle")
