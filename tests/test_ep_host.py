"""The expert-parallel exchange on CPU: its oracle against the single-process
layer, and the rank driver (``EPMoELayer``) over a two-rank gloo group.

"Serving MoE models with expert parallelism on 8xH200", section "Tensor
parallel vs expert parallel"; "Wide Expert Parallelism", section "All-to-all
communication: the essential tradeoff".  The exchange only moves rows: the
layer it computes must be the single-process layer on the concatenation of
the ranks' batches, and the rows each rank's experts see must be exactly the
single-process dispatch rows of those experts.

The driver's per-step arithmetic is injected: here a test-supplied set of
steps built from the oracle (``OracleOps``), so the exchange plumbing (count
exchange, split sizes, all-to-all-v both ways, regrouping, return order) is
what is under test.  The product path uses the C ABI's kernels instead
(``LibraryOps``); the GPU tests cover that.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layer_inputs(R, T_of, d=64, E=8, k=2, f=64, zipf=True, seed=0):
    from routing_dispatch_expert_softmax_b200 import workloads as wl
    cfg = wl.MoEConfig("ep", T=1, d=d, E=E, k=k, f=f, zipf_s=1.2 if zipf else None)
    w_g, bias = wl.make_router(cfg, "cpu", seed)
    w13, w2 = wl.make_experts(cfg, "cpu", seed)
    xs = [wl.make_hidden(cfg.with_T(T_of(r)), "cpu", 10 + r) for r in range(R)]
    f64 = lambda t: None if t is None else t.double().numpy()
    return dict(cfg=cfg, w_g=f64(w_g), bias=f64(bias), w13=f64(w13), w2=f64(w2),
                xs=[f64(x) for x in xs])


# ---------------------------------------------------------------- oracle pins
def test_recv_expert_labels_worked_example():
    # 2 sources x 3 local experts: source 0 sent 2 rows of e0, 0 of e1, 1 of
    # e2; source 1 sent 1, 2, 0
    got = oracle.ep_recv_experts([[2, 0, 1], [1, 2, 0]], 2, 3)
    assert got.tolist() == [0, 0, 2, 0, 1, 1]
    assert oracle.ep_recv_experts(np.zeros((4, 2)), 4, 2).size == 0


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_ep_oracle_equals_the_single_process_layer(R):
    inp = _layer_inputs(R, lambda r: 3 + 4 * r)
    cfg = inp["cfg"]
    ep = oracle.ep_forward(inp["xs"], inp["w_g"], inp["bias"], inp["w13"], inp["w2"], cfg.k)
    x_all = np.concatenate(inp["xs"], axis=0)
    one = oracle.moe_forward(x_all, inp["w_g"], inp["bias"], inp["w13"], inp["w2"], cfg.k)
    y = np.concatenate(ep["y"], axis=0)
    assert np.abs(y - one["y"]).max() <= 1e-12 * max(1.0, np.abs(one["y"]).max())
    # the rows rank r's experts see, regrouped, are the single-process rows
    # of those experts, bit for bit
    E_loc = cfg.E // R
    for r in range(R):
        lo, hi = one["offsets"][r * E_loc], one["offsets"][(r + 1) * E_loc]
        regrouped = ep["x_recv"][r][ep["regrouped"][r]]
        np.testing.assert_array_equal(regrouped, x_all[one["perm"][lo:hi]])
    # counts are conserved through the exchange
    recv = sum(rc.sum(axis=0) for rc in ep["recv_counts"])
    assert recv.sum() == one["counts"].sum()
    np.testing.assert_array_equal(np.concatenate([rc.sum(axis=0) for rc in ep["recv_counts"]]),
                                  one["counts"])


# ---------------------------------------------------------------- driver, gloo
class OracleOps:
    """The driver's steps done by the oracle on CPU tensors (fp64)."""

    def route(self, x, w_g, bias, k, f):
        L = oracle.router_logits(x.numpy(), w_g.numpy(), None if bias is None else bias.numpy())
        idx = oracle.topk_select_sorted(L.astype(np.float32), k)
        return torch.from_numpy(idx), torch.from_numpy(oracle.gate_weights(L, idx))

    def dispatch(self, idx, x, E, R, f):
        idx_h = idx.numpy()
        counts = oracle.expert_counts(idx_h, E)
        perm, row_of = oracle.dispatch_rows(idx_h, E)
        out = dict(counts=torch.from_numpy(counts),
                   offsets=torch.from_numpy(oracle.expert_offsets(counts)),
                   perm=torch.from_numpy(perm), row_of=torch.from_numpy(row_of),
                   x_perm=x[torch.from_numpy(perm).long()].contiguous(), status=None,
                   rank_offsets=None)
        if R > 1:
            out["rank_offsets"] = torch.from_numpy(oracle.virtual_ep_layout(idx_h, E, R)[1])
        return out

    def recv_experts(self, recv_counts, R, E_loc, N):
        lab = oracle.ep_recv_experts(recv_counts.numpy(), R, E_loc)
        assert lab.size == N
        return torch.from_numpy(lab)

    def ffn(self, x_em, offsets, w13, w2, E_loc):
        n = x_em.shape[0]
        z = oracle.expert_outputs(x_em.numpy(), np.arange(n), offsets.numpy(), w13.numpy(),
                                  w2.numpy())
        return torch.from_numpy(z)

    def combine(self, z, row_of, w, E):
        return torch.from_numpy(oracle.combine(z.numpy(), row_of.numpy(), w.numpy()))

    def ones(self, n, device):
        return torch.ones(n, 1, dtype=torch.float64)

    def check(self, ws):
        return 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ep_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    from routing_dispatch_expert_softmax_b200.ep import EPMoELayer, TorchDistComm
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = _layer_inputs(world, lambda r: 5 + 3 * r)
        cfg = inp["cfg"]
        E_loc = cfg.E // world
        t = lambda a: None if a is None else torch.from_numpy(a)
        lo, hi = rank * E_loc, (rank + 1) * E_loc
        layer = EPMoELayer(t(inp["w_g"]), t(inp["bias"]), t(inp["w13"][lo:hi]),
                           t(inp["w2"][lo:hi]), cfg.k, rank, world, ops=OracleOps(),
                           comm=TorchDistComm())
        keep = {}
        y = layer(t(inp["xs"][rank]), keep=keep)
        out[rank] = dict(y=y.numpy(), recv_counts=keep["recv_counts"].numpy(),
                         x_recv=keep["x_recv"].numpy(),
                         expert_of_row=keep["grp"]["expert_of_row"].numpy(),
                         send_rows=keep["send_rows"], recv_rows=keep["recv_rows"])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_over_gloo_matches_the_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        res = m.dict()
        mp.start_processes(_ep_worker, args=(world, _free_port(), res), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(res)
    inp = _layer_inputs(world, lambda r: 5 + 3 * r)
    cfg = inp["cfg"]
    ref = oracle.ep_forward(inp["xs"], inp["w_g"], inp["bias"], inp["w13"], inp["w2"], cfg.k)
    one = oracle.moe_forward(np.concatenate(inp["xs"]), inp["w_g"], inp["bias"], inp["w13"],
                             inp["w2"], cfg.k)
    for r in range(world):
        got = res[r]
        np.testing.assert_array_equal(got["recv_counts"], ref["recv_counts"][r].reshape(-1))
        np.testing.assert_array_equal(got["expert_of_row"], ref["expert_of_row"][r])
        np.testing.assert_array_equal(got["x_recv"], ref["x_recv"][r])
        assert sum(got["recv_rows"]) == ref["x_recv"][r].shape[0]
        np.testing.assert_allclose(got["y"], ref["y"][r], rtol=0, atol=1e-12)
    # rows sent equal rows received across the pair
    assert res[0]["send_rows"][1] == res[1]["recv_rows"][0]
    assert res[1]["send_rows"][0] == res[0]["recv_rows"][1]
    y = np.concatenate([res[r]["y"] for r in range(world)])
    np.testing.assert_allclose(y, one["y"], rtol=0, atol=1e-12)
