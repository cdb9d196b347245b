"""GPU parity of the expert-parallel exchange's kernels.

``moe_ep_recv_experts`` against the oracle's labels bit for bit; the
rank driver (``EPMoELayer`` over the C ABI) with R ranks emulated in one
process on one GPU -- every rank's phases run in turn and the all-to-alls
are done by slicing, so no rank ever waits on another -- against the
single-GPU layer on the concatenated batch; and ``EPMoELayer.forward`` over a
one-rank NCCL group.  "Serving MoE models with expert parallelism on
8xH200", section "Tensor parallel vs expert parallel"; "Wide Expert
Parallelism", section "All-to-all communication: the essential tradeoff".
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape
from routing_dispatch_expert_softmax_b200.ep import EPMoELayer, TorchDistComm

from parity_utils import assert_layer_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("R,E_loc", [(1, 8), (2, 3), (8, 32), (64, 16)])
def test_recv_expert_labels_match_the_oracle(R, E_loc):
    rng = np.random.default_rng(R * 100 + E_loc)
    counts = rng.integers(0, 40, (R, E_loc)).astype(np.int32)
    counts[0, 0] = 0  # empty segments
    N = int(counts.sum())
    out = torch.full((N + 5,), 77, dtype=torch.int32, device=DEV)
    moe.moe_ep_recv_experts(torch.from_numpy(counts).to(DEV), R, E_loc, N + 5, out)
    want = oracle.ep_recv_experts(counts, R, E_loc)
    np.testing.assert_array_equal(out[:N].cpu().numpy(), want)
    assert out[N:].cpu().tolist() == [-1] * 5  # rows beyond the counts' total


def test_recv_expert_labels_negative_count_marks_every_row():
    counts = torch.tensor([[3, -1], [2, 2]], dtype=torch.int32, device=DEV)
    out = torch.zeros(6, dtype=torch.int32, device=DEV)
    moe.moe_ep_recv_experts(counts, 2, 2, 6, out)
    assert out.cpu().tolist() == [-1] * 6


def _ranks(cfg, R, T_of, seed=0):
    x = [wl.make_hidden(cfg.with_T(T_of(r)), DEV, 20 + r) for r in range(R)]
    w_g, bias = wl.make_router(cfg, DEV, seed)
    w13, w2 = wl.make_experts(cfg, DEV, seed)
    E_loc = cfg.E // R
    layers = [EPMoELayer(w_g, bias, w13[r * E_loc:(r + 1) * E_loc].contiguous(),
                         w2[r * E_loc:(r + 1) * E_loc].contiguous(), cfg.k, r, R)
              for r in range(R)]
    return x, w_g, bias, w13, w2, layers


def _emulated_exchange(layers, xs):
    """All ranks' phases in turn; the all-to-alls by slicing device tensors."""
    R = len(layers)
    E, E_loc, k = layers[0].E, layers[0].E_loc, layers[0].k
    st = [layers[r].dispatch_phase(xs[r]) for r in range(R)]
    offs = [s["offsets"].cpu().long() for s in st]
    counts = [s["counts"] for s in st]
    grp = []
    for r in range(R):
        lo, hi = r * E_loc, (r + 1) * E_loc
        recv_counts = torch.cat([counts[s][lo:hi] for s in range(R)])
        x_recv = torch.cat([st[s]["x_perm"][offs[s][lo]:offs[s][hi]] for s in range(R)])
        grp.append(layers[r].expert_phase(x_recv, recv_counts))
    ys = []
    for s in range(R):
        parts = []
        for r in range(R):
            lo, hi = r * E_loc, (r + 1) * E_loc
            before = sum(int(offs[s2][hi] - offs[s2][lo]) for s2 in range(s))
            n = int(offs[s][hi] - offs[s][lo])
            parts.append(grp[r]["z_recv"][before:before + n])
        z_back = torch.cat(parts)
        assert z_back.shape[0] == st[s]["T"] * k
        ys.append(layers[s].combine_phase(st[s], z_back))
    return st, grp, ys


@pytest.mark.parametrize("cfg,R,T_of", [
    (wl.MoEConfig("ep-small", T=1, d=256, E=16, k=4, f=256, zipf_s=1.2), 4, lambda r: 9 + 7 * r),
    (wl.DEEPSEEK_V3_ROUTED, 8, lambda r: 8),
    (wl.QWEN3_30B_A3B_DECODE, 2, lambda r: 90 + 20 * r),
], ids=["small", "deepseek-8x8", "qwen-2ranks"])
def test_emulated_ranks_match_the_single_gpu_layer(cfg, R, T_of):
    xs, w_g, bias, w13, w2, layers = _ranks(cfg, R, T_of)
    st, grp, ys = _emulated_exchange(layers, xs)
    for r in range(R):
        assert layers[r].check(st[r]) == moe.MOE_OK
        assert layers[r].check(grp[r]) == moe.MOE_OK
    x_all = torch.cat(xs)
    T = x_all.shape[0]
    shape = MoEShape.of(T, cfg.d, cfg.E, cfg.k, cfg.f)
    ws = moe.workspace(shape)
    y1 = torch.empty(T, cfg.d, dtype=torch.bfloat16, device=DEV)
    idx1 = torch.empty(T, cfg.k, dtype=torch.int32, device=DEV)
    cnt1 = torch.empty(cfg.E, dtype=torch.int32, device=DEV)
    moe.moe_forward(x_all, w_g, bias, w13, w2, y1, shape, ws, idx1, None, cnt1)
    assert moe.moe_check(ws) == moe.MOE_OK
    # routing: every rank's selection is the single-GPU selection of its tokens
    # (both routers take each token's logits in the same fixed order up to 256
    # tokens per call)
    if T <= 256:
        assert torch.equal(torch.cat([s["idx"] for s in st]), idx1)
    idx_all = torch.cat([s["idx"] for s in st]).cpu().numpy()
    perm1, _ = oracle.dispatch_rows(idx_all, cfg.E)
    off1 = oracle.expert_offsets(oracle.expert_counts(idx_all, cfg.E))
    # the rows each rank's experts run on are the single-GPU dispatch rows of
    # those experts, bit for bit, and the counts add up
    E_loc = cfg.E // R
    for r in range(R):
        lo, hi = off1[r * E_loc], off1[(r + 1) * E_loc]
        want = x_all[torch.from_numpy(perm1[lo:hi]).long().to(DEV)]
        assert torch.equal(grp[r]["x_perm"], want)
        np.testing.assert_array_equal(grp[r]["offsets"].cpu().numpy(),
                                      off1[r * E_loc:(r + 1) * E_loc + 1] - lo)
    # outputs: the single-GPU layer's, within the layer tolerance
    assert_layer_close(torch.cat(ys), y1.float().cpu().numpy().astype(np.float64),
                       f"EP x{R} vs single GPU")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_forward_over_a_one_rank_nccl_group():
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV, torch.cuda.current_device()))
    try:
        cfg = wl.MoEConfig("ep-nccl", T=96, d=512, E=32, k=4, f=256, zipf_s=1.0)
        xs, w_g, bias, w13, w2, layers = _ranks(cfg, 1, lambda r: 96)
        layer = layers[0]
        layer.comm = TorchDistComm()
        keep = {}
        y = layer(xs[0], keep=keep)
        torch.cuda.synchronize()
        assert layer.check(keep["st"]) == moe.MOE_OK
        shape = MoEShape.of(96, cfg.d, cfg.E, cfg.k, cfg.f)
        ws = moe.workspace(shape)
        y1 = torch.empty_like(y)
        moe.moe_forward(xs[0], w_g, bias, w13, w2, y1, shape, ws)
        assert moe.moe_check(ws) == moe.MOE_OK
        assert_layer_close(y, y1.float().cpu().numpy().astype(np.float64), "EP x1 (NCCL)")
    finally:
        dist.destroy_process_group()
