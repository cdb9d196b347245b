"""GPU parity of token-deduplicated per-rank dispatch against the oracle:
every output is integer or a copied row, so the comparison is bit for bit."""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import routing_dispatch_expert_softmax_b200 as moe
from routing_dispatch_expert_softmax_b200 import workloads as wl
from routing_dispatch_expert_softmax_b200.binding import MoEShape

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(idx_np, E, R, d=64, x=None):
    T, k = idx_np.shape
    rows = T * min(k, R)
    shape = MoEShape.of(T, d, E, k, 64, R)
    ws = moe.workspace(shape)
    send = torch.empty(R, R, dtype=torch.int32, device=DEV)
    off = torch.empty(R + 1, dtype=torch.int32, device=DEV)
    tok = torch.full((max(rows, 1),), -7, dtype=torch.int32, device=DEV)
    mask = torch.zeros(max(rows, 1), dtype=torch.int32, device=DEV)
    row_of = torch.empty(T, R, dtype=torch.int32, device=DEV)
    xd = None if x is None else torch.zeros(max(rows, 1), d, dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch_dedup(torch.from_numpy(idx_np.astype(np.int32)).to(DEV), x, send, off, tok,
                           mask, shape, ws, rank_row_of=row_of, x_dedup=xd)
    st = moe.moe_check(ws)
    return st, send.cpu().numpy(), off.cpu().numpy(), tok.cpu().numpy(), \
        mask.cpu().numpy().view(np.uint32), row_of.cpu().numpy(), xd


def test_dedup_worked_example():
    path = os.path.join(os.path.dirname(__file__), "golden", "dedup_worked_example.json")
    with open(path) as fh:
        c = json.load(fh)
    st, S, off, tok, mask, row_of, _ = _run(np.array(c["idx"]), c["E"], c["R"])
    assert st == moe.MOE_OK
    n = off[-1]
    assert S.tolist() == c["send_counts"] and off.tolist() == c["rank_offsets"]
    assert tok[:n].tolist() == c["token_of"] and mask[:n].tolist() == c["slot_mask"]
    assert row_of.tolist() == c["rank_row_of"]


@pytest.mark.parametrize("T,E,k,R", [(1000, 256, 8, 8), (16384, 256, 8, 8), (777, 1024, 32, 64),
                                     (300, 64, 1, 2), (257, 128, 8, 16), (1, 256, 8, 8)])
def test_dedup_matches_oracle(T, E, k, R):
    rng = np.random.default_rng(T + E)
    logits = rng.normal(size=(T, E)) - 1.2 * np.log1p(rng.permutation(E))  # skewed popularity
    idx = oracle.topk_select_sorted(logits.astype(np.float32), k)
    d = 128
    x = wl.make_hidden(wl.MoEConfig("x", T=T, d=d, E=E, k=k, f=64), DEV, 3)
    st, S, off, tok, mask, row_of, xd = _run(idx, E, R, d, x)
    assert st == moe.MOE_OK
    S_o, off_o, tok_o, mask_o, row_of_o = oracle.dedup_layout(idx, E, R)
    n = int(off_o[-1])
    np.testing.assert_array_equal(S, S_o)
    np.testing.assert_array_equal(off, off_o)
    np.testing.assert_array_equal(tok[:n], tok_o)
    np.testing.assert_array_equal(mask[:n], mask_o)
    np.testing.assert_array_equal(row_of, row_of_o)
    assert torch.equal(xd[:n], x[torch.from_numpy(tok_o).long().to(DEV)])
    # fewer rows than the plain layout whenever a token has two experts on one rank
    S_plain, _ = oracle.virtual_ep_layout(idx, E, R)
    assert S.sum() <= S_plain.sum()


def test_dedup_records_bad_ids():
    idx = np.array([[0, 1], [2, 9], [5, 3]])
    st, S, off, tok, mask, row_of, _ = _run(idx, 8, 4)
    assert st == moe.MOE_ERR_DEVICE_CHECK
    # t0 -> r0; t1 -> r1 (id 9 is out of range and skipped); t2 -> r1, r2
    assert row_of.tolist() == [[0, -1, -1, -1], [-1, 1, -1, -1], [-1, 2, 3, -1]]
    assert off.tolist() == [0, 1, 3, 4, 4]
    assert tok[:4].tolist() == [0, 1, 2, 2] and mask[:4].tolist() == [3, 1, 2, 1]
