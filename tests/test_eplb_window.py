"""Host logic of the windowed expert-load statistics and the automatic
re-plan rule (``LoadWindow``, ``MoELayer.enable_auto_rebalance``), on CPU.

"vLLM Expert Parallel deployment" (EPLB section): load over a window of recent
steps, re-planned at a fixed interval with a configured number of extra
copies; "Serving MoE models with expert parallelism on 8xH200", section
"Routing imbalance": act when the busiest device carries more than about 1.3x
the mean.  The replica plan itself is the library's host call
(``moe_eplb_plan``), which needs no GPU; these tests write counts into the
window the way the layer's routing kernel would and check the decisions.
"""

import numpy as np
import torch

import oracle
from routing_dispatch_expert_softmax_b200.layer import LoadWindow, MoELayer, imbalance_factor


def test_window_sums_the_last_calls_only():
    w = LoadWindow(4, window=3, device="cpu")
    rows = [[1, 0, 0, 0], [0, 2, 0, 0], [0, 0, 3, 0], [0, 0, 0, 4], [5, 0, 0, 0]]
    for r in rows:
        w.next_slot().copy_(torch.tensor(r, dtype=torch.int32))
    np.testing.assert_array_equal(w.load(), np.array(rows[-3:]).sum(axis=0))
    w.reset()
    assert w.calls == 0 and w.load().sum() == 0


def test_imbalance_factor_matches_the_oracle():
    rng = np.random.default_rng(3)
    for _ in range(20):
        counts = rng.integers(0, 50, 32)
        for R in (1, 2, 4, 8):
            assert abs(imbalance_factor(counts, R) - oracle.imbalance_factor(counts, R)) < 1e-12


def _cpu_layer(E=8, d=64, f=64, k=2, R=2):
    g = torch.Generator().manual_seed(0)
    w_g = torch.randn(d, E, generator=g)
    w13 = torch.randn(E, 2 * f, d, generator=g).to(torch.bfloat16)
    w2 = torch.randn(E, d, f, generator=g).to(torch.bfloat16)
    return MoELayer(w_g, None, w13, w2, k, R)


def _record(layer, counts):
    layer.load_window.next_slot().copy_(torch.tensor(counts, dtype=torch.int32))
    layer._after_call()


def test_balanced_load_keeps_the_placement():
    layer = _cpu_layer()
    layer.enable_auto_rebalance(n_redundant=2, window=4, step_interval=4, threshold=1.3)
    for _ in range(8):
        _record(layer, [2] * 8)
    assert layer.physical_experts == 8 and layer._auto["replans"] == 0
    assert layer._auto["last_factor"] == 1.0


def test_skewed_load_replans_at_the_interval():
    layer = _cpu_layer()
    layer.enable_auto_rebalance(n_redundant=2, window=4, step_interval=4, threshold=1.3)
    skew = [10, 6, 1, 1, 1, 1, 1, 1]  # rank 0 (experts 0-3) holds 18 of 22 rows
    for i in range(3):
        _record(layer, skew)
        assert layer.physical_experts == 8  # not due yet
    _record(layer, skew)  # the 4th call: factor 18/11 > 1.3
    assert layer._auto["replans"] == 1 and layer.physical_experts == 10
    assert layer._auto["last_factor"] > 1.3
    # the plan is the library's plan for the window's load (4 x skew)
    p2l = layer._eplb["p2l"]
    want_p2l, _, _ = oracle.eplb_plan(np.array(skew) * 4, 2, 2)
    np.testing.assert_array_equal(p2l, want_p2l)
    # the window restarted over the 10 physical experts
    assert layer.load_window.ring.shape[1] == 10 and layer.load_window.calls == 0
    # physical counts map back to logical load (replicas summed)
    phys = np.zeros(10, dtype=np.int64)
    for p, e in enumerate(p2l):
        phys[p] = 1 + e
    _record(layer, phys.tolist())
    want = np.zeros(8, dtype=np.int64)
    np.add.at(want, p2l, phys)
    np.testing.assert_array_equal(layer.logical_load(), want)
