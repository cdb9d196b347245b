"""Pins for the fp64 oracle, against things other than the oracle itself.

Each check compares the oracle with a hand-worked example, a closed form, a
library routine doing a special case, an invariant, exact rational arithmetic
or brute force on tiny inputs.  The planted-mistake tests at the bottom plant
plausible bugs into the oracle (on the CPU) and confirm a pin catches each.
"""

import itertools
import json
import os
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from routing_dispatch_expert_softmax_b200 import workloads as wl


def _np(t):
    return t.float().numpy().astype(np.float64) if t is not None else None


# ---------------------------------------------------------------- selection
def test_topk_hand_worked_examples(golden):
    for case in golden["topk"]:
        L = np.array([case["logits"]], dtype=np.float32)
        k = case["k"]
        got = oracle.topk_select(L, k)[0].tolist()
        assert got == case["idx"], case["why"]
        assert oracle.topk_select_sorted(L, k)[0].tolist() == case["idx"]
        L64 = np.array([case["logits"]], dtype=np.float64)
        w = oracle.gate_weights(L64, np.array([case["idx"]]))[0]
        want = [eval(expr, {"exp": math.exp}) for expr in case["gates"]]
        np.testing.assert_allclose(w, want, rtol=0, atol=1e-12, err_msg=case["why"])


def _lexmax_topk(row, k):
    """Brute force over all ordered k-subsets: the selection is the
    lexicographically greatest sequence of (value, -index) pairs."""
    best = None
    for combo in itertools.permutations(range(len(row)), k):
        key = tuple((float(row[e]) + 0.0, -e) for e in combo)
        if best is None or key > best[0]:
            best = (key, combo)
    return list(best[1])


@pytest.mark.parametrize("kind", ["normal", "ties", "const"])
def test_topk_brute_force_tiny(kind):
    L = wl.make_logits(40, 6, seed=3, kind=kind).numpy()
    for k in (1, 2, 3, 6):
        a = oracle.topk_select(L, k)
        b = oracle.topk_select_sorted(L, k)
        np.testing.assert_array_equal(a, b)
        for t in range(0, 40, 7):
            assert a[t].tolist() == _lexmax_topk(L[t], k)


def test_topk_forms_agree_tie_heavy_wide():
    L = wl.make_logits(200, 16, seed=5, kind="ties").numpy()
    for k in (1, 4, 8, 16):
        np.testing.assert_array_equal(oracle.topk_select(L, k),
                                      oracle.topk_select_sorted(L, k))


def test_topk_signed_zero_ties():
    L = np.array([[-0.0, 0.0, -0.0, 0.0]], dtype=np.float32)
    assert oracle.topk_select(L, 2)[0].tolist() == [0, 1]
    L = np.array([[0.0, -0.0, -1.0, -0.0]], dtype=np.float32)
    assert oracle.topk_select_sorted(L, 3)[0].tolist() == [0, 1, 3]


def test_topk_rejects_bad_k():
    L = np.zeros((2, 4), np.float32)
    for k in (0, 5):
        with pytest.raises(ValueError):
            oracle.topk_select(L, k)


# ---------------------------------------------------------------- gates
def test_gates_sum_to_one_and_k_equals_E_is_softmax():
    L = wl.make_logits(64, 12, seed=1).numpy().astype(np.float64) * 3.0
    for k in (1, 2, 5, 12):
        idx = oracle.topk_select_sorted(L, k)
        w = oracle.gate_weights(L, idx)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert np.all(w > 0)
        assert np.all(np.diff(w, axis=1) <= 1e-15)  # slots in descending order
    idx = oracle.topk_select_sorted(L, 12)
    w = oracle.gate_weights(L, idx)
    ref = scipy.special.softmax(L, axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(ref, idx.astype(np.int64), 1),
                               rtol=1e-13, atol=0)


def test_gates_k2_closed_form_is_logistic():
    L = wl.make_logits(50, 7, seed=2).numpy().astype(np.float64) * 2.0
    idx = oracle.topk_select_sorted(L, 2)
    w = oracle.gate_weights(L, idx)
    a = np.take_along_axis(L, idx[:, :1].astype(np.int64), 1)[:, 0]
    b = np.take_along_axis(L, idx[:, 1:2].astype(np.int64), 1)[:, 0]
    np.testing.assert_allclose(w[:, 0], scipy.special.expit(a - b), rtol=1e-13)
    np.testing.assert_allclose(w[:, 1], scipy.special.expit(b - a), rtol=1e-12)


def test_gates_shift_invariant_and_large_logits_finite():
    L = wl.make_logits(16, 8, seed=4).numpy().astype(np.float64)
    idx = oracle.topk_select_sorted(L, 3)
    w0 = oracle.gate_weights(L, idx)
    w1 = oracle.gate_weights(L + 700.0, idx)  # exp(700+) would overflow unshifted
    np.testing.assert_allclose(w0, w1, rtol=1e-10)
    assert np.all(np.isfinite(w1))


# ---------------------------------------------------------------- counts / rows
def test_dispatch_hand_worked_example(golden):
    g = golden["dispatch"]
    idx = np.array(g["idx"], dtype=np.int32)
    counts = oracle.expert_counts(idx, g["E"])
    assert counts.tolist() == g["counts"]
    assert oracle.expert_offsets(counts).tolist() == g["offsets"]
    perm, row_of = oracle.dispatch_rows(idx, g["E"])
    assert perm.tolist() == g["perm"]
    assert row_of.tolist() == g["row_of"]
    S, ro = oracle.virtual_ep_layout(idx, g["E"], g["R"])
    assert S.tolist() == g["send_counts"]
    assert ro.tolist() == g["rank_offsets"]


def test_imbalance_hand_worked_example(golden):
    g = golden["imbalance"]
    assert oracle.imbalance_factor(np.array(g["counts"]), g["R"]) == pytest.approx(g["factor"])


@pytest.mark.parametrize("T,E,k,R", [(1, 8, 2, 2), (37, 16, 4, 4), (300, 32, 8, 8),
                                     (5, 4, 4, 2)])
def test_counts_offsets_perm_invariants(T, E, k, R):
    L = wl.make_logits(T, E, seed=T + E).numpy()
    idx = oracle.topk_select_sorted(L, k)
    counts = oracle.expert_counts(idx, E)
    # library routines for the special cases
    np.testing.assert_array_equal(counts, np.bincount(idx.reshape(-1), minlength=E))
    assert counts.sum() == T * k
    assert counts.mean() == pytest.approx(T * k / E)  # mean load B*k/E
    offsets = oracle.expert_offsets(counts)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    perm, row_of = oracle.dispatch_rows(idx, E)
    P = T * k
    assert sorted(row_of.reshape(-1).tolist()) == list(range(P))  # bijection
    for t in range(T):
        for j in range(k):
            r = row_of[t, j]
            assert perm[r] == t
            e = idx[t, j]
            assert offsets[e] <= r < offsets[e + 1]
    # rows equal a stable library sort of the pairs by (expert, token)
    flat_e = idx.reshape(-1)
    flat_t = np.repeat(np.arange(T), k)
    order = np.lexsort((flat_t, flat_e))
    np.testing.assert_array_equal(perm, flat_t[order])
    S, ro = oracle.virtual_ep_layout(idx, E, R)
    assert S.sum() == P
    chunk = -(-T // R)
    per_src = np.array([min(T, (s + 1) * chunk) - min(T, s * chunk) for s in range(R)])
    np.testing.assert_array_equal(S.sum(axis=1), per_src * k)
    np.testing.assert_array_equal(S.sum(axis=0), np.diff(ro))
    assert ro[0] == 0 and ro[-1] == P


def test_dispatch_then_combine_is_identity():
    T, d, E = 33, 24, 8
    x = np.random.default_rng(0).standard_normal((T, d))
    L = wl.make_logits(T, E, seed=9).numpy()
    # k = 1 with unit gates: bit-exact identity
    idx = oracle.topk_select_sorted(L, 1)
    perm, row_of = oracle.dispatch_rows(idx, E)
    y = oracle.combine(x[perm], row_of, np.ones((T, 1)))
    np.testing.assert_array_equal(y, x)
    # k = 3 with gates summing to 1: identity up to rounding
    idx = oracle.topk_select_sorted(L, 3)
    perm, row_of = oracle.dispatch_rows(idx, E)
    w = oracle.gate_weights(L, idx)
    y = oracle.combine(x[perm], row_of, w)
    np.testing.assert_allclose(y, x, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- FFN / layer
def test_silu_against_library():
    z = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(oracle.silu(z), z * scipy.special.expit(z), rtol=1e-14)


def test_router_logits_exact_rational():
    rng = np.random.default_rng(1)
    x = rng.integers(-8, 8, (3, 5)) / 8.0
    W = rng.integers(-8, 8, (5, 4)) / 16.0
    b = rng.integers(-4, 4, 4) / 4.0
    L = oracle.router_logits(x, W, b)
    for t in range(3):
        for e in range(4):
            exact = sum(Fraction(x[t, i]) * Fraction(W[i, e]) for i in range(5)) + Fraction(b[e])
            assert L[t, e] == float(exact)


def _small_layer(T, d, E, k, f, seed=0, zipf=None):
    cfg = wl.MoEConfig("pin", T=T, d=d, E=E, k=k, f=f, zipf_s=zipf)
    t = wl.make_layer(cfg, "cpu", seed)
    return cfg, {n: _np(v) for n, v in t.items()}


def test_single_expert_k1_is_plain_swiglu_ffn():
    cfg, t = _small_layer(T=9, d=32, E=1, k=1, f=48)
    out = oracle.moe_forward(t["x"], t["w_g"], None, t["w13"], t["w2"], k=1)
    x = torch.tensor(t["x"], dtype=torch.float64)
    Wg = torch.tensor(t["w13"][0, :48], dtype=torch.float64)
    Wu = torch.tensor(t["w13"][0, 48:], dtype=torch.float64)
    Wd = torch.tensor(t["w2"][0], dtype=torch.float64)
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(x, Wg))
        * torch.nn.functional.linear(x, Wu), Wd)
    np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(out["w"] == 1.0)


def test_k_equals_E_is_dense_gate_weighted_sum():
    cfg, t = _small_layer(T=11, d=32, E=4, k=4, f=16)
    out = oracle.moe_forward(t["x"], t["w_g"], None, t["w13"], t["w2"], k=4)
    x = torch.tensor(t["x"], dtype=torch.float64)
    p = torch.softmax(x @ torch.tensor(t["w_g"], dtype=torch.float64), dim=1)
    y = torch.zeros_like(x)
    for e in range(4):
        W = torch.tensor(t["w13"][e], dtype=torch.float64)
        Wd = torch.tensor(t["w2"][e], dtype=torch.float64)
        h = torch.nn.functional.silu(x @ W[:16].T) * (x @ W[16:].T)
        y += p[:, e:e + 1] * (h @ Wd.T)
    np.testing.assert_allclose(out["y"], y.numpy(), rtol=1e-11, atol=1e-12)


def test_layer_per_token_brute_force_with_bias():
    cfg, t = _small_layer(T=13, d=32, E=8, k=3, f=16, zipf=1.0)
    out = oracle.moe_forward(t["x"], t["w_g"], t["bias"], t["w13"], t["w2"], k=3)
    for tok in range(13):
        xt = t["x"][tok]
        L = xt @ t["w_g"] + t["bias"]
        L32 = L.astype(np.float32)
        order = sorted(range(8), key=lambda e: (-float(L32[e]), e))[:3]
        assert out["idx"][tok].tolist() == order
        ex = np.exp(L[order] - L.max())
        gates = ex / ex.sum()
        acc = np.zeros(32)
        for g, e in zip(gates, order):
            W = t["w13"][e]
            h = (xt @ W[:16].T) / (1 + np.exp(-(xt @ W[:16].T))) * (xt @ W[16:].T)
            acc += g * (h @ t["w2"][e].T)
        np.testing.assert_allclose(out["y"][tok], acc, rtol=1e-11, atol=1e-12)


def test_bias_skews_popularity_toward_low_rank():
    cfg = wl.MoEConfig("skew", T=4000, d=64, E=16, k=1, f=8, zipf_s=1.0)
    w_g, bias = wl.make_router(cfg, "cpu", 0)
    x = wl.make_hidden(cfg, "cpu", 0)
    L = oracle.router_logits(_np(x), _np(w_g), _np(bias))
    counts = oracle.expert_counts(oracle.topk_select_sorted(L, 1), 16)
    hottest = int(np.argmax(_np(bias)))
    assert counts[hottest] == counts.max()
    assert counts.max() > 3 * cfg.T / 16


def test_weight_bytes_match_memory_sizing():
    # Expert memory = N_experts * P_per_expert * bytes ("Expert Parallelism
    # for MoE Models", memory sizing), P_per_expert = 3*d*f for SwiGLU.
    assert wl.DEEPSEEK_V3_ROUTED.expert_bytes() * 256 == pytest.approx(22.55e9, rel=1e-3)
    assert wl.QWEN3_30B_A3B_DECODE.expert_bytes() * 128 == pytest.approx(1.208e9, rel=1e-3)
    assert wl.MIXTRAL_8X7B.expert_bytes() * 8 == pytest.approx(2.818e9, rel=1e-3)


# ---------------------------------------------------------------- planted mistakes
def _pins_fail(monkeypatch, name, bad, golden):
    monkeypatch.setattr(oracle.moe_oracle, name, bad)
    monkeypatch.setattr(oracle, name, bad)
    failures = 0
    for fn in (lambda: test_topk_hand_worked_examples(golden),
               lambda: test_dispatch_hand_worked_example(golden),
               lambda: test_single_expert_k1_is_plain_swiglu_ffn(),
               lambda: test_k_equals_E_is_dense_gate_weighted_sum(),
               lambda: test_layer_per_token_brute_force_with_bias(),
               lambda: test_gates_k2_closed_form_is_logistic(),
               lambda: test_counts_offsets_perm_invariants(37, 16, 4, 4)):
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def test_planted_tie_break_to_higher_index_is_caught(monkeypatch, golden):
    def bad(L, k):
        L = np.asarray(L)
        return (L.shape[1] - 1 - np.argsort(-L[:, ::-1], axis=1, kind="stable")[:, :k]).astype(np.int32)
    assert _pins_fail(monkeypatch, "topk_select_sorted", bad, golden) > 0


def test_planted_missing_renormalisation_is_caught(monkeypatch, golden):
    def bad(L, idx):
        L = np.asarray(L, dtype=np.float64)
        p = scipy.special.softmax(L, axis=1)
        return np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    assert _pins_fail(monkeypatch, "gate_weights", bad, golden) > 0


def test_planted_swapped_gate_up_is_caught(monkeypatch, golden):
    def bad(X, w13_e, w2_e):
        f = w13_e.shape[0] // 2
        X = np.asarray(X, np.float64)
        g = X @ np.asarray(w13_e[f:], np.float64).T
        u = X @ np.asarray(w13_e[:f], np.float64).T
        return (g / (1 + np.exp(-g)) * u) @ np.asarray(w2_e, np.float64).T
    assert _pins_fail(monkeypatch, "swiglu_ffn", bad, golden) > 0


def test_planted_token_descending_rows_are_caught(monkeypatch, golden):
    real = oracle.moe_oracle.dispatch_rows

    def bad(idx, E):
        idx = np.asarray(idx)
        perm, row_of = real(idx[::-1], E)
        T = idx.shape[0]
        return (T - 1 - perm).astype(np.int32), row_of[::-1].copy()
    assert _pins_fail(monkeypatch, "dispatch_rows", bad, golden) > 0


def test_planted_wrong_silu_sign_is_caught(monkeypatch, golden):
    def bad(z):
        z = np.asarray(z, np.float64)
        return z / (1.0 + np.exp(z))
    assert _pins_fail(monkeypatch, "silu", bad, golden) > 0


# ---------------------------------------------------------------- EPLB-style balancing
def _eplb_cases():
    path = os.path.join(os.path.dirname(__file__), "golden", "eplb_worked_examples.json")
    with open(path) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _eplb_cases(), ids=lambda c: str(c["load"]))
def test_eplb_plan_matches_hand_worked_examples(case):
    n = oracle.eplb_replicate(case["load"], case["n_redundant"])
    assert n.tolist() == case["copies"]
    p2l, off, phys = oracle.eplb_plan(case["load"], case["n_redundant"], case["R"])
    assert p2l.tolist() == case["phys_to_logical"]
    assert off.tolist() == case["rep_offsets"]
    assert phys.tolist() == case["rep_phys"]
    shares = {(e, i): s for e, i, s in oracle.eplb_shares(case["load"], n)}
    S = len(p2l) // case["R"]
    loads = [0] * case["R"]
    for e in range(len(case["load"])):
        for i in range(off[e + 1] - off[e]):
            loads[phys[off[e] + i] // S] += shares[(e, i)]
    assert loads == case["rank_loads"]


def test_eplb_replication_minimises_the_largest_load_per_copy():
    # brute force over every way to hand out the redundant copies
    rng = np.random.default_rng(3)
    for _ in range(40):
        E = int(rng.integers(2, 5))
        rd = int(rng.integers(0, 5))
        load = rng.integers(0, 30, E).tolist()
        n = oracle.eplb_replicate(load, rd)
        best = min(max(l / c for l, c in zip(load, comp))
                   for comp in itertools.product(range(1, rd + 2), repeat=E)
                   if sum(comp) == E + rd)
        assert max(l / c for l, c in zip(load, n)) == pytest.approx(best)


@pytest.mark.parametrize("seed", range(6))
def test_eplb_plan_invariants(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.choice([1, 2, 4, 8]))
    E = R * int(rng.integers(1, 9))
    rd = R * int(rng.integers(0, 3))
    load = (1000 * rng.zipf(1.3, E).clip(max=50)).tolist()
    p2l, off, phys = oracle.eplb_plan(load, rd, R)
    n = np.diff(off)
    assert n.sum() == E + rd and (n >= 1).all()
    assert sorted(phys.tolist()) == list(range(E + rd))        # every slot used once
    for e in range(E):
        assert (p2l[phys[off[e]:off[e + 1]]] == e).all()      # replicas map back
    assert sum(s for _, _, s in oracle.eplb_shares(load, n)) == sum(load)


def test_eplb_remap_conserves_counts_and_uses_t_mod_copies():
    rng = np.random.default_rng(7)
    E, k, T, R, rd = 16, 4, 300, 4, 4
    logits = rng.normal(size=(T, E)) - np.log(np.arange(1, E + 1))  # skewed popularity
    idx = oracle.topk_select_sorted(logits.astype(np.float32), k)
    counts = oracle.expert_counts(idx, E)
    p2l, off, phys = oracle.eplb_plan(counts, rd, R)
    idx_p = oracle.eplb_remap(idx, off, phys)
    counts_p = oracle.expert_counts(idx_p, E + rd)
    for e in range(E):
        assert counts_p[phys[off[e]:off[e + 1]]].sum() == counts[e]
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            assert idx_p[t, j] == phys[off[e] + t % (off[e + 1] - off[e])]
    # the balanced placement evens the per-rank rows out on this skewed batch
    assert (oracle.rank_loads(counts_p, R).max() <
            oracle.rank_loads(counts, R).max())


# ---------------------------------------------------------------- token-deduplicated dispatch
def test_dedup_layout_matches_hand_worked_example():
    path = os.path.join(os.path.dirname(__file__), "golden", "dedup_worked_example.json")
    with open(path) as fh:
        c = json.load(fh)
    S, off, tok, mask, row_of = oracle.dedup_layout(np.array(c["idx"]), c["E"], c["R"])
    assert S.tolist() == c["send_counts"]
    assert off.tolist() == c["rank_offsets"]
    assert tok.tolist() == c["token_of"]
    assert mask.tolist() == c["slot_mask"]
    assert row_of.tolist() == c["rank_row_of"]


def test_dedup_layout_reduces_to_the_plain_layout_for_k1_and_r1():
    rng = np.random.default_rng(5)
    T, E, R = 37, 16, 4
    idx = rng.integers(0, E, (T, 1))
    S, off, tok, mask, _ = oracle.dedup_layout(idx, E, R)
    S_plain, off_plain = oracle.virtual_ep_layout(idx, E, R)
    np.testing.assert_array_equal(S, S_plain)
    np.testing.assert_array_equal(off, off_plain)
    assert (mask == 1).all()
    # R = 1: every token once, all k slots local
    idx = oracle.topk_select_sorted(rng.normal(size=(T, E)).astype(np.float32), 3)
    S, off, tok, mask, _ = oracle.dedup_layout(idx, E, 1)
    assert S.tolist() == [[T]] and tok.tolist() == list(range(T)) and (mask == 7).all()


@pytest.mark.parametrize("seed", range(4))
def test_dedup_layout_invariants(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.choice([2, 4, 8]))
    E = R * int(rng.integers(1, 9))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.integers(1, 200))
    idx = oracle.topk_select_sorted(rng.normal(size=(T, E)).astype(np.float32), k)
    S, off, tok, mask, row_of = oracle.dedup_layout(idx, E, R)
    S_plain, _ = oracle.virtual_ep_layout(idx, E, R)
    assert (S <= S_plain).all() and (S > 0).sum() == (S_plain > 0).sum()
    per = E // R
    for t in range(T):
        rows = [row_of[t, r] for r in range(R) if row_of[t, r] >= 0]
        got = 0
        for row in rows:
            assert tok[row] == t
            assert (got & int(mask[row])) == 0            # slots split across ranks
            got |= int(mask[row])
        assert got == (1 << k) - 1                         # every slot goes somewhere
        for r in range(R):
            want = sum(1 << j for j in range(k) if idx[t, j] // per == r)
            assert (row_of[t, r] >= 0) == (want != 0)
            if want:
                assert mask[row_of[t, r]] == want
    for r in range(R):                                     # tokens ascending per rank
        seg = tok[off[r]:off[r + 1]]
        assert (np.diff(seg) > 0).all()


# ---------------------------------------------------------------- planted mistakes (EPLB, dedup)
def _eplb_pins_fail(monkeypatch, module, name, bad):
    monkeypatch.setattr(module, name, bad)
    monkeypatch.setattr(oracle, name, bad)
    failures = 0
    checks = [lambda c=c: test_eplb_plan_matches_hand_worked_examples(c) for c in _eplb_cases()]
    checks += [test_eplb_replication_minimises_the_largest_load_per_copy,
               test_eplb_remap_conserves_counts_and_uses_t_mod_copies]
    for fn in checks:
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def test_planted_replication_tie_to_higher_id_is_caught(monkeypatch):
    def bad(load, n_redundant):
        load = [int(v) for v in load]
        n = [1] * len(load)
        for _ in range(int(n_redundant)):
            best = 0
            for e in range(1, len(load)):
                if load[e] * n[best] >= load[best] * n[e]:  # ties to the higher id
                    best = e
            n[best] += 1
        return np.array(n, dtype=np.int64)
    assert _eplb_pins_fail(monkeypatch, oracle.eplb_oracle, "eplb_replicate", bad) > 0


def test_planted_placement_on_most_loaded_rank_is_caught(monkeypatch):
    real_shares = oracle.eplb_oracle.eplb_shares

    def bad(load, n, R):
        n = [int(c) for c in n]
        P = sum(n)
        S = P // R
        reps = sorted(real_shares(load, n), key=lambda r: (-r[2], r[0], r[1]))
        rank_load, rank_fill = [0] * R, [0] * R
        off = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
        phys, p2l = np.full(P, -1, np.int64), np.full(P, -1, np.int64)
        for e, i, share in reps:
            r = max((r for r in range(R) if rank_fill[r] < S), key=lambda r: (rank_load[r], -r))
            slot = r * S + rank_fill[r]
            rank_fill[r] += 1
            rank_load[r] += share
            phys[off[e] + i] = slot
            p2l[slot] = e
        return p2l, off, phys
    assert _eplb_pins_fail(monkeypatch, oracle.eplb_oracle, "eplb_place", bad) > 0


def test_planted_replica_choice_by_division_is_caught(monkeypatch):
    def bad(idx, off, phys):
        idx = np.asarray(idx, dtype=np.int64)
        out = np.empty_like(idx)
        for t in range(idx.shape[0]):
            for j in range(idx.shape[1]):
                e = idx[t, j]
                c = off[e + 1] - off[e]
                out[t, j] = phys[off[e] + min(t // 97, c - 1)]
        return out
    assert _eplb_pins_fail(monkeypatch, oracle.eplb_oracle, "eplb_remap", bad) > 0


def test_planted_dedup_mistakes_are_caught(monkeypatch):
    real = oracle.dedup_oracle.dedup_layout

    def reversed_masks(idx, E, R):
        S, off, tok, mask, row_of = real(idx, E, R)
        k = np.asarray(idx).shape[1]
        flip = np.array([int(format(int(m), f"0{k}b")[::-1], 2) for m in mask], dtype=np.uint32)
        return S, off, tok, flip, row_of

    def tokens_descending(idx, E, R):
        S, off, tok, mask, row_of = real(idx, E, R)
        tok, mask = tok.copy(), mask.copy()
        for r in range(R):
            tok[off[r]:off[r + 1]] = tok[off[r]:off[r + 1]][::-1]
            mask[off[r]:off[r + 1]] = mask[off[r]:off[r + 1]][::-1]
        return S, off, tok, mask, row_of

    for bad in (reversed_masks, tokens_descending):
        monkeypatch.setattr(oracle.dedup_oracle, "dedup_layout", bad)
        monkeypatch.setattr(oracle, "dedup_layout", bad)
        failures = 0
        for fn in (test_dedup_layout_matches_hand_worked_example,
                   lambda: test_dedup_layout_invariants(0),
                   lambda: test_dedup_layout_invariants(1)):
            try:
                fn()
            except (AssertionError, ValueError, IndexError):
                failures += 1
        assert failures > 0, bad.__name__


# ---------------------------------------------------------------- FP8 (E4M3) weights
# (code, value) worked out by hand from the E4M3 bit layout: sign | 4 exponent
# bits, bias 7 | 3 mantissa bits; exponent 0 holds the subnormals m/8 * 2^-6.
E4M3_HAND = [(0x00, 0.0), (0x80, -0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
             (0x08, 2.0 ** -6), (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0xB8, -1.0),
             (0x77, 240.0), (0x78, 256.0), (0x7E, 448.0), (0xFE, -448.0)]


def test_e4m3_decode_hand_values_and_library_cast():
    got = oracle.e4m3_decode(np.array([c for c, _ in E4M3_HAND], dtype=np.uint8))
    for (c, want), v in zip(E4M3_HAND, got):
        assert v == want and math.copysign(1.0, v) == math.copysign(1.0, want), hex(c)
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # the table lookup in dequantise_rows gives the element-wise decode
    rnd = np.random.default_rng(4).integers(0, 256, (7, 33), dtype=np.uint8)
    np.testing.assert_array_equal(oracle.dequantise_rows(rnd, np.full(7, 2.0)),
                                  2.0 * oracle.e4m3_decode(rnd))


def test_fp8_single_expert_worked_by_hand():
    # One expert (E = k = 1, gate weight 1), d = 2, f = 1, x = (1, 2).
    # W13 codes: gate row (0x38, 0x40) = (1, 2) with scale 1/2; up row
    # (0x3C, 0xB8) = (1.5, -1) with scale 2.  W2 codes: (0x40) = 2 with scale
    # 1/4, (0x38) = 1 with scale 1.
    #   g = (1*1 + 2*2) / 2 = 2.5,  u = 2 * (1.5 - 2) = -1,  h = silu(2.5) * u
    #   y = (2/4 * h, 1 * h)
    h = 2.5 / (1 + math.exp(-2.5)) * -1.0
    c13 = np.array([[[0x38, 0x40], [0x3C, 0xB8]]], dtype=np.uint8)
    c2 = np.array([[[0x40], [0x38]]], dtype=np.uint8)
    out = oracle.moe_forward_fp8(np.array([[1.0, 2.0]]), np.zeros((2, 1)), None, c13,
                                 np.array([[0.5, 2.0]]), c2, np.array([[0.25, 1.0]]), 1)
    np.testing.assert_allclose(out["y"], [[0.5 * h, h]], rtol=1e-15, atol=0)


def _fp8_case(seed=0, T=24, d=64, E=4, k=2, f=64):
    """Tiny layer with E4M3 weights and power-of-two row scales (so the
    dequantised weights are exact bf16 values)."""
    rng = np.random.default_rng(seed)
    cfg = wl.MoEConfig("fp8-tiny", T=T, d=d, E=E, k=k, f=f)
    x = _np(wl.make_hidden(cfg, "cpu", seed))
    w_g, bias = wl.make_router(cfg, "cpu", seed)
    c13, _, c2, _ = wl.make_experts_fp8(cfg, "cpu", seed)
    c13, c2 = c13.numpy(), c2.numpy()
    s13 = np.ldexp(1.0, rng.integers(-10, -5, (E, 2 * f))).astype(np.float32)
    s2 = np.ldexp(1.0, rng.integers(-10, -5, (E, d))).astype(np.float32)
    return cfg, x, _np(w_g), _np(bias), c13, s13, c2, s2


def _y_fp8(case, s13=None, s2=None):
    cfg, x, w_g, b, c13, S13, c2, S2 = case
    return oracle.moe_forward_fp8(x, w_g, b, c13, S13 if s13 is None else s13, c2,
                                  S2 if s2 is None else s2, cfg.k, select_dtype=None)["y"]


def test_fp8_layer_is_the_bf16_layer_on_library_dequantised_weights():
    cfg, x, w_g, b, c13, s13, c2, s2 = case = _fp8_case()

    def deq(c, s):  # torch's E4M3 cast, row scale broadcast over K, then bf16
        w = torch.from_numpy(c).view(torch.float8_e4m3fn).float() * torch.from_numpy(s)[..., None]
        w16 = w.to(torch.bfloat16)
        assert torch.equal(w16.float(), w)  # power-of-two scales keep it exact
        return _np(w16)

    ref = oracle.moe_forward(x, w_g, b, deq(c13, s13), deq(c2, s2), cfg.k,
                             select_dtype=None)["y"]
    np.testing.assert_array_equal(_y_fp8(case), ref)


def test_fp8_row_scales_act_on_output_rows():
    cfg, x, w_g, b, c13, s13, c2, s2 = case = _fp8_case(seed=1)
    y = _y_fp8(case)
    # W_down row r produces output column r: doubling its scale in every
    # expert doubles y[:, r] exactly and leaves the other columns alone.
    r = 5
    s2b = s2.copy()
    s2b[:, r] *= 2
    y2 = _y_fp8(case, s2=s2b)
    np.testing.assert_array_equal(y2[:, r], 2 * y[:, r])
    np.testing.assert_array_equal(np.delete(y2, r, 1), np.delete(y, r, 1))
    # Up row j scales h_j linearly: y is affine in that scale.
    j = 3
    ys = []
    for m in (1.0, 2.0, 3.0):
        s = s13.copy()
        s[:, cfg.f + j] *= m
        ys.append(_y_fp8(case, s13=s))
    np.testing.assert_allclose(ys[2] - ys[0], 2 * (ys[1] - ys[0]), rtol=0, atol=1e-12)
    assert np.abs(ys[1] - ys[0]).max() > 1e-6
    # Zeroing gate row j or up row j removes the same term h_j = silu(g_j) u_j.
    zg, zu = s13.copy(), s13.copy()
    zg[:, j] = 0
    zu[:, cfg.f + j] = 0
    np.testing.assert_allclose(_y_fp8(case, s13=zg), _y_fp8(case, s13=zu), rtol=0, atol=1e-12)


def _fp8_pins_fail(monkeypatch, name, bad):
    monkeypatch.setattr(oracle.fp8_oracle, name, bad)
    monkeypatch.setattr(oracle, name, bad)
    failures = 0
    for fn in (test_e4m3_decode_hand_values_and_library_cast,
               test_fp8_single_expert_worked_by_hand,
               test_fp8_layer_is_the_bf16_layer_on_library_dequantised_weights,
               test_fp8_row_scales_act_on_output_rows):
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def test_planted_fp8_mistakes_are_caught(monkeypatch):
    good_decode = oracle.fp8_oracle.e4m3_decode

    def bias8(codes):  # exponent bias 8 instead of 7
        return good_decode(codes) / 2

    def no_subnormals(codes):  # exponent field 0 read with an implicit leading 1
        c = np.asarray(codes, dtype=np.uint8)
        v = good_decode(c)
        e0 = ((c >> 3) & 0xF) == 0
        return np.where(e0, np.where(c >> 7, -1.0, 1.0) * np.ldexp(1 + (c & 7) / 8.0, -7), v)

    def per_column(codes, scale):  # the scale applied along K instead of the rows
        w = good_decode(codes)
        s = np.asarray(scale, dtype=np.float64)
        return w * np.resize(s, w.shape[-1])[None, :]

    assert _fp8_pins_fail(monkeypatch, "e4m3_decode", bias8) > 0
    monkeypatch.undo()
    assert _fp8_pins_fail(monkeypatch, "e4m3_decode", no_subnormals) > 0
    monkeypatch.undo()
    assert _fp8_pins_fail(monkeypatch, "dequantise_rows", per_column) > 0
