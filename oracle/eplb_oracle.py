"""Plain CPU oracle for expert load balancing (EPLB-style replica placement).

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests and bench.py's
CPU legs may use it; it shares nothing with the CUDA library.

What the pages fix, and the reading taken where they are silent:

* "Serving MoE models with expert parallelism on 8xH200", section "Routing
  imbalance": the per-expert load is measured, the busiest experts are given
  extra copies on devices that have room, and placement is reshuffled so that
  busy and idle experts share devices.
* "vLLM Expert Parallel deployment" (EPLB section): the balancer collects
  load over a window and redistributes expert-to-rank mappings; the number of
  redundant experts is a parameter (num_redundant_experts).

The pages give no algorithm.  Plainest reading, all in integers so every
decision is exact:

1. Replication: every expert starts with one copy; n_redundant times, the
   expert with the largest load per copy gets one more (ties: lower id).
2. Shares: replica i of expert e is credited load_e // n_e, plus one if
   i < load_e % n_e (so the shares sum to load_e).
3. Placement: the E + n_redundant replicas go to R ranks of S = (E+n_r)/R
   slots each, in order of decreasing share (ties: lower expert id, then
   lower replica index), each to the least-loaded rank that still has a free
   slot (ties: lower rank).  Rank r's physical slots are r*S .. r*S+S-1 in
   the order they were filled, so rank r owns a contiguous block of physical
   experts exactly as in the plain layout.
4. Replica choice: slot j of token t with logical expert e uses replica
   t mod n_e.
"""

from __future__ import annotations

import numpy as np

__all__ = ["eplb_replicate", "eplb_shares", "eplb_place", "eplb_plan", "eplb_remap",
           "rank_loads"]


def eplb_replicate(load, n_redundant):
    """Copies per expert (step 1)."""
    load = [int(v) for v in load]
    E = len(load)
    n = [1] * E
    for _ in range(int(n_redundant)):
        best = 0
        for e in range(1, E):
            # load[e]/n[e] > load[best]/n[best], compared exactly
            if load[e] * n[best] > load[best] * n[e]:
                best = e
        n[best] += 1
    return np.array(n, dtype=np.int64)


def eplb_shares(load, n):
    """Integer share of every replica (step 2): list of (expert, replica, share)."""
    out = []
    for e, (l, c) in enumerate(zip(load, n)):
        l, c = int(l), int(c)
        for i in range(c):
            out.append((e, i, l // c + (1 if i < l % c else 0)))
    return out


def eplb_place(load, n, R):
    """Greedy placement (step 3).  Returns (phys_to_logical, rep_offsets,
    rep_phys): replica i of expert e sits in physical slot
    rep_phys[rep_offsets[e] + i] and phys_to_logical of that slot is e."""
    n = [int(c) for c in n]
    P = sum(n)
    if P % R:
        raise ValueError("E + n_redundant must be a multiple of R")
    S = P // R
    reps = eplb_shares(load, n)
    reps.sort(key=lambda r: (-r[2], r[0], r[1]))
    rank_load = [0] * R
    rank_fill = [0] * R
    rep_offsets = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    rep_phys = np.full(P, -1, dtype=np.int64)
    phys_to_logical = np.full(P, -1, dtype=np.int64)
    for e, i, share in reps:
        r = min((r for r in range(R) if rank_fill[r] < S), key=lambda r: (rank_load[r], r))
        slot = r * S + rank_fill[r]
        rank_fill[r] += 1
        rank_load[r] += share
        rep_phys[rep_offsets[e] + i] = slot
        phys_to_logical[slot] = e
    return phys_to_logical, rep_offsets, rep_phys


def eplb_plan(load, n_redundant, R):
    """Replication then placement."""
    n = eplb_replicate(load, n_redundant)
    return eplb_place(load, n, R)


def eplb_remap(idx, rep_offsets, rep_phys):
    """Physical expert ids (step 4): idx_phys[t, j] = replica t mod n_e of e."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    out = np.empty_like(idx)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            c = rep_offsets[e + 1] - rep_offsets[e]
            out[t, j] = rep_phys[rep_offsets[e] + t % c]
    return out


def rank_loads(counts, R):
    """Rows per rank when rank r owns the contiguous block r of the experts."""
    counts = np.asarray(counts, dtype=np.int64)
    return counts.reshape(R, counts.shape[0] // R).sum(axis=1)
