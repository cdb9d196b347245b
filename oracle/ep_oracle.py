"""Plain CPU oracle of the expert-parallel exchange (R ranks, each holding
E/R whole experts and its own tokens).

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests and bench.py's
CPU legs may use it; it shares nothing with the CUDA library.

"Serving MoE models with expert parallelism on 8xH200", section "Tensor
parallel vs expert parallel": each device keeps whole experts, a token is
sent to the devices holding its selected experts, and the expert outputs are
sent back by a second exchange.  "Wide Expert Parallelism", sections "Expert
Parallelism: keep specialists whole" (contiguous blocks of experts per
device) and "All-to-all communication: the essential tradeoff".  "Expert
Parallelism for MoE Models", section "Mechanics of Token Routing and
All-to-All Communication": the representation travels to the expert and the
output travels back to the token's device.

Readings taken (the pages give no layout):

* rank r owns experts [r E/R, (r+1) E/R); each rank routes its own tokens;
* a rank sends, for each destination, the rows of its expert-major dispatch
  buffer that belong to the destination's experts (so they arrive ordered by
  local expert, then token) together with its per-expert row counts;
* the receiver keeps what it received ordered by source rank; for the
  expert FFN it regroups the rows by local expert, sources in rank order;
* outputs return in the order the rows were received, and the source sums
  its tokens' k rows with the gates.
"""

from __future__ import annotations

import numpy as np

from . import moe_oracle as M

__all__ = ["ep_recv_experts", "ep_forward"]


def ep_recv_experts(recv_counts, R, E_loc):
    """Local expert of every received row: rows come ordered by source rank,
    then local expert, recv_counts[s][e] rows of each."""
    recv_counts = np.asarray(recv_counts, dtype=np.int64).reshape(R, E_loc)
    labels = []
    for s in range(R):
        for e in range(E_loc):
            labels += [e] * int(recv_counts[s, e])
    return np.array(labels, dtype=np.int32)


def ep_forward(xs, w_g, bias, w13, w2, k, select_dtype=np.float32):
    """The layer over R ranks' token batches xs[0..R-1] (each (T_r, d)), the
    exchange carried out step by step.  Returns a dict of per-rank lists:
    y, idx, w, counts (per source), recv_counts, x_recv, expert_of_row,
    regrouped (received-row index of each regrouped row), z_recv."""
    R = len(xs)
    E = np.asarray(w_g).shape[1]
    if E % R:
        raise ValueError("R must divide E")
    E_loc = E // R
    out = {key: [] for key in ("idx", "w", "counts", "offsets", "row_of", "x_perm")}
    # 1. every rank routes and dispatches its own tokens, expert-major
    for x in xs:
        x = M._f64(x)
        L = M.router_logits(x, w_g, bias)
        Ls = L.astype(select_dtype) if select_dtype is not None else L
        idx = M.topk_select_sorted(Ls, k)
        counts = M.expert_counts(idx, E)
        offsets = M.expert_offsets(counts)
        perm, row_of = M.dispatch_rows(idx, E)
        out["idx"].append(idx)
        out["w"].append(M.gate_weights(L, idx))
        out["counts"].append(counts)
        out["offsets"].append(offsets)
        out["row_of"].append(row_of)
        out["x_perm"].append(x[np.asarray(perm, dtype=np.int64)])
    # 2. the exchange: rank r receives, from every source s in rank order,
    #    s's rows of r's experts and s's counts of them
    for key in ("recv_counts", "x_recv", "expert_of_row", "regrouped", "z_recv", "y"):
        out[key] = []
    for r in range(R):
        lo, hi = r * E_loc, (r + 1) * E_loc
        rc = np.stack([out["counts"][s][lo:hi] for s in range(R)])
        xr = np.concatenate([out["x_perm"][s][out["offsets"][s][lo]:out["offsets"][s][hi]]
                             for s in range(R)], axis=0)
        lab = ep_recv_experts(rc, R, E_loc)
        # 3. regroup by local expert (stable: sources in rank order) and run
        #    the local experts; outputs go back to received order
        order = np.argsort(lab, kind="stable")
        z = np.zeros((xr.shape[0], xr.shape[1]))
        for e in range(E_loc):
            rows = order[lab[order] == e]
            if rows.size:
                z[rows] = M.swiglu_ffn(xr[rows], w13[lo + e], w2[lo + e])
        out["recv_counts"].append(rc.astype(np.int32))
        out["x_recv"].append(xr)
        out["expert_of_row"].append(lab)
        out["regrouped"].append(order.astype(np.int64))
        out["z_recv"].append(z)
    # 4. the return exchange: source s gets back, from every rank r, the
    #    outputs of the rows it sent there, which restores its expert-major
    #    order; then the gate-weighted sum
    for s in range(R):
        parts = []
        for r in range(R):
            lo, hi = r * E_loc, (r + 1) * E_loc
            before = sum(int(out["counts"][s2][lo:hi].sum()) for s2 in range(s))
            n = int(out["counts"][s][lo:hi].sum())
            parts.append(out["z_recv"][r][before:before + n])
        z_back = np.concatenate(parts, axis=0) if parts else np.zeros((0, xs[s].shape[1]))
        out["y"].append(M.combine(z_back, out["row_of"][s], out["w"][s]))
    return out
