"""Plain CPU oracle for token-deduplicated per-rank dispatch.

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests and bench.py's
CPU legs may use it; it shares nothing with the CUDA library.

"Serving MoE models with expert parallelism on 8xH200", section "Tensor
parallel vs expert parallel", and "Expert Parallelism for MoE Models",
section "Mechanics of Token Routing and All-to-All Communication": a token's
representation travels to the devices holding its selected experts.  When
several of a token's k experts live on the same device the representation
only has to travel there once.  Readings taken (the pages give no layout):

* owner(e) = e // (E/R) and src(t) = t // ceil(T/R), as in the plain virtual
  expert-parallel layout;
* token t is sent once to every rank r that owns at least one of its
  selected experts; S'[s, r] counts those (token, rank) pairs by source;
* the send buffer is rank-major, tokens ascending inside a rank (a stable
  counting sort by destination rank); each row carries the token and a
  k-bit mask of the token's slots whose expert that rank owns;
* rank_row_of[t, r] is the row of (t, r), or -1 when t sends nothing to r.
"""

from __future__ import annotations

import numpy as np

__all__ = ["dedup_layout"]


def dedup_layout(idx, E, R):
    """Returns (S_dedup [R, R], rank_offsets [R + 1], token_of [rows],
    slot_mask [rows], rank_row_of [T, R])."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    if R < 1 or E % R != 0:
        raise ValueError("R must divide E")
    per = E // R
    chunk = -(-T // R) if T > 0 else 1
    # which of token t's slots land on rank r
    masks = np.zeros((T, R), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            masks[t, idx[t, j] // per] |= 1 << j
    S = np.zeros((R, R), dtype=np.int64)
    for t in range(T):
        for r in range(R):
            if masks[t, r]:
                S[t // chunk, r] += 1
    per_rank = S.sum(axis=0)
    rank_offsets = np.concatenate([[0], np.cumsum(per_rank)])
    token_of, slot_mask = [], []
    rank_row_of = np.full((T, R), -1, dtype=np.int64)
    for r in range(R):
        for t in range(T):
            if masks[t, r]:
                rank_row_of[t, r] = len(token_of)
                token_of.append(t)
                slot_mask.append(masks[t, r])
    return (S.astype(np.int32), rank_offsets.astype(np.int32),
            np.array(token_of, dtype=np.int32), np.array(slot_mask, dtype=np.uint32),
            rank_row_of.astype(np.int32))
