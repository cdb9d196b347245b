"""Plain fp64 CPU oracle for the routed mixture-of-experts layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` use it.  It shares no code,
tables or helpers with the CUDA library; it takes NumPy arrays and returns
NumPy arrays.

What the layer computes, and where each step comes from:

* "Wide Expert Parallelism" (llm-d), section "What is an MoE layer?": a small
  routing gate inspects every token and sends it to a few of the layer's
  experts; the DeepSeek example there picks 8 of 256.
* "Serving MoE models with expert parallelism on 8xH200", section "Tensor
  parallel vs expert parallel": tokens are dispatched to the holders of their
  selected experts, run through full-size expert GEMMs, and sent back by a
  second exchange; with 256 experts on 8 GPUs each GPU owns 32 whole experts.
* Same page, section "Batching: MoE needs bigger batches than you think": the
  mean load of an expert is B*k/E tokens per step.
* Same page, section "Routing imbalance": per-expert token counts per layer,
  and the busiest-GPU / mean ratio as the imbalance factor.
* "Expert Parallelism for MoE Models" (apxml), section "Mechanics of Token
  Routing and All-to-All Communication": a routing layer assigns each token
  to experts, the token representation travels to the expert and the output
  travels back.
* "Wide Expert Parallelism", section "Expert Parallelism: keep specialists
  whole": each device owns a contiguous block of whole experts.

The pages never write the layer's arithmetic down.  Where they are silent this
oracle takes the plainest reading consistent with them (each one is named at
the function that uses it):

* scoring is a softmax over the E linear router logits;
* the k largest logits are selected, ties going to the lower expert index,
  slots ordered by descending logit;
* the gate weights are the softmax renormalised over the k selected experts;
* an expert is a SwiGLU FFN: h = silu(x W_gate) * (x W_up), z = h W_down;
* the combine is the gate-weighted sum of the k expert outputs;
* rows inside an expert keep ascending token order;
* virtual expert-parallel rank r owns experts [r*E/R, (r+1)*E/R), and token t
  belongs to source rank t // ceil(T/R).

Weight layouts (the same as the library's, so tests pass the same arrays):
``w13[e]`` is (2f, d): rows 0..f-1 are W_gate[e] transposed, rows f..2f-1 are
W_up[e] transposed.  ``w2[e]`` is (d, f): W_down[e] transposed.  Everything is
widened to float64 on entry; bf16 and fp32 values widen exactly.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "router_logits",
    "topk_select",
    "topk_select_sorted",
    "gate_weights",
    "expert_counts",
    "expert_offsets",
    "dispatch_rows",
    "virtual_ep_layout",
    "silu",
    "swiglu_ffn",
    "expert_outputs",
    "combine",
    "moe_forward",
    "imbalance_factor",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def router_logits(x, w_g, bias=None):
    """Router scores L[t, e] = sum_i x[t, i] * W_g[i, e] + bias[e], in fp64.

    The routing gate of "Wide Expert Parallelism", section "What is an MoE
    layer?"; the optional per-expert bias is how skewed popularity is injected
    ("Serving MoE models ... on 8xH200", section "Routing imbalance").
    x: (T, d); w_g: (d, E); bias: (E,) or None.  Returns (T, E) float64.
    """
    x = _f64(x)
    w_g = _f64(w_g)
    out = x @ w_g
    if bias is not None:
        out = out + _f64(bias)[None, :]
    return out


def topk_select(logits, k):
    """Brute-force top-k by rank counting (the definition, O(E^2) per token).

    Reading where the pages are silent: expert e outranks e' when its logit is
    larger, or equal with a lower index.  rank(e) = #{e': L[e'] > L[e]} +
    #{e' < e: L[e'] == L[e]}; e is selected iff rank(e) < k and its slot is
    rank(e).  -0.0 and +0.0 compare equal (IEEE), so they tie.
    The selection decides an integer, so callers pass the logits in the
    precision the decision is taken in (fp32 for the library); they are
    compared exactly as given.
    Returns idx (T, k) int32 with idx[t, j] the expert in slot j.
    """
    L = np.asarray(logits)
    T, E = L.shape
    if not 1 <= k <= E:
        raise ValueError("k must lie in [1, E]")
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        row = L[t]
        for e in range(E):
            greater = int(np.count_nonzero(row > row[e]))
            equal_lower = int(np.count_nonzero(row[:e] == row[e]))
            r = greater + equal_lower
            if r < k:
                idx[t, r] = e
    return idx


def topk_select_sorted(logits, k):
    """Sort-based top-k under the same total order (descending value, then
    ascending index).  A second, independent form used to cross-check
    :func:`topk_select` and fast enough for large T."""
    L = np.asarray(logits)
    T, E = L.shape
    if not 1 <= k <= E:
        raise ValueError("k must lie in [1, E]")
    # Stable sort of -L keeps the lower index first among equal values.  The
    # negation maps +0/-0 to -0/+0, which still compare equal, so the stable
    # order among them is by index as required.
    order = np.argsort(-L.astype(np.float64), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gate_weights(logits, idx):
    """Gate weights: softmax over all E logits, then renormalised over the k
    selected experts, w[t, j] = p[idx[t, j]] / sum_j' p[idx[t, j']].

    Reading where the pages are silent (softmax scoring, renormalisation).
    The max is subtracted before exponentiation; the top slot then holds
    exp(0) = 1, so the denominator is never zero.  fp64 throughout.
    """
    L = _f64(logits)
    idx = np.asarray(idx)
    m = L.max(axis=1, keepdims=True)
    p = np.exp(L - m)
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def expert_counts(idx, E):
    """counts[e] = #{(t, j): idx[t, j] == e}, the per-expert token counts of
    "Serving MoE models ... on 8xH200", section "Routing imbalance"."""
    idx = np.asarray(idx).reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    for e in idx:
        counts[int(e)] += 1
    return counts.astype(np.int32)


def expert_offsets(counts):
    """Exclusive prefix sum, E + 1 entries; offsets[E] = T*k."""
    counts = np.asarray(counts, dtype=np.int64)
    off = np.zeros(counts.shape[0] + 1, dtype=np.int64)
    run = 0
    for e, c in enumerate(counts):
        off[e] = run
        run += int(c)
    off[-1] = run
    return off.astype(np.int32)


def dispatch_rows(idx, E):
    """The local form of the dispatch exchange: every (token, slot) pair gets
    a row of the expert-major buffer.

    Rows are ordered by (expert ascending, token ascending) -- a reading where
    the pages are silent.  A token never selects one expert twice, so the
    order is total.  Returns perm (P,) with perm[row] = token and row_of
    (T, k) with row_of[t, j] = row, P = T*k.
    Source: "Serving MoE models ... on 8xH200", section "Tensor parallel vs
    expert parallel" (tokens are dispatched to their experts' holders);
    "Expert Parallelism for MoE Models", section "Mechanics of Token Routing
    and All-to-All Communication".
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    offsets = expert_offsets(expert_counts(idx, E)).astype(np.int64)
    fill = offsets[:-1].copy()
    perm = np.zeros(T * k, dtype=np.int32)
    row_of = np.zeros((T, k), dtype=np.int32)
    for t in range(T):  # ascending token order inside each expert
        for j in range(k):
            e = int(idx[t, j])
            r = int(fill[e])
            fill[e] += 1
            perm[r] = t
            row_of[t, j] = r
    return perm, row_of


def virtual_ep_layout(idx, E, R):
    """Virtual expert-parallel layout on one device.

    owner(e) = e // (E/R): contiguous blocks of whole experts per rank ("Wide
    Expert Parallelism", section "Expert Parallelism: keep specialists whole";
    256 experts on 8 GPUs is 32 each in "Serving MoE models ... on 8xH200",
    section "Tensor parallel vs expert parallel").
    src(t) = t // ceil(T/R): a reading -- with data-parallel attention each
    rank serves its own requests, taken here as contiguous token blocks.
    S[s, r] counts the (token, slot) rows that source rank s sends to rank r;
    rank_offsets[r] = first row of rank r in the expert-major buffer.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    if R < 1 or E % R != 0:
        raise ValueError("R must divide E")
    per = E // R
    chunk = -(-T // R) if T > 0 else 1
    S = np.zeros((R, R), dtype=np.int64)
    for t in range(T):
        s = t // chunk
        for j in range(k):
            S[s, int(idx[t, j]) // per] += 1
    offsets = expert_offsets(expert_counts(idx, E)).astype(np.int64)
    rank_offsets = np.array([offsets[r * per] for r in range(R)] + [offsets[E]],
                            dtype=np.int64)
    return S.astype(np.int32), rank_offsets.astype(np.int32)


def silu(z):
    """silu(z) = z / (1 + exp(-z)), fp64."""
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(X, w13_e, w2_e):
    """One expert's SwiGLU FFN on the rows X (n, d), in fp64 with no rounding
    between the three products: z = (silu(X W_gate) * (X W_up)) W_down.

    The expert GEMMs of "Serving MoE models ... on 8xH200" (full-size expert
    GEMMs; gate and up projections stream the expert's weights, section
    "Batching ..."); the SwiGLU form is a reading where the pages are silent.
    w13_e: (2f, d) with gate rows first; w2_e: (d, f).
    """
    X = _f64(X)
    w13_e = _f64(w13_e)
    w2_e = _f64(w2_e)
    f = w13_e.shape[0] // 2
    g = X @ w13_e[:f].T
    u = X @ w13_e[f:].T
    return (silu(g) * u) @ w2_e.T


def expert_outputs(x, perm, offsets, w13, w2, ffn=None):
    """Run every expert's FFN (``ffn``, default swiglu_ffn) over its
    contiguous rows; returns Z (P, d)."""
    ffn = swiglu_ffn if ffn is None else ffn
    x = _f64(x)
    offsets = np.asarray(offsets, dtype=np.int64)
    E = offsets.shape[0] - 1
    P = int(offsets[-1])
    Z = np.zeros((P, x.shape[1]), dtype=np.float64)
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            Z[a:b] = ffn(x[np.asarray(perm[a:b], dtype=np.int64)], w13[e], w2[e])
    return Z


def combine(Z, row_of, w):
    """Return exchange plus combine: y[t] = sum_j w[t, j] * Z[row_of[t, j]].

    "Serving MoE models ... on 8xH200", section "Tensor parallel vs expert
    parallel" (results return through a second exchange); weighting by the
    gates is a reading where the pages are silent.  fp64.
    """
    Z = _f64(Z)
    w = _f64(w)
    row_of = np.asarray(row_of, dtype=np.int64)
    T, k = row_of.shape
    y = np.zeros((T, Z.shape[1]), dtype=np.float64)
    for j in range(k):
        y += w[:, j:j + 1] * Z[row_of[:, j]]
    return y


def imbalance_factor(counts, R):
    """Busiest virtual rank's row count divided by the mean per rank
    ("Serving MoE models ... on 8xH200", section "Routing imbalance")."""
    counts = np.asarray(counts, dtype=np.int64)
    E = counts.shape[0]
    per_rank = counts.reshape(R, E // R).sum(axis=1)
    mean = per_rank.mean()
    return float(per_rank.max() / mean) if mean > 0 else 0.0


def moe_forward(x, w_g, bias, w13, w2, k, R=0, select_dtype=np.float32,
                idx=None, ffn=None):
    """The whole layer, step by step, in the order the pages describe it.

    1. router logits in fp64;
    2. top-k selection, taken on the logits rounded to ``select_dtype`` (the
       precision the library takes the decision in) unless ``idx`` is given
       (the tests pass oracle-made alternatives for near-ties here);
    3. gates from the fp64 logits;
    4. counts, offsets, dispatch rows (and the virtual-EP layout if R > 1);
    5. expert SwiGLU FFNs on each expert's rows (``ffn`` replaces
       swiglu_ffn, e.g. with a quantised variant);
    6. gate-weighted combine.
    Returns a dict of every intermediate.
    """
    x = _f64(x)
    L = router_logits(x, w_g, bias)
    E = L.shape[1]
    if idx is None:
        Ls = L.astype(select_dtype) if select_dtype is not None else L
        idx = topk_select_sorted(Ls, k)
    idx = np.asarray(idx, dtype=np.int32)
    w = gate_weights(L, idx)
    counts = expert_counts(idx, E)
    offsets = expert_offsets(counts)
    perm, row_of = dispatch_rows(idx, E)
    out = dict(logits=L, idx=idx, w=w, counts=counts, offsets=offsets,
               perm=perm, row_of=row_of)
    if R and R > 1:
        S, rank_offsets = virtual_ep_layout(idx, E, R)
        out.update(send_counts=S, rank_offsets=rank_offsets)
    Z = expert_outputs(x, perm, offsets, w13, w2, ffn)
    out["z"] = Z
    out["y"] = combine(Z, row_of, w)
    return out
