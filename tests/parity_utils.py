"""Helpers shared by the parity tests: tolerances, the router-logit error
bound, and validation of selections when fp32 logits nearly tie."""

from __future__ import annotations

import numpy as np
import torch

U32 = 2.0 ** -24  # unit roundoff of fp32

# Layer-output tolerance (bf16 inputs, fp32 accumulation): relative L2 error
# <= 5e-3 and per element |got - ref| <= 2e-2 * (1 + |ref|).
REL_L2 = 5e-3
ELEM = 2e-2


def np64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_layer_close(got, ref, what=""):
    got = np64(got) if not isinstance(got, np.ndarray) else got.astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / nref if nref > 0 else np.linalg.norm(got)
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    viol = np.abs(got - ref) > ELEM * (1.0 + np.abs(ref))
    assert not viol.any(), (f"{what}: {int(viol.sum())} elements off; worst "
                            f"{np.max(np.abs(got - ref) / (1 + np.abs(ref))):.3e}")
    return rel


def logit_bound(x64, wg64, bias64=None):
    """Rigorous forward-error bound of an fp32 dot product of length d plus a
    bias add, valid for any summation order: gamma_{d+2} * (sum|x W| + |b|),
    gamma_n = n u / (1 - n u)."""
    d = x64.shape[1]
    n = d + 2
    gamma = n * U32 / (1 - n * U32)
    s = np.abs(x64) @ np.abs(wg64)
    if bias64 is not None:
        s = s + np.abs(bias64)[None, :]
    return gamma * s


def logit_bound_tensor_cores(x64, wg64, bias64=None):
    """Bound for the tensor-core router (T > 256).

    W_g is carried as three bf16 planes hi + mid + lo; every product of a
    bf16 x with a bf16 plane value is exact in fp32, and the planes leave a
    residual below 2^-24 |W| per term, counted as one more rounding.  The
    3d products are then accumulated in fp32 by the tensor cores.  Their
    adds are not guaranteed to round to nearest; the reading taken is that
    each add may truncate (round toward zero), whose relative error bound is
    2^-23 = 2u instead of u.  n = 3d + 4 covers the 3d - 1 adds of the
    products (in any grouping, the K partitions' partial sums included), the
    plane residual and the bias add, with two to spare; the standard bound
    with unit roundoff 2u is then
    gamma_n(2u) (sum|x W| + |b|), gamma_n(2u) = 2nu / (1 - 2nu)."""
    d = x64.shape[1]
    n = 3 * d + 4
    u2 = 2 * U32
    gamma = n * u2 / (1 - n * u2)
    s = np.abs(x64) @ np.abs(wg64)
    if bias64 is not None:
        s = s + np.abs(bias64)[None, :]
    return gamma * s


def selection_is_valid(L64_row, delta_row, sel):
    """True when some logits within [L - delta, L + delta] make `sel` (an
    ordered list of k experts) the top-k in that slot order."""
    sel = list(sel)
    if len(set(sel)) != len(sel):
        return False
    lo = L64_row - delta_row
    hi = L64_row + delta_row
    mask = np.zeros(L64_row.shape[0], dtype=bool)
    mask[sel] = True
    if (~mask).any() and hi[mask].min() < lo[~mask].max():
        return False
    for a, b in zip(sel[:-1], sel[1:]):
        if hi[a] < lo[b]:
            return False
    return True


def unique_selection(L64_row, delta_row, k):
    """The selected set if every logit-error-consistent choice gives the same
    set, else None."""
    order = np.argsort(-L64_row, kind="stable")
    top, rest = order[:k], order[k:]
    if rest.size == 0:
        return set(top.tolist())
    if (L64_row[top] - delta_row[top]).min() > (L64_row[rest] + delta_row[rest]).max():
        return set(top.tolist())
    return None


def order_by_logit(L64_row, sel):
    """Slot order of a selected set: descending logit, then ascending index."""
    return sorted(sel, key=lambda e: (-L64_row[e], e))


class LazyExperts:
    """Indexable view that widens one expert of a device tensor to float64 on
    the host when the oracle asks for it (keeps host memory to one expert)."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, e):
        return self.t[int(e)].float().cpu().numpy().astype(np.float64)


def token_sample(n=256, seed=0):
    """A seeded sample of n tokens of the batch that always includes tokens
    routed to the two hottest and the four coldest touched experts (the
    first two and the last token of each), and the first and last token."""
    def pick(idx_h, counts):
        rng = np.random.default_rng(seed)
        T = idx_h.shape[0]
        touched = np.nonzero(counts)[0]
        order = touched[np.argsort(-counts[touched], kind="stable")]
        must = {0, T - 1}
        for e in np.concatenate([order[:2], order[-4:]]):
            toks = np.nonzero((idx_h == e).any(1))[0]
            must.update(int(t) for t in toks[:2])
            must.add(int(toks[-1]))
        must = np.array(sorted(must), dtype=np.int64)
        rest = np.setdiff1d(np.arange(T), must)
        fill = rng.choice(rest, size=max(0, min(n - must.size, rest.size)), replace=False)
        return np.unique(np.concatenate([must, fill]))
    return pick
