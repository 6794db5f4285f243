"""Parity rules between the CUDA path and the fp64 oracle.

Scores (fp32 accumulation on the GPU against fp64 in the oracle) must satisfy, per row,
    |gpu - ref| <= RTOL * |ref| + ATOL_REL * max_s |ref[s]|        (RTOL 1e-3, ATOL_REL 1e-4)
Selected sets (routed heads, top-k tokens) must equal the oracle's, except for elements
whose oracle value lies within that tolerance of the oracle's cutoff (the h-th / k-th
largest value): those may be swapped for one another.
"""

from __future__ import annotations

import numpy as np

RTOL = 1e-3
ATOL_REL = 1e-4


def tol(ref_vals: np.ndarray, row_ref: np.ndarray) -> np.ndarray:
    scale = float(np.max(np.abs(row_ref))) if row_ref.size else 0.0
    return RTOL * np.abs(ref_vals) + ATOL_REL * scale


def check_scores(gpu: np.ndarray, ref: np.ndarray, what: str = "scores"):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = tol(ref, ref)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, (f"{what}: {bad.size} of {ref.size} outside tolerance; first at "
                           f"{bad[0]}: gpu {gpu[bad[0]]!r} ref {ref[bad[0]]!r} bound {bound[bad[0]]!r}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0


def check_selection(sel: np.ndarray, ref_vals: np.ndarray, k: int, what: str = "top-k",
                    ids: np.ndarray | None = None):
    """`sel`: GPU-selected ids (padding -1).  `ref_vals[i]`: oracle value of item ids[i]
    (ids default to 0..n-1).  Checks validity, count, padding and the cutoff rule."""
    n = ref_vals.shape[0]
    if ids is None:
        ids = np.arange(n)
    pos_of = {int(t): i for i, t in enumerate(ids)}
    sel = np.asarray(sel)
    m = min(n, k)
    valid = sel[:m]
    assert np.all(sel[m:] == -1), f"{what}: padding after {m} entries is not -1"
    assert np.all(valid >= 0), f"{what}: fewer than {m} valid entries"
    assert len(set(valid.tolist())) == m, f"{what}: duplicate entries"
    assert all(int(t) in pos_of for t in valid), f"{what}: entry outside the candidate range"
    if n <= k:
        assert set(valid.tolist()) == set(int(t) for t in ids), f"{what}: short row not complete"
        return 0
    order = np.lexsort((ids, -ref_vals))
    ref_set = set(int(ids[i]) for i in order[:k])
    cut = ref_vals[order[k - 1]]
    ctol = tol(np.array([cut]), ref_vals)[0]
    got = set(int(t) for t in valid)
    missing = ref_set - got
    extra = got - ref_set
    for t in missing:
        v = ref_vals[pos_of[t]]
        assert v <= cut + ctol, f"{what}: missed {t} (ref {v!r}, cutoff {cut!r}, tol {ctol!r})"
    for t in extra:
        v = ref_vals[pos_of[t]]
        assert v >= cut - ctol, f"{what}: extra {t} (ref {v!r}, cutoff {cut!r}, tol {ctol!r})"
    return len(missing)


def check_order(idx: np.ndarray, vals: np.ndarray, what: str = "order"):
    """GPU output rows are sorted by descending value, ties by ascending index."""
    m = int(np.sum(idx >= 0))
    v, i = vals[:m], idx[:m]
    for a in range(m - 1):
        assert v[a] > v[a + 1] or (v[a] == v[a + 1] and i[a] < i[a + 1]), \
            f"{what}: entries {a},{a + 1} out of order ({v[a]},{i[a]}) ({v[a + 1]},{i[a + 1]})"
    assert np.all(np.isneginf(vals[m:])), f"{what}: padding values are not -inf"
