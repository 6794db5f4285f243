"""Pins for the fp64 oracle: checks against facts fixed outside the oracle itself.

Each check takes the oracle module as an argument, so that the same checks can be
run against deliberately broken copies of the oracle (see test_oracle_mutations.py)
to show that a plausible mistake is caught.

Sources of truth used here:
  * the bf16 format itself: torch's own bf16 -> float64 conversion over all 65,536 bit
    patterns, and values fixed by the format (1.0, -2.0, the smallest subnormal, inf);
  * hand-worked examples of Eqs. (1), (2), (4), (7)-(12) in tests/golden/
    ("MISA: Mixture of Indexer Sparse Attention", Introduction and Methodology);
  * closed forms (the mean of an arithmetic progression of keys);
  * library routines for selection (heapq.nlargest) and a brute-force rank count;
  * structural invariants of the equations: h = H^I turns Eq. (9) into Eq. (1);
    k' >= P turns MISA-dagger into the dense TopK; scaling or sign-flipping w
    leaves the routed head set unchanged (|A| in Eq. 7).
"""

from __future__ import annotations

import heapq

import numpy as np

from tests.golden import fixtures


def _q(fx, H, d):
    return fx["q"].reshape(H, d)


# ----------------------------------------------------------------- hand-worked examples
def check_dense_hand(orc):
    fx = fixtures.load("eq1_dense_hand.txt")
    H, d, L = int(fx["H"][0]), int(fx["d"][0]), int(fx["L"][0])
    q, w, k = _q(fx, H, d), fx["w"], fx["k"].reshape(L, d)
    I = orc.dense_scores(q, w, k, L)
    assert np.array_equal(I, fx["I"]), (I, fx["I"])
    idx, vals = orc.topk(I, 3)
    assert list(idx) == [int(x) for x in fx["top3"]], idx
    assert np.array_equal(orc.token_scores(q, w, k, L, [0]), fx["routed_h0"])
    assert np.array_equal(orc.token_scores(q, w, k, L, [1]), fx["routed_h1"])


def check_router_hand(orc):
    fx = fixtures.load("eq7_router_hand.txt")
    H, d, B, L = int(fx["H"][0]), int(fx["d"][0]), int(fx["B"][0]), int(fx["L"][0])
    P = int(fx["pos"][0]) + 1
    q, w, k = _q(fx, H, d), fx["w"], fx["k"].reshape(L, d)
    kp = orc.pool_keys(k[:P], B)
    assert np.array_equal(kp, fx["kpool"].reshape(-1, d)), kp
    E = orc.router_energy(q, w, k, P, B)
    assert np.allclose(E, fx["E"], rtol=0, atol=1e-15), E
    assert list(orc.select_heads(E, H)) == [int(x) for x in fx["heads"]]
    r = orc.misa_row(q, w, k, P, B, 2, 5)
    assert list(r["heads"]) == [1, 0]
    assert np.array_equal(r["scores"], fx["routed_h2"]), r["scores"]
    assert list(r["idx"]) == [int(x) for x in fx["routed_h2_top5"]], r["idx"]
    assert np.array_equal(orc.dense_scores(q, w, k, P), fx["dense"])
    r1 = orc.misa_row(q, w, k, P, B, 1, 1)
    assert list(r1["heads"]) == [int(x) for x in fx["h1_heads"]]
    assert list(r1["idx"]) == [int(x) for x in fx["h1_misa_top1"]], r1["idx"]
    omega, _ = orc.topk(r1["scores"], 3)
    assert list(omega) == [int(x) for x in fx["h1_omega_k3"]], omega
    dg = orc.misa_dagger_row(q, w, k, P, omega, 1)
    assert list(dg["idx"]) == [int(x) for x in fx["h1_dagger_top1"]], dg["idx"]
    assert list(orc.dsa_row(q, w, k, P, 1)["idx"]) == [int(x) for x in fx["h1_dagger_top1"]]


# ----------------------------------------------------------------- closed forms
def check_pool_closed_form(orc):
    # keys k_s = s (every dim): block b's mean is the midpoint of its first and last index
    for L, B in [(10, 4), (64, 64), (65, 64), (7, 3), (1, 5), (130, 128)]:
        k = np.repeat(np.arange(L, dtype=np.float64)[:, None], 3, axis=1)
        kp = orc.pool_keys(k, B)
        M = -(-L // B)
        assert kp.shape == (M, 3)
        for b in range(M):
            first, last = b * B, min((b + 1) * B, L) - 1
            assert np.all(kp[b] == (first + last) / 2.0), (L, B, b, kp[b])
    # B = 1: pooling is the identity
    rng = np.random.default_rng(1)
    k = rng.standard_normal((37, 8))
    assert np.array_equal(orc.pool_keys(k, 1), k)


def check_router_closed_form(orc):
    """q_j = a_j * e_j, all keys equal to the all-ones vector: every pooled key is the
    all-ones vector, so E_j = |w_j| * ReLU(a_j) for any prefix length and block size."""
    H, d = 6, 6
    a = np.array([3.0, -1.0, 0.5, 2.0, 0.0, 1.5])
    w = np.array([0.25, 4.0, -2.0, -0.5, 1.0, 1.0])
    q = np.diag(a)
    k = np.ones((50, d))
    for P, B in [(1, 4), (5, 4), (8, 4), (50, 7), (50, 64)]:
        E = orc.router_energy(q, w, k, P, B)
        assert np.allclose(E, np.abs(w) * np.maximum(a, 0.0), rtol=1e-15, atol=0), (P, B, E)
    E = orc.router_energy(q, w, k, 50, 7)
    # E = [0.75, 0, 1.0, 1.0, 0, 1.5] -> descending with lower index first on ties
    assert list(orc.select_heads(E, 6)) == [5, 2, 3, 0, 1, 4]


def check_partial_block_router(orc):
    """A query whose prefix ends mid-block routes on the mean of the block's valid keys
    only.  Keys k_s = s * u with u a unit vector; the partial block {8, 9} of P = 10,
    B = 4 pools to 8.5 * u (a full-L pooling would give 9.5 * u, an unweighted sum 17 * u)."""
    d = 4
    u = np.array([1.0, 0.0, 0.0, 0.0])
    k = np.arange(12, dtype=np.float64)[:, None] * u[None, :]
    q = np.array([[1.0, 0, 0, 0]])
    w = np.array([1.0])
    E = orc.router_energy(q, w, k, 10, 4)
    # pooled keys of the prefix: 1.5, 5.5, 8.5 (times u); E = (1.5 + 5.5 + 8.5) / 3
    assert abs(E[0] - (1.5 + 5.5 + 8.5) / 3.0) < 1e-14, E


# ----------------------------------------------------------------- library routine / brute force
def check_topk_against_library(orc):
    rng = np.random.default_rng(2)
    for n, kk in [(1, 1), (5, 3), (40, 7), (200, 64), (13, 20), (300, 300)]:
        # quantised values so that ties are frequent
        s = np.round(rng.standard_normal(n) * 4) / 4
        idx, vals = orc.topk(s, kk)
        ref = heapq.nlargest(min(kk, n), range(n), key=lambda i: (s[i], -i))
        assert list(idx[:len(ref)]) == ref, (n, kk)
        assert np.all(idx[len(ref):] == -1) and np.all(np.isneginf(vals[len(ref):]))
        assert np.array_equal(vals[:len(ref)], s[ref])


def check_topk_brute_rank(orc):
    """Brute force: item i is selected iff fewer than k items beat it, where j beats i
    when s_j > s_i, or s_j == s_i and j < i."""
    rng = np.random.default_rng(3)
    for n, kk in [(9, 4), (16, 16), (25, 1), (30, 12)]:
        s = rng.integers(-3, 4, size=n).astype(np.float64)
        idx, _ = orc.topk(s, kk)
        chosen = set(int(i) for i in idx if i >= 0)
        for i in range(n):
            beats = sum(1 for j in range(n) if s[j] > s[i] or (s[j] == s[i] and j < i))
            assert (beats < kk) == (i in chosen), (n, kk, i)


# ----------------------------------------------------------------- invariants
def _rand_problem(seed, H=8, d=16, L=97):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H, d))
    w = rng.standard_normal(H)
    k = rng.standard_normal((L, d)) + 0.3 * rng.standard_normal((1, d))
    return q, w, k


def check_h_equals_H_is_dense(orc):
    for seed in range(4):
        q, w, k = _rand_problem(seed)
        H = q.shape[0]
        for P in (1, 17, 97):
            r = orc.misa_row(q, w, k, P, 8, H, 10)
            dd = orc.dsa_row(q, w, k, P, 10)
            assert np.array_equal(r["scores"], dd["scores"])
            assert np.array_equal(r["idx"], dd["idx"])


def check_dagger_limits(orc):
    for seed in range(4):
        q, w, k = _rand_problem(seed + 10)
        for P in (5, 60, 97):
            r = orc.misa_row(q, w, k, P, 8, 3, 10)
            # k' >= P: the candidate set is the whole prefix -> exactly the dense TopK
            cand, _ = orc.topk(r["scores"], max(P, 12))
            dg = orc.misa_dagger_row(q, w, k, P, cand, 10)
            assert np.array_equal(dg["idx"], orc.dsa_row(q, w, k, P, 10)["idx"])
            # k' = k: the re-rank keeps MISA's set (order may change)
            cand, _ = orc.topk(r["scores"], 10)
            dg = orc.misa_dagger_row(q, w, k, P, cand, 10)
            assert set(dg["idx"].tolist()) == set(r["idx"].tolist())


def check_router_w_invariance(orc):
    for seed in range(4):
        q, w, k = _rand_problem(seed + 20)
        E = orc.router_energy(q, w, k, 90, 8)
        heads = orc.select_heads(E, 3)
        E2 = orc.router_energy(q, 2.5 * w, k, 90, 8)
        assert np.allclose(E2, 2.5 * E, rtol=1e-13, atol=0)
        assert np.array_equal(orc.select_heads(E2, 3), heads)
        E3 = orc.router_energy(q, -w, k, 90, 8)
        assert np.array_equal(E3, E)
        perm = np.random.default_rng(seed).permutation(q.shape[0])
        E4 = orc.router_energy(q[perm], w[perm], k, 90, 8)
        assert np.allclose(E4, E[perm], rtol=1e-13, atol=0)


def check_causal_prefix(orc):
    """Keys after the query's position never influence its scores or its routing."""
    q, w, k = _rand_problem(30, L=80)
    k2 = k.copy()
    k2[50:] = 1e3
    r1 = orc.misa_row(q, w, k, 50, 8, 3, 10)
    r2 = orc.misa_row(q, w, k2, 50, 8, 3, 10)
    assert np.array_equal(r1["E"], r2["E"]) and np.array_equal(r1["idx"], r2["idx"])
    assert r1["scores"].shape == (50,)


# ----------------------------------------------------------------- input widening and reporting
def check_bf16_widening(orc):
    """bf16 bit patterns widen to the float64 value the bf16 format defines: compared with
    torch's bf16 -> float64 conversion on every non-NaN pattern, and with values the format
    fixes by hand (sign, exponent bias 127, 7 stored mantissa bits, subnormals)."""
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    with np.errstate(invalid="ignore"):   # the NaN patterns
        got = orc.bf16_bits_to_f64(bits)
    assert got.dtype == np.float64 and got.shape == (1 << 16,)
    keep = ~np.isnan(ref)
    assert np.array_equal(got[keep], ref[keep]), np.nonzero(got[keep] != ref[keep])[0][:5]
    assert np.all(np.isnan(got[~keep]))
    hand = {0x3F80: 1.0, 0xC000: -2.0, 0x3FC0: 1.5, 0x0001: 2.0 ** -133, 0x8000: -0.0,
            0x7F80: np.inf, 0xFF80: -np.inf, 0x4049: 3.140625, 0x0080: 2.0 ** -126}
    for b, v in hand.items():
        w = orc.bf16_bits_to_f64(np.array([b], dtype=np.uint16))[0]
        assert w == v and np.signbit(w) == np.signbit(v), (hex(b), w, v)
    # shape is kept for multi-dimensional inputs
    assert orc.bf16_bits_to_f64(np.full((2, 3), 0x3F80, dtype=np.uint16)).shape == (2, 3)


def check_recall_hand(orc):
    """recall = |sel intersect ref| / |ref| over valid (>= 0) ids: the fraction of the
    dense selection that the other selection recovers (the pages' token-recovery measure)."""
    assert orc.recall(np.array([5, 2, 9, 11]), np.array([2, 9, 7])) == 2 / 3
    # padding (-1) is not a token on either side
    assert orc.recall(np.array([-1, 4, -1]), np.array([4, 8, -1, -1])) == 1 / 2
    assert orc.recall(np.array([1, 2, 3]), np.array([3, 2, 1])) == 1.0
    assert orc.recall(np.array([-1, -1]), np.array([6, 7])) == 0.0


def check_dagger_candidate_set(orc):
    """Eq. (12) ranges over the set Omega_t: a repeated candidate id counts once and -1
    slots are empty.  Hand case: H = 1, d = 1, w = 1, q = 1, keys k_s = s, so I[s] = s.
    Candidates [3, 3, 1, -1, 3, 0] form {0, 1, 3}; TopK(., 2) = [3, 1].  Counting the
    repeats would return [3, 3]."""
    q = np.array([[1.0]])
    w = np.array([1.0])
    k = np.arange(6, dtype=np.float64)[:, None]
    dg = orc.misa_dagger_row(q, w, k, 6, np.array([3, 3, 1, -1, 3, 0]), 2)
    assert list(dg["idx"]) == [3, 1], dg["idx"]
    assert list(dg["vals"]) == [3.0, 1.0]
    assert list(dg["cand"]) == [0, 1, 3] and list(dg["scores"]) == [0.0, 1.0, 3.0]
    # fewer distinct candidates than k: padded with -1 / -inf
    dg = orc.misa_dagger_row(q, w, k, 6, np.array([2, 2, 2, -1]), 3)
    assert list(dg["idx"]) == [2, -1, -1] and np.all(np.isneginf(dg["vals"][1:]))
    # ids past the query's prefix (P = 4) are not tokens of Omega_t
    dg = orc.misa_dagger_row(q, w, k, 4, np.array([5, 1, 4, 2]), 2)
    assert list(dg["idx"]) == [2, 1], dg["idx"]


# ----------------------------------------------------------------- HISA-style block filter
def check_hisa_hand(orc):
    """Hand case of the head-axis reduction G[b] = sum_j A[j, b] (MISA page, "Key
    distinction from HISA"): H = 2, d = 2, B = 2, P = 7, q = I, w = (1, -0.5),
    keys (1,0) (3,0) (0,2) (0,4) (2,2) (0,0) (5,-1).  Pooled keys of the prefix:
    (2,0) (0,3) (1,1) and the partial block {6}: (5,-1).  A[0,:] = (2, 0, 1, 5),
    A[1,:] = (0, -1.5, -0.5, 0), so G = (2, -1.5, 0.5, 5).  Top-3 blocks: 3, 0, 2; their
    tokens 0 1 4 5 6 have dense scores 1 3 1 0 5, so TopK(., 2) = [6, 1]."""
    q = np.eye(2)
    w = np.array([1.0, -0.5])
    k = np.array([[1, 0], [3, 0], [0, 2], [0, 4], [2, 2], [0, 0], [5, -1], [9, 9]], float)
    assert np.array_equal(orc.block_scores(q, w, k, 7, 2), [2.0, -1.5, 0.5, 5.0])
    r = orc.hisa_row(q, w, k, 7, 2, 3, 2)
    assert list(r["blocks"]) == [3, 0, 2], r["blocks"]
    assert list(r["cand"]) == [0, 1, 4, 5, 6], r["cand"]
    assert list(r["scores"]) == [1.0, 3.0, 1.0, 0.0, 5.0], r["scores"]
    assert list(r["idx"]) == [6, 1] and list(r["vals"]) == [5.0, 3.0]
    # two blocks: 3 and 0 -> tokens 0 1 6; TopK(., 3) = [6, 1, 0]
    r = orc.hisa_row(q, w, k, 7, 2, 2, 3)
    assert list(r["blocks"]) == [3, 0] and list(r["idx"]) == [6, 1, 0], r["idx"]
    # more blocks than the prefix has: every token, padded past P
    r = orc.hisa_row(q, w, k, 3, 2, 5, 4)
    assert list(r["cand"]) == [0, 1, 2] and list(r["idx"]) == [1, 0, 2, -1], r["idx"]


def check_hisa_limits(orc):
    """m >= M keeps every block, so the filter is the dense TopK exactly; with B = 1 every
    block is one token and G is the dense score itself, so m = k returns DSA's selection."""
    for seed in range(4):
        q, w, k = _rand_problem(seed + 40)
        for P in (1, 30, 97):
            M = -(-P // 8)
            r = orc.hisa_row(q, w, k, P, 8, M, 10)
            assert np.array_equal(r["idx"], orc.dsa_row(q, w, k, P, 10)["idx"])
            assert np.array_equal(orc.block_scores(q, w, k, P, 1), orc.dense_scores(q, w, k, P))
            r1 = orc.hisa_row(q, w, k, P, 1, 10, 10)
            assert np.array_equal(r1["idx"], orc.dsa_row(q, w, k, P, 10)["idx"])


ALL_CHECKS = [
    check_hisa_hand, check_hisa_limits,
    check_bf16_widening, check_recall_hand, check_dagger_candidate_set,
    check_dense_hand, check_router_hand, check_pool_closed_form, check_router_closed_form,
    check_partial_block_router, check_topk_against_library, check_topk_brute_rank,
    check_h_equals_H_is_dense, check_dagger_limits, check_router_w_invariance,
    check_causal_prefix,
]
