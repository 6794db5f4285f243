"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch
each one.  The mutants are local copies of single oracle functions; the real oracle
is restored by monkeypatch after every test."""

import numpy as np
import pytest

import oracle.misa_oracle as orc
from tests import oracle_pins


def _relu_after_weight(q_t, w_t, k, P, heads):
    hs = np.sort(np.asarray(heads))
    return np.maximum(w_t[hs][:, None] * (q_t[hs] @ k[:P].T), 0.0).sum(axis=0)


def _no_relu(q_t, w_t, k, P, heads):
    hs = np.sort(np.asarray(heads))
    return (w_t[hs][:, None] * (q_t[hs] @ k[:P].T)).sum(axis=0)


def _transposed_q(q_t, w_t, k, P, heads):
    hs = np.sort(np.asarray(heads))
    qt = q_t.T if q_t.shape[0] == q_t.shape[1] else q_t[::-1]
    return (w_t[hs][:, None] * np.maximum(qt[hs] @ k[:P].T, 0.0)).sum(axis=0)


def _energy_no_abs(q_t, w_t, k, P, B):
    kp = orc.pool_keys(k[:P], B)
    return (w_t[:, None] * np.maximum(q_t @ kp.T, 0.0)).mean(axis=1)


def _energy_full_L(q_t, w_t, k, P, B):
    kp = orc.pool_keys(k, B)          # pools keys past the query's position
    return np.abs(w_t[:, None] * np.maximum(q_t @ kp.T, 0.0)).mean(axis=1)


def _energy_drop_partial(q_t, w_t, k, P, B):
    Pf = max(B, (P // B) * B)
    kp = orc.pool_keys(k[:Pf], B)
    return np.abs(w_t[:, None] * np.maximum(q_t @ kp.T, 0.0)).mean(axis=1)


def _pool_sum_over_B(k, B):
    P = k.shape[0]
    M = -(-P // B)
    return np.stack([k[b * B:min((b + 1) * B, P)].sum(axis=0) / B for b in range(M)])


def _topk_ties_high_index(scores, kk, index=None):
    n = scores.shape[0]
    if index is None:
        index = np.arange(n)
    order = np.lexsort((-index, -scores))
    take = order[:kk]
    idx = np.full(kk, -1, dtype=np.int64)
    vals = np.full(kk, -np.inf)
    idx[:take.shape[0]] = index[take]
    vals[:take.shape[0]] = scores[take]
    return idx, vals


def _heads_ascending(E, h):
    return np.argsort(E, kind="stable")[:h]


def _bf16_shift15(bits):
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)


def _bf16_as_fp16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _bf16_truncated_mantissa(bits):
    b = np.asarray(bits, dtype=np.uint16) & np.uint16(0xFFF0)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _recall_over_sel(sel, ref):
    a = set(int(x) for x in sel if x >= 0)
    b = set(int(x) for x in ref if x >= 0)
    return len(a & b) / max(1, len(a))


def _recall_counts_padding(sel, ref):
    a, b = set(int(x) for x in sel), set(int(x) for x in ref)
    return len(a & b) / max(1, len(b))


def _dagger_keeps_repeats(q_t, w_t, k, P, cand, kk):
    c = np.asarray(cand, dtype=np.int64)
    c = c[c >= 0]
    s_full = orc.dense_scores(q_t, w_t, k[c], c.shape[0])
    idx, vals = orc.topk(s_full, kk, index=c)
    return dict(idx=idx, vals=vals, cand=c, scores=s_full)


def _dagger_ignores_prefix(q_t, w_t, k, P, cand, kk):
    c = np.asarray(cand, dtype=np.int64)
    c = np.unique(c[c >= 0])
    s_full = orc.dense_scores(q_t, w_t, k[c], c.shape[0])
    idx, vals = orc.topk(s_full, kk, index=c)
    return dict(idx=idx, vals=vals, cand=c, scores=s_full)


def _block_scores_abs(q_t, w_t, k, P, B):
    kp = orc.pool_keys(k[:P], B)
    return np.abs(w_t[:, None] * np.maximum(q_t @ kp.T, 0.0)).sum(axis=0)


def _block_scores_drop_partial(q_t, w_t, k, P, B):
    Pf = max(B, (P // B) * B) if P >= B else P
    kp = orc.pool_keys(k[:Pf], B)
    return (w_t[:, None] * np.maximum(q_t @ kp.T, 0.0)).sum(axis=0)


def _block_scores_relu_after_sum(q_t, w_t, k, P, B):
    kp = orc.pool_keys(k[:P], B)
    return np.maximum((w_t[:, None] * (q_t @ kp.T)).sum(axis=0), 0.0)


def _hisa_lowest_blocks(q_t, w_t, k, P, B, m, kk):
    G = orc.block_scores(q_t, w_t, k, P, B)
    blocks = np.argsort(G, kind="stable")[:m]
    toks = [np.arange(b * B, min((b + 1) * B, P)) for b in sorted(int(b) for b in blocks)]
    cand = np.concatenate(toks).astype(np.int64)
    s = orc.dense_scores(q_t, w_t, k[cand], cand.shape[0])
    idx, vals = orc.topk(s, kk, index=cand)
    return dict(G=G, blocks=blocks, cand=cand, scores=s, idx=idx, vals=vals)


MUTANTS = [
    ("block_scores", _block_scores_abs),
    ("block_scores", _block_scores_drop_partial),
    ("block_scores", _block_scores_relu_after_sum),
    ("hisa_row", _hisa_lowest_blocks),
    ("bf16_bits_to_f64", _bf16_shift15),
    ("bf16_bits_to_f64", _bf16_as_fp16),
    ("bf16_bits_to_f64", _bf16_truncated_mantissa),
    ("recall", _recall_over_sel),
    ("recall", _recall_counts_padding),
    ("misa_dagger_row", _dagger_keeps_repeats),
    ("misa_dagger_row", _dagger_ignores_prefix),
    ("token_scores", _relu_after_weight),
    ("token_scores", _no_relu),
    ("token_scores", _transposed_q),
    ("router_energy", _energy_no_abs),
    ("router_energy", _energy_full_L),
    ("router_energy", _energy_drop_partial),
    ("pool_keys", _pool_sum_over_B),
    ("topk", _topk_ties_high_index),
    ("select_heads", _heads_ascending),
]


@pytest.mark.parametrize("name,fn", MUTANTS, ids=[f.__name__ for _, f in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setattr(orc, name, fn)
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, ValueError, IndexError, TypeError, KeyError):
            caught.append(check.__name__)
    assert caught, f"no pin caught the planted mistake {fn.__name__}"
