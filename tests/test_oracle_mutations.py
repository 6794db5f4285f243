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


MUTANTS = [
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
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin caught the planted mistake {fn.__name__}"
