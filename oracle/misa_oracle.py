"""fp64 CPU oracle for the MISA indexer path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this module.  The product path (the CUDA library and its
binding) never calls it, and this module imports nothing from that path.

What it computes, following "MISA: Mixture of Indexer Sparse Attention for
Long-Context LLM Inference" (picx.dev summary page):

  * Eq. (1)  DSA indexer score  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])
  * Eq. (2)  token selection    T_t = TopK(I[t,:], k)
  * Eq. (4)  block pooling of the prefix into M = ceil(P/B) pooled keys; the
             Pool operator is not given on the page (its defining equations are
             missing from the text), and is read here as the arithmetic mean of
             the block's keys.
  * Eq. (7)  router affinities A[t,j,b] = w[t,j] * ReLU(q[t,j] . kpool[b]) and
             head energy E[t,j] = (1/M) * sum_b |A[t,j,b]|
  * Eq. (8)  routed heads H_t = TopK_j(E[t,:], h)
  * Eq. (9)  routed score Ihat[t,s] = sum_{j in H_t} w[t,j] * ReLU(q[t,j] . k[s])
  * Eq. (10) final selection TopK_s(Ihat[t,:], k)
  * Eq. (11) MISA-dagger coarse candidates Omega_t = TopK_s(Ihat[t,:], k')
  * Eq. (12) MISA-dagger fine stage TopK over s in Omega_t of I[t,s]
  * the HISA-style token-axis filter the page contrasts MISA with ("Key distinction
    from HISA", Methodology section 1): the same affinities A[t,j,b], reduced across
    heads instead of across blocks, pick the top-m blocks; the original indexer then
    scores only the tokens of those blocks (the two-stage search the HISA abstract
    describes: block-level coarse filter, token-level refinement in the kept blocks).

Readings taken where the page is silent (each listed with its reason in the
design notes of the repository):
  * Causality: query t at absolute position pos[t] sees keys s in [0, pos[t]],
    so its prefix length is P = pos[t] + 1.
  * Router blocks are the blocks of the query's own prefix: B_b = [bB, min((b+1)B, P)),
    the last block possibly partial (its pooled key is the mean of its valid keys),
    and M in Eq. (7) is ceil(P / B).
  * TopK returns indices ordered by descending value; equal values keep the lower
    index first.  When fewer than k items exist, all are returned and the rest of
    the row is padded with -1 (values -inf).
  * MISA-dagger's fine stage recomputes the full all-head score I[t,s] for every
    candidate; ties there are broken by the lower token index s.  Omega_t is a set
    (Eq. 11 selects it by TopK, Eq. 12 ranges over s in Omega_t): a candidate list
    handed in with a repeated id counts that id once, and -1 marks an empty slot;
    ids outside the query's prefix [0, P) are not tokens of Omega_t and are dropped.
  * Precision: q and k are bf16 values, w is fp32; everything here is widened to
    float64 and computed in float64.

Every function works on one query row so that it can be read against the
equations directly; the batch helpers at the bottom only loop over rows.
Library primitives used as steps: numpy matrix products, means and sorts.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64", "pool_keys", "router_energy", "select_heads", "token_scores",
    "dense_scores", "topk", "misa_row", "dsa_row", "misa_dagger_row", "recall",
    "block_scores", "hisa_row",
]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- Eq. (4)
def pool_keys(k: np.ndarray, B: int) -> np.ndarray:
    """Mean-pool consecutive blocks of B keys (the last block may be shorter).

    k: float64 [P, d].  Returns float64 [ceil(P/B), d], row b = mean of k[bB : min((b+1)B, P)].
    """
    P = k.shape[0]
    M = -(-P // B)
    out = np.empty((M, k.shape[1]), dtype=np.float64)
    for b in range(M):
        out[b] = k[b * B: min((b + 1) * B, P)].mean(axis=0)
    return out


# --------------------------------------------------------------------------- Eq. (7)
def router_energy(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray, P: int, B: int) -> np.ndarray:
    """Head energy E[j] = (1/M) sum_b |w_j * ReLU(q_j . kpool_b)| over the query's prefix.

    q_t: [H, d] float64, w_t: [H] float64, k: [>=P, d] float64.  Returns float64 [H].
    """
    kpool = pool_keys(k[:P], B)                         # [M, d]
    A = w_t[:, None] * np.maximum(q_t @ kpool.T, 0.0)   # [H, M]
    return np.abs(A).mean(axis=1)


# --------------------------------------------------------------------------- Eq. (8)
def select_heads(E: np.ndarray, h: int) -> np.ndarray:
    """Indices of the h largest E[j], by descending E, equal E -> lower j first."""
    order = sorted(range(E.shape[0]), key=lambda j: (-E[j], j))
    return np.asarray(order[:h], dtype=np.int64)


# --------------------------------------------------------------------------- Eqs. (1), (9)
def token_scores(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray, P: int,
                 heads) -> np.ndarray:
    """sum_{j in heads} w_j * ReLU(q_j . k_s) for s < P.  Returns float64 [P].

    The head terms are summed in ascending j, so that heads = all H gives exactly
    the dense score of Eq. (1).
    """
    hs = np.sort(np.asarray(heads, dtype=np.int64))
    dots = q_t[hs] @ k[:P].T                             # [h, P]
    terms = w_t[hs][:, None] * np.maximum(dots, 0.0)
    out = np.zeros(P, dtype=np.float64)
    for r in range(hs.shape[0]):
        out += terms[r]
    return out


def dense_scores(q_t, w_t, k, P):
    """Eq. (1): all H heads."""
    return token_scores(q_t, w_t, k, P, np.arange(q_t.shape[0]))


# --------------------------------------------------------------------------- Eqs. (2), (10)
def topk(scores: np.ndarray, kk: int, index: np.ndarray | None = None):
    """The kk largest entries: (idx int64 [kk], vals float64 [kk]).

    Ordered by descending value; equal values -> lower index first.  `index`
    gives the token index of each entry (default: its position).  Short rows
    are padded with idx -1 and value -inf.
    """
    n = scores.shape[0]
    if index is None:
        index = np.arange(n, dtype=np.int64)
    order = np.lexsort((index, -scores))   # primary key: -score; secondary: token index
    take = order[:kk]
    idx = np.full(kk, -1, dtype=np.int64)
    vals = np.full(kk, -np.inf, dtype=np.float64)
    idx[:take.shape[0]] = index[take]
    vals[:take.shape[0]] = scores[take]
    return idx, vals


# --------------------------------------------------------------------------- full rows
def misa_row(q_t, w_t, k, P, B, h, kk):
    """MISA for one query: route (Eqs. 4, 7, 8), routed score (Eq. 9), TopK (Eq. 10)."""
    E = router_energy(q_t, w_t, k, P, B)
    heads = select_heads(E, h)
    s_hat = token_scores(q_t, w_t, k, P, heads)
    idx, vals = topk(s_hat, kk)
    return dict(E=E, heads=heads, scores=s_hat, idx=idx, vals=vals)


def dsa_row(q_t, w_t, k, P, kk):
    """Dense DSA indexer for one query (Eqs. 1-2)."""
    s = dense_scores(q_t, w_t, k, P)
    idx, vals = topk(s, kk)
    return dict(scores=s, idx=idx, vals=vals)


def misa_dagger_row(q_t, w_t, k, P, cand, kk):
    """MISA-dagger fine stage (Eq. 12) over the candidate set Omega_t given by `cand`.

    `cand` may list an id more than once and in any order; -1 marks an empty slot.
    Omega_t is the set of distinct ids in [0, P).  Returns idx / vals of the TopK, and
    the set itself ("cand", ascending) with the all-head scores of its members ("scores").
    """
    c = np.asarray(cand, dtype=np.int64)
    c = np.unique(c[(c >= 0) & (c < P)])                # Omega_t as a set, ascending
    s_full = dense_scores(q_t, w_t, k[c], c.shape[0])   # I[t, s] for s in Omega_t
    idx, vals = topk(s_full, kk, index=c)
    return dict(idx=idx, vals=vals, cand=c, scores=s_full)


# --------------------------------------------------------------------------- HISA-style filter
def block_scores(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray, P: int, B: int) -> np.ndarray:
    """Head-axis reduction of the router affinities: G[b] = sum_j A[j, b] with
    A[j, b] = w_j * ReLU(q_j . kpool_b) over the blocks of the query's prefix (the same
    blocks, partial last block included, as Eq. 7).  Returns float64 [ceil(P/B)]."""
    kpool = pool_keys(k[:P], B)                         # [M, d]
    A = w_t[:, None] * np.maximum(q_t @ kpool.T, 0.0)   # [H, M]
    G = np.zeros(kpool.shape[0], dtype=np.float64)
    for j in range(A.shape[0]):                         # sum over heads in ascending j
        G += A[j]
    return G


def hisa_row(q_t, w_t, k, P, B, m, kk):
    """Token-axis block filter for one query: keep the m blocks with the largest G[b]
    (ties: lower b), then TopK of the all-head score I[t,s] (Eq. 1) over the tokens of
    the kept blocks (ties: lower s).  Returns the block scores, the kept blocks (by
    descending G), the candidate tokens (ascending) with their scores, and idx / vals."""
    G = block_scores(q_t, w_t, k, P, B)
    blocks, _ = topk(G, m)
    blocks = blocks[blocks >= 0]
    toks = [np.arange(b * B, min((b + 1) * B, P)) for b in sorted(int(b) for b in blocks)]
    cand = np.concatenate(toks).astype(np.int64) if toks else np.zeros(0, dtype=np.int64)
    s = dense_scores(q_t, w_t, k[cand], cand.shape[0])
    idx, vals = topk(s, kk, index=cand)
    return dict(G=G, blocks=blocks, cand=cand, scores=s, idx=idx, vals=vals)


def recall(sel: np.ndarray, ref: np.ndarray) -> float:
    """|sel intersect ref| / |ref| over valid (non -1) entries."""
    a = set(int(x) for x in sel if x >= 0)
    b = set(int(x) for x in ref if x >= 0)
    return len(a & b) / max(1, len(b))
