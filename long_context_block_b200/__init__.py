"""MISA indexer hot path for NVIDIA B200 (sm_100a).

Kernels live in libmisa_b200.so (C ABI in include/misa.h); this package is a thin
binding plus two compositions of the entry points:

  misa_indexer  -- pool keys, route heads, routed score + top-k   (Eqs. 4, 7-10)
  misa_dagger   -- misa_indexer with k' candidates, then the all-head re-rank (Eqs. 11-12)
  hisa_indexer  -- the HISA-style token-axis block filter the pages contrast MISA with

Reference: "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
Inference" (picx.dev summary page, Methodology sections 1-2).
"""

from ._binding import (  # noqa: F401
    HEAD_DIM,
    LIB_PATH,
    MisaError,
    declared_symbols,
    dsa_score_topk,
    hisa_block_filter_topk,
    library,
    misa_check_device_status,
    misa_dagger_rerank,
    misa_pool_keys,
    misa_pool_keys_range,
    misa_route_heads,
    misa_score_rows,
    misa_score_topk,
    misa_score_topk_noalloc,
    misa_testing_score_rows_wait_expiry,
    misa_testing_score_rows_timed,
    misa_testing_score_simt,
    misa_workspace_size,
    workspace,
)


def misa_indexer(q, w, k, pos, B: int, h: int, topk: int, return_vals: bool = True,
                 k_pool=None):
    """MISA for a batch of queries: Eq. (4) pooling (skipped when k_pool is given),
    Eqs. (7)-(8) routing, Eqs. (9)-(10) routed scoring and top-k.

    Returns (idx, vals, heads)."""
    if k_pool is None:
        k_pool = misa_pool_keys(k, B)
    heads = misa_route_heads(q, w, k, k_pool, pos, B, h)
    idx, vals = misa_score_topk(q, w, k, heads, pos, topk, return_vals=True)
    return (idx, vals, heads) if return_vals else (idx, None, heads)


def misa_dagger(q, w, k, pos, B: int, h: int, topk: int, kprime: int, k_pool=None):
    """MISA-dagger: routed coarse top-k' (Eq. 11), then the all-head re-rank to top-k
    (Eq. 12).  Returns (idx, vals, cand, heads)."""
    if k_pool is None:
        k_pool = misa_pool_keys(k, B)
    heads = misa_route_heads(q, w, k, k_pool, pos, B, h)
    cand = misa_score_topk(q, w, k, heads, pos, kprime, return_vals=False)
    idx, vals = misa_dagger_rerank(q, w, k, pos, cand, topk)
    return idx, vals, cand, heads


def hisa_indexer(q, w, k, pos, B: int, m: int, topk: int, k_pool=None):
    """HISA-style block filter: pool with B (skipped when k_pool is given), keep each
    query's top-m blocks by head-summed affinity, top-k of the all-head scores of their
    tokens.  Returns (idx, vals, blocks)."""
    if k_pool is None:
        k_pool = misa_pool_keys(k, B)
    return hisa_block_filter_topk(q, w, k, k_pool, pos, B, m, topk, return_blocks=True)
