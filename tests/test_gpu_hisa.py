"""The HISA-style token-axis block filter against the fp64 oracle (GPU): the kept blocks
follow the cutoff rule on the oracle's head-summed block scores G (MISA page, "Key
distinction from HISA"), and the selected tokens follow it on the oracle's all-head
scores (Eq. 1) over the tokens of the blocks the GPU kept."""

import numpy as np
import pytest
import torch

import oracle.misa_oracle as orc
from synth import WORKLOADS, Workload, make_inputs, sample_rows
from tests import gpu_path
from tests import tolerance as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_block_b200 as M
    return M


def _check(M, x, B, m, topk, rows):
    wl = x.wl
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, B)
    idx, vals, blocks = M.hisa_indexer(q, w, k, pos, B, m, topk, k_pool=kp)
    M.misa_check_device_status(q.device)
    r = torch.as_tensor(np.asarray(rows), device=q.device)
    idx = idx.reshape(wl.rows, -1).index_select(0, r).cpu().numpy()
    vals = vals.reshape(wl.rows, -1).index_select(0, r).cpu().numpy()
    blocks = blocks.reshape(wl.rows, -1).index_select(0, r).cpu().numpy()
    kcache = {}
    swaps = 0
    for i, row in enumerate(rows):
        n, t = divmod(int(row), wl.T)
        if n not in kcache:
            kcache.clear()
            kcache[n] = orc.bf16_bits_to_f64(x.k_bits[n])
        kk = kcache[n]
        q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
        w_t = x.w[n, t].astype(np.float64)
        P = int(x.pos[n, t]) + 1
        G = orc.block_scores(q_t, w_t, kk, P, B)
        swaps += tl.check_selection(blocks[i], G, m, what=f"row {row} kept blocks")
        kept = blocks[i][blocks[i] >= 0]
        # the oracle's refinement over the blocks the GPU kept (a legitimate swap at the
        # block cutoff changes the candidate tokens, not the rule)
        toks = np.concatenate([np.arange(b * B, min((b + 1) * B, P)) for b in np.sort(kept)])
        s_ref = orc.dense_scores(q_t, w_t, kk[toks], toks.shape[0])
        tl.check_selection(idx[i], s_ref, topk, what=f"row {row} tokens", ids=toks)
        tl.check_order(idx[i], vals[i], what=f"row {row} order")
        sel = idx[i][idx[i] >= 0]
        pos_of = {int(s): j for j, s in enumerate(toks)}
        tl.check_scores(vals[i][:sel.size], s_ref[[pos_of[int(s)] for s in sel]],
                        what=f"row {row} values")
        if swaps == 0 and i < 4:   # same blocks as the oracle: the whole row equals hisa_row
            ref = orc.hisa_row(q_t, w_t, kk, P, B, m, topk)
            assert set(kept.tolist()) == set(ref["blocks"].tolist())
    return swaps


CASES = {
    "ragged_prefixes": dict(nseq=2, T=3, L=3000, H=64, B=128, m=6, topk=300),
    "partial_block_kept": dict(nseq=3, T=1, L=1000, H=32, B=128, m=3, topk=128),
    "more_blocks_than_prefix": dict(nseq=2, T=2, L=500, H=64, B=128, m=16, topk=64),
    "B1_is_token_topk": dict(nseq=1, T=2, L=700, H=16, B=1, m=64, topk=64),
    "H128_B64": dict(nseq=1, T=3, L=2500, H=128, B=64, m=10, topk=200),
    "topk_larger_than_candidates": dict(nseq=2, T=1, L=4000, H=64, B=128, m=2, topk=512),
}


@pytest.mark.parametrize("case", list(CASES))
def test_hisa_edge_cases(M, case):
    c = CASES[case]
    wl = Workload(name=case, nseq=c["nseq"], T=c["T"], L=c["L"], H=c["H"], d=128, h=8,
                  B=c["B"], topk=c["topk"], kprime=c["topk"], pos_mode="tail", drift=True,
                  needles=2)
    x = make_inputs(wl, seed=51)
    rng = np.random.default_rng(9)
    x.pos = rng.integers(0, wl.L, size=x.pos.shape).astype(np.int32)
    _check(M, x, c["B"], c["m"], c["topk"], np.arange(wl.rows))


@pytest.mark.parametrize("name", ["dsv32_decode_32k", "glm5_decode_128k"])
def test_hisa_full_size(M, name):
    """The decode workloads at full size with the page's HISA block size (B = 128) and
    m = 64 blocks (8192 candidate tokens, the MISA-dagger budget), every row checked for
    the 32K batch and the 128K batch."""
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0)
    _check(M, x, 128, 64, wl.topk, sample_rows(wl, 256, seed=0))
