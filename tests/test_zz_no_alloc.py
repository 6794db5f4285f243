"""misa_score_topk_noalloc against misa_score_topk (GPU).

The no-allocation entry point serves callers that cannot allocate device memory or
pass a workspace (allocator-free regions of a serving engine, plugins whose host
framework owns all device memory); it keeps its scratch in a fixed array inside the
library.  Here it is called through the C ABI twice in a row, on two different
inputs, and each result must match the workspace-based entry point within the
parity tolerance.  This file is collected last on purpose: a failure here leaves
every other test already run."""

import numpy as np
import pytest
import torch

from synth import WORKLOADS, make_inputs
from tests import gpu_path
from tests import tolerance as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_block_b200 as M
    return M


def _compare(idx, vals, ref_idx, ref_vals, topk):
    idx, vals = idx.cpu().numpy(), vals.cpu().numpy()
    ref_idx, ref_vals = ref_idx.cpu().numpy(), ref_vals.cpu().numpy()
    for r in range(idx.shape[0]):
        m = int((ref_idx[r] >= 0).sum())
        assert int((idx[r] >= 0).sum()) == m
        rv = ref_vals[r, :m].astype(np.float64)
        tl.check_scores(vals[r, :m], rv, what=f"row {r} values")
        if m == 0:
            continue
        cut = rv[m - 1]
        ctol = tl.tol(np.array([cut]), rv)[0]
        got = dict(zip(idx[r, :m].tolist(), vals[r, :m].tolist()))
        ref = dict(zip(ref_idx[r, :m].tolist(), rv.tolist()))
        for t in set(got) ^ set(ref):
            v = got.get(t, ref.get(t))
            assert abs(v - cut) <= ctol, f"row {r}: token {t} ({v}) differs away from the cutoff {cut}"


def test_noalloc_matches_workspace_entry_point_on_two_calls(M):
    shapes = [WORKLOADS["dsv32_decode_32k"].replace(nseq=4, L=8192),
              WORKLOADS["glm5_decode_128k"].replace(nseq=2, L=20000, topk=1024)]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, wl in enumerate(shapes):
        x = make_inputs(wl, seed=100 + call)
        q, w, k, pos = gpu_path.to_device(x)
        kp = M.misa_pool_keys(k, wl.B)
        heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
        ref_idx, ref_vals = M.misa_score_topk(q, w, k, heads, pos, wl.topk)
        idx = torch.full_like(ref_idx, -7)
        vals = torch.full_like(ref_vals, float("nan"))
        M.misa_score_topk_noalloc(q, w, k, heads, pos, wl.topk, idx=idx, vals=vals,
                                  device_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        _compare(idx.view(wl.rows, -1), vals.view(wl.rows, -1), ref_idx.view(wl.rows, -1),
                 ref_vals.view(wl.rows, -1), wl.topk)


def test_noalloc_matches_oracle_on_every_row_of_the_tiny_workload(M):
    """The entry point's own scorer and top-k against the fp64 oracle (not only against the
    workspace entry point): every row of the 16-query, 2K-key workload, with the oracle's
    routed scores under the heads the GPU routed (Eqs. 9-10)."""
    import oracle.misa_oracle as orc
    wl = WORKLOADS["tiny_2k"]
    x = make_inputs(wl, seed=0)
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    idx, vals = M.misa_score_topk_noalloc(q, w, k, heads, pos, wl.topk, device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    idx = idx.view(wl.rows, -1).cpu().numpy()
    vals = vals.view(wl.rows, -1).cpu().numpy()
    hh = heads.view(wl.rows, -1).cpu().numpy()
    kk = orc.bf16_bits_to_f64(x.k_bits[0])
    for t in range(wl.T):
        P = int(x.pos[0, t]) + 1
        s_ref = orc.token_scores(orc.bf16_bits_to_f64(x.q_bits[0, t]),
                                 x.w[0, t].astype(np.float64), kk, P, hh[t])
        tl.check_selection(idx[t], s_ref, wl.topk, what=f"row {t} set")
        tl.check_order(idx[t], vals[t], what=f"row {t} order")
        tl.check_scores(vals[t], s_ref[idx[t]], what=f"row {t} values")


def test_noalloc_rejects_calls_beyond_its_scratch(M):
    wl = WORKLOADS["dsv32_decode_32k"].replace(nseq=2, L=4096)
    x = make_inputs(wl, seed=7)
    q, w, k, pos = gpu_path.to_device(x)
    heads = torch.zeros((2, 1, wl.h), dtype=torch.int32, device="cuda")
    big_k = torch.zeros((2, (1 << 21) + 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MisaError) as e:
        M.misa_score_topk_noalloc(q, w, big_k, heads, pos, 16)
    assert e.value.status == 7
