"""Code paths the ordinary entry points take only in rare conditions, against the fp64
oracle (GPU): the CUDA-core scorer (the fallback of misa_score_topk / dsa_score_topk /
the MISA-dagger re-rank), the expiry path of the tensor-core scorer's bounded waits,
the h = H^I invariant (MISA page, Eq. 9 with every head routed is Eq. 1), the timed
scorer entry the benchmark's roofline uses, and the host-side rejection of a too-small
workspace and of misaligned or short buffers."""

import ctypes

import numpy as np
import pytest
import torch

import oracle.misa_oracle as orc
from synth import Workload, make_inputs
from tests import gpu_path
from tests import tolerance as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_block_b200 as M
    return M


def _wl(**kw):
    base = dict(name="paths", nseq=2, T=3, L=3000, H=64, d=128, h=8, B=64, topk=128,
                kprime=256, pos_mode="tail", drift=True, needles=4)
    base.update(kw)
    return Workload(**base)


def _random_pos(x, seed):
    rng = np.random.default_rng(seed)
    x.pos = rng.integers(0, x.wl.L, size=x.pos.shape).astype(np.int32)
    return x


@pytest.mark.parametrize("routed", [True, False], ids=["routed_eq9", "dense_eq1"])
def test_simt_scorer_matches_oracle(M, routed):
    wl = _wl()
    x = _random_pos(make_inputs(wl, seed=31), seed=2)
    q, w, k, pos = gpu_path.to_device(x)
    heads = None
    if routed:
        kp = M.misa_pool_keys(k, wl.B)
        heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    s = M.misa_testing_score_simt(q, w, k, heads, pos)
    M.misa_check_device_status(q.device)
    s = s.cpu().numpy()
    hh = heads.cpu().numpy() if routed else None
    for n in range(wl.nseq):
        kk = orc.bf16_bits_to_f64(x.k_bits[n])
        for t in range(wl.T):
            P = int(x.pos[n, t]) + 1
            q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
            w_t = x.w[n, t].astype(np.float64)
            ref = (orc.token_scores(q_t, w_t, kk, P, hh[n, t]) if routed
                   else orc.dense_scores(q_t, w_t, kk, P))
            tl.check_scores(s[n, t, :P], ref, what=f"simt row {n},{t}")
            assert np.all(np.isnan(s[n, t, P:])), "entries past the prefix were written"


def test_simt_scorer_gather_mode_matches_oracle(M):
    """The CUDA-core form of the MISA-dagger fine stage (Eq. 12): all-head scores of a
    given list of tokens per row."""
    wl = _wl()
    x = _random_pos(make_inputs(wl, seed=32), seed=3)
    q, w, k, pos = gpu_path.to_device(x)
    rng = np.random.default_rng(5)
    kprime = 300
    ids = np.zeros((wl.nseq, wl.T, kprime), dtype=np.int32)
    lens = np.zeros((wl.nseq, wl.T), dtype=np.int32)
    for n in range(wl.nseq):
        for t in range(wl.T):
            P = int(x.pos[n, t]) + 1
            m = min(P, int(rng.integers(1, kprime + 1)))
            ids[n, t, :m] = np.sort(rng.choice(P, size=m, replace=False))
            lens[n, t] = m
    g_ids = torch.from_numpy(ids).cuda()
    g_len = torch.from_numpy(lens).cuda()
    s = M.misa_testing_score_simt(q, w, k, None, pos, gather_ids=g_ids, gather_len=g_len)
    M.misa_check_device_status(q.device)
    s = s.cpu().numpy()
    for n in range(wl.nseq):
        kk = orc.bf16_bits_to_f64(x.k_bits[n])
        for t in range(wl.T):
            P = int(x.pos[n, t]) + 1
            q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
            d_ref = orc.dense_scores(q_t, x.w[n, t].astype(np.float64), kk, P)
            m = lens[n, t]
            tl.check_scores(s[n, t, :m], d_ref[ids[n, t, :m]], what=f"gather row {n},{t}")
            assert np.all(np.isnan(s[n, t, m:]))


@pytest.mark.parametrize("T", [1, 3], ids=["decode_form", "block_form"])
def test_h_equals_H_is_dense_dsa(M, T):
    """h = H^I = 64: every head is routed, so Eq. (9) is Eq. (1): the routed scores equal the
    dense scores within the parity tolerance and the top-k sets agree up to cutoff ties;
    both equal the oracle's."""
    wl = _wl(T=T, nseq=3, h=64, topk=200, kprime=400)
    x = _random_pos(make_inputs(wl, seed=33), seed=4)
    q, w, k, pos = gpu_path.to_device(x)
    out = gpu_path.run_all(M, q, w, k, pos, wl.B, wl.h, wl.topk, wl.kprime)
    rows = np.arange(wl.rows)
    host = gpu_path.rows_to_host(out, rows, wl.T)
    gpu_path.check_rows(x, host, rows, wl.B, wl.h, wl.topk, wl.kprime)
    for i in rows:
        n, t = divmod(int(i), wl.T)
        P = int(x.pos[n, t]) + 1
        assert sorted(host["heads"][i].tolist()) == list(range(64))
        d = host["s_dsa"][i, :P].astype(np.float64)
        tl.check_scores(host["s_misa"][i, :P], d, what=f"row {i}: MISA h=H vs DSA")
        tl.check_selection(host["idx"][i], d, wl.topk, what=f"row {i}: MISA h=H set vs DSA")


def _expiry_case(M, wl, seed, skip_tile):
    x = make_inputs(wl, seed=seed)
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    M.misa_check_device_status(q.device)
    nan = lambda: torch.full((wl.nseq, wl.T, wl.L), float("nan"), device=q.device)
    ref = M.misa_score_rows(q, w, k, heads, pos, scores=nan())
    # a short bound with nothing skipped: identical to the ordinary call, no status
    s = M.misa_testing_score_rows_wait_expiry(q, w, k, heads, pos, 20_000_000, -1,
                                              scores=nan())
    M.misa_check_device_status(q.device)
    assert torch.equal(torch.nan_to_num(s, nan=-7.0), torch.nan_to_num(ref, nan=-7.0))
    # one key tile never loaded: the waits for it run out (about 1 ms of SM clock each), the
    # kernel records the timeout, drains, frees its tensor memory and returns
    M.misa_testing_score_rows_wait_expiry(q, w, k, heads, pos, 2_000_000, skip_tile)
    with pytest.raises(M.MisaError) as e:
        M.misa_check_device_status(q.device)
    assert e.value.status == 4
    # the context is still usable: the next ordinary calls pass parity against the oracle
    out = gpu_path.run_all(M, q, w, k, pos, wl.B, wl.h, wl.topk, wl.kprime)
    rows = np.arange(wl.rows) if wl.rows <= 8 else np.arange(0, wl.rows, wl.rows // 8)
    host = gpu_path.rows_to_host(out, rows, wl.T)
    gpu_path.check_rows(x, host, rows, wl.B, wl.h, wl.topk, wl.kprime)


def test_bounded_wait_expiry_decode_form(M):
    wl = _wl(nseq=8, T=1, L=32768, topk=2048, kprime=8192)
    _expiry_case(M, wl, seed=41, skip_tile=1000)   # 8 x 256 tiles; one in the middle


def test_bounded_wait_expiry_block_form(M):
    wl = _wl(nseq=1, T=256, L=8192, topk=256, kprime=512)
    _expiry_case(M, wl, seed=42, skip_tile=5)


def test_workspace_too_small_and_bad_buffers_rejected(M):
    """Host validation on real allocations: a workspace one byte short, q or k 2 bytes off
    their 16-byte alignment, and a workspace or an idx buffer that runs past the end of its
    driver allocation are rejected before anything is enqueued (the outputs keep their
    contents)."""
    lib = M.library()
    wl = _wl(nseq=2, T=1, L=4096, topk=64)
    x = make_inputs(wl, seed=43)
    q, w, k, pos = gpu_path.to_device(x)
    heads = torch.zeros((2, 1, wl.h), dtype=torch.int32, device="cuda")
    idx = torch.full((2, 1, wl.topk), -7, dtype=torch.int32, device="cuda")
    need = M.misa_workspace_size(2, 2, 1, 64, 128, wl.L, 1, wl.h, wl.topk, wl.topk)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)

    def call(qp, kp_, idxp, wsp, wsb):
        return lib.misa_score_topk(qp, P(w), kp_, P(heads), P(pos), 2, 1, 64, 128, wl.L, wl.h,
                                   wl.topk, idxp, None, None, wsp, wsb, st)

    assert call(P(q), P(k), P(idx), P(ws), need - 1) == 5            # WORKSPACE_TOO_SMALL
    qbuf = torch.zeros(q.numel() + 8, dtype=torch.bfloat16, device="cuda")
    kbuf = torch.zeros(k.numel() + 8, dtype=torch.bfloat16, device="cuda")
    assert call(P(qbuf, 2), P(k), P(idx), P(ws), need) == 1          # q misaligned
    assert call(P(q), P(kbuf, 2), P(idx), P(ws), need) == 1          # k misaligned
    # buffers that run past the end of their driver allocation: a 2 MiB cudaMalloc of their
    # own (the range check sees driver allocations, so a tensor carved out of a caching
    # allocator's larger block is checked against that block instead)
    from cuda.bindings import runtime as cudart
    err, base = cudart.cudaMalloc(1 << 21)
    assert err == cudart.cudaError_t.cudaSuccess
    try:
        end = int(base) + (1 << 21)
        assert call(P(q), P(k), P(idx), ctypes.c_void_p(end - 1024), need) == 1   # workspace
        idx_bytes = 2 * wl.topk * 4
        short_idx = ctypes.c_void_p(end - idx_bytes + 4)                  # 4 bytes short
        # idx is checked before the workspace: a one-byte-short workspace would give 5
        assert call(P(q), P(k), short_idx, P(ws), need - 1) == 1
        # the no-allocation entry point applies the same buffer checks (a misaligned
        # device_status, checked after idx, keeps the call from launching either way)
        assert lib.misa_score_topk_noalloc(P(q), P(w), P(k), P(heads), P(pos), 2, 1, 64, 128,
                                           wl.L, wl.h, wl.topk, short_idx, None,
                                           ctypes.c_void_p(int(base) + 2), st) == 1
    finally:
        cudart.cudaFree(base)
    assert lib.misa_score_topk_noalloc(P(qbuf, 2), P(w), P(k), P(heads), P(pos), 2, 1, 64, 128,
                                       wl.L, wl.h, wl.topk, P(idx), None, None, st) == 1
    host_idx = torch.zeros_like(idx, device="cpu")
    assert lib.misa_score_topk_noalloc(P(q), P(w), P(k), P(heads), P(pos), 2, 1, 64, 128, wl.L,
                                       wl.h, wl.topk, P(host_idx), None, None, st) == 1
    torch.cuda.synchronize()
    assert bool((idx == -7).all())


@pytest.mark.parametrize("T", [1, 64], ids=["decode_form", "block_form"])
def test_timed_scorer_matches_score_rows(M, T):
    # the timed entry runs the same scorer as misa_score_rows: identical scores (the
    # same kernel on the same inputs), and a positive kernel time
    wl = _wl(T=T, L=4096, pos_mode="tail" if T == 1 else "causal")
    if T > 1:
        wl = wl.replace(L=T)
    x = make_inputs(wl, seed=5)
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    ref = M.misa_score_rows(q, w, k, heads, pos)
    out = torch.full_like(ref, float("nan"))
    ms = M.misa_testing_score_rows_timed(q, w, k, heads, pos, scores=out)
    M.misa_check_device_status(q.device)
    assert ms > 0.0
    P = pos.long() + 1
    valid = torch.arange(ref.shape[-1], device=ref.device)[None, None, :] < P[..., None]
    assert torch.equal(out[valid], ref[valid])
