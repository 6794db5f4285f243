"""Edge cases of the CUDA path against the fp64 oracle (GPU): ragged blocks, prefixes
shorter than a block or than k, h = 1 and h = H, k' = k, ties, zero and negative
weights, odd head counts, B = 1 and B > L, many rows, the largest k, bad device
input, and guard bands around every output."""

import numpy as np
import pytest
import torch

from synth import Workload, fp32_to_bf16_bits, make_inputs
from tests import gpu_path

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_block_b200 as M
    return M


def _wl(**kw):
    base = dict(name="edge", nseq=2, T=5, L=300, H=8, d=128, h=3, B=64, topk=40, kprime=80,
                pos_mode="tail", drift=True, needles=2)
    base.update(kw)
    return Workload(**base)


def _random_pos(x, seed, lo=0):
    rng = np.random.default_rng(seed)
    x.pos = rng.integers(lo, x.wl.L, size=x.pos.shape).astype(np.int32)
    return x


CASES = {
    "ragged_L_random_pos": dict(),
    "prefix_shorter_than_block": dict(L=50, B=64, topk=16, kprime=32),
    "prefix_shorter_than_k": dict(L=100, topk=256, kprime=512),
    "h1": dict(h=1),
    "h_equals_H": dict(h=8),
    "kprime_equals_k": dict(kprime=40),
    "H32_B128": dict(H=32, B=128, L=1000, h=8, topk=64, kprime=128),
    "H3_odd": dict(H=3, h=2, L=257, B=16),
    "H128_max_heads": dict(H=128, h=16, L=600, topk=100, kprime=200),
    "B1": dict(B=1, L=200, topk=20, kprime=40),
    "B_larger_than_L": dict(B=1024, L=300),
    "many_rows": dict(nseq=3, T=150, L=700, topk=50, kprime=100),
    "max_topk": dict(nseq=1, T=2, L=20000, topk=16384, kprime=16384, B=128),
    # re-rank over more candidates than the row top-k keeps resident (16384 > 8192)
    "dagger_wide_kprime": dict(nseq=1, T=2, L=20000, topk=2048, kprime=16384, B=128),
    # one query per sequence: the decode form of the scorer
    "decode_T1_ragged": dict(nseq=4, T=1, L=777, topk=64, kprime=128),
    "decode_T1_H16_B1": dict(nseq=3, T=1, L=300, H=16, h=5, B=1, topk=32, kprime=64),
    # a few queries per sequence (multi-token decode): narrow query blocks
    "mtp_T2": dict(nseq=3, T=2, L=900, topk=64, kprime=128),
    "mtp_T3_H16": dict(nseq=2, T=3, L=1500, H=16, h=4, topk=100, kprime=200),
    "mtp_T4_H64": dict(nseq=2, T=4, L=2000, H=64, h=8, topk=128, kprime=256),
    "mtp_T9_H32": dict(nseq=2, T=9, L=1200, H=32, h=8, topk=64, kprime=128),
    # many queries per sequence: tensor-core router and query-block scorer
    "blocks_two_seqs_H16": dict(nseq=2, T=64, L=1000, H=16, h=4, topk=64, kprime=128),
    "blocks_H64_B32": dict(nseq=1, T=40, L=3000, H=64, h=8, B=32, topk=128, kprime=256),
    # tensor-core router shapes: 16 queries per tile with a partial last tile, 4 per tile
    # over two sequences, and a prefix beyond 16K (512 pooled blocks)
    "route_tc_H8_partial_tile": dict(nseq=1, T=100, L=3000, H=8, h=3, topk=64, kprime=128),
    "route_tc_H32_two_seqs": dict(nseq=2, T=64, L=2000, H=32, h=8, B=32, topk=64, kprime=128),
    "prefill_32k_prefix": dict(nseq=1, T=64, L=32768, H=64, h=8, B=64, topk=2048,
                               kprime=4096),
}


@pytest.mark.parametrize("case", list(CASES))
def test_edge_case(M, case):
    wl = _wl(**CASES[case])
    x = make_inputs(wl, seed=11)
    if case not in ("prefix_shorter_than_k", "max_topk"):
        x = _random_pos(x, seed=5)
    q, w, k, pos = gpu_path.to_device(x)
    out = gpu_path.run_all(M, q, w, k, pos, wl.B, wl.h, wl.topk, wl.kprime)
    rows = np.arange(wl.rows)
    host = gpu_path.rows_to_host(out, rows, wl.T)
    gpu_path.check_rows(x, host, rows, wl.B, wl.h, wl.topk, wl.kprime)


def test_all_scores_tied_and_zero_weights(M):
    """Keys all equal and every q.k negative: every score is exactly 0 and every E is 0,
    so the selections must be the lowest indices (ties -> lower index)."""
    wl = _wl(nseq=1, T=3, L=500, H=8, h=3, topk=64, kprime=128)
    x = make_inputs(wl, seed=3)
    kv = np.full((128,), 0.05, dtype=np.float32)
    x.k_bits[:] = fp32_to_bf16_bits(kv)[None, None, :]
    qv = -np.abs((x.q_bits.astype(np.uint32) << 16).view(np.float32))
    x.q_bits = fp32_to_bf16_bits(qv)
    x.w[:] = 0.0
    x.w[0, 0, 2] = -1.5
    q, w, k, pos = gpu_path.to_device(x)
    out = gpu_path.run_all(M, q, w, k, pos, wl.B, wl.h, wl.topk, wl.kprime)
    assert torch.all(out["heads"].cpu() == torch.arange(3, dtype=torch.int32))
    for key in ("idx", "didx", "gidx"):
        assert torch.all(out[key].cpu() == torch.arange(64, dtype=torch.int32)), key
    assert torch.all(out["cand"].cpu() == torch.arange(128, dtype=torch.int32))


def test_bad_device_input_is_reported_not_faulting(M):
    """pos >= L and out-of-prefix candidates are clamped / skipped and reported through
    the workspace status word."""
    wl = _wl(nseq=1, T=2, L=256, topk=16, kprime=32)
    x = make_inputs(wl, seed=4)
    q, w, k, pos = gpu_path.to_device(x)
    bad_pos = pos.clone()
    bad_pos[0, 1] = 10_000
    kp = M.misa_pool_keys(k, wl.B)
    M.misa_route_heads(q, w, k, kp, bad_pos, wl.B, wl.h)
    with pytest.raises(M.MisaError) as e:
        M.misa_check_device_status(q.device)
    assert e.value.status == 6
    M.misa_check_device_status(q.device)  # cleared
    cand = torch.full((1, 2, 32), -1, dtype=torch.int32, device=q.device)
    cand[0, 0, 0] = 5
    cand[0, 0, 1] = 100_000
    idx, vals = M.misa_dagger_rerank(q, w, k, pos, cand, 16)
    with pytest.raises(M.MisaError):
        M.misa_check_device_status(q.device)
    assert idx[0, 0, 0].item() == 5 and idx[0, 0, 1].item() == -1


def test_guard_bands_untouched(M):
    wl = _wl(nseq=2, T=3, L=400, topk=32, kprime=64)
    x = make_inputs(wl, seed=9)
    q, w, k, pos = gpu_path.to_device(x)
    G = 1024
    rows = wl.rows

    def banded(n, dtype, fill):
        buf = torch.full((n + 2 * G,), fill, dtype=dtype, device=q.device)
        return buf, buf[G:G + n]

    kp_buf, kp = banded(2 * 7 * 128, torch.float32, 7.0)
    M.misa_pool_keys(k, wl.B, out=kp.view(2, 7, 128))
    h_buf, heads = banded(rows * wl.h, torch.int32, 77)
    e_buf, E = banded(rows * wl.H, torch.float32, 7.0)
    M.misa_route_heads(q, w, k, kp.view(2, 7, 128), pos, wl.B, wl.h, return_E=True,
                       heads=heads.view(2, 3, wl.h), E=E.view(2, 3, wl.H))
    i_buf, idx = banded(rows * wl.topk, torch.int32, 77)
    v_buf, vals = banded(rows * wl.topk, torch.float32, 7.0)
    M.misa_score_topk(q, w, k, heads.view(2, 3, wl.h), pos, wl.topk,
                      idx=idx.view(2, 3, wl.topk), vals=vals.view(2, 3, wl.topk))
    torch.cuda.synchronize()
    for buf, fill in ((kp_buf, 7.0), (h_buf, 77), (e_buf, 7.0), (i_buf, 77), (v_buf, 7.0)):
        assert torch.all(buf[:G] == fill) and torch.all(buf[-G:] == fill)


@pytest.mark.parametrize("T,pos_mode", [(3, "tail"), (70, "causal")])
def test_score_rows_entry_point(M, T, pos_mode):
    """misa_score_rows (scores without selection) against the oracle's Eq. (9) under the
    GPU's heads and Eq. (1), for decode-form rows and for query blocks (T >= 32)."""
    import oracle.misa_oracle as orc
    from tests import tolerance as tl
    wl = _wl(nseq=2, T=T, L=900, topk=32, kprime=64, pos_mode=pos_mode)
    x = make_inputs(wl, seed=13)
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    routed = M.misa_score_rows(q, w, k, heads, pos).cpu().numpy()
    dense = M.misa_score_rows(q, w, k, None, pos).cpu().numpy()
    hh = heads.cpu().numpy()
    for n in range(wl.nseq):
        kk = orc.bf16_bits_to_f64(x.k_bits[n])
        for t in range(T):
            P = int(x.pos[n, t]) + 1
            q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
            w_t = x.w[n, t].astype(np.float64)
            tl.check_scores(routed[n, t, :P], orc.token_scores(q_t, w_t, kk, P, hh[n, t]),
                            what=f"routed {n},{t}")
            tl.check_scores(dense[n, t, :P], orc.dense_scores(q_t, w_t, kk, P),
                            what=f"dense {n},{t}")


def test_tied_long_rows_exact_fallback(M):
    """Rows long enough for the histogram top-k whose scores are all equal: the crowded
    cutoff takes the exact fallback (inside the group kernel for k <= 4096, the separate
    overflow kernel above) and returns the lowest indices."""
    wl = _wl(nseq=2, T=1, L=10000, H=8, h=3, topk=2048, kprime=8192)
    x = make_inputs(wl, seed=5)
    x.k_bits[:] = fp32_to_bf16_bits(np.full((128,), 0.05, dtype=np.float32))[None, None, :]
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    for kk in (wl.topk, wl.kprime):
        idx = M.misa_score_topk(q, w, k, heads, pos, kk, return_vals=False)
        didx = M.dsa_score_topk(q, w, k, pos, kk, return_vals=False)
        ref = torch.arange(kk, dtype=torch.int32).expand(2, 1, kk)
        assert torch.equal(idx.cpu(), ref) and torch.equal(didx.cpu(), ref), kk


@pytest.mark.parametrize("L", [2000, 40000], ids=["one_cta_per_row", "cluster_split_rows"])
def test_dagger_candidates_any_order_with_repeats(M, L):
    """Eq. (12) re-scores the set Omega_t: candidates given shuffled, with repeated ids
    and empty slots, re-rank exactly like the oracle on the distinct ids (at L = 40000 the
    six rows' candidate ordering splits each prefix over a cluster of CTAs)."""
    import oracle.misa_oracle as orc
    from tests import tolerance as tl
    wl = _wl(nseq=2, T=3, L=L, topk=64, kprime=400)
    x = make_inputs(wl, seed=21)
    rng = np.random.default_rng(8)
    cand = np.full((wl.nseq, wl.T, wl.kprime), -1, dtype=np.int32)
    for n in range(wl.nseq):
        for t in range(wl.T):
            P = int(x.pos[n, t]) + 1
            ids = rng.choice(P, size=300, replace=False)
            rep = rng.choice(ids, size=60)                 # repeated ids
            row = np.concatenate([ids, rep, np.full(40, -1)]).astype(np.int32)
            cand[n, t] = rng.permutation(row)
    q, w, k, pos = gpu_path.to_device(x)
    idx, vals = M.misa_dagger_rerank(q, w, k, pos, torch.from_numpy(cand).to(q.device), wl.topk)
    M.misa_check_device_status(q.device)
    idx, vals = idx.cpu().numpy(), vals.cpu().numpy()
    for n in range(wl.nseq):
        kk = orc.bf16_bits_to_f64(x.k_bits[n])
        for t in range(wl.T):
            P = int(x.pos[n, t]) + 1
            q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
            w_t = x.w[n, t].astype(np.float64)
            d_ref = orc.dense_scores(q_t, w_t, kk, P)
            dg = orc.misa_dagger_row(q_t, w_t, kk, P, cand[n, t], wl.topk)   # Omega_t as a set
            assert len(set(idx[n, t].tolist())) == wl.topk
            tl.check_selection(idx[n, t], dg["scores"], wl.topk, what=f"dagger {n},{t}",
                               ids=dg["cand"])
            tl.check_order(idx[n, t], vals[n, t], what=f"dagger order {n},{t}")
            tl.check_scores(vals[n, t], d_ref[idx[n, t]], what=f"dagger vals {n},{t}")


@pytest.mark.parametrize("B", [64, 512])
def test_pool_keys_range_refreshes_only_changed_blocks(M, B):
    """Eq. (4) kept up to date: after keys in a token range change, the refresh rewrites
    exactly the blocks meeting that range; the result equals a full re-pool bit for bit
    (same kernel arithmetic) and the oracle's pooled keys within tolerance.  B = 512 takes
    the form where a CTA's warps share one block."""
    import oracle.misa_oracle as orc
    from tests import tolerance as tl
    wl = _wl(nseq=3, T=1, L=1000, B=B)
    x = make_inputs(wl, seed=17)
    _, _, k, _ = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, B)
    rng = np.random.default_rng(4)
    for s0, s1 in ((130, 131), (990, 1000), (0, 64), (300, 700), (999, 1000), (500, 500)):
        new = rng.standard_normal((wl.nseq, s1 - s0, 128)).astype(np.float32) / np.sqrt(128)
        x.k_bits[:, s0:s1] = fp32_to_bf16_bits(new)
        _, _, k, _ = gpu_path.to_device(x)
        b0, b1 = s0 // B, -(-s1 // B)
        kp[:, :b0] = 7.0   # blocks outside the range must not be written
        kp[:, b1:] = 7.0
        M.misa_pool_keys_range(k, B, kp, s0, s1)
        full = M.misa_pool_keys(k, B)
        got = kp.cpu().numpy()
        assert np.all(got[:, :b0] == 7.0) and np.all(got[:, b1:] == 7.0), (s0, s1)
        assert torch.equal(kp[:, b0:b1], full[:, b0:b1]), (s0, s1)
        for n in range(wl.nseq):
            ref = orc.pool_keys(orc.bf16_bits_to_f64(x.k_bits[n]), B)
            for b in range(b0, b1):
                tl.check_scores(got[n, b], ref[b], what=f"block {n},{b} after [{s0},{s1})")
        kp = full


def test_decode_with_kept_pooled_keys(M):
    """A decode loop that appends one key per step and refreshes only its block routes
    and selects exactly like re-pooling every step."""
    B = 64
    wl = _wl(nseq=2, T=1, L=700, B=B, topk=64, kprime=128)
    x = make_inputs(wl, seed=23)
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, B)
    for p in range(600, 700, 7):
        pos.fill_(p)
        x.k_bits[:, p] = fp32_to_bf16_bits(
            np.random.default_rng(p).standard_normal((wl.nseq, 128)).astype(np.float32) / 12)
        _, _, k, _ = gpu_path.to_device(x)
        M.misa_pool_keys_range(k, B, kp, p, p + 1)
        full = M.misa_pool_keys(k, B)
        assert torch.equal(kp, full), p
        h1 = M.misa_route_heads(q, w, k, kp, pos, B, wl.h)
        h2 = M.misa_route_heads(q, w, k, full, pos, B, wl.h)
        assert torch.equal(h1, h2), p


@pytest.mark.parametrize("T,L,topk", [(300, 5000, 3000), (300, 10000, 8192)])
def test_tied_rows_many_queries(M, T, L, topk):
    """Many rows of equal scores longer than the row top-k's candidate room: the crowded
    cutoff takes the exact radix select and returns the lowest indices."""
    wl = _wl(nseq=1, T=T, L=L, H=8, h=3, topk=topk, kprime=topk)
    x = make_inputs(wl, seed=6)
    x.k_bits[:] = fp32_to_bf16_bits(np.full((128,), 0.05, dtype=np.float32))[None, None, :]
    q, w, k, pos = gpu_path.to_device(x)
    kp = M.misa_pool_keys(k, wl.B)
    heads = M.misa_route_heads(q, w, k, kp, pos, wl.B, wl.h)
    idx = M.misa_score_topk(q, w, k, heads, pos, topk, return_vals=False)
    ref = torch.arange(topk, dtype=torch.int32).expand(1, T, topk)
    assert torch.equal(idx.cpu(), ref)


def test_tied_candidates_exact_rerank(M):
    """12000 tied candidates re-ranked to 8192: exact fallback over an index map."""
    wl = _wl(nseq=2, T=1, L=13000, H=8, h=3, topk=8192, kprime=12000)
    x = make_inputs(wl, seed=7)
    x.k_bits[:] = fp32_to_bf16_bits(np.full((128,), 0.05, dtype=np.float32))[None, None, :]
    q, w, k, pos = gpu_path.to_device(x)
    rng = np.random.default_rng(3)
    cand = np.stack([rng.permutation(12000) for _ in range(2)]).astype(np.int32)[:, None, :]
    idx, _ = M.misa_dagger_rerank(q, w, k, pos, torch.from_numpy(cand).to(q.device), 8192)
    ref = torch.arange(8192, dtype=torch.int32).expand(2, 1, 8192)
    assert torch.equal(idx.cpu(), ref)
