"""Helpers for the GPU parity tests: move seeded inputs to the device, run every
entry point of the CUDA path through the C ABI, and check the outputs of sampled
rows against the fp64 oracle with the rules in tests/tolerance.py."""

from __future__ import annotations

import numpy as np
import torch

import oracle.misa_oracle as orc
from tests import tolerance as tl


def to_device(x, device="cuda"):
    q = torch.from_numpy(np.ascontiguousarray(x.q_bits).view(np.int16)).to(device).view(torch.bfloat16)
    k = torch.from_numpy(np.ascontiguousarray(x.k_bits).view(np.int16)).to(device).view(torch.bfloat16)
    w = torch.from_numpy(np.ascontiguousarray(x.w)).to(device)
    pos = torch.from_numpy(np.ascontiguousarray(x.pos).astype(np.int32)).to(device)
    return q, w, k, pos


def run_all(M, q, w, k, pos, B, h, topk, kprime, want_scores=True):
    """Every entry point once; returns host numpy arrays."""
    nseq, T, H, d = q.shape
    L = k.shape[1]
    kp = M.misa_pool_keys(k, B)
    heads, E = M.misa_route_heads(q, w, k, kp, pos, B, h, return_E=True)
    s_misa = torch.full((nseq, T, L), float("nan"), device=q.device) if want_scores else None
    s_dsa = torch.full((nseq, T, L), float("nan"), device=q.device) if want_scores else None
    idx, vals = M.misa_score_topk(q, w, k, heads, pos, topk, scores=s_misa)
    didx, dvals = M.dsa_score_topk(q, w, k, pos, topk, scores=s_dsa)
    cand = M.misa_score_topk(q, w, k, heads, pos, kprime, return_vals=False)
    gidx, gvals = M.misa_dagger_rerank(q, w, k, pos, cand, topk)
    torch.cuda.synchronize()
    M.misa_check_device_status(q.device)
    out = dict(kp=kp, heads=heads, E=E, idx=idx, vals=vals, didx=didx, dvals=dvals, cand=cand,
               gidx=gidx, gvals=gvals, s_misa=s_misa, s_dsa=s_dsa)
    return out


def rows_to_host(out, rows, T):
    """Pull only the sampled rows (flat ids) to the host."""
    r = torch.as_tensor(np.asarray(rows), device=out["heads"].device)
    host = {}
    for key in ("heads", "E", "idx", "vals", "didx", "dvals", "cand", "gidx", "gvals", "s_misa",
                "s_dsa"):
        t = out[key]
        if t is None:
            host[key] = None
            continue
        flat = t.reshape(-1, t.shape[-1])
        host[key] = flat.index_select(0, r).cpu().numpy()
    host["kp"] = out["kp"].cpu().numpy()
    return host


def check_rows(x, host, rows, B, h, topk, kprime, check_pool=True):
    """Compare sampled rows with the oracle.  Returns summary statistics."""
    nseq, T, H, d = x.q_bits.shape
    stats = dict(rows=len(rows), head_swaps=0, token_swaps=0, dsa_swaps=0, dagger_swaps=0,
                 recall_misa=[], recall_dagger=[], max_err_ratio=0.0)
    if check_pool:
        for n in sorted(set(int(r) // T for r in rows)):
            ref = orc.pool_keys(orc.bf16_bits_to_f64(x.k_bits[n]), B)
            for b in range(ref.shape[0]):
                tl.check_scores(host["kp"][n, b], ref[b], what=f"pooled key seq {n} block {b}")
    kcache = {}
    for i, row in enumerate(rows):
        n, t = divmod(int(row), T)
        if n not in kcache:
            kcache.clear()
            kcache[n] = orc.bf16_bits_to_f64(x.k_bits[n])
        k = kcache[n]
        q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
        w_t = x.w[n, t].astype(np.float64)
        P = int(x.pos[n, t]) + 1
        tag = f"row {row}"
        # router: E and the head set (Eqs. 7-8)
        E_ref = orc.router_energy(q_t, w_t, k, P, B)
        stats["max_err_ratio"] = max(stats["max_err_ratio"],
                                     tl.check_scores(host["E"][i], E_ref, what=f"{tag} E"))
        stats["head_swaps"] += tl.check_selection(host["heads"][i], E_ref, h, what=f"{tag} heads")
        assert list(host["heads"][i]) == sorted(host["heads"][i], key=lambda j: (-host["E"][i][j], j))
        # routed scores under the GPU's heads (Eq. 9) and their top-k (Eq. 10)
        gh = host["heads"][i]
        s_ref = orc.token_scores(q_t, w_t, k, P, gh)
        if host["s_misa"] is not None:
            stats["max_err_ratio"] = max(stats["max_err_ratio"], tl.check_scores(
                host["s_misa"][i, :P], s_ref, what=f"{tag} routed scores"))
        stats["token_swaps"] += tl.check_selection(host["idx"][i], s_ref, topk, what=f"{tag} MISA top-k")
        tl.check_order(host["idx"][i], host["vals"][i], what=f"{tag} MISA order")
        sel = host["idx"][i][host["idx"][i] >= 0]
        tl.check_scores(host["vals"][i][:sel.size], s_ref[sel], what=f"{tag} MISA vals")
        # dense DSA (Eqs. 1-2)
        d_ref = orc.dense_scores(q_t, w_t, k, P)
        if host["s_dsa"] is not None:
            stats["max_err_ratio"] = max(stats["max_err_ratio"], tl.check_scores(
                host["s_dsa"][i, :P], d_ref, what=f"{tag} dense scores"))
        stats["dsa_swaps"] += tl.check_selection(host["didx"][i], d_ref, topk, what=f"{tag} DSA top-k")
        tl.check_order(host["didx"][i], host["dvals"][i], what=f"{tag} DSA order")
        dsel = host["didx"][i][host["didx"][i] >= 0]
        tl.check_scores(host["dvals"][i][:dsel.size], d_ref[dsel], what=f"{tag} DSA vals")
        # MISA-dagger: coarse candidates (Eq. 11) then all-head re-rank (Eq. 12)
        tl.check_selection(host["cand"][i], s_ref, kprime, what=f"{tag} MISA-dagger candidates")
        dg = orc.misa_dagger_row(q_t, w_t, k, P, host["cand"][i], topk)
        stats["dagger_swaps"] += tl.check_selection(host["gidx"][i], dg["scores"], topk,
                                                    what=f"{tag} MISA-dagger top-k",
                                                    ids=dg["cand"])
        tl.check_order(host["gidx"][i], host["gvals"][i], what=f"{tag} MISA-dagger order")
        gsel = host["gidx"][i][host["gidx"][i] >= 0]
        tl.check_scores(host["gvals"][i][:gsel.size], d_ref[gsel], what=f"{tag} MISA-dagger vals")
        ref_dense_top = orc.topk(d_ref, topk)[0]
        stats["recall_misa"].append(orc.recall(host["idx"][i], ref_dense_top))
        stats["recall_dagger"].append(orc.recall(host["gidx"][i], ref_dense_top))
    stats["recall_misa"] = float(np.mean(stats["recall_misa"]))
    stats["recall_dagger"] = float(np.mean(stats["recall_dagger"]))
    return stats
