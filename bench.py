"""Benchmark of the MISA indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the MISA path over one batch of synthetic input that is
already resident in HBM: block pooling (Eq. 4), head routing (Eqs. 7-8), routed
scoring and top-k (Eqs. 9-10).  The dense DSA indexer (Eqs. 1-2) and MISA-dagger
(coarse top-k' + all-head re-rank, Eqs. 11-12) run the same number of steps on the
same inputs, timed separately, and are reported beside it.  Rank 0 prints one JSON
line.  Throughput unit: query x prefix-token pairs scored per second.

Inputs are larger than L2 (126 MB) and two copies are used alternately, so no step
reads keys another step left in L2.

`--impl reference` times the fp64 CPU oracle (the parity reference) on a bounded
sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import WORKLOADS, make_inputs  # noqa: E402

METRIC = "indexer query×prefix-tokens/s at 32K–128K (MISA h=8 vs dense); % of roofline"
UNIT = "query×prefix-tokens/s"
DEFAULT_WORKLOAD = "dsv32_decode_32k"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's elapsed time (every rank passes its own; a collective that all ranks
    take in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, tag: int):
        self.gpu = gpu_id            # nvidia-smi --id value (the device UUID)
        self.proc = None
        out_dir = os.environ.get("MISA_BENCH_LOG_DIR")   # keep the raw samples there if set
        if out_dir:
            self.path = os.path.join(out_dir, f"clocks_rank{tag}.csv")
        else:
            fd, self.path = tempfile.mkstemp(prefix=f"misa_clocks_rank{tag}_", suffix=".csv")
            os.close(fd)

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path) or ".", exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.STDOUT)
            time.sleep(0.5)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def block_form(wl) -> bool:
    """Whether the scorer shares key tiles among the queries of a sequence (any T > 1)."""
    return wl.T >= 2


def misa_step_launches(wl) -> int:
    """Kernels one MISA step launches, following the library's dispatch: pooling, the router
    (one kernel, or three on tcgen05 for many queries per sequence), the scorer's
    gather/offsets kernel and the scorer, then the top-k: one kernel, except histogrammed
    rows longer than 40960 scores or with k > 3072, which take a scatter and a group kernel
    (and an overflow kernel above k = 4096); rows of several queries per sequence longer
    than 16384 scores first take a histogram pass."""
    qt = 128 // wl.H if (128 % wl.H == 0 and wl.H >= 8) else 0
    route_tc = qt > 0 and wl.T >= 4 * qt and (wl.nseq == 1 or wl.T % qt == 0)
    n = 1 + (3 if route_tc else 1)
    n += 2
    hist_path = wl.rows <= 1024 and wl.L >= 8192 and not block_form(wl)
    hist_kernel = wl.rows <= 1024 and wl.L > 16384 and block_form(wl)
    if hist_kernel:
        n += 1
    if (hist_path or hist_kernel) and not (wl.L <= 40960 and wl.topk <= 3072):
        n += 2 + (wl.topk > 4096)
    else:
        n += 1
    return n


def algorithmic_flops_score(wl) -> float:
    """Multiply-add work of Eq. (9) over every causal (query, key) pair: 2 * h * d each."""
    return 2.0 * wl.h * wl.d * wl.query_prefix_tokens()


def algorithmic_bytes_score(wl) -> float:
    """Bytes the routed scoring kernel (misa_score_rows, the scorer misa_score_topk runs)
    must move: every key of every query's prefix, 256 B per token (decode rows do not
    share keys; the queries of a prefill sequence share its keys), each query's routed
    head vectors, weights and head ids (h * (256 + 4 + 4) B), and one fp32 score written
    per query x prefix-token."""
    P = wl.positions().astype(np.int64) + 1
    if wl.T == 1:
        keys = float(P.sum()) * wl.d * 2
    else:
        keys = float(wl.nseq) * wl.L * wl.d * 2
    return keys + wl.rows * wl.h * (wl.d * 2 + 4 + 4) + 4.0 * wl.query_prefix_tokens()


def run_reference(args, wl):
    """fp64 CPU oracle on a bounded sample: each step = one query row of the workload."""
    rank, world, _ = _dist_env()
    if rank != 0:
        return 0
    import oracle.misa_oracle as orc
    from threadpoolctl import threadpool_info
    x = make_inputs(wl, seed=0)
    rows = list(range(wl.rows))
    T = wl.T

    def one(row):
        n, t = divmod(row, T)
        k = orc.bf16_bits_to_f64(x.k_bits[n])
        q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
        P = int(x.pos[n, t]) + 1
        orc.misa_row(q_t, x.w[n, t].astype(np.float64), k, P, wl.B, wl.h, wl.topk)
        return P

    for i in range(args.warmup):
        one(rows[i % len(rows)])
    t0 = time.perf_counter()
    units = 0
    for i in range(args.steps):
        units += one(rows[(args.warmup + i) % len(rows)])
    dt = time.perf_counter() - t0
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    val = units / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "nseq": wl.nseq, "T": wl.T, "L": wl.L, "H": wl.H,
                   "h": wl.h, "B": wl.B, "topk": wl.topk, "path": "MISA (pool+route+score+top-k)"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads,
                         "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{args.steps} query rows of {wl.name} (one row per step), "
                                   "fp64 numpy oracle"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def cpu_baseline(wl, budget_s: float = 10.0):
    """Time the oracle's MISA path on the host cores: passes over the workload's query
    rows until the time budget is used (at least one row)."""
    import oracle.misa_oracle as orc
    from threadpoolctl import threadpool_info
    x = make_inputs(wl, seed=0)
    units, rows_done = 0, 0
    t0 = time.perf_counter()
    for it in range(1 << 30):
        row = it % x.wl.rows
        n, t = divmod(row, x.wl.T)
        k = orc.bf16_bits_to_f64(x.k_bits[n])
        q_t = orc.bf16_bits_to_f64(x.q_bits[n, t])
        P = int(x.pos[n, t]) + 1
        orc.misa_row(q_t, x.w[n, t].astype(np.float64), k, P, wl.B, wl.h, wl.topk)
        units += P
        rows_done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    return {"value": units / dt, "unit": UNIT, "cores": threads,
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows_done} query rows of {wl.name} ({units} query x prefix-token pairs), "
                      f"full MISA path in fp64 numpy, {dt:.1f} s"}


EXTRA_WORKLOADS = ("dsv32_prefill_16k", "glm5_decode_128k", "dagger_128k")


def _roofline(wl, ms_score_kernel, peaks, traffic):
    """Roofline object of the routed scorer: its bound is whichever of the kernel's
    algorithmic flops and bytes takes longer at the measured peaks."""
    flops = algorithmic_flops_score(wl)
    score_bytes = algorithmic_bytes_score(wl)
    form = "block form" if block_form(wl) else "decode form"
    common = {"kernel": f"score_tc_kernel (routed scoring, {form})", "traffic": traffic,
              "algorithmic_flops": flops, "algorithmic_bytes": score_bytes,
              "avg_ms": ms_score_kernel}
    if flops / (peaks["bf16"] * 1e12) > score_bytes / (peaks["hbm"] * 1e9):
        achieved = flops / (ms_score_kernel * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16"],
                "peak_source": peaks["source"] + " bf16 dense (burst)", **common}
    achieved = score_bytes / (ms_score_kernel * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": achieved / peaks["hbm"], "peak_source": peaks["source"] + " HBM copy",
            **common}


def measure_workload(M, wl, args, dev, world, rank, peaks, headline: bool):
    """Time MISA, dense DSA, MISA-dagger (and, for decode, MISA with kept pooled keys) on
    one workload with two resident input copies used alternately; also the routed scorer
    alone (for the roofline), recall against DSA and the clocks during the MISA region.
    The headline workload also gets the end-to-end number.  Returns (result, misa_ms)."""
    import torch
    import torch.distributed as dist

    x = make_inputs(wl, seed=rank)
    q_h = torch.from_numpy(x.q_bits.view(np.int16)).pin_memory()
    k_h = torch.from_numpy(x.k_bits.view(np.int16)).pin_memory()
    w_h = torch.from_numpy(x.w).pin_memory()
    pos_h = torch.from_numpy(x.pos.astype(np.int32)).pin_memory()
    sets = []
    for _ in range(2):   # two resident copies, used alternately (each larger than L2)
        sets.append((q_h.to(dev).view(torch.bfloat16), w_h.to(dev),
                     k_h.to(dev).view(torch.bfloat16), pos_h.to(dev)))
    nseq, T, H, d = wl.nseq, wl.T, wl.H, wl.d
    M_blocks = -(-wl.L // wl.B)
    kp = [torch.empty((nseq, M_blocks, d), dtype=torch.float32, device=dev) for _ in range(2)]
    heads = torch.empty((nseq, T, wl.h), dtype=torch.int32, device=dev)
    idx = torch.empty((nseq, T, wl.topk), dtype=torch.int32, device=dev)
    vals = torch.empty((nseq, T, wl.topk), dtype=torch.float32, device=dev)
    cand = torch.empty((nseq, T, wl.kprime), dtype=torch.int32, device=dev)
    gidx = torch.empty_like(idx)
    gvals = torch.empty_like(vals)
    didx = torch.empty_like(idx)
    dvals = torch.empty_like(vals)
    units = wl.query_prefix_tokens()
    stream = torch.cuda.current_stream()

    ev_calls = []   # per timed step: events around pool, route, routed score + top-k

    def misa_step(i, record=False):
        q, w, k, pos = sets[i % 2]
        if record:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(stream)
        M.misa_pool_keys(k, wl.B, out=kp[i % 2])
        if record:
            ev[1].record(stream)
        M.misa_route_heads(q, w, k, kp[i % 2], pos, wl.B, wl.h, heads=heads)
        if record:
            ev[2].record(stream)
        M.misa_score_topk(q, w, k, heads, pos, wl.topk, idx=idx, vals=vals)
        if record:
            ev[3].record(stream)
            ev_calls.append(ev)

    def dagger_step(i):
        q, w, k, pos = sets[i % 2]
        M.misa_pool_keys(k, wl.B, out=kp[i % 2])
        M.misa_route_heads(q, w, k, kp[i % 2], pos, wl.B, wl.h, heads=heads)
        M.misa_score_topk(q, w, k, heads, pos, wl.kprime, return_vals=False, idx=cand)
        M.misa_dagger_rerank(q, w, k, pos, cand, wl.topk, idx=gidx, vals=gvals)

    def dsa_step(i):
        q, w, k, pos = sets[i % 2]
        M.dsa_score_topk(q, w, k, pos, wl.topk, idx=didx, vals=dvals)

    # HISA-style block filter (decode workloads): the page's HISA block size B = 128 and
    # m = k' / B blocks, so its token refinement re-scores as many tokens as MISA-dagger's
    hisa_B = 128
    hisa_m = max(1, wl.kprime // hisa_B)
    hisa_on = T == 1
    if hisa_on:
        kp_h = [torch.empty((nseq, -(-wl.L // hisa_B), d), dtype=torch.float32, device=dev)
                for _ in range(2)]
        hidx = torch.empty_like(idx)
        hvals = torch.empty_like(vals)

    def hisa_step(i):
        q, w, k, pos = sets[i % 2]
        M.misa_pool_keys(k, hisa_B, out=kp_h[i % 2])
        M.hisa_block_filter_topk(q, w, k, kp_h[i % 2], pos, hisa_B, hisa_m, wl.topk, idx=hidx,
                                 vals=hvals)

    def kept_pool_step(i):
        # decode with the pooled keys kept between steps: each sequence's newest key (the
        # query's own position, L - 1) is the only change, so only its block is re-pooled
        q, w, k, pos = sets[i % 2]
        M.misa_pool_keys_range(k, wl.B, kp[i % 2], wl.L - 1, wl.L)
        M.misa_route_heads(q, w, k, kp[i % 2], pos, wl.B, wl.h, heads=heads)
        M.misa_score_topk(q, w, k, heads, pos, wl.topk, idx=idx, vals=vals)

    if args.only:
        # one path's steps and nothing else (for profiler captures); prints no bench line
        fn = {"misa": misa_step, "dagger": dagger_step, "dsa": dsa_step,
              "kept": kept_pool_step, "hisa": hisa_step}[args.only]
        for i in range(args.warmup + args.steps):
            fn(i)
        torch.cuda.synchronize()
        M.misa_check_device_status(dev)
        return {"only": args.only, "workload": wl.name, "steps": args.warmup + args.steps}, None

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(step_fn, steps, warmup, load_s=0.0, **kw):
        for i in range(warmup):
            step_fn(i)
        if load_s > 0:   # untimed steady-state load so the clock sampler sees this kernel mix
            torch.cuda.synchronize()
            t_end = time.perf_counter() + load_s
            i = warmup
            while time.perf_counter() < t_end:
                for _ in range(20):
                    step_fn(i)
                    i += 1
                torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            step_fn(warmup + i, **kw)
        e1.record(stream)
        barrier()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        return ms / steps

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    with ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid,
                      f"{rank}_{wl.name}") as clk:
        ms_misa = timed(misa_step, args.steps, args.warmup, load_s=2.0 if headline else 1.0,
                        record=True)
    clocks = clk.summary()
    M.misa_check_device_status(dev)
    per_call = [[e[j].elapsed_time(e[j + 1]) for j in range(3)] for e in ev_calls]
    call_ms = [sum(c[j] for c in per_call) / len(per_call) for j in range(3)]
    ms_dagger = timed(dagger_step, args.steps, args.warmup)
    ms_dsa = timed(dsa_step, args.steps, args.warmup)
    decode = T == 1 and bool(np.all(x.pos == wl.L - 1))
    ms_kept = timed(kept_pool_step, args.steps, args.warmup) if decode else None
    ms_hisa = timed(hisa_step, args.steps, args.warmup) if hisa_on else None

    # selection agreement with dense DSA on the same inputs (outside the timed regions): the
    # fraction of DSA's k tokens that MISA and MISA-dagger also select, averaged over rows
    misa_step(0)
    dsa_step(0)
    dagger_step(0)
    if hisa_on:
        hisa_step(0)
    torch.cuda.synchronize()

    def recall(sel, ref):
        r = ref.reshape(-1, ref.shape[-1]).long()
        s_ = sel.reshape(-1, sel.shape[-1]).long()
        out = []
        for r0 in range(0, r.shape[0], 1024):   # bounded memory for many rows
            rr, ss = r[r0:r0 + 1024], s_[r0:r0 + 1024]
            mask = torch.zeros((rr.shape[0], wl.L + 1), dtype=torch.bool, device=dev)
            mask.scatter_(1, torch.where(rr >= 0, rr, wl.L), True)
            hit = mask.gather(1, torch.where(ss >= 0, ss, wl.L)) & (ss >= 0)
            n_ref = (rr >= 0).sum(1).clamp(min=1)
            out.append(hit.sum(1).float() / n_ref.float())
        return float(torch.cat(out).mean().item())

    recalls = {"misa": recall(idx, didx), "misa_dagger": recall(gidx, didx)}
    if hisa_on:
        recalls["hisa_block_filter"] = recall(hidx, didx)
    # the routed scoring kernel alone (the scorer of misa_score_topk with the same launch
    # configuration), on the heads the MISA steps routed: CUDA events around that kernel's
    # launch, inside the library (the gather kernel before it is left out), averaged over
    # the steps; and the whole misa_score_rows call (gather + scoring kernel) for reference
    score_buf = torch.empty((nseq, T, wl.L), dtype=torch.float32, device=dev)

    def score_step(i):
        q, w, k, pos = sets[i % 2]
        M.misa_score_rows(q, w, k, heads, pos, scores=score_buf)

    ms_score_call = timed(score_step, args.steps, args.warmup)

    def score_kernel(i):
        q, w, k, pos = sets[i % 2]
        return M.misa_testing_score_rows_timed(q, w, k, heads, pos, scores=score_buf)

    for i in range(args.warmup):
        score_kernel(i)
    kernel_ms = [score_kernel(i) for i in range(args.steps)]
    ms_score_kernel = sum(kernel_ms) / len(kernel_ms)
    del score_buf
    M.misa_check_device_status(dev)

    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        with open(tfile) as f:
            traffic = json.load(f).get(wl.name, {}).get("score_tc_kernel")
    res = {
        "value": units * world / (ms_misa * 1e-3), "unit": UNIT, "ms_per_step": ms_misa,
        "config": {"workload": wl.name, "nseq": nseq, "T": T, "L": wl.L, "H": H, "d": d,
                   "h": wl.h, "B": wl.B, "topk": wl.topk, "kprime": wl.kprime},
        "roofline": _roofline(wl, ms_score_kernel, peaks, traffic),
        "paths": {
            "misa": {"value": units * world / (ms_misa * 1e-3), "ms_per_step": ms_misa,
                     "ms_pool": call_ms[0], "ms_route": call_ms[1], "ms_score_topk": call_ms[2],
                     "ms_score_kernel_alone": ms_score_kernel,
                     "ms_score_rows_call": ms_score_call},
            "dsa": {"value": units * world / (ms_dsa * 1e-3), "ms_per_step": ms_dsa},
            "misa_dagger": {"value": units * world / (ms_dagger * 1e-3),
                            "ms_per_step": ms_dagger},
            "speedup_misa_vs_dsa": ms_dsa / ms_misa,
            "speedup_dagger_vs_dsa": ms_dsa / ms_dagger,
            "recall_vs_dsa": recalls,
        },
        "clocks": clocks,
        "l2": "inputs > L2 (keys %.0f MB, q %.0f MB), two resident copies used alternately"
              % (x.k_bits.nbytes / 1e6, x.q_bits.nbytes / 1e6),
    }
    if not decode and wl.kprime >= int(np.mean(x.pos)) + 1:
        res["paths"]["misa_dagger"]["note"] = (
            f"k'={wl.kprime} is at least the mean causal prefix: the re-rank re-scores about "
            "every prefix token with all heads (MISA-dagger is a decode method)")
    if ms_hisa is not None:
        res["paths"]["hisa_block_filter"] = {
            "value": units * world / (ms_hisa * 1e-3), "ms_per_step": ms_hisa,
            "speedup_vs_dsa": ms_dsa / ms_hisa, "B": hisa_B, "m": hisa_m,
            "step": "pool (B=128) + head-summed block scores + top-m blocks + all-head "
                    "re-score of their tokens + top-k"}
    if ms_kept is not None:
        res["paths"]["misa_kept_pool"] = {
            "value": units * world / (ms_kept * 1e-3), "ms_per_step": ms_kept,
            "speedup_vs_dsa": ms_dsa / ms_kept,
            "step": "refresh the newest key's pooled block + route + routed score + top-k"}

    if headline:
        # end to end through the public API: pinned host inputs -> device -> MISA -> host
        idx_h = torch.empty((nseq, T, wl.topk), dtype=torch.int32).pin_memory()
        e2e_dev = [torch.empty_like(t) for t in sets[0]]

        def e2e_step(i):
            for dst, src in zip(e2e_dev, (q_h, w_h, k_h, pos_h)):
                dst.view(src.dtype).copy_(src, non_blocking=True)
            q, w, k, pos = e2e_dev
            out_idx, _, _ = M.misa_indexer(q, w, k, pos, wl.B, wl.h, wl.topk)
            idx_h.copy_(out_idx, non_blocking=True)

        ms_e2e = timed(e2e_step, max(3, args.steps // 2), 3)
        h2d = sum(t.numel() * t.element_size() for t in (q_h, w_h, k_h, pos_h))
        d2h = idx_h.numel() * idx_h.element_size()
        res["e2e"] = {"value": units * world / (ms_e2e * 1e-3), "unit": UNIT,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del sets, kp
    torch.cuda.empty_cache()
    return res, ms_misa


def run_cuda(args, wl):
    import torch
    import torch.distributed as dist
    rank, world, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=dev)
    import long_context_block_b200 as M
    peaks = _peaks()

    head, ms_misa = measure_workload(M, wl, args, dev, world, rank, peaks, headline=True)
    if args.only:
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(head))
        return 0
    extra = {}
    if args.all_configs and wl.name == DEFAULT_WORKLOAD:
        for name in EXTRA_WORKLOADS:   # the other configs of the metric, same steps
            r, _ = measure_workload(M, WORKLOADS[name], args, dev, world, rank, peaks,
                                    headline=False)
            extra[name] = r

    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_misa,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(head["config"], path="MISA: pool + route + routed score + top-k",
                       l2=head["l2"], parallelism="replicas" if world > 1 else "single"),
        "roofline": head["roofline"],
        "paths": head["paths"],
        "e2e": head["e2e"],
        "gpu_launches": misa_step_launches(wl) * args.steps,
        "clocks": head["clocks"],
    }
    if extra:
        line["configs"] = extra
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override an integer field of the workload (e.g. T=8192), for "
                         "smaller profiling runs; the JSON line names the result")
    ap.add_argument("--no-all-configs", dest="all_configs", action="store_false",
                    help="time only the headline workload (by default the 32K decode run also "
                         "times the 16K prefill, GLM-5 128K and MISA-dagger 128K workloads "
                         "and reports them under 'configs')")
    ap.add_argument("--only", choices=["misa", "dagger", "dsa", "kept", "hisa"],
                    help="run only this path's warm-up + timed steps, untimed, and print no "
                         "bench line (for profiler captures)")
    args = ap.parse_args()
    if not args.only:
        args.warmup = max(3, args.warmup)
    wl = WORKLOADS[args.workload]
    for kv in args.set:
        field, value = kv.split("=", 1)
        wl = wl.replace(**{field: int(value)})
    if args.set:
        wl = wl.replace(name=wl.name + "[" + ",".join(args.set) + "]")
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_cuda(args, wl)


if __name__ == "__main__":
    sys.exit(main())
