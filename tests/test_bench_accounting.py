"""The roofline accounting of bench.py against the figures derived by hand from the workload
shapes: algorithmic bytes of the decode scorer, flops of the prefill scorer, the number of
query x prefix-token units, and which form (and so which bound) each workload takes."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import WORKLOADS  # noqa: E402


def test_decode_32k_bytes():
    wl = WORKLOADS["dsv32_decode_32k"]
    # 32 rows x 32768 prefix keys x (256 B of key + 4 B of score) + 32 x 8 x (256 + 4 + 4)
    expect = 32 * 32768 * (256 + 4) + 32 * 8 * 264
    assert bench.algorithmic_bytes_score(wl) == expect
    assert abs(expect / 1e6 - 272.70) < 0.01
    assert wl.query_prefix_tokens() == 32 * 32768


def test_prefill_16k_flops_and_units():
    wl = WORKLOADS["dsv32_prefill_16k"]
    pairs = 16384 * 16385 // 2   # causal pairs: sum over t of (t + 1)
    assert wl.query_prefix_tokens() == pairs
    assert bench.algorithmic_flops_score(wl) == 2.0 * 8 * 128 * pairs
    assert abs(bench.algorithmic_flops_score(wl) / 1e9 - 274.9) < 0.1
    # keys of the one sequence are read once for all its queries
    assert bench.algorithmic_bytes_score(wl) == 16384 * 256 + 16384 * 8 * 264 + 4.0 * pairs


def test_bound_follows_arithmetic_intensity():
    peaks = {"hbm": 6557.4, "bf16": 1629.0}
    for name, bound in (("dsv32_decode_32k", "hbm"), ("glm5_decode_128k", "hbm"),
                        ("dsv32_mtp_32k", "hbm"), ("dsv32_draft16_32k", "hbm"),
                        ("dsv32_prefill_16k", "tensor")):
        wl = WORKLOADS[name]
        t_flops = bench.algorithmic_flops_score(wl) / (peaks["bf16"] * 1e12)
        t_bytes = bench.algorithmic_bytes_score(wl) / (peaks["hbm"] * 1e9)
        assert ("tensor" if t_flops > t_bytes else "hbm") == bound, name


def test_forms_and_launch_counts():
    assert not bench.block_form(WORKLOADS["dsv32_decode_32k"])
    assert bench.block_form(WORKLOADS["dsv32_mtp_32k"])
    # decode 32K: pool, router, scorer prep + scorer, one row top-k
    assert bench.misa_step_launches(WORKLOADS["dsv32_decode_32k"]) == 5
    # 128K decode rows exceed the row top-k's 40960: scatter + group
    assert bench.misa_step_launches(WORKLOADS["glm5_decode_128k"]) == 6
    # 4 queries per sequence over 32K: histogram pass + row top-k
    assert bench.misa_step_launches(WORKLOADS["dsv32_mtp_32k"]) == 6
    # prefill: three tensor-core router kernels (hi/lo split, partial blocks, GEMM + top-h)
    assert bench.misa_step_launches(WORKLOADS["dsv32_prefill_16k"]) == 7


def test_roofline_object_from_a_kernel_time():
    # 32K decode: HBM-bound; achieved = algorithmic bytes / kernel time, frac against the
    # measured copy peak; the traffic figure passes through unchanged
    peaks = {"hbm": 6557.4, "bf16": 1629.0, "source": "measured"}
    wl = WORKLOADS["dsv32_decode_32k"]
    r = bench._roofline(wl, 0.0544, peaks, 274656768)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 274656768
    assert abs(r["achieved"] - bench.algorithmic_bytes_score(wl) / 0.0544e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6557.4) < 1e-12 and 0.7 < r["frac"] < 0.8
    # 16K prefill: tensor-bound against the bf16 burst peak
    wl = WORKLOADS["dsv32_prefill_16k"]
    r = bench._roofline(wl, 0.3057, peaks, None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] is None
    assert abs(r["achieved"] - bench.algorithmic_flops_score(wl) / 0.3057e-3 / 1e12) < 1e-6
    assert 0.5 < r["frac"] < 0.6
