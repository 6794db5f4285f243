"""CUDA path against the fp64 oracle on the five seeded workloads (GPU).

Every entry point runs through the C ABI at the workload's full size, in the same
launch configuration the benchmark times.  The oracle checks every row of the tiny
and 32K-decode workloads and a seeded sample of 256 query rows of the others (all
rows where there are fewer)."""

import json
import os

import numpy as np
import pytest
import torch

from synth import WORKLOADS, make_inputs, sample_rows
from tests import gpu_path

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import long_context_block_b200 as M
    return M


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_parity(M, name):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0)
    q, w, k, pos = gpu_path.to_device(x)
    out = gpu_path.run_all(M, q, w, k, pos, wl.B, wl.h, wl.topk, wl.kprime)
    rows = sample_rows(wl, 256, seed=0)
    host = gpu_path.rows_to_host(out, rows, wl.T)
    del out
    stats = gpu_path.check_rows(x, host, rows, wl.B, wl.h, wl.topk, wl.kprime)
    out_dir = os.environ.get("MISA_TEST_LOG_DIR")   # keep the statistics there if set
    if out_dir:
        os.makedirs(out_dir, exist_ok=True)
        with open(os.path.join(out_dir, f"parity_{name}.json"), "w") as f:
            json.dump(stats, f)
    print(name, stats)
