"""The seeded input generator: determinism, shapes, bf16 rounding and the planted
needle geometry (CPU only)."""

import numpy as np
import torch

from synth import WORKLOADS, fp32_to_bf16_bits, make_inputs, sample_rows


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 1e-30],
                                 dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(fp32_to_bf16_bits(x), ref)


def test_generator_deterministic_and_shaped():
    wl = WORKLOADS["tiny_2k"]
    a = make_inputs(wl, seed=0)
    b = make_inputs(wl, seed=0)
    c = make_inputs(wl, seed=1)
    assert a.q_bits.shape == (1, 16, 64, 128) and a.k_bits.shape == (1, 2048, 128)
    assert a.w.shape == (1, 16, 64) and a.pos.shape == (1, 16)
    assert list(a.pos[0]) == list(range(2032, 2048))
    assert np.array_equal(a.q_bits, b.q_bits) and np.array_equal(a.k_bits, b.k_bits)
    assert not np.array_equal(a.k_bits, c.k_bits)
    assert wl.query_prefix_tokens() == sum(range(2033, 2049))


def test_needles_have_cosine_point_eight():
    wl = WORKLOADS["dsv32_decode_32k"].replace(nseq=2, L=4096)
    x = make_inputs(wl, seed=0)
    q = (x.q_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    k = (x.k_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for n in range(2):
        for s in x.needle_pos[n]:
            ks = k[n, s] / np.linalg.norm(k[n, s])
            qh = q[n, 0] / np.linalg.norm(q[n, 0], axis=1, keepdims=True)
            assert abs(np.max(qh @ ks) - 0.8) < 0.01


def test_sample_rows():
    assert len(sample_rows(WORKLOADS["dsv32_prefill_16k"])) == 256
    assert list(sample_rows(WORKLOADS["glm5_decode_128k"])) == list(range(8))
    r1 = sample_rows(WORKLOADS["dsv32_prefill_16k"], seed=0)
    r2 = sample_rows(WORKLOADS["dsv32_prefill_16k"], seed=0)
    assert np.array_equal(r1, r2) and np.all(np.diff(r1) > 0)
