"""Seeded input generator: rounding, prefix property and value ranges (no GPU)."""
import numpy as np
import torch

from selective_state_space_10_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0], np.float32)])
    bits, vals = inputs.round_to_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16)
    assert np.array_equal(bits, ref.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vals, ref.float().numpy())


def test_prefix_property():
    long = inputs.sequence(2, 50, 3, 4, 8, 1, "bf16", seed=7)
    short = inputs.sequence(2, 30, 3, 4, 8, 1, "bf16", seed=7)
    s = long.token_slice(0, 30)
    for k in ("x", "dt", "B", "C"):
        assert np.array_equal(getattr(s, k), getattr(short, k)), k
    assert np.array_equal(s.bits["x"], short.bits["x"])


def test_value_ranges():
    w = inputs.BY_NAME["mamba2_130m_prefill"]
    s = inputs.workload_sequence(w, seqlen=512)
    assert s.x.shape == (1, 512, 24, 64) and s.B.shape == (1, 512, 1, 128)
    assert s.dt.min() >= 1e-3 - 1e-9 and s.dt.max() <= 0.1 + 1e-9
    assert (s.A < 0).all() and s.A.min() >= -16.0 - 1e-4 and s.A.max() <= -1.0 + 1e-6
    assert abs(s.x.std() - 1.0) < 0.02
    assert abs(s.B.std() * np.sqrt(128) - 1.0) < 0.05
    for k in ("x", "B", "C"):
        assert s.bits[k].dtype == np.uint16


def test_decode_tokens_differ_per_step():
    w = inputs.BY_NAME["mamba2_2.7b_decode_b256"]
    from dataclasses import replace
    w = replace(w, batch=2)
    t0, t1 = inputs.decode_token(w, 0), inputs.decode_token(w, 1)
    assert t0.x.shape == (2, 1, 80, 64)
    assert not np.array_equal(t0.x, t1.x)
    assert np.array_equal(t0.A, t1.A) and np.array_equal(t0.D, t1.D)
