"""The seeded input recipe (CPU): shapes, outlier channels, factor and logit ranges,
determinism, and the bf16 packing both sides read."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import workloads as wl


@pytest.mark.parametrize("name", wl.ORDER)
def test_recipe(name):
    w = wl.WORKLOADS[name]
    M, N = min(w.M, 256), min(w.N, 64)
    inp = wl.make_inputs(name, seed=0, M=M, N=N)
    assert inp.X.shape == (M, w.K) and inp.X.dtype == np.uint16
    assert inp.W.shape == (N, w.K) and inp.W.dtype == np.uint16
    assert inp.A.shape == (8, 8) and inp.B.shape == (w.nb, 4, 4)
    assert inp.g_lo.shape == inp.g_hi.shape == (w.nb,)
    # outlier channels: the stated fraction of K, distinct, scaled within the stated range
    n_out = max(1, int(round(w.outlier_frac * w.K)))
    ch = inp.outlier_channels
    assert len(ch) == n_out == len(np.unique(ch))
    x = wl.bf16_bits_to_f32(inp.X)
    rest = np.setdiff1d(np.arange(w.K), ch)
    base = np.abs(x[:, rest]).mean()
    ratio = np.abs(x[:, ch]).mean(axis=0) / base
    assert ratio.min() > 0.5 * w.outlier_lo and ratio.max() < 2.0 * w.outlier_hi
    # factors near identity with 0.1 spread, logits in [1, 4], weights at 0.02
    assert abs((inp.A - np.eye(8)).std() - 0.1) < 0.04
    assert abs((inp.B - np.eye(4)[None]).std() - 0.1) < 0.03
    assert inp.g_lo.min() >= 1.0 and inp.g_hi.max() <= 4.0
    assert abs(wl.bf16_bits_to_f32(inp.W).std() - 0.02) < 0.002


def test_deterministic_and_seeded():
    a = wl.make_inputs("tiny", seed=3)
    b = wl.make_inputs("tiny", seed=3)
    c = wl.make_inputs("tiny", seed=4)
    assert np.array_equal(a.X, b.X) and np.array_equal(a.W, b.W) and np.array_equal(a.B, b.B)
    assert not np.array_equal(a.X, c.X)
    # X is drawn first: the activations do not depend on how many weight rows follow
    d = wl.make_inputs("tiny", seed=3, N=7)
    assert np.array_equal(a.X, d.X)


def test_bf16_packing_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 100000),
        # exact ties between two bf16 values: round to the even mantissa
        (np.arange(1, 2001, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.5, 3.0e38, -3.0e38, 1e-40], dtype=np.float32),
    ]).astype(np.float32)
    ours = wl.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = wl.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(v).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("s", [1, 2, 4, 8, 16, 32])
def test_random_factors_shapes_and_spread(s):
    t = 32 // s
    A, B, g_lo, g_hi = wl.random_factors(5, seed=1, shared=s)
    assert A.shape == (s, s) and B.shape == (5, t, t)
    if s >= 4:
        assert abs((A - np.eye(s)).std() - 0.1 * min(1.0, np.sqrt(8.0 / s))) < 0.05
    assert np.all((g_lo >= 1.0) & (g_lo <= 4.0)) and np.all((g_hi >= 1.0) & (g_hi <= 4.0))
