"""Pins of the oracle's dt transform and gated group RMSNorm against library
routines (torch's softplus, silu and rms_norm on the CPU, in fp64) and
closed forms (softplus(0) = ln 2, the clamp, unit RMS, scale invariance)."""
import math

import numpy as np
import pytest
import torch

import oracle


def test_softplus_closed_forms_and_library():
    v = np.array([-50.0, -3.0, 0.0, 0.5, 3.0, 30.0])
    got = oracle.dt_transform(v, softplus=True)
    assert got[2] == pytest.approx(math.log(2.0), rel=1e-15)
    assert got[0] == pytest.approx(math.exp(-50.0), rel=1e-12)       # e^v for v << 0
    assert got[-1] == pytest.approx(30.0, rel=1e-12)                  # v for v >> 0
    ref = torch.nn.functional.softplus(torch.from_numpy(v), threshold=1000.0).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-14)


def test_bias_per_head_then_clamp():
    rng = np.random.default_rng(1)
    dt = rng.standard_normal((7, 5))
    bias = rng.standard_normal(5)
    got = oracle.dt_transform(dt, bias, softplus=True, dt_min=0.2, dt_max=0.9)
    ref = np.clip(np.log1p(np.exp(dt + bias[None, :])), 0.2, 0.9)
    np.testing.assert_allclose(got, ref, rtol=1e-14)
    assert got.min() >= 0.2 and got.max() <= 0.9
    np.testing.assert_array_equal(oracle.dt_transform(dt), dt)       # identity by default


def test_gated_rmsnorm_matches_torch_rms_norm():
    rng = np.random.default_rng(2)
    rows, G, gs = 6, 4, 16
    y = rng.standard_normal((rows, G * gs))
    z = rng.standard_normal((rows, G * gs))
    w = rng.standard_normal(G * gs)
    got = oracle.gated_rmsnorm(y, z, w, gs, eps=1e-5)
    g = torch.from_numpy(y) * torch.nn.functional.silu(torch.from_numpy(z))
    ref = torch.nn.functional.rms_norm(g.view(rows, G, gs), (gs,), eps=1e-5).reshape(rows, -1)
    np.testing.assert_allclose(got, (ref * torch.from_numpy(w)).numpy(), rtol=1e-12, atol=1e-12)


def test_gated_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(3)
    y = rng.standard_normal((3, 32))
    z = rng.standard_normal((3, 32))
    out = oracle.gated_rmsnorm(y, z, np.ones(32), 8, eps=0.0)
    ms = np.mean(out.reshape(3, 4, 8) ** 2, axis=-1)
    np.testing.assert_allclose(ms, 1.0, rtol=1e-13)
    out2 = oracle.gated_rmsnorm(5.0 * y, z, np.ones(32), 8, eps=0.0)
    np.testing.assert_allclose(out2, out, rtol=1e-13)
