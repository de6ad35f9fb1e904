"""The seeded input generator: determinism, distributions and bf16 rounding."""
import numpy as np
import torch

from hybrid_mamba_ssm_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1e-40, 3.0e38, np.inf, -np.inf], np.float32)])
    bits = inputs.bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = inputs.bf16_values(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_scan_inputs_are_seeded_and_in_range():
    a = inputs.make_scan_inputs(7, [100, 28], 4, 16, 8, 2, dtype="bf16", init_state=True)
    b = inputs.make_scan_inputs(7, [100, 28], 4, 16, 8, 2, dtype="bf16", init_state=True)
    np.testing.assert_array_equal(a.x.bits, b.x.bits)
    np.testing.assert_array_equal(a.h0, b.h0)
    assert a.cu_seqlens.tolist() == [0, 100, 128]
    assert a.x.values.shape == (128, 4, 16) and a.B.values.shape == (128, 2, 8)
    assert a.dt.min() >= 1e-3 and a.dt.max() <= 0.1 and a.dt.dtype == np.float32
    assert (a.A < 0).all() and (a.A >= -16).all() and (a.A <= -1).all()
    assert a.h0.shape == (2, 4, 16, 8)
    np.testing.assert_array_equal(inputs.bf16_values(a.x.bits), a.x.values)


def test_mixed_lengths_in_range():
    lens = inputs.mixed_seqlens(inputs.workload_seed("mixed_varlen"))
    assert len(lens) == 8 and min(lens) >= 512 and max(lens) <= 16384
