"""The method's own special cases through the GPU entry points, against the
oracle (the recurrence of the deep-research note, section "1. Selective SSM
的直觉"):

* dt = 0: no input enters and nothing decays, so the state is unchanged
  (bit for bit) and y = C.h0 + D x;
* A = 0: no decay, the state is a plain cumulative sum of dt x B^T, over a
  long sequence so that it grows;
* values beyond the fp16 range of the tensor-core operands (a large carried
  state, bf16 inputs of 1e5): the CUDA-core kernels and decode stay exact in
  fp32; the tensor-core kernel writes SSM_ERR_RANGE to the status word.

Each case runs on the tensor-core shape (bf16, head_dim 64, d_state 128,
chunk 128, even heads per group) and on a CUDA-core shape.
"""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import (TOL, Guarded, dev_f32, dev_tensor, guarded_like, oracle_scan,
                               rel_err, scan_on_gpu, to_np)

pytestmark = pytest.mark.gpu

SSM_ERR_RANGE = 7

# (dtype, head_dim, d_state, chunk): the tensor-core shape, and CUDA-core ones
TC = ("bf16", 64, 128, 128)
SIMT = [("f32", 64, 128, 128), ("bf16", 32, 64, 64)]
SHAPES = [TC] + SIMT


def _inputs(seed, lens, shape, H=8, G=2):
    dtype, P, N, _ = shape
    return synth.make_scan_inputs(seed, lens, H, P, N, G, dtype=dtype, init_state=True)


def _scaled(t, k):
    return synth.store(t.values * np.float32(k), t.dtype)


@pytest.mark.parametrize("shape", SHAPES)
def test_scan_dt_zero_keeps_the_state(shape):
    inp = _inputs(101, [300, 129], shape)
    inp.dt[:] = 0.0
    y, hT = scan_on_gpu(inp, chunk=shape[3], y_dtype=torch.float32)
    np.testing.assert_array_equal(to_np(hT), inp.h0.astype(np.float64))
    y_ref, h_ref = oracle_scan(inp)
    np.testing.assert_array_equal(h_ref, inp.h0.astype(np.float64))   # the oracle agrees
    assert rel_err(to_np(y), y_ref) < TOL


@pytest.mark.parametrize("shape", SHAPES)
def test_scan_A_zero_is_a_cumulative_sum(shape):
    inp = _inputs(102, [8192 + 77], shape)
    inp.A[:] = 0.0
    y, hT = scan_on_gpu(inp, chunk=shape[3], y_dtype=torch.float32)
    y_ref, h_ref = oracle_scan(inp)
    assert np.abs(h_ref).max() > 3.0          # the sum has grown well past h0
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(hT), h_ref) < TOL
    hg = to_np(hT)
    for s in range(hg.shape[0]):
        for h in range(hg.shape[1]):
            assert rel_err(hg[s, h], h_ref[s, h]) < TOL


def _large_state_inputs(shape):
    """A = 0 and dt = 8 over 8192 tokens with x ~ N(0, 100^2): the carried
    state reaches ~1e5..1e6 (beyond fp16) while x, the decay-masked C.B^T
    entries (|C.B| dt ~ 100) and dt x (< 1e4) stay inside it."""
    inp = _inputs(103, [8192], shape)
    inp.A[:] = 0.0
    inp.dt[:] = 8.0
    inp.x = _scaled(inp.x, 100.0)
    return inp


@pytest.mark.parametrize("shape", SIMT)
def test_scan_state_beyond_fp16_range_cuda_cores(shape):
    inp = _large_state_inputs(shape)
    y, hT = scan_on_gpu(inp, chunk=shape[3], y_dtype=torch.float32)
    y_ref, h_ref = oracle_scan(inp)
    assert np.abs(h_ref).max() > 1e5
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(hT), h_ref) < TOL


def test_scan_state_beyond_fp16_range_tensor_cores_reports_range():
    inp = _large_state_inputs(TC)
    y, hT = scan_on_gpu(inp, chunk=128, y_dtype=torch.float32, expect_status=SSM_ERR_RANGE)
    # the final state comes from x, B and the decay weights only, all in range
    y_ref, h_ref = oracle_scan(inp)
    assert np.abs(h_ref).max() > 1e5
    assert rel_err(to_np(hT), h_ref) < TOL


def _huge_inputs(shape, where):
    """Some bf16 entries of x (or C) at +-1e5, beyond fp16's 65504."""
    inp = _inputs(104, [400], shape)
    t = getattr(inp, where)
    v = t.values.copy()
    flat = v.reshape(-1)
    idx = np.random.default_rng(7).choice(flat.size, 64, replace=False)
    flat[idx] = np.where(np.arange(64) % 2 == 0, 1e5, -1e5)
    setattr(inp, where, synth.store(v, t.dtype))
    return inp


@pytest.mark.parametrize("where", ["x", "C"])
def test_scan_bf16_inputs_beyond_fp16_cuda_cores(where):
    shape = ("bf16", 32, 64, 64)
    inp = _huge_inputs(shape, where)
    y, hT = scan_on_gpu(inp, chunk=64, y_dtype=torch.float32)
    y_ref, h_ref = oracle_scan(inp)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(hT), h_ref) < TOL


@pytest.mark.parametrize("where", ["x", "C"])
def test_scan_bf16_inputs_beyond_fp16_tensor_cores_report_range(where):
    inp = _huge_inputs(TC, where)
    y, hT = scan_on_gpu(inp, chunk=128, y_dtype=torch.float32, expect_status=SSM_ERR_RANGE)
    if where == "C":   # C enters only y: the final state is still valid
        _, h_ref = oracle_scan(inp)
        assert rel_err(to_np(hT), h_ref) < TOL


def _decode(inp_state, steps, A, D, dtype="bf16", H=8, P=64, N=128, G=2, batch=3, seed=0,
            dt_value=None, x_scale=None, huge_x=False):
    import oracle
    from hybrid_mamba_ssm_b200 import ssm
    st_g = guarded_like(dev_f32(inp_state))
    y_g = Guarded((batch, H, P), torch.float32)
    At, Dt = dev_f32(A), dev_f32(D)
    ref = inp_state.astype(np.float64)
    ey = 0.0
    for k in range(steps):
        s = synth.make_decode_step(seed + k, batch, H, P, N, G, dtype)
        if dt_value is not None:
            s.dt[:] = dt_value
        if x_scale is not None:
            s.x = _scaled(s.x, x_scale)
        if huge_x:
            v = s.x.values.copy()
            v.reshape(-1)[::97] = 1e5
            s.x = synth.store(v, s.x.dtype)
        ssm.ssm_state_update(st_g.t, dev_tensor(s.x), dev_f32(s.dt), At, dev_tensor(s.B),
                             dev_tensor(s.C), Dt, y=y_g.t)
        yr, ref = oracle.state_update(ref, s.x.values, s.dt, A, s.B.values, s.C.values, D)
        torch.cuda.synchronize()
        ey = max(ey, rel_err(to_np(y_g.t), yr))
    st_g.check("state")
    y_g.check("y")
    return to_np(st_g.t), ref, ey


def test_decode_dt_zero_keeps_the_state():
    A, D = synth.make_head_params(201, 8)
    h0 = synth.make_state(202, (3, 8, 64, 128))
    got, ref, ey = _decode(h0, 3, A, D, seed=203, dt_value=0.0)
    np.testing.assert_array_equal(got, h0.astype(np.float64))
    assert ey < TOL


def test_decode_A_zero_is_a_cumulative_sum():
    A, D = synth.make_head_params(211, 8)
    A[:] = 0.0
    h0 = synth.make_state(212, (3, 8, 64, 128))
    got, ref, ey = _decode(h0, 64, A, D, seed=213)
    assert rel_err(got, ref) < TOL and ey < TOL


def test_decode_state_and_inputs_beyond_fp16_range():
    """Decode computes in fp32 throughout: a state of ~1e6 and bf16 inputs of
    1e5 are exact to fp32 rounding."""
    A, D = synth.make_head_params(221, 8)
    A[:] = 0.0
    h0 = (synth.make_state(222, (3, 8, 64, 128)) * np.float32(1e7)).astype(np.float32)
    got, ref, ey = _decode(h0, 8, A, D, seed=223, dt_value=8.0, x_scale=100.0, huge_x=True)
    assert np.abs(ref).max() > 1e5
    assert rel_err(got, ref) < TOL and ey < TOL
