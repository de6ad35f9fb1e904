"""Decode (ssm_state_update) against the fp64 oracle, element by element."""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, Guarded, dev_f32, dev_tensor, guarded_like, rel_err, to_np

pytestmark = pytest.mark.gpu


def run_steps(batch, H, P, N, G, dtype, y_dtype, steps, seed, use_D=True, sample=None):
    import oracle
    from hybrid_mamba_ssm_b200 import ssm
    A, D = synth.make_head_params(seed, H)
    state0 = synth.make_state(seed + 1, (batch, H, P, N))
    st_g = guarded_like(dev_f32(state0))
    st_gpu = st_g.t
    At, Dt = dev_f32(A), (dev_f32(D) if use_D else None)
    y_g = Guarded((batch, H, P), y_dtype)
    ref = state0.astype(np.float64)
    bs = slice(None) if sample is None else sample
    worst_y = worst_s = 0.0
    for k in range(steps):
        inp = synth.make_decode_step(seed + 100 + k, batch, H, P, N, G, dtype)
        y = ssm.ssm_state_update(st_gpu, dev_tensor(inp.x), dev_f32(inp.dt), At,
                                 dev_tensor(inp.B), dev_tensor(inp.C), Dt, y=y_g.t)
        y_ref, ref_new = oracle.state_update(ref[bs], inp.x.values[bs], inp.dt[bs], A,
                                             inp.B.values[bs], inp.C.values[bs],
                                             D if use_D else None)
        ref = ref_new if sample is None else _put(ref, bs, ref_new)
        worst_y = max(worst_y, rel_err(to_np(y)[bs], y_ref, bf16=y_dtype == torch.bfloat16))
    torch.cuda.synchronize()
    st_g.check("state")
    y_g.check("y")
    worst_s = rel_err(to_np(st_gpu)[bs], ref[bs])
    return worst_y, worst_s


def _put(full, bs, part):
    full = full.copy()
    full[bs] = part
    return full


@pytest.mark.parametrize("batch,H,P,N,G", [
    (1, 1, 1, 16, 1), (3, 4, 16, 16, 1), (2, 4, 64, 128, 2), (5, 6, 33, 32, 3),
    (2, 8, 100, 64, 4), (1, 2, 256, 256, 1), (4, 16, 64, 128, 8)])
@pytest.mark.parametrize("dtype,y_dtype", [("bf16", torch.float32), ("f32", torch.float32),
                                           ("bf16", torch.bfloat16)])
def test_decode_small_shapes(batch, H, P, N, G, dtype, y_dtype):
    wy, ws = run_steps(batch, H, P, N, G, dtype, y_dtype, steps=4, seed=batch * 7 + P)
    assert ws < TOL, ws
    assert wy < TOL, wy


def test_decode_without_D():
    wy, ws = run_steps(2, 4, 64, 128, 2, "bf16", torch.float32, steps=3, seed=5, use_D=False)
    assert ws < TOL and wy < TOL


def test_decode_ultra_shape_sampled():
    """The timed decode launch (batch 64, 256 heads, 64 x 128 state, 8 groups)
    for 20 consecutive steps; the oracle follows 6 batch rows of all heads."""
    wy, ws = run_steps(64, 256, 64, 128, 8, "bf16", torch.float32, steps=20,
                       seed=synth.workload_seed("decode_ultra"), sample=[0, 1, 17, 32, 50, 63])
    assert ws < TOL, ws
    assert wy < TOL, wy
