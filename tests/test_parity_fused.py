"""The fused steps on either side of the scan, on the GPU against the fp64
oracle: the dt transform (bias, softplus, clamp) applied inside the prefill
(tensor-core and CUDA-core kernels), decode and speculative-decode kernels,
and the gated group RMSNorm."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, dev_f32, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu

LIMIT = (1e-3, 0.1)


@pytest.mark.parametrize("dtype,P,N,G,chunk", [("bf16", 64, 128, 2, 128), ("f32", 32, 64, 2, 64)])
def test_scan_with_raw_dt(dtype, P, N, G, chunk):
    from hybrid_mamba_ssm_b200 import ssm
    lens, H = [300, 77], 8
    inp = synth.make_scan_inputs(301, lens, H, P, N, G, dtype=dtype, init_state=True)
    raw, bias = synth.make_raw_dt(302, (sum(lens), H), H)
    pool = dev_f32(inp.h0)
    y = ssm.ssd_chunk_scan_slots(dev_tensor(inp.x), dev_f32(raw), dev_f32(inp.A),
                                 dev_tensor(inp.B), dev_tensor(inp.C), dev_f32(inp.D), pool, None,
                                 cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda(),
                                 chunk_size=chunk, y_dtype=torch.float32,
                                 dt_bias=dev_f32(bias), dt_softplus=True, dt_limit=LIMIT)
    torch.cuda.synchronize()
    dt = oracle.dt_transform(raw, bias, softplus=True, dt_min=LIMIT[0], dt_max=LIMIT[1])
    y_ref, h_ref = oracle.scan(inp.x.values, dt, inp.A, inp.B.values, inp.C.values, inp.D,
                               inp.h0, cu_seqlens=inp.cu_seqlens)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(pool), h_ref) < TOL


def test_decode_with_raw_dt_softplus_only():
    from hybrid_mamba_ssm_b200 import ssm
    batch, H, P, N, G = 6, 16, 64, 128, 4
    A, D = synth.make_head_params(311, H)
    st0 = synth.make_state(312, (batch, H, P, N))
    step = synth.make_decode_step(313, batch, H, P, N, G)
    raw, bias = synth.make_raw_dt(314, (batch, H), H)
    state = dev_f32(st0)
    y = ssm.ssm_state_update_slots(state, None, dev_tensor(step.x), dev_f32(raw), dev_f32(A),
                                   dev_tensor(step.B), dev_tensor(step.C), dev_f32(D),
                                   y_dtype=torch.float32, dt_bias=dev_f32(bias), dt_softplus=True)
    torch.cuda.synchronize()
    dt = oracle.dt_transform(raw, bias, softplus=True)
    y_ref, s_ref = oracle.state_update(st0, step.x.values, dt, A, step.B.values, step.C.values, D)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(state), s_ref) < TOL


def test_multi_with_raw_dt():
    from hybrid_mamba_ssm_b200 import ssm
    batch, ntok, H, P, N, G = 3, 4, 8, 64, 128, 2
    A, D = synth.make_head_params(321, H)
    st0 = synth.make_state(322, (batch, H, P, N))
    steps = [synth.make_decode_step(323 + k, batch, H, P, N, G) for k in range(ntok)]
    raw, bias = synth.make_raw_dt(330, (batch, ntok, H), H)
    stk = lambda f: torch.stack([dev_tensor(f(s)) for s in steps], dim=1).contiguous()
    npk = lambda f: np.stack([f(s) for s in steps], axis=1)
    state = dev_f32(st0)
    acc = np.array([4, 0, 2], dtype=np.int32)
    y, _ = ssm.ssm_state_update_multi(state, stk(lambda s: s.x), dev_f32(raw), dev_f32(A),
                                      stk(lambda s: s.B), stk(lambda s: s.C), dev_f32(D),
                                      accept_len=torch.from_numpy(acc).cuda(),
                                      y_dtype=torch.float32, dt_bias=dev_f32(bias),
                                      dt_softplus=True, dt_limit=LIMIT)
    torch.cuda.synchronize()
    dt = oracle.dt_transform(raw, bias, softplus=True, dt_min=LIMIT[0], dt_max=LIMIT[1])
    y_ref, _, new_ref = oracle.state_update_multi(st0, npk(lambda s: s.x.values), dt, A,
                                                  npk(lambda s: s.B.values),
                                                  npk(lambda s: s.C.values), D, accept_len=acc)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(state), new_ref) < TOL


@pytest.mark.parametrize("dtype,out,gs", [("bf16", "bf16", 1024), ("bf16", "f32", 2048),
                                          ("f32", "f32", 256), ("bf16", "bf16", 8192)])
def test_gated_rmsnorm(dtype, out, gs):
    from hybrid_mamba_ssm_b200 import ssm
    rows, dim = 37, 8192
    y, z, w = synth.make_gate(341, rows, dim, dtype)
    got = ssm.ssm_gated_rmsnorm(dev_tensor(y), dev_tensor(z), dev_f32(w), gs, eps=1e-5,
                                out_dtype=torch.bfloat16 if out == "bf16" else torch.float32)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(y.values, z.values, w, gs, eps=1e-5)
    assert rel_err(to_np(got), ref, bf16=(out == "bf16")) < 1e-5


def test_gated_rmsnorm_in_place_full_rows():
    """In place on y at the prefill shape (16384 x 8192, groups of 1024);
    sampled rows against the oracle."""
    from hybrid_mamba_ssm_b200 import ssm
    rows, dim, gs = 16384, 8192, 1024
    y, z, w = synth.make_gate(351, rows, dim, "bf16")
    yd = dev_tensor(y)
    ssm.ssm_gated_rmsnorm(yd, dev_tensor(z), dev_f32(w), gs, eps=1e-5, out=yd)
    torch.cuda.synchronize()
    pick = np.random.default_rng(352).choice(rows, 64, replace=False)
    ref = oracle.gated_rmsnorm(y.values[pick], z.values[pick], w, gs, eps=1e-5)
    assert rel_err(to_np(yd[torch.from_numpy(pick).cuda()]), ref, bf16=True) < 1e-5
