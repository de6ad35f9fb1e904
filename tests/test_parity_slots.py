"""Slot-indexed state pools on the GPU against the fp64 oracle: prefill and
decode read and write pool rows in place; rows not named are left bit for
bit; has_initial_state = 0 starts from zero; padding and invalid slots."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, dev_f32, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,P,N,G,chunk", [("bf16", 64, 128, 2, 128),   # tensor-core kernel
                                               ("f32", 32, 64, 2, 64)])     # CUDA-core kernel
def test_scan_slots_against_oracle(dtype, P, N, G, chunk):
    from hybrid_mamba_ssm_b200 import ssm
    lens = [300, 0, 129, 64]
    H, max_slots = 8, 7
    inp = synth.make_scan_inputs(31, lens, H, P, N, G, dtype=dtype)
    pool0 = synth.make_state(32, (max_slots, H, P, N))
    slots = np.array([5, 2, 0, 6], dtype=np.int32)
    has = np.array([1, 0, 1, 0], dtype=np.int32)
    pool = dev_f32(pool0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = ssm.ssd_chunk_scan_slots(dev_tensor(inp.x), dev_f32(inp.dt), dev_f32(inp.A),
                                 dev_tensor(inp.B), dev_tensor(inp.C), dev_f32(inp.D), pool,
                                 torch.from_numpy(slots).cuda(), torch.from_numpy(has).cuda(),
                                 cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda(),
                                 chunk_size=chunk, y_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    y_ref, pool_ref = oracle.scan_slots(pool0, slots, has, inp.x.values, inp.dt, inp.A,
                                        inp.B.values, inp.C.values, inp.D,
                                        cu_seqlens=inp.cu_seqlens)
    got = to_np(pool)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(got[slots], pool_ref[slots]) < TOL
    untouched = [r for r in range(max_slots) if r not in slots]
    np.testing.assert_array_equal(got[untouched], pool0[untouched].astype(np.float64))
    np.testing.assert_array_equal(got[2], 0.0)   # empty sequence without initial state


def test_decode_slots_against_oracle():
    from hybrid_mamba_ssm_b200 import ssm
    H, P, N, G, max_slots = 16, 64, 128, 4, 9
    slots = np.array([4, -1, 8, 0, -1, 3], dtype=np.int32)
    batch = slots.shape[0]
    A, D = synth.make_head_params(41, H)
    pool0 = synth.make_state(42, (max_slots, H, P, N))
    pool = dev_f32(pool0)
    ref = pool0.astype(np.float64)
    sl = torch.from_numpy(slots).cuda()
    for k in range(3):
        st = synth.make_decode_step(43 + k, batch, H, P, N, G)
        y = torch.full((batch, H, P), 7.0, device="cuda")
        ssm.ssm_state_update_slots(pool, sl, dev_tensor(st.x), dev_f32(st.dt), dev_f32(A),
                                   dev_tensor(st.B), dev_tensor(st.C), dev_f32(D), y=y)
        y_ref, ref = oracle.state_update_slots(ref, slots, st.x.values, st.dt, A, st.B.values,
                                               st.C.values, D)
        live = slots >= 0
        assert rel_err(to_np(y)[live], y_ref[live]) < TOL
        assert (to_np(y)[~live] == 7.0).all()          # padding rows untouched
    torch.cuda.synchronize()
    got = to_np(pool)
    assert rel_err(got, ref) < TOL
    untouched = [r for r in range(max_slots) if r not in slots]
    np.testing.assert_array_equal(got[untouched], pool0[untouched].astype(np.float64))


def test_slot_out_of_range_reported_and_skipped():
    from hybrid_mamba_ssm_b200 import ssm
    H, P, N, G = 4, 64, 128, 2
    inp = synth.make_scan_inputs(51, [128, 128], H, P, N, G, dtype="bf16")
    pool0 = synth.make_state(52, (3, H, P, N))
    pool = dev_f32(pool0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    n, L = 2, 128
    ssm.ssd_chunk_scan_slots(dev_tensor(inp.x).view(n, L, H, P), dev_f32(inp.dt).view(n, L, H),
                             dev_f32(inp.A), dev_tensor(inp.B).view(n, L, G, N),
                             dev_tensor(inp.C).view(n, L, G, N), dev_f32(inp.D), pool,
                             torch.tensor([1, 3], dtype=torch.int32, device="cuda"),
                             status=status)
    torch.cuda.synchronize()
    assert status.item() == 6
    got = to_np(pool)
    np.testing.assert_array_equal(got[[0, 2]], pool0[[0, 2]].astype(np.float64))
    assert not np.array_equal(got[1], pool0[1])   # the valid sequence was processed
