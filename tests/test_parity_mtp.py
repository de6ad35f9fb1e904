"""Speculative (multi-token) decode on the GPU against the fp64 oracle: draft
outputs, intermediate states, both commit flows (scatter of an intermediate
state, and an in-place replay with accept_len), slot pools with padding, bad
accept lengths, and the conv1d window over draft tokens."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, dev_f32, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu


def _draft(seed, batch, ntok, H, P, N, G, dtype="bf16"):
    """ntok decode-step input sets stacked along a token axis."""
    steps = [synth.make_decode_step(seed + k, batch, H, P, N, G, dtype) for k in range(ntok)]
    stack = lambda f: np.stack([f(s) for s in steps], axis=1)
    x = stack(lambda s: s.x.values)
    dt = stack(lambda s: s.dt)
    B = stack(lambda s: s.B.values)
    C = stack(lambda s: s.C.values)
    if dtype == "bf16":
        dev = lambda f: torch.stack([dev_tensor(f(s)) for s in steps], dim=1).contiguous()
        xd, Bd, Cd = dev(lambda s: s.x), dev(lambda s: s.B), dev(lambda s: s.C)
    else:
        xd, Bd, Cd = dev_f32(x), dev_f32(B), dev_f32(C)
    return (x, dt, B, C), (xd, dev_f32(dt), Bd, Cd)


@pytest.mark.parametrize("dtype,P,N,G", [("bf16", 64, 128, 4), ("f32", 32, 64, 2)])
def test_verify_then_scatter_commit(dtype, P, N, G):
    from hybrid_mamba_ssm_b200 import ssm
    batch, ntok, H = 5, 4, 8
    A, D = synth.make_head_params(201, H)
    st0 = synth.make_state(202, (batch, H, P, N))
    (x, dt, B, C), (xd, dtd, Bd, Cd) = _draft(210, batch, ntok, H, P, N, G, dtype)
    state = dev_f32(st0)
    y, inter = ssm.ssm_state_update_multi(state, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D),
                                          y_dtype=torch.float32, want_inter=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(state), st0)      # verify only reads the state
    acc = np.array([0, 1, 2, 4, 3], dtype=np.int32)
    y_ref, inter_ref, new_ref = oracle.state_update_multi(st0, x, dt, A, B, C, D, accept_len=acc)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(inter), inter_ref) < TOL
    ssm.ssm_state_commit(inter, torch.from_numpy(acc).cuda(), state)
    torch.cuda.synchronize()
    got = to_np(state)
    assert rel_err(got, new_ref) < TOL
    np.testing.assert_array_equal(got[0], st0[0])         # nothing accepted
    np.testing.assert_array_equal(got[3], to_np(inter)[3, 3])


def test_replay_commit_in_place():
    """Verify without intermediates, then replay the draft with accept_len."""
    from hybrid_mamba_ssm_b200 import ssm
    batch, ntok, H, P, N, G = 6, 3, 16, 64, 128, 8
    A, D = synth.make_head_params(221, H)
    st0 = synth.make_state(222, (batch, H, P, N))
    (x, dt, B, C), (xd, dtd, Bd, Cd) = _draft(230, batch, ntok, H, P, N, G)
    state = dev_f32(st0)
    y, _ = ssm.ssm_state_update_multi(state, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D))
    acc = np.array([3, 0, 1, 2, 3, 1], dtype=np.int32)
    out, _ = ssm.ssm_state_update_multi(state, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D),
                                        accept_len=torch.from_numpy(acc).cuda(), want_y=False)
    torch.cuda.synchronize()
    assert out is None
    y_ref, _, new_ref = oracle.state_update_multi(st0, x, dt, A, B, C, D, accept_len=acc)
    assert rel_err(to_np(y), y_ref, bf16=True) < TOL
    got = to_np(state)
    assert rel_err(got, new_ref) < TOL
    np.testing.assert_array_equal(got[1], st0[1])


def test_multi_one_token_equals_decode_step():
    from hybrid_mamba_ssm_b200 import ssm
    batch, H, P, N, G = 4, 8, 64, 128, 2
    A, D = synth.make_head_params(241, H)
    st0 = synth.make_state(242, (batch, H, P, N))
    (_, _, _, _), (xd, dtd, Bd, Cd) = _draft(243, batch, 1, H, P, N, G)
    s1, s2 = dev_f32(st0), dev_f32(st0)
    y1 = ssm.ssm_state_update(s1, xd[:, 0].contiguous(), dtd[:, 0].contiguous(), dev_f32(A),
                              Bd[:, 0].contiguous(), Cd[:, 0].contiguous(), dev_f32(D),
                              y_dtype=torch.float32)
    y2, _ = ssm.ssm_state_update_multi(s2, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D),
                                       accept_len=torch.ones(batch, dtype=torch.int32,
                                                             device="cuda"),
                                       y_dtype=torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(y2)[:, 0], to_np(y1), rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(to_np(s2), to_np(s1), rtol=1e-6, atol=1e-6)


def test_multi_slots_padding_and_bad_accept():
    from hybrid_mamba_ssm_b200 import ssm
    H, P, N, G, ntok, max_slots = 8, 64, 128, 2, 3, 7
    slots = np.array([5, -1, 0, 2], dtype=np.int32)
    acc = np.array([2, 1, 9, 3], dtype=np.int32)           # row 2: beyond ntok
    batch = slots.shape[0]
    A, D = synth.make_head_params(251, H)
    pool0 = synth.make_state(252, (max_slots, H, P, N))
    (x, dt, B, C), (xd, dtd, Bd, Cd) = _draft(260, batch, ntok, H, P, N, G)
    pool = dev_f32(pool0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((batch, ntok, H, P), 7.0, device="cuda")
    ssm.ssm_state_update_multi(pool, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D),
                               slot_idx=torch.from_numpy(slots).cuda(),
                               accept_len=torch.from_numpy(acc).cuda(), y=y, status=status)
    torch.cuda.synchronize()
    assert status.item() == 6
    got, yn = to_np(pool), to_np(y)
    for b in (0, 3):
        y_ref, _, new_ref = oracle.state_update_multi(
            pool0[slots[b]][None], x[b:b + 1], dt[b:b + 1], A, B[b:b + 1], C[b:b + 1], D,
            accept_len=acc[b:b + 1])
        assert rel_err(yn[b], y_ref[0]) < TOL
        assert rel_err(got[slots[b]], new_ref[0]) < TOL
    assert (yn[1] == 7.0).all() and (yn[2] == 7.0).all()   # padding row, rejected row
    np.testing.assert_array_equal(got[[0, 1, 3, 4, 6]], pool0[[0, 1, 3, 4, 6]])


@pytest.mark.parametrize("dim", [640, 102])
def test_conv_multi_verify_and_commit(dim):
    from hybrid_mamba_ssm_b200 import ssm
    batch, ntok, width = 4, 5, 4
    w = synth.make_conv_inputs(271, [1], dim, width, "bf16")
    st0 = synth.make_conv_inputs(272, [1] * batch, dim, width, "bf16").state
    xs = synth.make_conv_inputs(273, [batch * ntok], dim, width, "bf16").x
    xv = xs.values.reshape(batch, ntok, dim)
    xd = dev_tensor(xs).view(batch, ntok, dim)
    state = dev_tensor(st0)
    y = ssm.causal_conv1d_update_multi(xd, dev_f32(w.weight), dev_f32(w.bias), state)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(state), st0.values)   # verify only reads
    acc = np.array([0, 2, 5, 1], dtype=np.int32)
    y_ref, new_ref = oracle.causal_conv1d_update_multi(xv, w.weight, w.bias, st0.values,
                                                       accept_len=acc)
    assert rel_err(to_np(y), y_ref, bf16=True) < 1e-5
    ssm.causal_conv1d_update_multi(xd, dev_f32(w.weight), dev_f32(w.bias), state,
                                   accept_len=torch.from_numpy(acc).cuda(), want_y=False)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(state), new_ref)


@pytest.mark.parametrize("ntok", [1, 2, 5, 8, 9])
@pytest.mark.parametrize("dtype,P", [("bf16", 64), ("f32", 48)])
def test_verify_only_against_oracle(ntok, dtype, P):
    """y-only verify (the pass that reads the state without stepping it), with
    slots, a padding row and the dt transform; 9 tokens take the stepping
    kernel, fewer the state-space-duality form."""
    from hybrid_mamba_ssm_b200 import ssm
    H, N, G, max_slots = 8, 128, 2, 5
    slots = np.array([3, -1, 0], dtype=np.int32)
    batch = slots.shape[0]
    A, D = synth.make_head_params(281 + ntok, H)
    pool0 = synth.make_state(282, (max_slots, H, P, N))
    (x, _, B, C), (xd, _, Bd, Cd) = _draft(283 + ntok, batch, ntok, H, P, N, G, dtype)
    raw, bias = synth.make_raw_dt(284, (batch, ntok, H), H)
    pool = dev_f32(pool0)
    y = torch.full((batch, ntok, H, P), 7.0, device="cuda")
    ssm.ssm_state_update_multi(pool, xd, dev_f32(raw), dev_f32(A), Bd, Cd, dev_f32(D),
                               slot_idx=torch.from_numpy(slots).cuda(), y=y,
                               dt_bias=dev_f32(bias), dt_softplus=True, dt_limit=(1e-3, 0.1))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(pool), pool0.astype(np.float64))   # only read
    dt = oracle.dt_transform(raw, bias, softplus=True, dt_min=1e-3, dt_max=0.1)
    live = slots >= 0
    y_ref, _, _ = oracle.state_update_multi(pool0[slots[live]], x[live], dt[live], A, B[live],
                                            C[live], D)
    yn = to_np(y)
    assert rel_err(yn[live], y_ref) < TOL
    assert (yn[~live] == 7.0).all()


def test_verify_only_many_slices():
    """The y-only verify at a size where every SM runs many (row, head)
    slices: 24 rows of 128 heads in 8 groups, a shuffled slot map with
    padding rows between live ones; all heads against the oracle."""
    from hybrid_mamba_ssm_b200 import ssm
    H, P, N, G, ntok, max_slots = 128, 64, 128, 8, 4, 30
    rng = np.random.default_rng(291)
    slots = rng.permutation(max_slots)[:24].astype(np.int32)
    slots[[5, 17]] = -1                                   # padding rows
    batch = slots.shape[0]
    A, D = synth.make_head_params(292, H)
    pool0 = synth.make_state(293, (max_slots, H, P, N))
    (x, dt, B, C), (xd, dtd, Bd, Cd) = _draft(294, batch, ntok, H, P, N, G, "bf16")
    pool = dev_f32(pool0)
    y = torch.full((batch, ntok, H, P), 7.0, device="cuda")
    ssm.ssm_state_update_multi(pool, xd, dtd, dev_f32(A), Bd, Cd, dev_f32(D),
                               slot_idx=torch.from_numpy(slots).cuda(), y=y)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(pool), pool0.astype(np.float64))   # only read
    live = slots >= 0
    y_ref, _, _ = oracle.state_update_multi(pool0[slots[live]], x[live], dt[live], A, B[live],
                                            C[live], D)
    yn = to_np(y)
    assert rel_err(yn[live], y_ref) < TOL
    assert (yn[~live] == 7.0).all()
