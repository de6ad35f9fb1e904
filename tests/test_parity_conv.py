"""Causal depthwise conv1d on the GPU against the fp64 oracle: packed and
batched prefill (ragged channel blocks, sequences shorter than the window,
empty sequences, several 64-token tiles), the carried conv state (bit for bit:
it holds inputs verbatim), slot pools, and the one-token decode update."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import dev_f32, dev_tensor, rel_err, to_np

pytestmark = pytest.mark.gpu

# fp32 accumulation of at most 8 products against fp64: a few fp32 ulps.
CONV_TOL = 1e-5


def _torch_dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def _act(a):
    return "silu" if a else None


@pytest.mark.parametrize("width", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("dtype,y_dtype", [("bf16", "bf16"), ("bf16", "f32"), ("f32", "f32")])
@pytest.mark.parametrize("with_state,act", [(True, True), (False, False)])
@pytest.mark.parametrize("dim", [640, 102])      # vectorised path / scalar path (ragged)
def test_conv_prefill_packed(width, dtype, y_dtype, with_state, act, dim):
    from hybrid_mamba_ssm_b200 import ssm
    lens = [300, 0, 1, 2, 129, 64, 5]
    inp = synth.make_conv_inputs(71 + width, lens, dim, width, dtype)
    state = dev_tensor(inp.state) if with_state else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = ssm.causal_conv1d_fwd(dev_tensor(inp.x), dev_f32(inp.weight), dev_f32(inp.bias),
                              conv_state=state,
                              cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda(),
                              activation=_act(act), y_dtype=_torch_dtype(y_dtype), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    y_ref, st_ref = oracle.causal_conv1d(inp.x.values, inp.weight, inp.bias, _act(act),
                                         inp.state.values if with_state else None,
                                         cu_seqlens=inp.cu_seqlens)
    assert rel_err(to_np(y), y_ref, bf16=(y_dtype == "bf16")) < CONV_TOL
    if with_state:
        np.testing.assert_array_equal(to_np(state), st_ref)


def test_conv_prefill_batched_bf16():
    from hybrid_mamba_ssm_b200 import ssm
    nseq, L, dim, width = 3, 200, 1056, 4
    inp = synth.make_conv_inputs(81, [L] * nseq, dim, width, "bf16")
    state = dev_tensor(inp.state)
    y = ssm.causal_conv1d_fwd(dev_tensor(inp.x).view(nseq, L, dim), dev_f32(inp.weight),
                              dev_f32(inp.bias), conv_state=state)
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.causal_conv1d(inp.x.values, inp.weight, inp.bias, "silu",
                                         inp.state.values, cu_seqlens=inp.cu_seqlens)
    assert y.shape == (nseq, L, dim)
    assert rel_err(to_np(y).reshape(-1, dim), y_ref, bf16=True) < CONV_TOL
    np.testing.assert_array_equal(to_np(state), st_ref)


def _oracle_conv_slots(pool, slots, has, x, weight, bias, act, cu):
    """Gather / oracle / scatter around oracle.causal_conv1d for a pool."""
    st = pool[slots].copy()
    if has is not None:
        st[np.asarray(has) == 0] = 0.0
    y, new = oracle.causal_conv1d(x, weight, bias, act, st, cu_seqlens=cu)
    out = pool.astype(np.float64).copy()
    out[slots] = new
    return y, out


def test_conv_prefill_slots():
    from hybrid_mamba_ssm_b200 import ssm
    lens, dim, width, max_slots = [70, 2, 0, 130], 512, 4, 6
    inp = synth.make_conv_inputs(91, lens, dim, width, "bf16")
    pool0 = synth.make_conv_inputs(92, [1] * max_slots, dim, width, "bf16").state
    slots = np.array([4, 0, 5, 2], dtype=np.int32)
    has = np.array([1, 0, 0, 1], dtype=np.int32)
    pool = dev_tensor(pool0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = ssm.causal_conv1d_fwd(dev_tensor(inp.x), dev_f32(inp.weight), dev_f32(inp.bias),
                              conv_state=pool, cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda(),
                              slot_idx=torch.from_numpy(slots).cuda(),
                              has_initial_state=torch.from_numpy(has).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    y_ref, pool_ref = _oracle_conv_slots(pool0.values, slots, has, inp.x.values, inp.weight,
                                         inp.bias, "silu", inp.cu_seqlens)
    assert rel_err(to_np(y), y_ref, bf16=True) < CONV_TOL
    np.testing.assert_array_equal(to_np(pool), pool_ref)
    np.testing.assert_array_equal(to_np(pool)[5], 0.0)   # empty sequence, fresh slot


def test_conv_prefill_bad_slot_skips_sequence():
    from hybrid_mamba_ssm_b200 import ssm
    lens, dim, width = [64, 100], 256, 4
    inp = synth.make_conv_inputs(93, lens, dim, width, "bf16")
    pool0 = synth.make_conv_inputs(94, [1] * 3, dim, width, "bf16").state
    pool = dev_tensor(pool0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((sum(lens), dim), 7.0, dtype=torch.bfloat16, device="cuda")
    ssm.causal_conv1d_fwd(dev_tensor(inp.x), dev_f32(inp.weight), dev_f32(inp.bias),
                          conv_state=pool, cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda(),
                          slot_idx=torch.tensor([3, 1], dtype=torch.int32, device="cuda"),
                          y=y, status=status)
    torch.cuda.synchronize()
    assert status.item() == 6
    yn = to_np(y)
    assert (yn[:64] == 7.0).all()                        # skipped sequence: no y
    got = to_np(pool)
    np.testing.assert_array_equal(got[[0, 2]], pool0.values[[0, 2]])
    y_ref, pool_ref = _oracle_conv_slots(pool0.values, [1], None, inp.x.values[64:],
                                         inp.weight, inp.bias, "silu",
                                         np.array([0, 100], dtype=np.int32))
    assert rel_err(yn[64:], y_ref, bf16=True) < CONV_TOL
    np.testing.assert_array_equal(got[1], pool_ref[1])


@pytest.mark.parametrize("width", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv_update_steps(width, dtype):
    from hybrid_mamba_ssm_b200 import ssm
    batch, dim = 5, 800
    inp = synth.make_conv_inputs(101 + width, [1] * batch, dim, width, dtype)
    state = dev_tensor(inp.state)
    ref = inp.state.values.astype(np.float64)
    for k in range(width + 2):                   # enough steps to roll the window through
        xk = synth.make_conv_inputs(110 + k, [batch], dim, width, dtype).x
        y = ssm.causal_conv1d_update(dev_tensor(xk), dev_f32(inp.weight), dev_f32(inp.bias),
                                     state)
        y_ref, ref = oracle.causal_conv1d_update(xk.values, inp.weight, inp.bias, ref)
        assert rel_err(to_np(y), y_ref, bf16=(dtype == "bf16")) < CONV_TOL
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(state), ref)


def test_conv_update_slots_with_padding():
    from hybrid_mamba_ssm_b200 import ssm
    dim, width, max_slots = 512, 4, 7
    slots = np.array([6, -1, 0, 3, -1], dtype=np.int32)
    batch = slots.shape[0]
    w = synth.make_conv_inputs(121, [1], dim, width, "bf16")
    pool0 = synth.make_conv_inputs(122, [1] * max_slots, dim, width, "bf16").state
    pool = dev_tensor(pool0)
    ref = pool0.values.astype(np.float64)
    live = slots >= 0
    for k in range(3):
        xk = synth.make_conv_inputs(123 + k, [batch], dim, width, "bf16").x
        y = torch.full((batch, dim), 7.0, dtype=torch.bfloat16, device="cuda")
        ssm.causal_conv1d_update(dev_tensor(xk), dev_f32(w.weight), dev_f32(w.bias), pool,
                                 slot_idx=torch.from_numpy(slots).cuda(), y=y)
        y_ref, new = oracle.causal_conv1d_update(xk.values[live], w.weight, w.bias,
                                                 ref[slots[live]])
        ref[slots[live]] = new
        yn = to_np(y)
        assert rel_err(yn[live], y_ref, bf16=True) < CONV_TOL
        assert (yn[~live] == 7.0).all()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(pool), ref)


def test_conv_prefill_then_decode_matches_one_prefill():
    """Prefill of L tokens then 3 decode tokens equals one prefill of L+3."""
    from hybrid_mamba_ssm_b200 import ssm
    L, dim, width = 150, 384, 4
    inp = synth.make_conv_inputs(131, [L + 3], dim, width, "f32")
    xd = dev_tensor(inp.x)
    state = torch.zeros((1, dim, width - 1), device="cuda")
    w, b = dev_f32(inp.weight), dev_f32(inp.bias)
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    y0 = ssm.causal_conv1d_fwd(xd[:L].contiguous(), w, b, conv_state=state, cu_seqlens=cu)
    ys = [ssm.causal_conv1d_update(xd[L + k:L + k + 1].contiguous(), w, b, state)
          for k in range(3)]
    torch.cuda.synchronize()
    got = np.concatenate([to_np(y0)] + [to_np(v) for v in ys])
    y_ref, _ = oracle.causal_conv1d(inp.x.values, inp.weight, inp.bias, "silu",
                                    np.zeros((1, dim, width - 1)))
    assert rel_err(got, y_ref) < CONV_TOL


def test_conv_full_size_prefill_4x4096():
    """The benchmark's conv shape: 4 x 4096 tokens of 128*64 + 2*8*128 channels."""
    from hybrid_mamba_ssm_b200 import ssm
    dim = synth.conv_dim(128, 64, 8, 128)
    inp = synth.make_conv_inputs(141, [4096] * 4, dim, 4, "bf16")
    state = dev_tensor(inp.state)
    y = ssm.causal_conv1d_fwd(dev_tensor(inp.x), dev_f32(inp.weight), dev_f32(inp.bias),
                              conv_state=state, cu_seqlens=torch.from_numpy(inp.cu_seqlens).cuda())
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.causal_conv1d(inp.x.values, inp.weight, inp.bias, "silu",
                                         inp.state.values, cu_seqlens=inp.cu_seqlens)
    assert rel_err(to_np(y), y_ref, bf16=True) < CONV_TOL
    np.testing.assert_array_equal(to_np(state), st_ref)
