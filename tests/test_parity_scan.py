"""Prefill (ssd_chunk_scan) against the fp64 oracle, element by element.

Small cases compare every element and span several chunks plus a ragged tail;
the full-size workloads run in the benchmark's launch configuration and
compare sampled heads, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, oracle_scan, rel_err, scan_on_gpu, to_np

pytestmark = pytest.mark.gpu


def check(inp, chunk=128, y_dtype=torch.bfloat16, heads=None, initial_state=True,
          use_D=True, inplace=False, varlen=None):
    y, hT = scan_on_gpu(inp, chunk=chunk, y_dtype=y_dtype, initial_state=initial_state,
                        use_D=use_D, inplace=inplace, varlen=varlen)
    y_ref, h_ref = oracle_scan(inp, heads=heads, use_D=use_D, initial_state=initial_state)
    yg, hg = to_np(y), to_np(hT)
    if heads is not None:
        yg, hg = yg[:, heads], hg[:, heads]
    ey = rel_err(yg, y_ref, bf16=y_dtype == torch.bfloat16)
    eh = rel_err(hg, h_ref)
    # per (sequence, head) slice of the final state
    ehs = max(rel_err(hg[s, k], h_ref[s, k]) for s in range(hg.shape[0]) for k in range(hg.shape[1])
              if np.abs(h_ref[s, k]).max() > 0)
    return ey, eh, ehs


def test_tiny_f32_workload():
    w = synth.WORKLOADS["tiny_f32"]
    inp = synth.make_scan_inputs(synth.workload_seed("tiny_f32"), w["seqlens"], w["nheads"],
                                 w["head_dim"], w["d_state"], w["ngroups"], dtype="f32")
    ey, eh, ehs = check(inp, chunk=w["chunk"], y_dtype=torch.float32)
    assert ey < 1e-4 and eh < 1e-4, (ey, eh)


@pytest.mark.parametrize("seqlens,H,P,N,G,chunk", [
    ([300], 4, 16, 16, 1, 64),
    ([257, 128], 4, 32, 64, 2, 128),
    ([1, 129], 2, 64, 128, 1, 128),
    ([640], 8, 64, 128, 2, 128),
    ([400, 3, 0, 200], 8, 64, 128, 4, 128),
    ([333], 4, 128, 128, 2, 64),
    ([200], 2, 64, 32, 1, 128),
])
@pytest.mark.parametrize("dtype,y_dtype", [("bf16", torch.bfloat16), ("bf16", torch.float32),
                                           ("f32", torch.float32)])
def test_scan_small_shapes(seqlens, H, P, N, G, chunk, dtype, y_dtype):
    inp = synth.make_scan_inputs(sum(seqlens) + H * 3 + P, seqlens, H, P, N, G, dtype=dtype,
                                 init_state=True)
    ey, eh, ehs = check(inp, chunk=chunk, y_dtype=y_dtype)
    assert ey < TOL and eh < TOL and ehs < TOL, (ey, eh, ehs)


def test_scan_zero_initial_state_and_no_D():
    inp = synth.make_scan_inputs(11, [384], 8, 64, 128, 2, dtype="bf16", init_state=True)
    ey, eh, _ = check(inp, initial_state=False, use_D=False, y_dtype=torch.float32)
    assert ey < TOL and eh < TOL, (ey, eh)


def test_scan_in_place_state():
    inp = synth.make_scan_inputs(12, [256, 300], 8, 64, 128, 2, dtype="bf16", init_state=True)
    ey, eh, _ = check(inp, inplace=True, y_dtype=torch.float32)
    assert ey < TOL and eh < TOL, (ey, eh)


def test_scan_empty_sequences_keep_initial_state():
    inp = synth.make_scan_inputs(13, [0, 0], 4, 64, 128, 1, dtype="bf16", init_state=True)
    y, hT = scan_on_gpu(inp, varlen=True)
    np.testing.assert_array_equal(to_np(hT), inp.h0.astype(np.float64))


def test_bad_cu_seqlens_reported_on_device():
    from hybrid_mamba_ssm_b200 import ssm
    inp = synth.make_scan_inputs(14, [100, 60], 4, 64, 128, 1, dtype="bf16")
    from tests.gpu_helpers import dev_f32, dev_tensor
    cu = torch.tensor([0, 120, 160], dtype=torch.int32, device="cuda")   # sums to 160, T=160
    bad = torch.tensor([0, 170, 160], dtype=torch.int32, device="cuda")  # decreasing
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (dev_tensor(inp.x), dev_f32(inp.dt), dev_f32(inp.A), dev_tensor(inp.B),
            dev_tensor(inp.C), dev_f32(inp.D))
    ssm.ssd_chunk_scan(*args, cu_seqlens=cu, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ssm.ssd_chunk_scan(*args, cu_seqlens=bad, status=status)
    torch.cuda.synchronize()
    assert status.item() == 6


def test_scan_many_short_sequences_tensor_core():
    """Packed sequences of 1..9 tokens and a few longer ones on the
    tensor-core path: chunks restart at every sequence start, most chunks are
    ragged, and several sequences share a 128-token TMA tile."""
    rng = np.random.default_rng(15)
    lens = [int(v) for v in rng.integers(1, 10, 40)] + [130, 0, 257, 1]
    inp = synth.make_scan_inputs(15, lens, 8, 64, 128, 2, dtype="bf16", init_state=True)
    ey, eh, ehs = check(inp, y_dtype=torch.float32, varlen=True)
    assert ey < TOL and eh < TOL and ehs < TOL, (ey, eh, ehs)


@pytest.mark.parametrize("dt", [0.1, 0.2])
def test_scan_large_dt_decays_to_zero(dt):
    """Large dt with A at its most negative: long decays push exp(cs) toward
    0 inside a chunk.  At dt 0.1 a 32-token block decays by e^-51 (factorised
    path); at 0.2 by e^-102, beyond the factorised path's bound, so the mask
    takes one exp per element.  Neither may overflow or produce NaN."""
    inp = synth.make_scan_inputs(16, [512], 4, 64, 128, 1, dtype="bf16", init_state=True)
    inp.dt[:] = dt
    inp.A[:] = -16.0
    ey, eh, _ = check(inp, y_dtype=torch.float32)
    assert ey < TOL and eh < TOL, (ey, eh)


@pytest.mark.parametrize("nseq", [64, 65])   # longest-first order, and index order
@pytest.mark.parametrize("dtype,P,N", [("bf16", 64, 128), ("f32", 32, 64)])
def test_scan_packed_order_both_sides_of_cutoff(nseq, dtype, P, N):
    """Packed batches of up to 64 sequences are swept longest first (each CTA
    ranks the lengths), larger ones in index order.  Lengths with ties,
    empty sequences and ragged tails, on the tensor-core and CUDA-core
    kernels; every element against the oracle, empty sequences bit-exact."""
    rng = np.random.default_rng(16 + nseq)
    lens = [int(v) for v in rng.integers(0, 300, nseq)]
    lens[3] = lens[7] = 0
    lens[10] = lens[11] = lens[12] = 129
    inp = synth.make_scan_inputs(17 + nseq, lens, 4, P, N, 2, dtype=dtype, init_state=True)
    y, hT = scan_on_gpu(inp, y_dtype=torch.float32, varlen=True)
    y_ref, h_ref = oracle_scan(inp)
    assert rel_err(to_np(y), y_ref) < TOL
    assert rel_err(to_np(hT), h_ref) < TOL
    for s in (3, 7):
        np.testing.assert_array_equal(to_np(hT)[s], inp.h0[s].astype(np.float64))
