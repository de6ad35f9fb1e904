"""ssd_chunk_scan_noalloc, the scan whose workspace is the library's built-in
scratch, against ssd_chunk_scan (the caller's workspace, or none) on the same
inputs: two calls in a row, each bit-identical to the caller-workspace call
(the same chunk arithmetic in the same order) and within the tests' tolerance
of the oracle on sampled heads.  The Python binding must not allocate either.

This file is collected last, so the entry point is also exercised after every
other test has run in the same process; it must pass alone as well."""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, dev_f32, dev_tensor, oracle_scan, rel_err, to_np

pytestmark = pytest.mark.gpu


def _dev_inputs(inp, nseq, L, H, G, P=64, N=128):
    x = dev_tensor(inp.x).view(nseq, L, H, P)
    B = dev_tensor(inp.B).view(nseq, L, G, N)
    C = dev_tensor(inp.C).view(nseq, L, G, N)
    dt = dev_f32(inp.dt).view(nseq, L, H)
    h0 = None if inp.h0 is None else dev_f32(inp.h0)
    return x, dt, dev_f32(inp.A), B, C, dev_f32(inp.D), h0


@pytest.mark.parametrize("nseq,L,H,G,init", [
    (4, 4096, 128, 8, False),   # the 4 x 4096 prefill: the built-in scratch is used
    (2, 1000, 16, 2, True),     # one wave of chains: no workspace needed
])
def test_noalloc_matches_ssd_chunk_scan(nseq, L, H, G, init):
    from hybrid_mamba_ssm_b200 import ssm
    P, N = 64, 128
    inp = synth.make_scan_inputs(900 + H, [L] * nseq, H, P, N, G, dtype="bf16", init_state=init)
    x, dt, A, B, C, D, h0 = _dev_inputs(inp, nseq, L, H, G)
    need = ssm.ssd_chunk_scan_workspace_size(nseq, L, H, P, N, G, 128)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
    y_ref = torch.empty((nseq, L, H, P), dtype=torch.float32, device="cuda")
    h_ref = torch.empty((nseq, H, P, N), dtype=torch.float32, device="cuda")
    ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, y=y_ref, final_state=h_ref, workspace=ws)

    outs = [(torch.full_like(y_ref, float("nan")), torch.full_like(h_ref, float("nan")))
            for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    before = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    for y, hT in outs:   # two calls in a row, reusing the scratch
        ssm.ssd_chunk_scan_noalloc(x, dt, A, B, C, y, hT, D=D, initial_state=h0, status=status)
    after = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    torch.cuda.synchronize()
    assert after == before, "the binding allocated device memory"
    assert int(status.item()) == 0
    for y, hT in outs:
        assert torch.equal(y, y_ref)
        assert torch.equal(hT, h_ref)

    heads = [0, H // 2 + 1, H - 1]
    y_o, h_o = oracle_scan(inp, heads=heads)
    for y, hT in outs:
        yg = to_np(y).reshape(nseq * L, H, P)[:, heads]
        assert rel_err(yg, y_o) < TOL
        assert rel_err(to_np(hT)[:, heads], h_o) < TOL


def test_noalloc_needs_preallocated_outputs():
    from hybrid_mamba_ssm_b200 import ssm
    inp = synth.make_scan_inputs(950, [256], 4, 64, 128, 2, dtype="bf16")
    x, dt, A, B, C, D, _ = _dev_inputs(inp, 1, 256, 4, 2)
    with pytest.raises(ValueError):
        ssm.ssd_chunk_scan_noalloc(x, dt, A, B, C, None)
