"""The balanced schedule of the tensor-core scan (fixed-length batches with a
workspace): the chains of (sequence, head pair) laid end to end are cut into
one run per SM, and the carried state crosses each cut through the caller's
workspace.  It performs the same chunk arithmetic in the same order as one
CTA per chain, so its results must be bit-identical to that schedule's, and
match the oracle.  The cut is made only when there are more chains than SMs
(otherwise each chain is already its own critical path), so every run spans
parts of two or more chains.  Shapes cover a 4 x 4096 batch, a ragged last
chunk, runs that hold several whole chains (short sequences), and nonzero
initial states."""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, Guarded, dev_f32, dev_tensor, oracle_scan, rel_err, to_np

pytestmark = pytest.mark.gpu


def _run(inp, nseq, L, H, G, workspace, y_dtype=torch.bfloat16):
    from hybrid_mamba_ssm_b200 import ssm
    P, N = 64, 128
    x = dev_tensor(inp.x).view(nseq, L, H, P)
    B = dev_tensor(inp.B).view(nseq, L, G, N)
    C = dev_tensor(inp.C).view(nseq, L, G, N)
    dt = dev_f32(inp.dt).view(nseq, L, H)
    A, D = dev_f32(inp.A), dev_f32(inp.D)
    h0 = None if inp.h0 is None else dev_f32(inp.h0)
    yg = Guarded((nseq, L, H, P), y_dtype)
    hg = Guarded((nseq, H, P, N), torch.float32)
    wsg = None
    if workspace:
        n = ssm.ssd_chunk_scan_workspace_size(nseq, L, H, P, N, G, 128)
        assert n > 0, "the balanced schedule should apply to this shape"
        wsg = Guarded((n,), torch.uint8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, y=yg.t, final_state=hg.t, status=status,
                       workspace=None if wsg is None else wsg.t)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    yg.check("y")
    hg.check("final_state")
    if wsg is not None:
        wsg.check("workspace")
    return yg.t.clone(), hg.t.clone()


@pytest.mark.parametrize("nseq,L,H,G,init", [
    (4, 4096, 128, 8, False),     # 256 chains of 32 chunks, runs of ~55
    (2, 8192, 160, 8, True),      # 160 chains of 64 chunks, runs of ~69
    (5, 1000, 64, 4, True),       # ragged last chunk (8 chunks, the last of 104 tokens)
    (64, 256, 16, 2, True),       # 512 chains of 2 chunks: several whole chains per run
])
def test_balanced_schedule_is_bit_identical(nseq, L, H, G, init):
    inp = synth.make_scan_inputs(400 + L + H, [L] * nseq, H, 64, 128, G, dtype="bf16",
                                 init_state=init)
    y0, h0 = _run(inp, nseq, L, H, G, workspace=False)
    y1, h1 = _run(inp, nseq, L, H, G, workspace=True)
    assert torch.equal(y0, y1)
    assert torch.equal(h0, h1)


def test_balanced_schedule_matches_oracle():
    nseq, L, H, G = 4, 2000, 96, 4   # 192 chains
    inp = synth.make_scan_inputs(411, [L] * nseq, H, 64, 128, G, dtype="bf16", init_state=True)
    y, hT = _run(inp, nseq, L, H, G, workspace=True, y_dtype=torch.float32)
    heads = list(range(0, 24)) + [50, 95]   # one whole group, and heads of two others
    y_ref, h_ref = oracle_scan(inp, heads=heads)
    yg = to_np(y).reshape(nseq * L, H, 64)[:, heads]
    assert rel_err(yg, y_ref) < TOL
    assert rel_err(to_np(hT)[:, heads], h_ref) < TOL


def test_python_binding_allocates_the_workspace_by_default():
    """Without a workspace argument the binding allocates one where the shapes
    can use it; the result is bit-identical to passing one explicitly, and to
    passing none (one CTA per chain)."""
    from hybrid_mamba_ssm_b200 import ssm
    nseq, L, H, G = 2, 8192, 160, 8
    inp = synth.make_scan_inputs(421, [L] * nseq, H, 64, 128, G, dtype="bf16", init_state=True)
    x = dev_tensor(inp.x).view(nseq, L, H, 64)
    B = dev_tensor(inp.B).view(nseq, L, G, 128)
    C = dev_tensor(inp.C).view(nseq, L, G, 128)
    dt = dev_f32(inp.dt).view(nseq, L, H)
    A, D, h0 = dev_f32(inp.A), dev_f32(inp.D), dev_f32(inp.h0)
    y_auto, h_auto = ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0)
    y_none, h_none = ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, workspace=None)
    torch.cuda.synchronize()
    assert ssm.ssd_chunk_scan_workspace_size(nseq, L, H, 64, 128, G) > 0
    assert torch.equal(y_auto, y_none) and torch.equal(h_auto, h_none)
    with pytest.raises(ValueError):
        ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, workspace="always")
