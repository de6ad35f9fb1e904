"""The timeout path of the pipelined kernels' bounded waits, made to run out on
purpose without faulting or hanging the GPU: the testing hooks of
include/ssm_testing.h launch the tensor-core scan and the conv1d bulk-copy
ring with a producer that issues nothing and a 1 ms wait limit.  Every CTA's
first wait then expires with nothing in flight; the kernel must report
SSM_ERR_TIMEOUT on the status word, return promptly, and leave the context
usable (a normal call afterwards still matches the oracle)."""
import time

import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import TOL, dev_f32, dev_tensor, oracle_scan, rel_err, scan_on_gpu, to_np

pytestmark = pytest.mark.gpu

SSM_ERR_TIMEOUT = 5


def _normal_scan_still_works():
    inp = synth.make_scan_inputs(301, [300], 8, 64, 128, 2, dtype="bf16", init_state=True)
    y, hT = scan_on_gpu(inp, y_dtype=torch.float32)
    y_ref, h_ref = oracle_scan(inp)
    assert rel_err(to_np(y), y_ref) < TOL and rel_err(to_np(hT), h_ref) < TOL


@pytest.mark.parametrize("wait_ns", [1_000_000, 20_000_000])
def test_scan_stalled_producer_times_out(wait_ns):
    from hybrid_mamba_ssm_b200 import ssm
    nseq, L, H, G = 2, 512, 8, 2
    inp = synth.make_scan_inputs(302, [L] * nseq, H, 64, 128, G, dtype="bf16")
    x = dev_tensor(inp.x).view(nseq, L, H, 64)
    B = dev_tensor(inp.B).view(nseq, L, G, 128)
    C = dev_tensor(inp.C).view(nseq, L, G, 128)
    dt = dev_f32(inp.dt).view(nseq, L, H)
    A = dev_f32(inp.A)
    y = torch.empty_like(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ssm.testing_scan_stalled(x, dt, A, B, C, y, status, wait_ns=wait_ns)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == SSM_ERR_TIMEOUT
    assert elapsed < 5.0, elapsed            # one expired wait per thread, not one per chunk
    _normal_scan_still_works()


def test_conv1d_stalled_producer_times_out():
    from hybrid_mamba_ssm_b200 import ssm
    nseq, L, dim, K = 2, 1024, 2048, 4
    rng = np.random.default_rng(303)
    x = torch.from_numpy(rng.standard_normal((nseq, L, dim), dtype=np.float32)).to(
        torch.bfloat16).cuda()
    w = torch.from_numpy(rng.standard_normal((dim, K), dtype=np.float32)).cuda()
    y = torch.empty_like(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ssm.testing_conv1d_stalled(x, w, y, status, wait_ns=1_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == SSM_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    # the same kernel with its producer running gives the convolution
    y2 = ssm.causal_conv1d_fwd(x, w, None, activation=None)
    torch.cuda.synchronize()
    xf = x.float().cpu().numpy()
    ref = np.zeros_like(xf)
    wn = w.cpu().numpy()
    for k in range(K):
        shift = K - 1 - k
        ref[:, shift:, :] += wn[:, k] * xf[:, :L - shift, :]
    got = y2.float().cpu().numpy()
    assert np.abs(got - ref).max() / np.abs(ref).max() < 1e-2
    _normal_scan_still_works()
