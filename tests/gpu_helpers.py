"""Helpers for the GPU parity tests: move seeded inputs to the device and
compare CUDA results with the fp64 oracle.

Error metric (the 2e-3 bound on y and the final state): for a result tensor
r and the oracle's value o (fp64),

    err = max |r - o| / max |o|

over the tensor (and, where stated, over each (sequence, head) slice).  A bf16
output cannot be closer to o than its own rounding, so for bf16 y each
element's deviation first has half a bf16 ulp of o taken off:
max(|r - o| - ulp_bf16(o)/2, 0).
"""
import numpy as np
import torch

from hybrid_mamba_ssm_b200 import inputs as synth

TOL = 2e-3

# Canary guard bands: every output buffer a parity test hands to the library
# sits between two GUARD-byte bands filled with SENTINEL; after the call the
# bands must be untouched (no stray write before or after an output, e.g. by a
# TMA store of a partial tile or a slot-indexed write).
GUARD = 4096
SENTINEL = 0x5A


class Guarded:
    """A device tensor of ``shape`` inside a larger buffer with guard bands."""

    def __init__(self, shape, dtype, device="cuda", init=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        g = GUARD // es
        self.buf = torch.empty(n + 2 * g, dtype=dtype, device=device)
        self.buf.view(torch.uint8).fill_(SENTINEL)
        self.t = self.buf[g:g + n].view(*shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, name="output"):
        b = self.buf.view(torch.uint8)
        head, tail = b[:GUARD], b[b.numel() - GUARD:]
        assert bool((head == SENTINEL).all()), f"write before {name}"
        assert bool((tail == SENTINEL).all()), f"write after {name}"


def guarded_like(t, init=True):
    """A guarded copy of tensor t (its contents copied in when init)."""
    return Guarded(tuple(t.shape), t.dtype, t.device, init=t if init else None)


def dev_tensor(t: synth.Tensor16, device="cuda"):
    if t.bits is None:
        return torch.from_numpy(np.ascontiguousarray(t.values)).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(torch.bfloat16).to(device)


def dev_f32(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def ulp_bf16(o):
    a = np.abs(np.asarray(o, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return np.exp2(e - 7)


def rel_err(r, o, bf16=False):
    r = np.asarray(r, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    denom = np.max(np.abs(o))
    if denom == 0:
        return float(np.max(np.abs(r)))
    d = np.abs(r - o)
    if bf16:
        d = np.maximum(d - 0.5 * ulp_bf16(o), 0.0)
    return float(np.max(d) / denom)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def scan_on_gpu(inp: synth.ScanInputs, chunk=128, y_dtype=torch.bfloat16, varlen=None,
                initial_state=True, inplace=False, use_D=True, expect_status=0, workspace=False):
    """Run ssd_chunk_scan on the inputs; returns (y, final_state) tensors.

    y and the final state are written into guarded buffers whose guard bands
    are checked after the call; the device status word must read
    ``expect_status`` (0 unless a test provokes a device-side status).  With
    ``workspace`` a fixed-length call also gets the (guarded) scan workspace,
    as bench.py passes it, where the shapes can use one."""
    from hybrid_mamba_ssm_b200 import ssm
    T, nseq = inp.T, inp.nseq
    lens = np.diff(inp.cu_seqlens)
    equal = len(set(lens.tolist())) <= 1
    if varlen is None:
        varlen = not equal
    x = dev_tensor(inp.x)
    Bt, Ct = dev_tensor(inp.B), dev_tensor(inp.C)
    dt = dev_f32(inp.dt)
    A, D = dev_f32(inp.A), dev_f32(inp.D) if use_D else None
    H, P = x.shape[1], x.shape[2]
    G, N = Bt.shape[1], Bt.shape[2]
    h0g = None
    if initial_state and inp.h0 is not None:
        h0g = guarded_like(dev_f32(inp.h0))
    h0 = None if h0g is None else h0g.t
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    yg = Guarded((T, H, P), y_dtype)
    if inplace and h0g is not None:
        hg = h0g
    else:
        hg = Guarded((nseq, H, P, N), torch.float32)
    if varlen:
        cu = torch.from_numpy(inp.cu_seqlens.astype(np.int32)).cuda()
        y, hT = ssm.ssd_chunk_scan(x, dt, A, Bt, Ct, D, h0, cu_seqlens=cu, chunk_size=chunk,
                                   y=yg.t, final_state=hg.t, status=status)
    else:
        L = int(lens[0]) if nseq else 0
        wsg = None
        if workspace:
            n = ssm.ssd_chunk_scan_workspace_size(nseq, L, H, P, N, G, chunk)
            wsg = Guarded((n,), torch.uint8) if n else None
        y, hT = ssm.ssd_chunk_scan(x.view(nseq, L, H, P), dt.view(nseq, L, H), A,
                                   Bt.view(nseq, L, G, N), Ct.view(nseq, L, G, N), D, h0,
                                   chunk_size=chunk, y=yg.t.view(nseq, L, H, P),
                                   final_state=hg.t, status=status,
                                   workspace=None if wsg is None else wsg.t)
        y = y.view(T, H, P)
        if wsg is not None:
            torch.cuda.synchronize()
            wsg.check("workspace")
    torch.cuda.synchronize()
    yg.check("y")
    hg.check("final_state")
    if h0g is not None:
        h0g.check("initial_state")
    assert int(status.item()) == expect_status, (int(status.item()), expect_status)
    return y, hT


def oracle_scan(inp: synth.ScanInputs, heads=None, use_D=True, initial_state=True):
    """Oracle y [T, k, P] and final state [nseq, k, P, N] for the heads listed.

    The chosen heads are gathered into one sub-problem with one group per head
    (B, C of each head's own group), so a single oracle call covers them.
    """
    import oracle
    H = inp.x.values.shape[1]
    G = inp.B.values.shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    groups = [h // (H // G) for h in heads]
    h0 = inp.h0 if initial_state else None
    y, hT = oracle.scan(inp.x.values[:, heads], inp.dt[:, heads], inp.A[heads],
                        inp.B.values[:, groups], inp.C.values[:, groups],
                        inp.D[heads] if use_D else None,
                        None if h0 is None else h0[:, heads],
                        cu_seqlens=inp.cu_seqlens.astype(np.int64))
    return y, hT
