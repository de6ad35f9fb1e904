"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no arithmetic of the scan itself: it only draws random
numbers with numpy's PCG64 and rounds them to the storage type.  Both the CUDA
path and the CPU oracle consume what it returns, so the two see bit-identical
values: bf16 tensors are handed out both as raw bf16 bit patterns (for the GPU)
and as the exact float32 values those bits encode (for the oracle).

Distributions follow the Nemotron-shaped workloads the library is measured on:
x, B, C ~ N(0, 1); dt = clamp(softplus(z - 3), 1e-3, 0.1) with z ~ N(0, 1);
A = -exp(U(0, ln 16)) per head; D ~ N(0, 1) per head; initial states ~ N(0, 0.1)
(standard deviation 0.1) where a workload asks for a nonzero start.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


def bf16_bits(a) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16.  NaN stays NaN.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    out = rounded.astype(np.uint16)
    out[nan] = np.uint16(0x7FC0)
    return out


def bf16_values(bits) -> np.ndarray:
    """The float32 values encoded by bfloat16 bit patterns (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


@dataclass
class Tensor16:
    """A tensor stored as bf16 (``bits``) or fp32; ``values`` are exact fp32."""
    values: np.ndarray
    bits: np.ndarray | None = None   # uint16 bf16 patterns, or None for fp32

    @property
    def dtype(self) -> str:
        return "f32" if self.bits is None else "bf16"


def store(a32: np.ndarray, dtype: str) -> Tensor16:
    """Store float32 values as ``dtype`` ("bf16" rounds to nearest even)."""
    return _store(a32, dtype)


def _store(a32: np.ndarray, dtype: str) -> Tensor16:
    if dtype == "f32":
        return Tensor16(values=np.ascontiguousarray(a32, dtype=np.float32))
    if dtype == "bf16":
        bits = bf16_bits(a32)
        return Tensor16(values=bf16_values(bits), bits=bits)
    raise ValueError(f"unknown storage dtype {dtype!r}")


def draw_dt(rng: np.random.Generator, shape) -> np.ndarray:
    """dt = clamp(softplus(z - 3), 1e-3, 0.1), z ~ N(0, 1), stored fp32."""
    z = rng.standard_normal(shape)
    sp = np.logaddexp(0.0, z - 3.0)
    return np.clip(sp, 1e-3, 0.1).astype(np.float32)


def draw_A(rng: np.random.Generator, nheads: int) -> np.ndarray:
    """A = -exp(U(0, ln 16)) per head, stored fp32."""
    return (-np.exp(rng.uniform(0.0, math.log(16.0), nheads))).astype(np.float32)


@dataclass
class ScanInputs:
    """Inputs of one prefill (chunked scan) call over packed sequences."""
    cu_seqlens: np.ndarray          # int32 [nseq+1]
    x: Tensor16                     # [T, H, P]
    dt: np.ndarray                  # fp32 [T, H]
    A: np.ndarray                   # fp32 [H]
    B: Tensor16                     # [T, G, N]
    C: Tensor16                     # [T, G, N]
    D: np.ndarray                   # fp32 [H]
    h0: np.ndarray | None           # fp32 [nseq, H, P, N] or None
    dims: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def nseq(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)


def make_scan_inputs(seed: int, seqlens, nheads: int, head_dim: int,
                     d_state: int, ngroups: int, dtype: str = "bf16",
                     init_state: bool = False, state_std: float = 0.1,
                     A=None, D=None) -> ScanInputs:
    """Draw inputs for packed sequences of the given lengths.

    The draw order is fixed (x, B, C, dt, A, D, h0) so that a seed names one
    input set.  ``A``/``D`` may be passed in to share per-head parameters with
    a later decode phase.
    """
    seqlens = [int(s) for s in seqlens]
    rng = np.random.Generator(np.random.PCG64(seed))
    T = sum(seqlens)
    H, P, N, G = nheads, head_dim, d_state, ngroups
    x = _store(rng.standard_normal((T, H, P), dtype=np.float32), dtype)
    B = _store(rng.standard_normal((T, G, N), dtype=np.float32), dtype)
    C = _store(rng.standard_normal((T, G, N), dtype=np.float32), dtype)
    dt = draw_dt(rng, (T, H))
    A_ = draw_A(rng, H) if A is None else np.asarray(A, dtype=np.float32)
    D_ = rng.standard_normal(H).astype(np.float32) if D is None else np.asarray(D, dtype=np.float32)
    h0 = None
    if init_state:
        h0 = (state_std * rng.standard_normal((len(seqlens), H, P, N))).astype(np.float32)
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    return ScanInputs(cu_seqlens=cu, x=x, dt=dt, A=A_, B=B, C=C, D=D_, h0=h0,
                      dims=dict(H=H, P=P, N=N, G=G, dtype=dtype))


@dataclass
class DecodeInputs:
    """Per-token inputs of one decode step (state and A, D live elsewhere)."""
    x: Tensor16      # [batch, H, P]
    dt: np.ndarray   # fp32 [batch, H]
    B: Tensor16      # [batch, G, N]
    C: Tensor16      # [batch, G, N]


def make_decode_step(seed: int, batch: int, nheads: int, head_dim: int,
                     d_state: int, ngroups: int, dtype: str = "bf16") -> DecodeInputs:
    rng = np.random.Generator(np.random.PCG64(seed))
    x = _store(rng.standard_normal((batch, nheads, head_dim), dtype=np.float32), dtype)
    B = _store(rng.standard_normal((batch, ngroups, d_state), dtype=np.float32), dtype)
    C = _store(rng.standard_normal((batch, ngroups, d_state), dtype=np.float32), dtype)
    dt = draw_dt(rng, (batch, nheads))
    return DecodeInputs(x=x, dt=dt, B=B, C=C)


def make_raw_dt(seed: int, shape, nheads: int):
    """Raw projection dt ~ N(0, 1) (fp32, shape [..., nheads]) and a per-head
    dt_bias ~ U(-3.5, -2.5): softplus(dt + dt_bias) then spans the usual
    clamp range [1e-3, 0.1] and beyond it on both sides."""
    rng = np.random.Generator(np.random.PCG64(seed))
    raw = rng.standard_normal(tuple(shape), dtype=np.float32)
    bias = rng.uniform(-3.5, -2.5, nheads).astype(np.float32)
    return raw, bias


def make_gate(seed: int, rows: int, dim: int, dtype: str = "bf16"):
    """Scan output y and gate z ~ N(0, 1), and an RMSNorm weight ~ U(0.5, 1.5)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    y = _store(rng.standard_normal((rows, dim), dtype=np.float32), dtype)
    z = _store(rng.standard_normal((rows, dim), dtype=np.float32), dtype)
    w = rng.uniform(0.5, 1.5, dim).astype(np.float32)
    return y, z, w


def make_head_params(seed: int, nheads: int):
    """Per-head (A, D) for a decode workload."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return draw_A(rng, nheads), rng.standard_normal(nheads).astype(np.float32)


def make_state(seed: int, shape, std: float = 0.1) -> np.ndarray:
    """An fp32 state ~ N(0, std^2) of the given shape."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (std * rng.standard_normal(shape, dtype=np.float32)).astype(np.float32)


@dataclass
class ConvInputs:
    """Inputs of one causal depthwise conv1d call over packed sequences."""
    x: Tensor16              # [T, dim]
    weight: np.ndarray       # fp32 [dim, width]
    bias: np.ndarray         # fp32 [dim]
    state: Tensor16          # [nseq, dim, width-1], same storage as x
    cu_seqlens: np.ndarray   # int32 [nseq+1]


def conv_dim(nheads: int, head_dim: int, ngroups: int, d_state: int) -> int:
    """Channels of the short convolution: x (nheads*head_dim), B and C
    (ngroups*d_state each) side by side."""
    return nheads * head_dim + 2 * ngroups * d_state


def make_conv_inputs(seed: int, seqlens, dim: int, width: int = 4,
                     dtype: str = "bf16") -> ConvInputs:
    """x, state ~ N(0, 1); weight, bias ~ U(-1/sqrt(width), 1/sqrt(width))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = [int(v) for v in seqlens]
    T = sum(lens)
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    x = _store(rng.standard_normal((T, dim), dtype=np.float32), dtype)
    bound = 1.0 / np.sqrt(width)
    weight = rng.uniform(-bound, bound, (dim, width)).astype(np.float32)
    bias = rng.uniform(-bound, bound, dim).astype(np.float32)
    state = _store(rng.standard_normal((len(lens), dim, width - 1), dtype=np.float32), dtype)
    return ConvInputs(x=x, weight=weight, bias=bias, state=state, cu_seqlens=cu)


def mixed_seqlens(seed: int, nseq: int = 8, lo: int = 512, hi: int = 16384):
    """Sequence lengths drawn uniformly from the integers lo..hi."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return [int(v) for v in rng.integers(lo, hi + 1, size=nseq)]


# Workloads (seed = 1000 + workload id).  Names describe the shapes.
WORKLOADS = {
    "tiny_f32": dict(id=0, seqlens=[256], nheads=4, head_dim=16, d_state=16,
                     ngroups=1, chunk=64, dtype="f32", init_state=False),
    "decode_ultra": dict(id=1, batch=64, nheads=256, head_dim=64, d_state=128,
                         ngroups=8, dtype="bf16", steps=1000),
    "prefill_4x4096": dict(id=2, seqlens=[4096] * 4, nheads=128, head_dim=64,
                           d_state=128, ngroups=8, chunk=128, dtype="bf16",
                           init_state=False),
    "prefill_ultra_32k": dict(id=3, seqlens=[32768], nheads=256, head_dim=64,
                              d_state=128, ngroups=8, chunk=128, dtype="bf16",
                              init_state=True),
    "mixed_varlen": dict(id=4, nseq=8, lo=512, hi=16384, nheads=128, head_dim=64,
                         d_state=128, ngroups=8, chunk=128, dtype="bf16",
                         init_state=True, decode_steps=128),
}


def workload_seed(name: str) -> int:
    return 1000 + WORKLOADS[name]["id"]
