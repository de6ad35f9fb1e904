"""Python binding of libssm (include/ssm.h): argument marshalling only.

Torch tensors supply device memory and the current CUDA stream; every step of
the scan runs in the library's kernels.  Importing this module loads
``libssm.so`` and raises ImportError if it is missing or cannot be loaded --
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm.so")

SSM_F32, SSM_BF16, SSM_F16 = 0, 1, 2
STATUS_NAMES = {0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED",
                3: "SSM_ERR_MISALIGNED", 4: "SSM_ERR_CUDA", 5: "SSM_ERR_TIMEOUT",
                6: "SSM_ERR_DEVICE_INPUT", 7: "SSM_ERR_RANGE", 8: "SSM_ERR_INTERNAL"}
SSM_ERR_TIMEOUT, SSM_ERR_DEVICE_INPUT, SSM_ERR_RANGE = 5, 6, 7
EXPORTS = ("ssd_chunk_scan", "ssd_chunk_scan_workspace_size", "ssm_state_update",
           "ssd_chunk_scan_slots", "ssm_state_update_slots", "causal_conv1d_fwd",
           "causal_conv1d_update", "ssm_state_update_multi", "ssm_state_commit",
           "causal_conv1d_update_multi", "ssm_gated_rmsnorm", "ssm_status_string",
           "ssm_version", "ssm_testing_scan_stalled", "ssm_testing_conv1d_stalled")
ACTIVATIONS = {None: 0, "none": 0, "silu": 1}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libssm.so is not built ({LIB_PATH}); run "
                          "`python -m hybrid_mamba_ssm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ssd_chunk_scan.restype = i
    lib.ssd_chunk_scan.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp,
                                   vp, vp, i, vp, vp, vp, sz, vp, vp]
    lib.ssd_chunk_scan_noalloc.restype = i
    lib.ssd_chunk_scan_noalloc.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp,
                                           vp, vp, i, vp, vp, vp, vp]
    lib.ssd_chunk_scan_workspace_size.restype = sz
    lib.ssd_chunk_scan_workspace_size.argtypes = [i] * 7
    lib.ssm_state_update.restype = i
    lib.ssm_state_update.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, i,
                                     vp, vp]
    lib.ssd_chunk_scan_slots.restype = i
    lib.ssd_chunk_scan_slots.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp,
                                         vp, i, vp, i, vp, vp, i, vp, vp, vp]
    lib.ssm_state_update_slots.restype = i
    lib.ssm_state_update_slots.argtypes = [i, i, i, i, i, i, vp, i, vp, i, vp, vp, vp, vp, vp,
                                           vp, vp, vp, i, vp, vp, vp]
    lib.causal_conv1d_fwd.restype = i
    lib.causal_conv1d_fwd.argtypes = [i, i, vp, i, i, i, vp, vp, vp, i, vp, i, vp, vp, i, vp,
                                      vp, vp]
    lib.causal_conv1d_update.restype = i
    lib.causal_conv1d_update.argtypes = [i, i, i, i, vp, vp, vp, i, vp, i, vp, i, vp, vp, vp]
    lib.ssm_state_update_multi.restype = i
    lib.ssm_state_update_multi.argtypes = [i, i, i, i, i, i, i, vp, i, vp, vp, vp, vp, vp, vp,
                                           vp, vp, vp, vp, i, vp, vp, vp]
    lib.ssm_state_commit.restype = i
    lib.ssm_state_commit.argtypes = [i, i, i, i, i, vp, vp, vp, i, vp, vp, vp]
    lib.causal_conv1d_update_multi.restype = i
    lib.causal_conv1d_update_multi.argtypes = [i, i, i, i, i, vp, vp, vp, i, vp, i, vp, vp, i,
                                               vp, vp, vp]
    lib.ssm_gated_rmsnorm.restype = i
    lib.ssm_gated_rmsnorm.argtypes = [i, i, i, i, vp, i, vp, vp, ctypes.c_float, i, vp, vp]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_status_string.argtypes = [i]
    lib.ssm_version.restype = i
    u64 = ctypes.c_ulonglong
    lib.ssm_testing_scan_stalled.restype = i
    lib.ssm_testing_scan_stalled.argtypes = [i, i, i, i, vp, vp, vp, vp, vp, vp, u64, vp, vp]
    lib.ssm_testing_conv1d_stalled.restype = i
    lib.ssm_testing_conv1d_stalled.argtypes = [i, i, i, i, vp, vp, vp, u64, vp, vp]
    return lib


lib = _load()


class DtParams(ctypes.Structure):
    """ssm_dt_params: dt <- clamp(softplus(dt + dt_bias[h])) inside the kernels."""
    _fields_ = [("dt_bias", ctypes.c_void_p), ("softplus", ctypes.c_int), ("clamp", ctypes.c_int),
                ("dt_min", ctypes.c_float), ("dt_max", ctypes.c_float)]


def _dt_params(dt_bias, dt_softplus, dt_limit):
    """A DtParams reference for the keyword arguments, or None when dt is final."""
    if dt_bias is None and not dt_softplus and dt_limit is None:
        return None
    _dev(dt_bias, "dt_bias", torch.float32)
    lo, hi = dt_limit if dt_limit is not None else (0.0, 0.0)
    p = DtParams(None if dt_bias is None else dt_bias.data_ptr(), int(bool(dt_softplus)),
                 int(dt_limit is not None), float(lo), float(hi))
    return ctypes.byref(p)


class Rounding(ctypes.Structure):
    """ssm_rounding: stochastic rounding of an fp16 state pool (Philox-4x32)."""
    _fields_ = [("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64),
                ("philox_rounds", ctypes.c_int)]


def _state_format(pool, rounding):
    """(state dtype code, ssm_rounding reference or None) of a state pool.
    rounding: None (nearest even) or (seed, offset[, philox_rounds=10])."""
    if pool.dtype == torch.float32:
        return SSM_F32, None
    if pool.dtype != torch.float16:
        raise TypeError(f"state pool must be float32 or float16, got {pool.dtype}")
    if rounding is None:
        return SSM_F16, None
    seed, offset = int(rounding[0]), int(rounding[1])
    rounds = int(rounding[2]) if len(rounding) > 2 else 10
    return SSM_F16, ctypes.byref(Rounding(seed, offset, rounds))


class SSMError(RuntimeError):
    """A libssm entry point returned a nonzero status."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.ssm_status_string(status).decode()}")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SSMError(status, where)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return SSM_BF16
    if t == torch.float32:
        return SSM_F32
    raise TypeError(f"unsupported dtype {t}; use torch.bfloat16 or torch.float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def ssd_chunk_scan(x, dt, A, B, C, D=None, initial_state=None, cu_seqlens=None,
                   chunk_size: int = 128, y=None, final_state=None, y_dtype=None,
                   return_final_state: bool = True, status=None, stream=None, workspace="auto"):
    """Chunked SSD prefill scan.

    x  : [nseq, L, H, P] (fixed length) or [T, H, P] with ``cu_seqlens``
    dt : [nseq, L, H] or [T, H], fp32
    A  : [H] fp32;  D : [H] fp32 or None
    B, C : [nseq, L, G, N] or [T, G, N], same dtype as x
    initial_state : [nseq, H, P, N] fp32 or None (zeros); may be ``final_state``
    cu_seqlens : int32 [nseq+1] CUDA tensor of packed offsets, or None
    y / final_state : optional preallocated outputs
    workspace : CUDA tensor of at least ssd_chunk_scan_workspace_size(...) bytes (a
        fixed-length batch then runs the balanced schedule), None for none, or
        "auto" (the default): one is allocated through torch when these shapes
        can use it
    Returns (y, final_state) -- final_state is None if not requested.
    """
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32)
        T, H, P = x.shape
        nseq = cu_seqlens.shape[0] - 1
        seqlen = T
    else:
        nseq, L, H, P = x.shape
        T, seqlen = nseq * L, L
    G, N = B.shape[-2], B.shape[-1]
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(B, "B", x.dtype)
    _dev(C, "C", x.dtype)
    _dev(D, "D", torch.float32)
    _dev(initial_state, "initial_state", torch.float32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype, device=x.device)
    _dev(y, "y", y_dtype)
    if final_state is None and return_final_state:
        final_state = torch.empty((nseq, H, P, N), dtype=torch.float32, device=x.device)
    _dev(final_state, "final_state", torch.float32)
    _dev(status, "status", torch.int32)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError('workspace must be a CUDA tensor, None or "auto"')
        n = 0 if cu_seqlens is not None else ssd_chunk_scan_workspace_size(
            nseq, seqlen, H, P, N, G, chunk_size)
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device) if n else None
    _dev(workspace, "workspace")
    st = lib.ssd_chunk_scan(nseq, seqlen, _ptr(cu_seqlens), H, P, N, G, int(chunk_size),
                            in_code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                            _ptr(D), _ptr(initial_state), _dtype_code(y.dtype), _ptr(y),
                            _ptr(final_state), _ptr(workspace),
                            0 if workspace is None else workspace.numel() * workspace.element_size(),
                            _ptr(status), _stream(stream))
    _check(st, "ssd_chunk_scan")
    return y, final_state


def ssd_chunk_scan_noalloc(x, dt, A, B, C, y, final_state=None, D=None, initial_state=None,
                           cu_seqlens=None, chunk_size: int = 128, status=None, stream=None):
    """ssd_chunk_scan with its workspace taken from the library's built-in
    scratch; nothing here allocates, so y (and final_state, if wanted) must be
    given.  Layouts as for ssd_chunk_scan.  For callers that must not allocate
    device memory (a pool owned by another framework, or no allocator at
    hand).  The first call on a device looks up the scratch's address; calls
    whose launches overlap on the GPU race on the one scratch per device."""
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32)
        T, H, P = x.shape
        nseq = cu_seqlens.shape[0] - 1
        seqlen = T
    else:
        nseq, seqlen, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(B, "B", x.dtype)
    _dev(C, "C", x.dtype)
    _dev(D, "D", torch.float32)
    _dev(initial_state, "initial_state", torch.float32)
    if y is None:
        raise ValueError("ssd_chunk_scan_noalloc: y must be preallocated")
    _dev(y, "y", y.dtype)
    _dev(final_state, "final_state", torch.float32)
    _dev(status, "status", torch.int32)
    st = lib.ssd_chunk_scan_noalloc(nseq, seqlen, _ptr(cu_seqlens), H, P, N, G, int(chunk_size),
                                    in_code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                    _ptr(D), _ptr(initial_state), _dtype_code(y.dtype), _ptr(y),
                                    _ptr(final_state), _ptr(status), _stream(stream))
    _check(st, "ssd_chunk_scan_noalloc")
    return y, final_state


def ssd_chunk_scan_workspace_size(nseq, seqlen, nheads, head_dim, d_state, ngroups,
                                  chunk_size=128) -> int:
    """Bytes of optional workspace ssd_chunk_scan can use for these shapes on the
    current device (the balanced schedule of fixed-length batches); 0 if none."""
    return int(lib.ssd_chunk_scan_workspace_size(nseq, seqlen, nheads, head_dim, d_state,
                                                 ngroups, chunk_size))


def ssm_state_update(state, x, dt, A, B, C, D=None, y=None, y_dtype=None, stream=None):
    """One-token decode update, in place on ``state`` [batch, H, P, N] fp32.

    x : [batch, H, P];  dt : [batch, H] fp32;  A, D : [H] fp32;
    B, C : [batch, G, N] (same dtype as x).  Returns y [batch, H, P].
    """
    _dev(state, "state", torch.float32)
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    batch, H, P, N = state.shape
    G = B.shape[-2]
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(B, "B", x.dtype)
    _dev(C, "C", x.dtype)
    _dev(D, "D", torch.float32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.empty((batch, H, P), dtype=y_dtype, device=state.device)
    _dev(y, "y", y_dtype)
    st = lib.ssm_state_update(batch, H, P, N, G, in_code, _ptr(state), _ptr(x), _ptr(dt),
                              _ptr(A), _ptr(B), _ptr(C), _ptr(D), _dtype_code(y.dtype),
                              _ptr(y), _stream(stream))
    _check(st, "ssm_state_update")
    return y


def ssd_chunk_scan_slots(x, dt, A, B, C, D, state_pool, slot_idx, has_initial_state=None,
                         cu_seqlens=None, chunk_size: int = 128, y=None, y_dtype=None,
                         status=None, stream=None, dt_bias=None, dt_softplus=False,
                         dt_limit=None, rounding=None):
    """Chunked SSD prefill whose states live in a pool, updated in place.

    state_pool : [max_slots, H, P, N] fp32; sequence s starts from
        state_pool[slot_idx[s]] (or zero where has_initial_state[s] == 0) and
        its final state is written back to the same row.
    slot_idx, has_initial_state : int32 CUDA tensors [nseq] (slot_idx None:
        sequence s uses row s).
    dt_bias [H] fp32, dt_softplus, dt_limit (lo, hi): transform the raw dt
        inside the kernel (dt <- clamp(softplus(dt + dt_bias))).
    state_pool may be float16; rounding = (seed, offset[, philox_rounds])
        then rounds the written states stochastically (None: nearest even).
    Other arguments as for ssd_chunk_scan.  Returns y.
    """
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32)
        T, H, P = x.shape
        nseq = cu_seqlens.shape[0] - 1
        seqlen = T
    else:
        nseq, L, H, P = x.shape
        seqlen = L
    G, N = B.shape[-2], B.shape[-1]
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(B, "B", x.dtype)
    _dev(C, "C", x.dtype)
    _dev(D, "D", torch.float32)
    _dev(state_pool, "state_pool")
    sd, rnd = _state_format(state_pool, rounding)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(has_initial_state, "has_initial_state", torch.int32)
    _dev(status, "status", torch.int32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype, device=x.device)
    _dev(y, "y", y_dtype)
    dtp = _dt_params(dt_bias, dt_softplus, dt_limit)
    st = lib.ssd_chunk_scan_slots(nseq, seqlen, _ptr(cu_seqlens), H, P, N, G, int(chunk_size),
                                  in_code, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                  dtp, _ptr(state_pool), sd, rnd, state_pool.shape[0], _ptr(slot_idx),
                                  _ptr(has_initial_state), _dtype_code(y.dtype), _ptr(y),
                                  _ptr(status), _stream(stream))
    _check(st, "ssd_chunk_scan_slots")
    return y


def ssm_state_update_slots(state_pool, slot_idx, x, dt, A, B, C, D=None, y=None, y_dtype=None,
                           status=None, stream=None, dt_bias=None, dt_softplus=False,
                           dt_limit=None, rounding=None):
    """One-token decode update of pool rows: batch row b updates
    state_pool[slot_idx[b]] in place (slot_idx[b] < 0: padding row, skipped;
    slot_idx None: row b).  state_pool may be float16, with rounding =
    (seed, offset[, philox_rounds]) for stochastic rounding (None: nearest).
    Returns y [batch, H, P] (padding rows left as they were)."""
    _dev(state_pool, "state_pool")
    sd, rnd = _state_format(state_pool, rounding)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    batch, H, P = x.shape
    N = state_pool.shape[-1]
    G = B.shape[-2]
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(B, "B", x.dtype)
    _dev(C, "C", x.dtype)
    _dev(D, "D", torch.float32)
    _dev(status, "status", torch.int32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.zeros((batch, H, P), dtype=y_dtype, device=x.device)
    _dev(y, "y", y_dtype)
    dtp = _dt_params(dt_bias, dt_softplus, dt_limit)
    st = lib.ssm_state_update_slots(batch, H, P, N, G, in_code, _ptr(state_pool), sd, rnd,
                                    state_pool.shape[0], _ptr(slot_idx), _ptr(x), _ptr(dt),
                                    _ptr(A), _ptr(B), _ptr(C), _ptr(D), dtp, _dtype_code(y.dtype),
                                    _ptr(y), _ptr(status), _stream(stream))
    _check(st, "ssm_state_update_slots")
    return y


def _activation(activation) -> int:
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(map(str, ACTIVATIONS))}")
    return ACTIVATIONS[activation]


def causal_conv1d_fwd(x, weight, bias=None, conv_state=None, cu_seqlens=None,
                      activation="silu", slot_idx=None, has_initial_state=None, y=None,
                      y_dtype=None, status=None, stream=None):
    """Causal depthwise conv1d over whole sequences (prefill), channels-last.

    x : [nseq, L, dim] or, with cu_seqlens (int32 [nseq+1]), packed [T, dim];
        bf16 or fp32.
    weight : [dim, width] fp32 (width <= 8); bias : [dim] fp32 or None.
    conv_state : [rows, dim, width-1] in x's dtype, or None; read as the
        history before each sequence and overwritten with its last width-1
        inputs.  rows = nseq, or the pool size when slot_idx is given.
    slot_idx, has_initial_state : int32 [nseq] or None.
    Returns y shaped like x.
    """
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    if cu_seqlens is not None:
        _dev(cu_seqlens, "cu_seqlens", torch.int32)
        T, dim = x.shape
        nseq, seqlen = cu_seqlens.shape[0] - 1, T
    else:
        nseq, seqlen, dim = x.shape
    _dev(weight, "weight", torch.float32)
    width = weight.shape[-1]
    _dev(bias, "bias", torch.float32)
    _dev(conv_state, "conv_state", x.dtype)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(has_initial_state, "has_initial_state", torch.int32)
    _dev(status, "status", torch.int32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype, device=x.device)
    _dev(y, "y", y_dtype)
    max_slots = conv_state.shape[0] if (conv_state is not None and slot_idx is not None) else 0
    st = lib.causal_conv1d_fwd(nseq, seqlen, _ptr(cu_seqlens), dim, width, in_code, _ptr(x),
                               _ptr(weight), _ptr(bias), _activation(activation),
                               _ptr(conv_state), max_slots, _ptr(slot_idx),
                               _ptr(has_initial_state), _dtype_code(y.dtype), _ptr(y),
                               _ptr(status), _stream(stream))
    _check(st, "causal_conv1d_fwd")
    return y


def causal_conv1d_update(x, weight, bias, conv_state, activation="silu", slot_idx=None,
                         y=None, y_dtype=None, status=None, stream=None):
    """One decode token per batch row; conv_state [rows, dim, width-1] rolls in
    place (rows = batch, or the pool size when slot_idx is given; a negative
    slot marks a padding row).  x : [batch, dim].  Returns y [batch, dim]."""
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    batch, dim = x.shape
    _dev(weight, "weight", torch.float32)
    width = weight.shape[-1]
    _dev(bias, "bias", torch.float32)
    _dev(conv_state, "conv_state", x.dtype)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(status, "status", torch.int32)
    if y_dtype is None:
        y_dtype = x.dtype if y is None else y.dtype
    if y is None:
        y = torch.zeros((batch, dim), dtype=y_dtype, device=x.device)
    _dev(y, "y", y_dtype)
    max_slots = conv_state.shape[0] if (conv_state is not None and slot_idx is not None) else 0
    st = lib.causal_conv1d_update(batch, dim, width, in_code, _ptr(x), _ptr(weight), _ptr(bias),
                                  _activation(activation), _ptr(conv_state), max_slots,
                                  _ptr(slot_idx), _dtype_code(y.dtype), _ptr(y), _ptr(status),
                                  _stream(stream))
    _check(st, "causal_conv1d_update")
    return y


def ssm_state_update_multi(state, x, dt, A, B, C, D=None, slot_idx=None, accept_len=None,
                           inter_states=None, y=None, y_dtype=None, want_y=True,
                           want_inter=False, status=None, stream=None, dt_bias=None,
                           dt_softplus=False, dt_limit=None):
    """Speculative decode: ntok draft tokens per batch row from the row's state.

    state : [rows, H, P, N] fp32 (rows = batch, or a pool with slot_idx);
    x : [batch, ntok, H, P]; dt : [batch, ntok, H]; B, C : [batch, ntok, G, N].
    accept_len : int32 [batch] or None -- rewrite each row with its state after
    accept_len[b] tokens (None: the state is only read).
    Returns (y or None, inter_states or None); inter_states [batch, ntok, H, P,
    N] fp32 holds the state after each draft token when want_inter is set.
    """
    _dev(state, "state", torch.float32)
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    batch, ntok, H, P = x.shape
    N = state.shape[-1]
    G = B.shape[-2]
    for t, n, d in ((dt, "dt", torch.float32), (A, "A", torch.float32), (B, "B", x.dtype),
                    (C, "C", x.dtype), (D, "D", torch.float32), (slot_idx, "slot_idx", torch.int32),
                    (accept_len, "accept_len", torch.int32), (status, "status", torch.int32)):
        _dev(t, n, d)
    if want_inter and inter_states is None:
        inter_states = torch.empty((batch, ntok, H, P, N), dtype=torch.float32, device=x.device)
    _dev(inter_states, "inter_states", torch.float32)
    if want_y and y is None:
        y = torch.empty((batch, ntok, H, P), dtype=y_dtype or x.dtype, device=x.device)
    if y is not None:
        _dev(y, "y")
    y_code = _dtype_code(y.dtype) if y is not None else in_code
    max_slots = state.shape[0] if slot_idx is not None else 0
    st = lib.ssm_state_update_multi(batch, ntok, H, P, N, G, in_code, _ptr(state), max_slots,
                                    _ptr(slot_idx), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                    _ptr(D), _dt_params(dt_bias, dt_softplus, dt_limit),
                                    _ptr(accept_len), _ptr(inter_states), y_code,
                                    _ptr(y), _ptr(status), _stream(stream))
    _check(st, "ssm_state_update_multi")
    return y, inter_states


def ssm_state_commit(inter_states, accept_len, state, slot_idx=None, status=None, stream=None):
    """state row of b <- inter_states[b, accept_len[b] - 1] (unchanged where 0)."""
    _dev(inter_states, "inter_states", torch.float32)
    _dev(accept_len, "accept_len", torch.int32)
    _dev(state, "state", torch.float32)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(status, "status", torch.int32)
    batch, ntok, H, P, N = inter_states.shape
    max_slots = state.shape[0] if slot_idx is not None else 0
    st = lib.ssm_state_commit(batch, ntok, H, P, N, _ptr(inter_states), _ptr(accept_len),
                              _ptr(state), max_slots, _ptr(slot_idx), _ptr(status),
                              _stream(stream))
    _check(st, "ssm_state_commit")


def causal_conv1d_update_multi(x, weight, bias, conv_state, activation="silu", slot_idx=None,
                               accept_len=None, y=None, y_dtype=None, want_y=True,
                               status=None, stream=None):
    """ntok draft tokens per batch row through the causal conv1d.  x : [batch,
    ntok, dim]; conv_state [rows, dim, width-1] is rewritten with the window
    after accept_len[b] tokens (None: only read).  Returns y or None."""
    _dev(x, "x")
    in_code = _dtype_code(x.dtype)
    batch, ntok, dim = x.shape
    _dev(weight, "weight", torch.float32)
    width = weight.shape[-1]
    _dev(bias, "bias", torch.float32)
    _dev(conv_state, "conv_state", x.dtype)
    _dev(slot_idx, "slot_idx", torch.int32)
    _dev(accept_len, "accept_len", torch.int32)
    _dev(status, "status", torch.int32)
    if want_y and y is None:
        y = torch.empty((batch, ntok, dim), dtype=y_dtype or x.dtype, device=x.device)
    if y is not None:
        _dev(y, "y")
    y_code = _dtype_code(y.dtype) if y is not None else in_code
    max_slots = conv_state.shape[0] if (conv_state is not None and slot_idx is not None) else 0
    st = lib.causal_conv1d_update_multi(batch, ntok, dim, width, in_code, _ptr(x), _ptr(weight),
                                        _ptr(bias), _activation(activation), _ptr(conv_state),
                                        max_slots, _ptr(slot_idx), _ptr(accept_len), y_code,
                                        _ptr(y), _ptr(status), _stream(stream))
    _check(st, "causal_conv1d_update_multi")
    return y


def ssm_gated_rmsnorm(y, z, weight, group_size: int, eps: float = 1e-5, out=None,
                      out_dtype=None, stream=None):
    """out = (y * silu(z)) / rms over groups of group_size channels * weight.
    y, z : [rows, dim] (or any shape whose last axis is dim); weight [dim] fp32.
    out may be y itself.  Returns out."""
    _dev(y, "y")
    _dev(z, "z")
    _dev(weight, "weight", torch.float32)
    dim = y.shape[-1]
    rows = y.numel() // dim if dim else 0
    if out is None:
        out = torch.empty(y.shape, dtype=out_dtype or y.dtype, device=y.device)
    _dev(out, "out")
    st = lib.ssm_gated_rmsnorm(rows, dim, int(group_size), _dtype_code(y.dtype), _ptr(y),
                               _dtype_code(z.dtype), _ptr(z), _ptr(weight), float(eps),
                               _dtype_code(out.dtype), _ptr(out), _stream(stream))
    _check(st, "ssm_gated_rmsnorm")
    return out


# ---------------------------------------------------------------------------
# Testing hooks (include/ssm_testing.h): the pipelined kernels with a stalled
# producer and a short wait limit, to exercise their timeout path.
# ---------------------------------------------------------------------------
def testing_scan_stalled(x, dt, A, B, C, y, status, wait_ns: int = 1_000_000, stream=None):
    """Tensor-core scan kernel whose producer issues nothing: every CTA's first
    bounded wait expires after ``wait_ns`` and the kernel writes
    SSM_ERR_TIMEOUT to ``status``.  x [nseq, L, H, 64] bf16, dt [nseq, L, H],
    B, C [nseq, L, G, 128] bf16, y like x (meaningless output)."""
    for t, n in ((x, "x"), (y, "y"), (B, "B"), (C, "C")):
        _dev(t, n, torch.bfloat16)
    _dev(dt, "dt", torch.float32)
    _dev(A, "A", torch.float32)
    _dev(status, "status", torch.int32)
    nseq, L, H, _ = x.shape
    G = B.shape[-2]
    st = lib.ssm_testing_scan_stalled(nseq, L, H, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                      _ptr(y), int(wait_ns), _ptr(status), _stream(stream))
    _check(st, "ssm_testing_scan_stalled")


def testing_conv1d_stalled(x, weight, y, status, wait_ns: int = 1_000_000, stream=None):
    """Bulk-copy ring conv1d kernel whose producer issues nothing (see
    testing_scan_stalled).  x, y [nseq, L, dim] bf16, weight [dim, width] fp32."""
    _dev(x, "x", torch.bfloat16)
    _dev(y, "y", torch.bfloat16)
    _dev(weight, "weight", torch.float32)
    _dev(status, "status", torch.int32)
    nseq, L, dim = x.shape
    st = lib.ssm_testing_conv1d_stalled(nseq, L, dim, weight.shape[1], _ptr(x), _ptr(weight),
                                        _ptr(y), int(wait_ns), _ptr(status), _stream(stream))
    _check(st, "ssm_testing_conv1d_stalled")
