"""fp64 CPU oracle of the Mamba-2 selective state-space recurrence.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it; the product path never does.  It shares
no code with the CUDA library and does not import the ``hybrid_mamba_ssm_b200``
package.

The arithmetic lives in ``ssm_oracle.c`` (plain sequential C, double
precision, OpenMP over (sequence, head)).  This module compiles it with gcc,
loads it with ctypes and only marshals numpy arrays to and from it.

Source of the definition: the selective-SSM recurrence of the note
"Mamba 与 Nemotron 系列模型深度调研" (section "1. Selective SSM 的直觉"),
restated for decode in the modeling_nemotron_h.py walk-through (section
"Decode 阶段").  Per token t, head h, group g = h // (H // G):
``h <- exp(dt*A_h) * h + dt * x (outer) B`` and ``y = h . C + D_h * x``, the
output reading the updated state.

Every function here is pinned against results that do not come from this
code: tests/test_oracle.py (a brute-force evaluation of the structured
semiseparable (SSD) matrix form, closed forms for dt = 0, A = 0, d_state = 1
and time-invariant inputs, split-and-carry, and linearity),
tests/test_oracle_conv.py (numpy's correlate, the logistic function) and
tests/test_oracle_mtp.py (the matrix form over each draft prefix, correlate
over [conv state, draft inputs]) and tests/test_oracle_fused.py (torch's
softplus, silu and rms_norm; closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into oracle/libssm_oracle.so (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.oracle_scan.restype = ctypes.c_int
            lib.oracle_scan.argtypes = [
                ctypes.c_int, _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_state_update.restype = ctypes.c_int
            lib.oracle_state_update.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.oracle_causal_conv1d.restype = ctypes.c_int
            lib.oracle_causal_conv1d.argtypes = [
                ctypes.c_int, _i64p, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, ctypes.c_int,
                _dp, _dp]
            u32p = ctypes.POINTER(ctypes.c_uint32)
            lib.oracle_philox4x32.restype = None
            lib.oracle_philox4x32.argtypes = [u32p, u32p, ctypes.c_int, u32p]
            lib.oracle_sr_fp16.restype = ctypes.c_double
            lib.oracle_sr_fp16.argtypes = [ctypes.c_float, ctypes.c_uint32]
            lib.oracle_round_state_f16.restype = None
            lib.oracle_round_state_f16.argtypes = [ctypes.c_long, _dp, _i64p, ctypes.c_uint64,
                                                   ctypes.c_uint64, ctypes.c_int, _dp]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def scan(x, dt, A, B, C, D=None, h0=None, cu_seqlens=None):
    """Sequential recurrence over (possibly packed) sequences, in fp64.

    x  : [T, H, P] or [nseq, L, H, P]
    dt : [T, H]    or [nseq, L, H]
    A  : [H]
    B, C : [T, G, N] or [nseq, L, G, N]
    D  : [H] or None (zero skip term)
    h0 : [nseq, H, P, N] or None (zero initial state)
    cu_seqlens : [nseq+1] offsets for packed input, or None (then x is either
        [nseq, L, H, P], or [T, H, P] holding one sequence).

    Returns (y, h_final): y shaped like x, h_final [nseq, H, P, N], both fp64.
    """
    x = _f64(x)
    batched = x.ndim == 4
    if batched:
        nseq, L, H, P = x.shape
        T = nseq * L
        cu = np.arange(nseq + 1, dtype=np.int64) * L
    else:
        T, H, P = x.shape
        if cu_seqlens is None:
            cu = np.array([0, T], dtype=np.int64)
        else:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        nseq = cu.shape[0] - 1
    B64, C64 = _f64(B), _f64(C)
    G, N = B64.shape[-2], B64.shape[-1]
    Bf = B64.reshape(T, G, N)
    Cf = C64.reshape(T, G, N)
    dtf = _f64(dt).reshape(T, H)
    Af = _f64(A).reshape(H)
    Df = None if D is None else _f64(D).reshape(H)
    xf = x.reshape(T, H, P)
    if h0 is None:
        state = np.zeros((nseq, H, P, N), dtype=np.float64)
    else:
        state = _f64(h0).reshape(nseq, H, P, N).copy()
    y = np.zeros((T, H, P), dtype=np.float64)
    rc = _load().oracle_scan(int(nseq), cu.ctypes.data_as(_i64p), H, P, N, G,
                             _ptr(xf), _ptr(dtf), _ptr(Af), _ptr(Bf), _ptr(Cf),
                             _ptr(Df), _ptr(state), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_scan rejected its arguments (status {rc})")
    return y.reshape(x.shape), state


def state_update(state, x, dt, A, B, C, D=None):
    """One decode step of the recurrence for a batch, in fp64.

    state : [batch, H, P, N]  (not modified; the updated copy is returned)
    x : [batch, H, P]   dt : [batch, H]   A : [H]   B, C : [batch, G, N]
    Returns (y [batch, H, P], new_state [batch, H, P, N]).
    """
    st = _f64(state).copy()
    batch, H, P, N = st.shape
    xf, dtf, Af = _f64(x), _f64(dt), _f64(A)
    Bf, Cf = _f64(B), _f64(C)
    G = Bf.shape[1]
    Df = None if D is None else _f64(D)
    y = np.zeros((batch, H, P), dtype=np.float64)
    rc = _load().oracle_state_update(batch, H, P, N, G, _ptr(st), _ptr(xf),
                                     _ptr(dtf), _ptr(Af), _ptr(Bf), _ptr(Cf),
                                     _ptr(Df), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_state_update rejected its arguments ({rc})")
    return y, st


def scan_slots(pool, slot_idx, has_initial, x, dt, A, B, C, D=None, cu_seqlens=None):
    """The scan over sequences whose states are rows of a pool (the slot_idx ->
    ssm_pool design of the MAX nemotron_h article, section 8): sequence s
    starts from pool[slot_idx[s]] (zero where has_initial[s] == 0) and writes
    its final state back to that row; other rows are untouched.

    Returns (y, new_pool), fp64.  Pure gather / scan / scatter around scan().
    """
    pool = _f64(pool)
    slots = np.asarray(slot_idx, dtype=np.int64)
    h0 = pool[slots].copy()
    if has_initial is not None:
        h0[np.asarray(has_initial) == 0] = 0.0
    y, hT = scan(x, dt, A, B, C, D, h0, cu_seqlens=cu_seqlens)
    out = pool.copy()
    out[slots] = hT
    return y, out


def state_update_slots(pool, slot_idx, x, dt, A, B, C, D=None):
    """One decode step on pool rows: batch row b updates pool[slot_idx[b]];
    rows with a negative slot are padding (no update, y row NaN).

    Returns (y, new_pool), fp64.
    """
    pool = _f64(pool)
    slots = np.asarray(slot_idx, dtype=np.int64)
    live = slots >= 0
    out = pool.copy()
    batch = slots.shape[0]
    H, P = pool.shape[1], pool.shape[2]
    y = np.full((batch, H, P), np.nan)
    if live.any():
        yl, st = state_update(pool[slots[live]], _f64(x)[live], _f64(dt)[live], A,
                              _f64(B)[live], _f64(C)[live], D)
        y[live] = yl
        out[slots[live]] = st
    return y, out


def causal_conv1d(x, weight, bias=None, activation="silu", state=None, cu_seqlens=None):
    """Causal depthwise conv1d over (packed) sequences, channels-last, in fp64.

    x : [T, dim]; weight : [dim, K]; bias : [dim] or None;
    activation : "silu" or None; state : [nseq, dim, K-1] or None (zeros
    before each sequence start, and no state returned).
    Returns (y [T, dim], new_state [nseq, dim, K-1] or None).
    """
    xf = _f64(x)
    T, dim = xf.shape
    wf = _f64(weight)
    K = wf.shape[1]
    if K - 1 > 64:
        raise ValueError("conv width above 65 is not supported by the oracle")
    cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
          else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64)))
    nseq = cu.shape[0] - 1
    bf = None if bias is None else _f64(bias)
    st = None if state is None else _f64(state).reshape(nseq, dim, K - 1).copy()
    y = np.zeros((T, dim), dtype=np.float64)
    rc = _load().oracle_causal_conv1d(nseq, cu.ctypes.data_as(_i64p), dim, K, _ptr(xf),
                                      _ptr(wf), _ptr(bf), 1 if activation == "silu" else 0,
                                      _ptr(st), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_causal_conv1d rejected its arguments ({rc})")
    return y, st


def causal_conv1d_update(x, weight, bias, state, activation="silu"):
    """One decode token per row: window = [state (K-1 values), x] -> y; the
    state rolls by one (drops its oldest value, appends x).

    x : [batch, dim]; state : [batch, dim, K-1].  Returns (y, new_state), fp64.
    """
    xf = _f64(x)
    batch = xf.shape[0]
    cu = np.arange(batch + 1, dtype=np.int64)
    return causal_conv1d(xf, weight, bias, activation, state, cu_seqlens=cu)


def state_update_multi(state, x, dt, A, B, C, D=None, accept_len=None):
    """Speculative (multi-token) decode: each batch row runs its ntok draft
    tokens in order from its state (the MTP / speculative-decoding item of
    the deep-research note, "MTP / speculative decoding": candidate tokens
    produce intermediate states, and the accepted count decides which one
    becomes the row's state).

    state : [batch, H, P, N]; x : [batch, ntok, H, P]; dt : [batch, ntok, H];
    B, C : [batch, ntok, G, N]; accept_len : [batch] ints in [0, ntok] or None.
    Returns (y [batch, ntok, H, P], inter [batch, ntok, H, P, N] -- the state
    after each draft token --, new_state [batch, H, P, N]: the state after
    accept_len[b] tokens, i.e. the input state where accept_len[b] == 0 or
    where accept_len is None).  fp64; a loop of state_update calls.
    """
    st = _f64(state).copy()
    xf, dtf, Bf, Cf = _f64(x), _f64(dt), _f64(B), _f64(C)
    batch, ntok = xf.shape[0], xf.shape[1]
    ys, inter = [], []
    cur = st.copy()
    for k in range(ntok):
        yk, cur = state_update(cur, xf[:, k], dtf[:, k], A, Bf[:, k], Cf[:, k], D)
        ys.append(yk)
        inter.append(cur.copy())
    y = np.stack(ys, axis=1) if ntok else np.zeros(xf.shape)
    inter = (np.stack(inter, axis=1) if ntok
             else np.zeros((batch, 0) + st.shape[1:]))
    new = st.copy()
    if accept_len is not None:
        acc = np.asarray(accept_len, dtype=np.int64)
        for b in range(batch):
            if acc[b] > 0:
                new[b] = inter[b, acc[b] - 1]
    return y, inter, new


def causal_conv1d_update_multi(x, weight, bias, state, activation="silu", accept_len=None):
    """ntok draft tokens per batch row through the causal conv1d, in order
    from the row's conv state.  x : [batch, ntok, dim]; state : [batch, dim,
    K-1].  Returns (y [batch, ntok, dim], new_state): the conv state after
    accept_len[b] tokens (unchanged where 0, or everywhere when accept_len is
    None).  fp64; a loop of causal_conv1d_update calls.
    """
    xf = _f64(x)
    batch, ntok = xf.shape[0], xf.shape[1]
    st = _f64(state).copy()
    cur = st.copy()
    ys, states = [], []
    for k in range(ntok):
        yk, cur = causal_conv1d_update(xf[:, k], weight, bias, cur, activation)
        ys.append(yk)
        states.append(cur.copy())
    y = np.stack(ys, axis=1) if ntok else np.zeros(xf.shape)
    new = st.copy()
    if accept_len is not None:
        acc = np.asarray(accept_len, dtype=np.int64)
        for b in range(batch):
            if acc[b] > 0:
                new[b] = states[acc[b] - 1][b]
    return y, new


def dt_transform(dt, dt_bias=None, softplus=False, dt_min=None, dt_max=None):
    """The step size the recurrence uses, from the projection's raw dt
    (the dt_bias input of the TensorRT MambaPlugin in the deep-research
    note, "TensorRT Plugin 做 selective state update"; softplus then the
    time-step clamp of the Mamba-2 mixer): per (token, head h)

        v = dt + dt_bias[h];  v = log(1 + e^v) if softplus;  clamp to [dt_min, dt_max]

    dt : [..., H] (last axis = heads).  fp64, numpy only.
    """
    v = _f64(dt).copy()
    if dt_bias is not None:
        v = v + _f64(dt_bias)
    if softplus:
        v = np.logaddexp(0.0, v)
    if dt_min is not None:
        v = np.maximum(v, float(dt_min))
    if dt_max is not None:
        v = np.minimum(v, float(dt_max))
    return v


def gated_rmsnorm(y, z, weight, group_size, eps=1e-5):
    """Gated group RMSNorm after the scan, gate first (norm_before_gate =
    False; the _gated_group_rmsnorm step of the MAX nemotron_h article,
    section 5.4 item 4): per row and per group of group_size channels,

        g = y * silu(z),   out = g / sqrt(mean_group(g^2) + eps) * weight

    y, z : [rows, dim]; weight : [dim].  fp64, numpy only.
    """
    yf, zf, wf = _f64(y), _f64(z), _f64(weight)
    rows, dim = yf.shape
    if dim % group_size:
        raise ValueError("dim must be a multiple of group_size")
    g = yf * zf / (1.0 + np.exp(-zf))
    gg = g.reshape(rows, dim // group_size, group_size)
    ms = np.mean(gg * gg, axis=-1, keepdims=True)
    out = (gg / np.sqrt(ms + eps)).reshape(rows, dim) * wf
    return out


def philox4x32(counter, key, rounds=10):
    """Philox-4x32 of one 4-word counter under a 2-word key -> 4 words."""
    u32 = ctypes.c_uint32
    c = (u32 * 4)(*[int(v) & 0xFFFFFFFF for v in counter])
    k = (u32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    out = (u32 * 4)()
    _load().oracle_philox4x32(c, k, int(rounds), out)
    return [int(v) for v in out]


def sr_fp16(v, r16):
    """Stochastic rounding of the fp32 value v to fp16 with 16 random bits r16."""
    return _load().oracle_sr_fp16(float(np.float32(v)), int(r16) & 0xFFFF)


def round_state_f16(values, elem_index, seed, offset, rounds=10):
    """fp16 values (as fp64) a pool stores for state values written at pool
    elements elem_index, under stochastic rounding with (seed, offset)."""
    v = _f64(values).ravel()
    e = np.ascontiguousarray(np.asarray(elem_index, dtype=np.int64).ravel())
    out = np.empty_like(v)
    _load().oracle_round_state_f16(v.size, _ptr(v), e.ctypes.data_as(_i64p), int(seed),
                                   int(offset), int(rounds), _ptr(out))
    return out.reshape(np.shape(values))


def round_state_f16_nearest(values):
    """fp16 values (as fp64) of state values rounded to fp32 then to the
    nearest fp16 (ties to even)."""
    return _f64(values).astype(np.float32).astype(np.float16).astype(np.float64)


def state_update_slots_f16(pool16, slot_idx, x, dt, A, B, C, D=None, rounding=None):
    """One decode step on an fp16 pool: rows are read as fp16, updated in fp64
    (state_update), and written back rounded to fp16 -- stochastically with
    rounding = (seed, offset[, rounds]), else to nearest.  Padding rows
    (slot < 0) are skipped.  Returns (y, new_pool), fp64."""
    pool = np.asarray(pool16, dtype=np.float16).astype(np.float64)
    slots = np.asarray(slot_idx, dtype=np.int64)
    live = slots >= 0
    batch = slots.shape[0]
    H, P, N = pool.shape[1:]
    y = np.full((batch, H, P), np.nan)
    out = pool.copy()
    if live.any():
        yl, st = state_update(pool[slots[live]], _f64(x)[live], _f64(dt)[live], A,
                              _f64(B)[live], _f64(C)[live], D)
        y[live] = yl
        if rounding is None:
            out[slots[live]] = round_state_f16_nearest(st)
        else:
            row = H * P * N
            idx = slots[live][:, None] * row + np.arange(row)[None, :]
            out[slots[live]] = round_state_f16(st.reshape(-1, row), idx, *rounding).reshape(st.shape)
    return y, out
