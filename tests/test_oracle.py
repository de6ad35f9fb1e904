"""Pins of the fp64 CPU oracle against results that do not come from it.

Each test states what fixes the expected value:
  * the structured-semiseparable ("state space duality") matrix form of the
    scan, evaluated by brute force on tiny inputs (Mamba-2 as described in the
    note "Mamba 与 Nemotron 系列模型深度调研", section "2. Mamba block 的常见路径"
    and the conclusion list "核心结论");
  * closed forms of the recurrence: dt = 0, A = 0 (plain cumulative sum),
    time-invariant inputs (geometric series), and d_state = 1 solved by
    variation of parameters with cumprod/cumsum (the SM1 item of the Mamba tag
    page);
  * structural properties: splitting a sequence and carrying the state,
    linearity in (x, h0), packing of independent sequences;
  * shape facts printed for the Nemotron-3 Ultra Mamba layer (golden file).

A plausible mistake in the oracle -- a dropped D or input term, the output
reading the old state, a wrong decay sign or index, a transposed head_dim /
d_state, a wrong head-to-group map -- fails at least one of these; the planted
mutant test at the end checks that claim on compiled copies of the oracle.
"""
import json
import math
import os
import re
import subprocess
import ctypes

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_problem(rng, T, H, P, N, G, h0=True, dt_scale=1.0):
    x = rng.standard_normal((T, H, P))
    B = rng.standard_normal((T, G, N))
    C = rng.standard_normal((T, G, N))
    dt = dt_scale * rng.uniform(0.01, 0.3, (T, H))
    A = -rng.uniform(0.2, 3.0, H)
    D = rng.standard_normal(H)
    h = 0.5 * rng.standard_normal((1, H, P, N)) if h0 else None
    return x, dt, A, B, C, D, h


def ssd_matrix_form(x, dt, A, B, C, D, h0):
    """Brute-force evaluation of the semiseparable-matrix view of the scan.

    For head h with group g: y = M x + D x + (decay-to-i of h0) . C, where
    M[i, j] = (C_i . B_j) * exp(sum_{k=j+1..i} dt_k A) * dt_j for j <= i, and
    the final state is sum_j exp(sum_{k>j} dt_k A) dt_j x_j (outer) B_j plus the
    fully decayed h0.  Built from cumulative sums of dt*A, with no recurrence.
    """
    T, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    hpg = H // G
    y = np.zeros((T, H, P))
    hT = np.zeros((H, P, N))
    for h in range(H):
        g = h // hpg
        seg = np.concatenate([[0.0], np.cumsum(dt[:, h] * A[h])])  # seg[i+1] = sum_{k<=i}
        M = np.zeros((T, T))
        for i in range(T):
            for j in range(i + 1):
                M[i, j] = (C[i, g] @ B[j, g]) * math.exp(seg[i + 1] - seg[j + 1]) * dt[j, h]
        y[:, h, :] = M @ x[:, h, :] + D[h] * x[:, h, :]
        if h0 is not None:
            for i in range(T):
                y[i, h, :] += math.exp(seg[i + 1]) * (h0[0, h] @ C[i, g])
        for j in range(T):
            hT[h] += math.exp(seg[T] - seg[j + 1]) * dt[j, h] * np.outer(x[j, h], B[j, g])
        if h0 is not None:
            hT[h] += math.exp(seg[T]) * h0[0, h]
    return y, hT[None]


@pytest.mark.parametrize("T,H,P,N,G", [(1, 1, 1, 1, 1), (9, 2, 3, 5, 1),
                                       (13, 4, 4, 3, 2), (16, 6, 2, 7, 3)])
def test_matches_semiseparable_matrix_form(T, H, P, N, G):
    rng = np.random.default_rng(T * 100 + H)
    x, dt, A, B, C, D, h0 = rand_problem(rng, T, H, P, N, G)
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    y_ref, hT_ref = ssd_matrix_form(x, dt, A, B, C, D, h0)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(hT, hT_ref, rtol=1e-11, atol=1e-11)


def test_dt_zero_leaves_state_and_reads_it():
    rng = np.random.default_rng(1)
    x, dt, A, B, C, D, h0 = rand_problem(rng, 7, 3, 4, 5, 1)
    dt[:] = 0.0
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    np.testing.assert_array_equal(hT, h0)
    # y_t = h0 . C_t + D x_t
    expect = np.einsum("hpn,tn->thp", h0[0], C[:, 0]) + D[None, :, None] * x
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-13)


def test_A_zero_is_a_cumulative_sum():
    rng = np.random.default_rng(2)
    T, H, P, N = 11, 2, 3, 4
    x, dt, A, B, C, D, h0 = rand_problem(rng, T, H, P, N, 1)
    A[:] = 0.0
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    inc = dt[:, :, None, None] * x[:, :, :, None] * B[:, 0][:, None, None, :]
    states = h0[0][None] + np.cumsum(inc, axis=0)          # [T, H, P, N]
    np.testing.assert_allclose(hT[0], states[-1], rtol=1e-12, atol=1e-12)
    y_expect = np.einsum("thpn,tn->thp", states, C[:, 0]) + D[None, :, None] * x
    np.testing.assert_allclose(y, y_expect, rtol=1e-12, atol=1e-12)


def test_d_state_one_closed_form_cumprod_cumsum():
    """d_state = 1 solved by variation of parameters with cumprod/cumsum:
    h_t = P_t (h_0 + sum_{s<=t} dt_s B_s x_s / P_s),  P_t = prod_{k<=t} a_k."""
    rng = np.random.default_rng(3)
    T, H, P = 24, 3, 5
    x, dt, A, B, C, D, h0 = rand_problem(rng, T, H, P, 1, 1)
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    a = np.exp(dt * A[None, :])                     # [T, H]
    Pt = np.cumprod(a, axis=0)                      # [T, H]
    u = dt[:, :, None] * B[:, 0, 0][:, None, None] * x / Pt[:, :, None]
    hs = Pt[:, :, None] * (h0[0, :, :, 0][None] + np.cumsum(u, axis=0))  # [T,H,P]
    np.testing.assert_allclose(hT[0, :, :, 0], hs[-1], rtol=1e-11, atol=1e-12)
    y_expect = hs * C[:, 0, 0][:, None, None] + D[None, :, None] * x
    np.testing.assert_allclose(y, y_expect, rtol=1e-11, atol=1e-12)


def test_time_invariant_inputs_geometric_series():
    """Constant dt, B, C, x: h_t = a^t h0 + (1 - a^t)/(1 - a) * dt x B^T."""
    rng = np.random.default_rng(4)
    T, H, P, N = 40, 2, 3, 4
    x1 = rng.standard_normal((H, P))
    B1 = rng.standard_normal(N)
    C1 = rng.standard_normal(N)
    dt1 = np.array([0.05, 0.2])
    A = np.array([-1.5, -0.3])
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((1, H, P, N))
    x = np.broadcast_to(x1, (T, H, P))
    B = np.broadcast_to(B1, (T, 1, N))
    C = np.broadcast_to(C1, (T, 1, N))
    dt = np.broadcast_to(dt1, (T, H))
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    a = np.exp(dt1 * A)
    for t in (1, 2, 17, T):
        at = a ** t
        ht = (at[:, None, None] * h0[0]
              + ((1 - at) / (1 - a) * dt1)[:, None, None] * x1[:, :, None] * B1[None, None, :])
        yt = ht @ C1 + D[:, None] * x1
        np.testing.assert_allclose(y[t - 1], yt, rtol=1e-12, atol=1e-12)
        if t == T:
            np.testing.assert_allclose(hT[0], ht, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("k", [0, 1, 9, 20])
def test_split_and_carry_equals_one_run(k):
    rng = np.random.default_rng(5)
    x, dt, A, B, C, D, h0 = rand_problem(rng, 20, 4, 3, 6, 2)
    y, hT = oracle.scan(x, dt, A, B, C, D, h0)
    y1, h1 = oracle.scan(x[:k], dt[:k], A, B[:k], C[:k], D, h0)
    y2, h2 = oracle.scan(x[k:], dt[k:], A, B[k:], C[k:], D, h1)
    np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h2, hT, rtol=1e-13, atol=1e-13)


def test_linear_in_x_and_initial_state():
    rng = np.random.default_rng(6)
    x1, dt, A, B, C, D, h01 = rand_problem(rng, 15, 2, 4, 3, 1)
    x2 = rng.standard_normal(x1.shape)
    h02 = rng.standard_normal(h01.shape)
    al, be = 0.7, -1.9
    y, hT = oracle.scan(al * x1 + be * x2, dt, A, B, C, D, al * h01 + be * h02)
    ya, ha = oracle.scan(x1, dt, A, B, C, D, h01)
    yb, hb = oracle.scan(x2, dt, A, B, C, D, h02)
    np.testing.assert_allclose(y, al * ya + be * yb, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(hT, al * ha + be * hb, rtol=1e-12, atol=1e-12)


def test_packed_sequences_are_independent():
    rng = np.random.default_rng(7)
    lens = [5, 0, 12, 1]
    T = sum(lens)
    x, dt, A, B, C, D, _ = rand_problem(rng, T, 4, 2, 3, 2, h0=False)
    h0 = rng.standard_normal((len(lens), 4, 2, 3))
    cu = np.concatenate([[0], np.cumsum(lens)])
    y, hT = oracle.scan(x, dt, A, B, C, D, h0, cu_seqlens=cu)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        ys, hs = oracle.scan(x[a:b], dt[a:b], A, B[a:b], C[a:b], D, h0[s:s + 1])
        np.testing.assert_array_equal(y[a:b], ys)
        np.testing.assert_array_equal(hT[s], hs[0])
    # a zero-length sequence returns its initial state untouched
    np.testing.assert_array_equal(hT[1], h0[1])


def test_decode_steps_match_matrix_form():
    """T decode updates in a row reach the matrix-form result of the scan."""
    rng = np.random.default_rng(8)
    T, H, P, N, G = 6, 4, 3, 5, 2
    x, dt, A, B, C, D, h0 = rand_problem(rng, T, H, P, N, G)
    y_ref, hT_ref = ssd_matrix_form(x, dt, A, B, C, D, h0)
    st = h0.copy()
    for t in range(T):
        yt, st = oracle.state_update(st, x[t:t + 1], dt[t:t + 1], A, B[t:t + 1],
                                     C[t:t + 1], D)
        np.testing.assert_allclose(yt[0], y_ref[t], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(st, hT_ref, rtol=1e-11, atol=1e-11)


def test_no_D_means_zero_skip_term():
    rng = np.random.default_rng(9)
    x, dt, A, B, C, D, h0 = rand_problem(rng, 5, 2, 2, 2, 1)
    y0, h0a = oracle.scan(x, dt, A, B, C, None, h0)
    y1, h0b = oracle.scan(x, dt, A, B, C, np.zeros_like(D), h0)
    np.testing.assert_array_equal(y0, y1)
    np.testing.assert_array_equal(h0a, h0b)


def test_rejects_bad_arguments():
    rng = np.random.default_rng(10)
    x, dt, A, B, C, D, h0 = rand_problem(rng, 4, 3, 2, 2, 1)
    with pytest.raises(ValueError):   # 3 heads, 2 groups
        oracle.scan(x, dt, A, np.concatenate([B, B], 1), np.concatenate([C, C], 1), D, h0)
    with pytest.raises(ValueError):   # offsets must not decrease
        oracle.scan(x, dt, A, B, C, D, np.zeros((2, 3, 2, 2)), cu_seqlens=[0, 3, 2])


def test_ultra_layer_state_shape_golden():
    """Shape facts printed for the Nemotron-3 Ultra Mamba layer."""
    with open(os.path.join(HERE, "golden", "ultra_mamba_layer.json")) as f:
        g = json.load(f)
    H, P, N, G, K = g["mamba_num_heads"], g["head_dim"], g["ssm_state_size"], g["n_groups"], g["conv_kernel"]
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, H, P)).astype(np.float32)
    B = rng.standard_normal((1, G, N)).astype(np.float32)
    C = rng.standard_normal((1, G, N)).astype(np.float32)
    y, st = oracle.state_update(np.zeros((1, H, P, N)), x, np.full((1, H), 0.01),
                                -np.ones(H), B, C, np.zeros(H))
    assert st.shape[1:] == tuple(g["ssm_states_shape_per_batch"])
    assert st[0].size == g["ssm_state_elements"]
    assert st[0].astype(np.float32).nbytes == g["ssm_state_bytes_fp32"]
    assert H * P + 2 * G * N == g["conv_dim"]
    assert y.shape == (1, H, P)


# ---------------------------------------------------------------------------
# Planted mistakes: compile mutated copies of the oracle and check that the
# pins above reject each one.
# ---------------------------------------------------------------------------
MUTANTS = {
    "drop_input_term": ("row[n] * decay + bv[n] * dt * xv[p]", "row[n] * decay"),
    "wrong_decay_sign": ("exp(A * dt)", "exp(-A * dt)"),
    "output_reads_old_state": (
        "row[n] = row[n] * decay + bv[n] * dt * xv[p];\n            acc += row[n] * cv[n];",
        "acc += row[n] * cv[n];\n            row[n] = row[n] * decay + bv[n] * dt * xv[p];"),
    "drop_skip_term": ("yv[p] = acc + D * xv[p];", "yv[p] = acc;"),
    "c_indexes_b": ("acc += row[n] * cv[n];", "acc += row[n] * bv[n];"),
    "wrong_group_map": ("const int g = h / heads_per_group;\n        double *hs",
                        "const int g = h % G;\n        double *hs"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")).read()
    assert old in src, f"mutant {name}: pattern not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistakes(tmp_path, name, monkeypatch):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    lib = ctypes.CDLL(so)
    saved = oracle._lib
    real = oracle._load()
    for fn in ("oracle_scan", "oracle_state_update"):
        getattr(lib, fn).restype = getattr(real, fn).restype
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
    lib.oracle_num_threads.restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for pin in (lambda: test_matches_semiseparable_matrix_form(13, 4, 4, 3, 2),
                test_dt_zero_leaves_state_and_reads_it,
                test_A_zero_is_a_cumulative_sum,
                test_d_state_one_closed_form_cumprod_cumsum,
                test_time_invariant_inputs_geometric_series):
        try:
            pin()
        except AssertionError:
            caught.append(pin)
    monkeypatch.setattr(oracle, "_lib", saved)
    assert caught, f"no pin rejects the planted mistake {name!r}"


# ---------------------------------------------------------------------------
# Slot-indexed state pools (gather / scan / scatter around the recurrence)
# ---------------------------------------------------------------------------
def test_slot_pool_scan_identity_and_permutation():
    rng = np.random.default_rng(12)
    lens = [7, 0, 12]
    T = sum(lens)
    x, dt, A, B, C, D, _ = rand_problem(rng, T, 4, 3, 5, 2, h0=False)
    cu = np.concatenate([[0], np.cumsum(lens)])
    pool = rng.standard_normal((6, 4, 3, 5))
    slots = [4, 1, 0]
    has = [1, 1, 0]
    y, new_pool = oracle.scan_slots(pool, slots, has, x, dt, A, B, C, D, cu_seqlens=cu)
    h0 = np.stack([pool[4], pool[1], np.zeros_like(pool[0])])
    y_ref, hT_ref = oracle.scan(x, dt, A, B, C, D, h0, cu_seqlens=cu)
    np.testing.assert_array_equal(y, y_ref)
    np.testing.assert_array_equal(new_pool[[4, 1, 0]], hT_ref)
    np.testing.assert_array_equal(new_pool[[2, 3, 5]], pool[[2, 3, 5]])   # untouched rows
    np.testing.assert_array_equal(new_pool[1], pool[1])   # empty sequence keeps its slot


def test_slot_pool_decode_padding_rows():
    rng = np.random.default_rng(13)
    pool = rng.standard_normal((5, 2, 3, 4))
    slots = np.array([3, -1, 0])
    x = rng.standard_normal((3, 2, 3))
    dt = rng.uniform(0.01, 0.1, (3, 2))
    A = -rng.uniform(0.5, 2, 2)
    B = rng.standard_normal((3, 1, 4))
    C = rng.standard_normal((3, 1, 4))
    D = rng.standard_normal(2)
    y, new_pool = oracle.state_update_slots(pool, slots, x, dt, A, B, C, D)
    yr, st = oracle.state_update(pool[[3, 0]], x[[0, 2]], dt[[0, 2]], A, B[[0, 2]], C[[0, 2]], D)
    np.testing.assert_array_equal(y[[0, 2]], yr)
    assert np.isnan(y[1]).all()
    np.testing.assert_array_equal(new_pool[[3, 0]], st)
    np.testing.assert_array_equal(new_pool[[1, 2, 4]], pool[[1, 2, 4]])
