"""Pins of the oracle's speculative (multi-token) decode against results that do
not come from the decode step it loops over:
  * every draft token's output and intermediate state against the
    semiseparable (SSD) matrix form of the scan over the row's first k draft
    tokens, evaluated by brute force with the row's state as h0;
  * the committed state is the matrix-form final state over the accepted
    prefix, and the input state bit for bit when nothing is accepted;
  * the multi-token conv1d against numpy's correlate of the row's conv state
    followed by its draft inputs, and its committed state against that
    sequence's last K-1 entries.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle import ssd_matrix_form


def _mtp_problem(seed, batch, ntok, H, P, N, G):
    rng = np.random.default_rng(seed)
    st = 0.5 * rng.standard_normal((batch, H, P, N))
    x = rng.standard_normal((batch, ntok, H, P))
    dt = rng.uniform(0.01, 0.3, (batch, ntok, H))
    A = -rng.uniform(0.2, 3.0, H)
    B = rng.standard_normal((batch, ntok, G, N))
    C = rng.standard_normal((batch, ntok, G, N))
    D = rng.standard_normal(H)
    return st, x, dt, A, B, C, D


@pytest.mark.parametrize("batch,ntok,H,P,N,G", [(2, 1, 2, 3, 4, 1), (3, 4, 4, 2, 5, 2),
                                                (1, 6, 3, 4, 3, 3)])
def test_drafts_match_matrix_form(batch, ntok, H, P, N, G):
    st, x, dt, A, B, C, D = _mtp_problem(batch * 7 + ntok, batch, ntok, H, P, N, G)
    y, inter, new = oracle.state_update_multi(st, x, dt, A, B, C, D)
    np.testing.assert_array_equal(new, st)          # no accept_len: state untouched
    for b in range(batch):
        y_ref, _ = ssd_matrix_form(x[b], dt[b], A, B[b], C[b], D, st[b][None])
        np.testing.assert_allclose(y[b], y_ref, rtol=1e-11, atol=1e-11)
        for k in range(1, ntok + 1):
            _, h_ref = ssd_matrix_form(x[b, :k], dt[b, :k], A, B[b, :k], C[b, :k], D,
                                       st[b][None])
            np.testing.assert_allclose(inter[b, k - 1], h_ref[0], rtol=1e-11, atol=1e-11)


def test_commit_selects_the_accepted_prefix():
    batch, ntok, H, P, N, G = 5, 4, 2, 3, 4, 1
    st, x, dt, A, B, C, D = _mtp_problem(11, batch, ntok, H, P, N, G)
    acc = np.array([0, 1, 2, 4, 3])
    _, _, new = oracle.state_update_multi(st, x, dt, A, B, C, D, accept_len=acc)
    np.testing.assert_array_equal(new[0], st[0])
    for b in range(1, batch):
        a = acc[b]
        _, h_ref = ssd_matrix_form(x[b, :a], dt[b, :a], A, B[b, :a], C[b, :a], D, st[b][None])
        np.testing.assert_allclose(new[b], h_ref[0], rtol=1e-11, atol=1e-11)


def _np_conv_rows(state, x, w, b):
    """Per row and channel: correlation of [state, draft inputs] (library routine)."""
    batch, ntok, dim = x.shape
    K = w.shape[1]
    out = np.zeros((batch, ntok, dim))
    for r in range(batch):
        for c in range(dim):
            seq = np.concatenate([state[r, c], x[r, :, c]])
            out[r, :, c] = np.correlate(seq, w[c], mode="valid") + b[c]
    return out


@pytest.mark.parametrize("K", [1, 2, 4, 6])
def test_conv_drafts_match_numpy_correlate(K):
    rng = np.random.default_rng(K)
    batch, ntok, dim = 3, 5, 4
    x = rng.standard_normal((batch, ntok, dim))
    w = rng.standard_normal((dim, K))
    b = rng.standard_normal(dim)
    st = rng.standard_normal((batch, dim, K - 1))
    acc = np.array([0, 2, 5])
    y, new = oracle.causal_conv1d_update_multi(x, w, b, st, activation=None, accept_len=acc)
    np.testing.assert_allclose(y, _np_conv_rows(st, x, w, b), rtol=1e-13, atol=1e-13)
    for r in range(batch):
        seq = np.concatenate([st[r], x[r, :acc[r]].T], axis=1)     # [dim, K-1+a]
        np.testing.assert_array_equal(new[r], seq[:, seq.shape[1] - (K - 1):])
