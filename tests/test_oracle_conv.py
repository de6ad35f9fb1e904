"""Pins of the oracle's causal depthwise conv1d against numpy's correlate,
the logistic function, and its own split-and-carry / decode-step structure."""
import numpy as np
import pytest

import oracle


def _np_causal(x, w, b):
    """Per channel: zero-padded correlation (library routine)."""
    T, dim = x.shape
    K = w.shape[1]
    out = np.zeros((T, dim))
    for c in range(dim):
        xp = np.concatenate([np.zeros(K - 1), x[:, c]])
        out[:, c] = np.correlate(xp, w[c], mode="valid") + (b[c] if b is not None else 0.0)
    return out


@pytest.mark.parametrize("T,dim,K", [(1, 3, 4), (17, 5, 4), (9, 2, 2), (6, 3, 1), (30, 4, 7)])
def test_matches_numpy_correlate(T, dim, K):
    rng = np.random.default_rng(T + dim + K)
    x = rng.standard_normal((T, dim))
    w = rng.standard_normal((dim, K))
    b = rng.standard_normal(dim)
    y, _ = oracle.causal_conv1d(x, w, b, activation=None)
    np.testing.assert_allclose(y, _np_causal(x, w, b), rtol=1e-13, atol=1e-13)


def test_silu_is_v_times_logistic():
    from scipy.special import expit
    rng = np.random.default_rng(1)
    x = rng.standard_normal((20, 3)) * 3
    w = rng.standard_normal((3, 4))
    b = rng.standard_normal(3)
    y, _ = oracle.causal_conv1d(x, w, b, activation="silu")
    pre = _np_causal(x, w, b)
    np.testing.assert_allclose(y, pre * expit(pre), rtol=1e-13, atol=1e-13)


def test_impulse_response_is_the_kernel():
    K, dim = 4, 2
    w = np.arange(1.0, 1.0 + dim * K).reshape(dim, K)
    x = np.zeros((8, dim))
    x[2] = 1.0
    y, _ = oracle.causal_conv1d(x, w, None, activation=None)
    for c in range(dim):
        np.testing.assert_array_equal(y[2:2 + K, c], w[c][::-1])
        assert (y[:2, c] == 0).all() and (y[2 + K:, c] == 0).all()


@pytest.mark.parametrize("k", [0, 1, 2, 3, 11, 20])
def test_split_and_carry(k):
    rng = np.random.default_rng(2)
    T, dim, K = 20, 4, 4
    x = rng.standard_normal((T, dim))
    w = rng.standard_normal((dim, K))
    b = rng.standard_normal(dim)
    st0 = rng.standard_normal((1, dim, K - 1))
    y, st = oracle.causal_conv1d(x, w, b, "silu", st0)
    y1, s1 = oracle.causal_conv1d(x[:k], w, b, "silu", st0)
    y2, s2 = oracle.causal_conv1d(x[k:], w, b, "silu", s1)
    np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(s2, st, rtol=0, atol=0)
    # the state is the last K-1 inputs (older state values when the sequence is short)
    np.testing.assert_array_equal(st[0], x[-(K - 1):].T)


def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(3)
    T, dim, K = 9, 5, 4
    x = rng.standard_normal((T, dim))
    w = rng.standard_normal((dim, K))
    b = rng.standard_normal(dim)
    st0 = rng.standard_normal((1, dim, K - 1))
    y, st = oracle.causal_conv1d(x, w, b, "silu", st0)
    s = st0
    for t in range(T):
        yt, s = oracle.causal_conv1d_update(x[t:t + 1], w, b, s)
        np.testing.assert_allclose(yt[0], y[t], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(s, st)


def test_packed_sequences_independent():
    rng = np.random.default_rng(4)
    lens = [5, 0, 2, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, dim, K = cu[-1], 3, 4
    x = rng.standard_normal((T, dim))
    w = rng.standard_normal((dim, K))
    st0 = rng.standard_normal((len(lens), dim, K - 1))
    y, st = oracle.causal_conv1d(x, w, None, "silu", st0, cu_seqlens=cu)
    for s in range(len(lens)):
        a, bnd = cu[s], cu[s + 1]
        ys, ss = oracle.causal_conv1d(x[a:bnd], w, None, "silu", st0[s:s + 1])
        np.testing.assert_array_equal(y[a:bnd], ys)
        np.testing.assert_array_equal(st[s], ss[0])
