"""Pins of the oracle's window statistics and decode attention against
textbook loops written here.

Attention as the KVSlimmer deep dive states it (§数学主线三): e = q k^T / sqrt(d),
alpha = softmax(e), o = sum alpha v. The window average (reading R1) and the
causal window positions (reading R8) are checked element by element.
"""

import math

import numpy as np
import pytest

import oracle


def loop_attention_row(q, K, V, ln, upto):
    d = len(q)
    e = [sum(q[c] * K[t][c] for c in range(d)) / math.sqrt(d) + ln[t] for t in range(upto + 1)]
    m = max(e)
    w = [math.exp(x - m) for x in e]
    z = sum(w)
    a = [x / z for x in w]
    o = [sum(a[t] * V[t][c] for t in range(upto + 1)) for c in range(len(V[0]))]
    return a, o


@pytest.mark.parametrize("length,W,G", [(12, 4, 2), (5, 4, 1), (3, 4, 2), (9, 1, 3)])
def test_window_statistics_by_loops(length, W, G):
    rng = np.random.default_rng(length * 10 + W)
    d = 3
    Q = rng.normal(size=(G, W, d)) * 2
    K = rng.normal(size=(length, d))
    V = rng.normal(size=(length, d))
    ln = np.log(rng.integers(1, 4, size=length).astype(np.float64))
    alpha_bar, o_bar = oracle.window_statistics(Q, K, V, ln, length, W)
    rows, outs = [], []
    for g in range(G):
        for j in range(W):
            pos = length - W + j
            if pos < 0:
                continue
            a, o = loop_attention_row(Q[g, j], K, V, ln, pos)
            rows.append(a + [0.0] * (length - pos - 1))
            outs.append(o)
    np.testing.assert_allclose(alpha_bar, np.mean(rows, axis=0), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(o_bar, np.mean(outs, axis=0), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(alpha_bar.sum(), 1.0, rtol=1e-12)
    np.testing.assert_allclose(o_bar, alpha_bar @ V, rtol=1e-10, atol=1e-14)


def test_causal_window_masks_future_positions():
    rng = np.random.default_rng(0)
    Q = rng.normal(size=(1, 4, 3))
    K = rng.normal(size=(10, 3))
    V = rng.normal(size=(10, 3))
    A, _ = oracle.window_attention(Q, K, V, None, 10, 4)
    for j in range(4):
        pos = 10 - 4 + j
        assert np.all(A[j, pos + 1:] == 0)
        assert np.all(A[j, :pos + 1] > 0)


def test_empty_cache_window():
    alpha_bar, o_bar = oracle.window_statistics(np.ones((2, 4, 3)), np.zeros((0, 3)),
                                                np.zeros((0, 3)), None, 0, 4)
    assert alpha_bar.shape == (0,) and np.all(o_bar == 0)


@pytest.mark.parametrize("length", [1, 7, 40])
def test_decode_attention_by_loops(length):
    rng = np.random.default_rng(length)
    d, G = 5, 3
    q = rng.normal(size=(G, d)) * 3
    K = rng.normal(size=(length, d))
    V = rng.normal(size=(length, d))
    ln = np.log(rng.integers(1, 5, size=length).astype(np.float64))
    out = oracle.decode_attention(q, K, V, ln, length)
    for g in range(G):
        _, o = loop_attention_row(q[g], K, V, ln, length - 1)
        np.testing.assert_allclose(out[g], o, rtol=1e-12, atol=1e-14)


def test_decode_step_appends_then_attends():
    rng = np.random.default_rng(2)
    K = rng.normal(size=(1, 2, 6, 4))
    V = rng.normal(size=(1, 2, 6, 4))
    cache = oracle.cache_from_arrays(K, V, np.array([[6, 4]]))
    q = rng.normal(size=(1, 4, 4))
    kn, vn = rng.normal(size=(2, 1, 2, 4))
    out, cache = oracle.decode_step(cache, q, kn, vn)
    assert list(cache.lengths()[0]) == [7, 5]
    for h, L in ((0, 6), (1, 4)):
        Kf = np.vstack([K[0, h, :L], kn[0, h][None]])
        Vf = np.vstack([V[0, h, :L], vn[0, h][None]])
        for g in range(2):
            _, o = loop_attention_row(q[0, 2 * h + g], Kf, Vf, [0.0] * (L + 1), L)
            np.testing.assert_allclose(out[0, 2 * h + g], o, rtol=1e-12)


def test_decode_over_an_empty_cache_is_zero():
    out = oracle.decode_attention(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 4)), None, 0)
    assert out.shape == (2, 4) and np.all(out == 0)
