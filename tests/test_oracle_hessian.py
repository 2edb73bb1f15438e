"""Pins of the oracle's attention derivatives against finite differences.

The KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
§数学主线三) gives the Key gradient, the Hessian blocks and the sensitivities
ds_i/de_j of attention for the loss L = E^T o. Here the loss is evaluated by a
plain textbook attention written in this file and differentiated numerically;
the oracle's closed forms must agree.
"""

import math

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def textbook_attention(q, K, V, counts=None):
    """o = sum_t a_t v_t with a_t = c_t exp(q.k_t/sqrt d) / sum_s c_s exp(q.k_s/sqrt d)."""
    d = len(q)
    n = len(K)
    counts = [1.0] * n if counts is None else counts
    w = []
    for t in range(n):
        s = sum(q[c] * K[t][c] for c in range(d)) / math.sqrt(d)
        w.append(counts[t] * math.exp(s))
    z = sum(w)
    return np.array([sum(w[t] * V[t][c] for t in range(n)) / z for c in range(len(V[0]))])


def loss(q, K, V, E, counts=None):
    return float(np.dot(E, textbook_attention(q, K, V, counts)))


def fd_gradient(q, K, V, E, i, h=1e-5):
    g = np.zeros(K.shape[1])
    for a in range(K.shape[1]):
        Kp, Km = K.copy(), K.copy()
        Kp[i, a] += h
        Km[i, a] -= h
        g[a] = (loss(q, Kp, V, E) - loss(q, Km, V, E)) / (2 * h)
    return g


def fd_hessian(f, K, i, j, h=1e-4):
    d = K.shape[1]
    H = np.zeros((d, d))
    for a in range(d):
        for b in range(d):
            vals = []
            for sa, sb in ((1, 1), (1, -1), (-1, 1), (-1, -1)):
                Kx = K.copy()
                Kx[i, a] += sa * h
                Kx[j, b] += sb * h
                vals.append(f(Kx))
            H[a, b] = (vals[0] - vals[1] - vals[2] + vals[3]) / (4 * h * h)
    return H


def _case(seed, n=5, d=4, qscale=2.0):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=d) * qscale
    K = rng.normal(size=(n, d))
    V = rng.normal(size=(n, d + 1))
    E = rng.normal(size=d + 1)
    return q, K, V, E


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_key_gradient_matches_finite_difference(seed):
    q, K, V, E = _case(seed)
    for i in range(K.shape[0]):
        np.testing.assert_allclose(oracle.key_gradient(q, K, V, E, i), fd_gradient(q, K, V, E, i),
                                   rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_hessian_blocks_match_finite_difference(seed):
    q, K, V, E = _case(seed)
    f = lambda Kx: loss(q, Kx, V, E)  # noqa: E731
    for i, j in [(0, 0), (1, 2), (2, 1), (3, 3), (3, 4)]:
        np.testing.assert_allclose(oracle.hessian_block(q, K, V, E, i, j), fd_hessian(f, K, i, j),
                                   rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("seed,peaked", [(6, False), (7, False), (8, True)])
def test_pair_norms_equal_norms_of_numerical_sensitivities(seed, peaked):
    """With E = unit vectors, the FD Hessian gives each component of ds_i/de_j;
    their norms are |c11|, |c12|, |c22| and must equal what score_head uses for a
    one-query window (where the window average is exact)."""
    n, d = 6, 4
    q, K, V, _ = _case(seed, n=n, d=d, qscale=3.0)
    V = V[:, :d]
    m = 2                                   # pair (m, m+1) = (2, 3)
    dv = V.shape[1]
    if peaked:                              # 1/2 < alpha_m < 0.8: alpha (1 - 2 alpha) < 0
        for s in np.linspace(0.0, 20.0, 401):
            K[m] = s * q / np.linalg.norm(q)
            if oracle.softmax(oracle.attention_logits(q, K))[m] > 0.65:
                break
    alpha_chk = oracle.softmax(oracle.attention_logits(q, K))
    assert (alpha_chk[m] > 0.5) == peaked

    def sens_vector(i, j):
        vec = np.zeros(dv)
        for c in range(dv):
            E = np.zeros(dv)
            E[c] = 1.0
            H = fd_hessian(lambda Kx: loss(q, Kx, V, E), K, i, j)
            # h_ij = (1/d) (E^T ds_i/de_j) q q^T  -> read the scalar off the largest entry
            a = int(np.argmax(np.abs(q)))
            vec[c] = H[a, a] * d / (q[a] * q[a])
        return vec

    c11 = sens_vector(m, m)
    c22 = sens_vector(m + 1, m + 1)
    c12 = sens_vector(m, m + 1)
    # one window query at the last position attends every key
    hs = oracle.score_head(K, V, None, n, cand_begin=m, n_recent=n - m - 2,
                           Q_heads=q.reshape(1, 1, d), W=1)
    np.testing.assert_allclose(hs.n11[0], np.linalg.norm(c11), rtol=1e-4)
    np.testing.assert_allclose(hs.n22[0], np.linalg.norm(c22), rtol=1e-4)
    np.testing.assert_allclose(hs.n12[0], np.linalg.norm(c12), rtol=1e-4)
    # sign structure of the pages' vectors: c11, c22 along (v - o); c12 along -(v_m + v_m1 - 2o)
    alpha = oracle.softmax(oracle.attention_logits(q, K))
    o = alpha @ V
    r11, r22, r12 = oracle.forward_vectors(alpha[m], alpha[m + 1], V[m], V[m + 1], o)
    np.testing.assert_allclose(r11, c11, rtol=1e-4, atol=1e-7)
    np.testing.assert_allclose(r22, c22, rtol=1e-4, atol=1e-7)
    np.testing.assert_allclose(r12, c12, rtol=1e-4, atol=1e-7)


def test_hessian_of_shared_key_group_matches_expanded_cache():
    """A merged group (count n, mean value, log n bias) has exactly the Hessian of
    the expanded cache in which its n positions share one key and keep their own
    values (the Value rule reading)."""
    rng = np.random.default_rng(11)
    d, dv = 4, 5
    q = rng.normal(size=d) * 2.0
    k_group = rng.normal(size=d)
    K_other = rng.normal(size=(3, d))
    V_group = rng.normal(size=(3, dv))       # three original positions in the group
    V_other = rng.normal(size=(3, dv))
    E = rng.normal(size=dv)

    def expanded_loss(Kx):
        K_exp = np.vstack([Kx[0:1].repeat(3, axis=0), Kx[1:]])
        V_exp = np.vstack([V_group, V_other])
        return loss(q, K_exp, V_exp, E)

    K_merged = np.vstack([k_group[None], K_other])
    V_merged = np.vstack([V_group.mean(axis=0)[None], V_other])
    log_n = np.array([math.log(3.0), 0.0, 0.0, 0.0])
    for i, j in [(0, 0), (0, 1), (2, 2)]:
        H_fd = fd_hessian(expanded_loss, K_merged, i, j)
        H_or = oracle.hessian_block(q, K_merged, V_merged, E, i, j, log_n=log_n)
        np.testing.assert_allclose(H_or, H_fd, rtol=1e-4, atol=1e-6)


# ----------------------------------------------------------- reading B of the window

@pytest.mark.parametrize("seed", [0, 1])
def test_per_query_norms_are_the_mean_of_each_querys_numerical_sensitivities(seed):
    """Reading B: with several window queries, N11, N12, N22 are the means over the
    queries of the norms of that query's own sensitivity vectors (each from a finite-
    difference Hessian of its own attention-output loss, causal as the window is)."""
    n, d, W = 7, 4, 3
    rng = np.random.default_rng(50 + seed)
    K = rng.normal(size=(n, d))
    V = rng.normal(size=(n, d))
    Qw = rng.normal(size=(1, W, d)) * 2.0          # one query head, W window queries
    m = 1                                           # pair (1, 2): visible to every query
    per_q = []
    for j in range(W):
        pos = n - W + j
        q = Qw[0, j]
        Kq, Vq = K[:pos + 1].copy(), V[:pos + 1]

        def sens_vector(i, k):
            vec = np.zeros(d)
            for c in range(d):
                E = np.zeros(d)
                E[c] = 1.0
                H = fd_hessian(lambda Kx: loss(q, Kx, Vq, E), Kq, i, k)
                a = int(np.argmax(np.abs(q)))
                vec[c] = H[a, a] * d / (q[a] * q[a])
            return vec

        per_q.append([np.linalg.norm(sens_vector(m, m)), np.linalg.norm(sens_vector(m, m + 1)),
                      np.linalg.norm(sens_vector(m + 1, m + 1))])
    want = np.mean(np.array(per_q), axis=0)
    hs = oracle.score_head(K, V, None, n, cand_begin=m, n_recent=n - m - 2, Q_heads=Qw, W=W,
                           stats="per_query")
    np.testing.assert_allclose([hs.n11[0], hs.n12[0], hs.n22[0]], want, rtol=2e-4)


def test_per_query_norms_equal_the_mean_reading_for_one_query():
    rng = np.random.default_rng(9)
    K, V = rng.normal(size=(20, 6)), rng.normal(size=(20, 6))
    Q = rng.normal(size=(1, 1, 6)) * 2.0
    a = oracle.score_head(K, V, None, 20, 2, 1, Q, 1)
    b = oracle.score_head(K, V, None, 20, 2, 1, Q, 1, stats="per_query")
    np.testing.assert_allclose(b.n11, a.n11, rtol=1e-13)
    np.testing.assert_allclose(b.n12, a.n12, rtol=1e-13)
    np.testing.assert_allclose(b.n22, a.n22, rtol=1e-13)
    np.testing.assert_allclose(b.score, a.score, rtol=1e-12)


def test_per_query_norms_differ_from_the_mean_reading_for_several_queries():
    # norms are convex: the mean of norms is at least the norm of the mean residual,
    # and differs from it once the queries attend differently
    rng = np.random.default_rng(10)
    K, V = rng.normal(size=(40, 6)), rng.normal(size=(40, 6))
    Q = rng.normal(size=(2, 4, 6)) * 3.0
    a = oracle.score_head(K, V, None, 40, 2, 4, Q, 4)
    b = oracle.score_head(K, V, None, 40, 2, 4, Q, 4, stats="per_query")
    assert np.max(np.abs(b.n12 - a.n12) / (a.n12 + 1e-300)) > 1e-3
    with pytest.raises(ValueError):
        oracle.score_head(K, V, None, 40, 2, 4, Q, 4, stats="median")
