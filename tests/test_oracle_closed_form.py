"""Pins of the oracle's merge weights and scores.

The KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程")
states the second-order pair objective (§数学主线二) and the forward-only merged
Key (§数学主线四). The oracle's weights must equal a numerical minimiser of that
objective, its score the objective's minimum value, and its forward-only form
must follow from the Hessian form under the pages' angle relation.
"""

import numpy as np
import pytest
from scipy.optimize import minimize

import oracle


def _objective(k, a, b, n11, n12, n22):
    # the pages' scalar objective with the forward-only effective scalars (N11, -N12, N22)
    return oracle.pair_objective(k, a, b, n11, -n12, n22)


@pytest.mark.parametrize("seed", range(6))
def test_weights_and_score_match_numerical_minimiser(seed):
    rng = np.random.default_rng(seed)
    d = 8
    a, b = rng.normal(size=d), rng.normal(size=d)
    n11, n22 = rng.uniform(0.1, 2.0, size=2)
    n12 = rng.uniform(0.0, 0.45) * min(n11, n22) * (1 if seed % 2 else 3)
    w_b, score, degen, D = oracle.weight_and_score(n11, n12, n22, a, b)
    assert not degen and D > 0
    res = minimize(lambda k: _objective(k, a, b, n11, n12, n22), rng.normal(size=d),
                   method="BFGS", options={"gtol": 1e-12})
    k_num = res.x
    np.testing.assert_allclose(a + w_b * (b - a), k_num, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(score, res.fun, rtol=1e-7, atol=1e-10)


def test_score_can_be_negative_and_still_minimum():
    # N12 large relative to sqrt(N11 N22) but D > 0: the minimum is negative
    a, b = np.zeros(3), np.array([1.0, 0.0, 0.0])
    n11, n12, n22 = 1.0, 2.2, 4.0      # N12^2 > N11 N22, D = 0.6
    w_b, score, degen, _ = oracle.weight_and_score(n11, n12, n22, a, b)
    assert not degen and score < 0
    k = a + w_b * (b - a)
    np.testing.assert_allclose(score, _objective(k, a, b, n11, n12, n22), rtol=1e-12)
    for t in np.linspace(-3, 3, 61):
        assert _objective(k + t * np.array([0.3, -0.2, 0.5]), a, b, n11, n12, n22) >= score - 1e-12


def test_equal_self_terms_without_coupling_reduce_to_plain_average():
    """N12 = 0 and N11 = N22: the merged key is (k_m + k_m1) / 2, the plain
    average of §数学主线二."""
    rng = np.random.default_rng(3)
    a, b = rng.normal(size=5), rng.normal(size=5)
    w_b, _, degen, _ = oracle.weight_and_score(0.7, 0.0, 0.7, a, b)
    assert not degen
    np.testing.assert_allclose(a + w_b * (b - a), (a + b) / 2, rtol=0, atol=1e-15)


@pytest.mark.parametrize("lam", [0.3, 1.0, 5.0, -2.0])
def test_hessian_form_with_forward_scalars_equals_forward_only_form(lam):
    rng = np.random.default_rng(4)
    a, b = rng.normal(size=6), rng.normal(size=6)
    n11, n12, n22 = 1.3, 0.2, 0.6
    k_g = oracle.merged_key_hessian_form(lam * n11, -lam * n12, lam * n22, a, b)
    w_m, w_m1 = oracle.forward_only_weights(n11, n12, n22)
    np.testing.assert_allclose(w_m + w_m1, 1.0, rtol=1e-15)
    np.testing.assert_allclose(k_g, w_m * a + w_m1 * b, rtol=1e-13)
    w_b, _, _, _ = oracle.weight_and_score(n11, n12, n22, a, b)
    np.testing.assert_allclose(a + w_b * (b - a), w_m * a + w_m1 * b, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("seed", range(4))
def test_angle_relation_eliminates_E(seed):
    """If cos(E,c11) = cos(E,c22) = -cos(E,c12), the exact scalars g_ij = E^T c_ij
    of §数学主线四 give the same merged key as the forward-only norms.

    c12 lies along (v_m - o) + (v_m1 - o), so the relation holds exactly only when
    the two residuals are parallel; that case is built here (alpha < 1/2 keeps
    c11 and c22 pointing the same way)."""
    rng = np.random.default_rng(10 + seed)
    d = 7
    alpha_m, alpha_m1 = rng.uniform(0.01, 0.3, size=2)
    o, x = rng.normal(size=(2, d))
    v_m, v_m1 = o + x, o + rng.uniform(0.2, 3.0) * x
    c11, c22, c12 = oracle.forward_vectors(alpha_m, alpha_m1, v_m, v_m1, o)
    E = rng.normal(size=d)
    cos = lambda u: (E @ u) / (np.linalg.norm(E) * np.linalg.norm(u))  # noqa: E731
    np.testing.assert_allclose([cos(c11), cos(c22)], [-cos(c12)] * 2, rtol=1e-12)
    g11, g22, g12 = E @ c11, E @ c22, E @ c12
    a, b = rng.normal(size=(2, 5))
    k_exact = oracle.merged_key_hessian_form(g11, g12, g22, a, b)
    w_m, w_m1 = oracle.forward_only_weights(np.linalg.norm(c11), np.linalg.norm(c12),
                                            np.linalg.norm(c22))
    np.testing.assert_allclose(k_exact, w_m * a + w_m1 * b, rtol=1e-10, atol=1e-12)


def test_degenerate_pairs_use_the_average_scored_by_the_objective():
    rng = np.random.default_rng(5)
    a, b = rng.normal(size=4), rng.normal(size=4)
    cases = [(0.2, 0.5, 0.3),            # D < 0: concave, no minimiser
             (0.0, 0.0, 0.0),            # all zero (attention underflow)
             (1.0, 0.5, 0.0),            # D = 0
             (np.nan, 0.1, 0.2)]         # non-finite term
    for n11, n12, n22 in cases:
        w_b, score, degen, _ = oracle.weight_and_score(n11, n12, n22, a, b)
        assert degen
        assert w_b == 0.5
        if np.isfinite(n11):
            np.testing.assert_allclose(score, _objective((a + b) / 2, a, b, n11, n12, n22),
                                       rtol=1e-12, atol=1e-15)


def test_identical_keys_merge_to_themselves_exactly():
    k = np.array([0.1, -2.5, 3.75, 1e-3])
    K = np.vstack([k, k, k + 1, k + 1])
    V = np.arange(16, dtype=np.float64).reshape(4, 4)
    m = oracle.merge_compact_head(K, V, None, 4, 0, 0, np.array([True, True]), np.array([0.731, 5.2]))
    assert np.array_equal(m.K[0], k)
    assert np.array_equal(m.K[1], k + 1)


def test_merged_keys_of_a_scored_head_are_objective_minimisers():
    """score_head -> select all -> merge_compact_head: each merged key is the
    numerical minimiser of its own pair's objective."""
    rng = np.random.default_rng(21)
    length, d = 24, 5
    K = rng.normal(size=(length, d))
    V = rng.normal(size=(length, d))
    Q = rng.normal(size=(2, 4, d)) * 3
    hs = oracle.score_head(K, V, None, length, 2, 4, Q, 4)
    P = hs.score.shape[0]
    m = oracle.merge_compact_head(K, V, None, length, 2, 4, np.ones(P, bool), hs.w_b)
    for p in range(P):
        a, b = K[2 + 2 * p], K[3 + 2 * p]
        if hs.degenerate[p]:
            np.testing.assert_allclose(m.k_merged[p], (a + b) / 2, rtol=1e-14)
            continue
        res = minimize(lambda k: _objective(k, a, b, hs.n11[p], hs.n12[p], hs.n22[p]), np.zeros(d),
                       method="BFGS", options={"gtol": 1e-14})
        np.testing.assert_allclose(m.k_merged[p], res.x, rtol=1e-5, atol=1e-7)
        np.testing.assert_allclose(m.K[m.out_offset[p]], res.x, rtol=1e-5, atol=1e-7)


# ----------------------------------------------------------------- diagonal-only ablation

def _diagonal_objective(k, a, b, n11, n22):
    # the objective without the coupling term, written out by hand
    return n11 * np.sum((k - a) ** 2) + n22 * np.sum((k - b) ** 2)


@pytest.mark.parametrize("seed", range(5))
def test_diagonal_form_matches_numerical_minimiser(seed):
    """form="diagonal" (g12 = 0): weight and score are the minimiser and minimum of
    N11 |k - k_a|^2 + N22 |k - k_b|^2, whatever N12 is."""
    rng = np.random.default_rng(100 + seed)
    d = 6
    a, b = rng.normal(size=d), rng.normal(size=d)
    n11, n22 = rng.uniform(0.05, 3.0, size=2)
    n12 = rng.uniform(0.0, 2.0)
    w_b, score, degen, D = oracle.weight_and_score(n11, n12, n22, a, b, form="diagonal")
    assert not degen and D == pytest.approx(n11 + n22)
    res = minimize(lambda k: _diagonal_objective(k, a, b, n11, n22), rng.normal(size=d),
                   method="BFGS", options={"gtol": 1e-12})
    np.testing.assert_allclose(a + w_b * (b - a), res.x, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(score, res.fun, rtol=1e-7, atol=1e-10)


@pytest.mark.parametrize("seed", range(5))
def test_full_form_never_loses_to_diagonal_on_the_full_objective(seed):
    """The full form minimises the coupled objective, so the diagonal form's merged key
    can only do as well or worse on it (the quantity the ablation measures)."""
    rng = np.random.default_rng(200 + seed)
    d = 16
    a, b = rng.normal(size=(64, d)), rng.normal(size=(64, d))
    n11, n22 = rng.uniform(0.05, 2.0, size=(2, 64))
    n12 = rng.uniform(0.0, 0.45, size=64) * np.minimum(n11, n22)
    w_f, s_f, deg_f, _ = oracle.weight_and_score(n11, n12, n22, a, b)
    w_d, _, deg_d, _ = oracle.weight_and_score(n11, n12, n22, a, b, form="diagonal")
    assert not deg_f.any() and not deg_d.any()
    for i in range(64):
        f_full_at_diag = _objective(a[i] + w_d[i] * (b[i] - a[i]), a[i], b[i], n11[i], n12[i], n22[i])
        assert s_f[i] <= f_full_at_diag + 1e-12 * max(1.0, abs(f_full_at_diag))
    # and with some coupling present the diagonal key is strictly worse somewhere
    assert np.any(np.abs(w_f - w_d) > 1e-6)


def test_diagonal_form_equals_full_form_without_coupling():
    rng = np.random.default_rng(7)
    a, b = rng.normal(size=(10, 4)), rng.normal(size=(10, 4))
    n11, n22 = rng.uniform(0.1, 2.0, size=(2, 10))
    full = oracle.weight_and_score(n11, np.zeros(10), n22, a, b)
    diag = oracle.weight_and_score(n11, np.zeros(10), n22, a, b, form="diagonal")
    np.testing.assert_allclose(full[0], diag[0], rtol=1e-15)
    np.testing.assert_allclose(full[1], diag[1], rtol=1e-15)


def test_diagonal_form_degenerate_pair_is_the_plain_average():
    a, b = np.zeros(3), np.ones(3)
    w_b, score, degen, _ = oracle.weight_and_score(0.0, 0.3, 0.0, a, b, form="diagonal")
    assert degen and w_b == 0.5 and score == 0.0
    with pytest.raises(ValueError):
        oracle.weight_and_score(1.0, 0.0, 1.0, a, b, form="cosine")
