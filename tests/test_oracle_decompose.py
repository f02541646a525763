"""Pins of the decomposition oracle (oracle/decompose.py) to facts the BiLoCo
README's "Decomposition" section and the mathematics fix, independent of the
oracle's own formulas: exact recovery of a binary rank-one matrix, the
Pythagorean decrease of the residual that only the Frobenius-optimal
coefficient gives, brute-force maximisation of u^T R v over sign vectors, the
normal equations of the least-squares refit, and special cases."""

import itertools

import numpy as np
import pytest

from oracle import decompose as od


def _signs(rng, *shape):
    return (2 * rng.integers(0, 2, shape) - 1).astype(np.float64)


def test_binary_rank_one_is_recovered_exactly():
    rng = np.random.default_rng(0)
    N, K = 20, 33                                    # K odd: v . v0 is never zero
    u, v = _signs(rng, N), _signs(rng, K)
    W = 0.37 * np.outer(u, v)
    for T in (1, 3):
        out = od.decompose(W, 1, T, _signs(rng, 1, K))
        fit = np.outer(out["U"][:, 0], out["V"][:, 0]) * out["alpha"][0]
        assert np.max(np.abs(fit - W)) < 1e-13
        assert np.max(np.abs(out["R"])) < 1e-13
        assert abs(abs(out["alpha"][0]) - 0.37) < 1e-13


def test_deflation_decreases_the_residual_by_pythagoras():
    # ||R - a u v^T||^2 = ||R||^2 - 2 a u^T R v + a^2 N K, which equals
    # ||R||^2 - a^2 N K exactly when a is the Frobenius-optimal coefficient
    rng = np.random.default_rng(1)
    N, K, r = 48, 40, 12
    W = rng.standard_normal((N, K))
    out = od.decompose(W, r, 4, _signs(rng, r, K), refit=False)
    n = out["greedy_norms"]
    assert np.all(np.diff(n) <= 1e-12)
    drop = n[:-1] ** 2 - n[1:] ** 2
    np.testing.assert_allclose(drop, out["alpha_greedy"] ** 2 * N * K, rtol=1e-10)


def test_each_coefficient_is_frobenius_optimal():
    rng = np.random.default_rng(2)
    N, K, r = 24, 30, 5
    W = rng.standard_normal((N, K))
    R = W.copy()
    v0 = _signs(rng, r, K)
    for i in range(r):
        u, v, a = od.peel_term(R, v0[i], 3)
        f = lambda x: np.linalg.norm(R - x * np.outer(u, v))
        assert f(a) < f(a + 1e-4) and f(a) < f(a - 1e-4)
        R = R - a * np.outer(u, v)


def test_sign_steps_maximise_over_all_sign_vectors():
    # u = sign(R v) maximises u^T (R v) over every u in {+-1}^N (brute force), and
    # the alternation never lowers u^T R v
    rng = np.random.default_rng(3)
    N, K = 8, 6
    R = rng.standard_normal((N, K))
    v0 = _signs(rng, K)
    u1, v1, _ = od.peel_term(R, v0, 1)
    Rv0 = R @ od.sign_pm1(v0)
    best_u = max(itertools.product((-1.0, 1.0), repeat=N), key=lambda s: np.dot(s, Rv0))
    assert np.dot(u1, Rv0) == pytest.approx(np.dot(best_u, Rv0))
    Rtu = R.T @ u1
    best_v = max(itertools.product((-1.0, 1.0), repeat=K), key=lambda s: np.dot(s, Rtu))
    assert np.dot(v1, Rtu) == pytest.approx(np.dot(best_v, Rtu))
    vals = []
    for T in range(1, 6):
        u, v, _ = od.peel_term(R, v0, T)
        vals.append(u @ R @ v)
    assert all(b >= a - 1e-12 for a, b in zip(vals, vals[1:]))


def test_refit_satisfies_the_normal_equations():
    # the least-squares residual is orthogonal to every fitted term, and no worse
    # than the greedy one
    rng = np.random.default_rng(4)
    N, K, r = 64, 48, 10
    W = rng.standard_normal((N, K)).astype(np.float32)
    out = od.decompose(W, r, 3, _signs(rng, r, K))
    U, V, R = out["U"].astype(np.float64), out["V"].astype(np.float64), out["R"]
    inner = np.einsum("ni,nk,ki->i", U, R, V)
    assert np.max(np.abs(inner)) < 1e-9 * np.linalg.norm(W) * np.sqrt(N * K)
    assert np.linalg.norm(R) <= out["greedy_norms"][-1] + 1e-12
    # the fit is exactly W - R
    np.testing.assert_allclose((U * out["alpha"]) @ V.T, W.astype(np.float64) - R, atol=1e-12)


def test_special_cases():
    rng = np.random.default_rng(5)
    # one term: the refit coefficient is the greedy one
    W = rng.standard_normal((16, 24))
    out = od.decompose(W, 1, 2, _signs(rng, 1, 24))
    assert out["alpha"][0] == pytest.approx(out["alpha_greedy"][0], rel=1e-12)
    # a zero matrix: every sign is +1 (sign(0) = +1) and every coefficient 0; the
    # three terms repeat, so G is singular and the refit is the zero solution
    out = od.decompose(np.zeros((8, 8)), 3, 2, _signs(rng, 3, 8))
    assert np.all(out["U"] == 1) and np.all(out["V"] == 1)
    assert np.all(out["alpha_greedy"] == 0) and np.all(out["alpha"] == 0)
    assert np.all(out["R"] == 0)
    # r = 0: the residual is W itself
    W = rng.standard_normal((8, 12))
    out = od.decompose(W, 0, 2, np.zeros((0, 12)))
    np.testing.assert_array_equal(out["R"], W)
