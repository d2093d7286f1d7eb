"""Pins of the oracle's optimizer steps (CPU): closed forms under a constant gradient, and
special cases that reduce to plain gradient descent."""
import numpy as np

import oracle


def test_sgd_momentum_constant_gradient_closed_form():
    rng = np.random.default_rng(1)
    W0 = rng.standard_normal(37)
    G = rng.standard_normal(37)
    lr, mu, n = 0.05, 0.9, 12
    W, m = W0.copy(), np.zeros(37)
    for _ in range(n):
        W, m = oracle.sgd_momentum(W, m, G, lr, mu)
    # m_k = G (1 - mu^k) / (1 - mu);  W_n = W_0 - lr G sum_k (1 - mu^k) / (1 - mu)
    s = sum((1 - mu ** k) / (1 - mu) for k in range(1, n + 1))
    np.testing.assert_allclose(m, G * (1 - mu ** n) / (1 - mu), rtol=1e-12)
    np.testing.assert_allclose(W, W0 - lr * G * s, rtol=1e-12, atol=1e-14)


def test_sgd_momentum_zero_is_gradient_descent_and_decay():
    W0 = np.array([1.0, -2.0, 0.5])
    G = np.array([0.1, 0.2, -0.3])
    W, m = oracle.sgd_momentum(W0, np.zeros(3), G, 0.1, 0.0)
    np.testing.assert_allclose(W, W0 - 0.1 * G, rtol=1e-15)
    W, _ = oracle.sgd_momentum(W0, np.zeros(3), np.zeros(3), 0.1, 0.9, wd=0.01)
    np.testing.assert_allclose(W, W0 * (1 - 0.1 * 0.01), rtol=1e-15)


def test_adam_constant_gradient_closed_form():
    """With a constant gradient the bias-corrected moments are exactly G and G^2, so every step
    moves W by lr G / (|G| + eps)."""
    rng = np.random.default_rng(2)
    W0 = rng.standard_normal(29)
    G = rng.standard_normal(29)
    lr, b1, b2, eps, n = 1e-3, 0.9, 0.999, 1e-8, 7
    W, m, v = W0.copy(), np.zeros(29), np.zeros(29)
    for t in range(1, n + 1):
        W, m, v = oracle.adam(W, m, v, G, lr, b1, b2, eps, t)
    np.testing.assert_allclose(m, G * (1 - b1 ** n), rtol=1e-12)
    np.testing.assert_allclose(v, G * G * (1 - b2 ** n), rtol=1e-12)
    np.testing.assert_allclose(W, W0 - n * lr * G / (np.abs(G) + eps), rtol=1e-10, atol=1e-15)


def test_adam_first_step_is_sign_descent():
    G = np.array([3.0, -1e-3, 0.0])
    W, _, _ = oracle.adam(np.zeros(3), np.zeros(3), np.zeros(3), G, 0.01, 0.9, 0.999, 1e-8, 1)
    np.testing.assert_allclose(W, [-0.01 * 3 / (3 + 1e-8), 0.01 * 1e-3 / (1e-3 + 1e-8), 0.0],
                               rtol=1e-12)
