"""Pins of the oracle's LM-head loss (cross-entropy on cached logits with a noisy vocabulary
slab; Dust page, "간섭(interference) 줄이기").  Routes: a library log-sum-exp, the softmax
derivative of cross-entropy, shift invariance, and the slab boundaries."""
import numpy as np
from scipy.special import logsumexp, softmax

import oracle


def _logits(seed, N, V, scale=2.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((N, V)) * scale, rng.integers(0, V, size=N).astype(np.int32)


def test_clean_loss_is_library_cross_entropy():
    z, y = _logits(1, 9, 40)
    _, clean = oracle.noisy_logits_ce(z, y, 8, 16, K=2, sigma=0.1, seed=3)
    np.testing.assert_allclose(clean, logsumexp(z, axis=1) - z[np.arange(9), y], rtol=1e-13)


def test_noisy_loss_equals_logsumexp_of_shifted_logits():
    z, y = _logits(2, 7, 64)
    v0, S, K, sigma, seed = 16, 32, 3, 0.2, 0x5EED0009
    loss, _ = oracle.noisy_logits_ce(z, y, v0, S, K, sigma, seed, layer_id=5, draw_offset=2,
                                     token_offset=9)
    a = oracle.noise(seed, 5, 7, 64, K, draw_offset=2, token_offset=9)
    for i in range(K):
        zp = z.copy()
        zp[:, v0:v0 + S] += sigma * a[i][:, v0:v0 + S]
        ref = logsumexp(zp, axis=1) - zp[np.arange(7), y]
        np.testing.assert_allclose(loss[i], ref, rtol=1e-12)


def test_small_sigma_derivative_is_softmax_minus_onehot():
    """(l(s) - l(-s)) / 2s -> sum over the slab of (p_v - [v = y]) a_v as s -> 0."""
    z, y = _logits(3, 6, 48, scale=1.0)
    y[:3] = 20       # targets inside the slab ...
    y[3:] = 2        # ... and outside it
    v0, S, K, s, seed = 16, 16, 2, 1e-4, 0x5EED000A
    lp, _ = oracle.noisy_logits_ce(z, y, v0, S, K, s, seed)
    lm, _ = oracle.noisy_logits_ce(z, y, v0, S, K, -s, seed)
    a = oracle.noise(seed, 0, 6, 48, K)
    p = softmax(z, axis=1)
    onehot = np.zeros_like(p)
    onehot[np.arange(6), y] = 1.0
    d = (p - onehot)[:, v0:v0 + S]
    ref = np.einsum("tv,itv->it", d, a[:, :, v0:v0 + S])
    np.testing.assert_allclose((lp - lm) / (2 * s), ref, rtol=1e-5, atol=1e-9)


def test_shift_invariance_and_empty_slab():
    z, y = _logits(4, 5, 32)
    l1, c1 = oracle.noisy_logits_ce(z, y, 0, 32, 2, 0.3, 7)
    l2, c2 = oracle.noisy_logits_ce(z + 17.0, y, 0, 32, 2, 0.3, 7)
    np.testing.assert_allclose(l1, l2, rtol=1e-11)
    np.testing.assert_allclose(c1, c2, rtol=1e-11)
    l0, c0 = oracle.noisy_logits_ce(z, y, 8, 0, 2, 0.3, 7)     # no slab: no perturbation
    np.testing.assert_allclose(l0, np.broadcast_to(c0, l0.shape), rtol=1e-14)
