"""Pins of the oracle's attention-internal reward c_s = -<ghat_s, delta_o_s> and of the
credit equation on a given reward (CPU).  Besides closed forms, the whole chain is pinned
against the mathematics of a V perturbation: with a causal mixing o_s = sum_t P[s, t] v_t, a
perturbation v_t -> v_t + sigma a_t changes the output by delta_o_s = sigma sum_t P[s, t] a_t,
and the estimate built from the reward, the undiscounted credit (gamma = 1) and the
output-error equation has expectation sum_{s >= t} P[s, t] G_s = (P^T G)_t, the exact
gradient with respect to v_t when G_s is the error at the attention output."""
import numpy as np

import oracle


def test_reward_closed_forms():
    rng = np.random.default_rng(1)
    N, d, K = 7, 12, 3
    G = rng.standard_normal((N, d))
    alpha = np.array([0.5, -2.0, 3.0])
    dO = -alpha[:, None, None] * G[None]            # anti-aligned with G: c = alpha |G|^2
    c = oracle.attn_reward(G, dO)
    np.testing.assert_allclose(c, alpha[:, None] * (G * G).sum(1)[None], rtol=1e-13)
    # orthogonal to G at every token: zero reward
    Q = rng.standard_normal((K, N, d))
    Q -= ((Q * G[None]).sum(-1) / (G * G).sum(-1)[None])[..., None] * G[None]
    np.testing.assert_allclose(oracle.attn_reward(G, Q), 0.0, atol=1e-12)
    # a change at one (draw, token) only rewards that (draw, token)
    E = np.zeros((K, N, d))
    E[2, 4] = G[4]
    c = oracle.attn_reward(G, E)
    assert c[2, 4] == -(G[4] * G[4]).sum() and np.count_nonzero(c) == 1


def test_discounted_credit_special_cases():
    rng = np.random.default_rng(2)
    K, N = 3, 40
    c = rng.standard_normal((K, N))
    cu = np.array([0, 1, 17, 18, 40], dtype=np.int32)
    np.testing.assert_allclose(oracle.discounted_credit(c, cu, 0.0), c, rtol=0, atol=0)
    r1 = oracle.discounted_credit(c, cu, 1.0)
    for a, b in zip(cu[:-1], cu[1:]):
        np.testing.assert_allclose(r1[:, a:b], np.cumsum(c[:, a:b][:, ::-1], axis=1)[:, ::-1],
                                   rtol=1e-13)
    # the backward recurrence r_t = c_t + gamma r_{t+1}, restarted at segment ends
    g = 0.8
    ref = c.copy()
    ends = set(int(e) - 1 for e in cu[1:])
    for t in range(N - 2, -1, -1):
        if t not in ends:
            ref[:, t] += g * ref[:, t + 1]
    np.testing.assert_allclose(oracle.discounted_credit(c, cu, g), ref, rtol=1e-12)
    # centred losses give the loss credit
    loss = rng.standard_normal((K, N))
    np.testing.assert_allclose(oracle.discounted_credit(loss.mean(0) - loss, cu, g),
                               oracle.credit(loss, cu, g), rtol=1e-12, atol=1e-14)


def test_v_perturbation_estimate_has_the_backprop_expectation():
    N, d, K, sigma, seed = 6, 4, 40000, 1e-3, 0x5EED00A7
    rng = np.random.default_rng(3)
    P = np.tril(rng.random((N, N)) + 0.1)
    P /= P.sum(1, keepdims=True)                   # causal, rows sum to one
    G = rng.standard_normal((N, d))                # error at the attention output
    a = oracle.noise(seed, 2, N, d, K)             # [K, N, d] noise on the values
    dO = sigma * np.einsum("st,itk->isk", P, a)    # change of the attention output
    c = oracle.attn_reward(G, dO)
    cu = np.array([0, N], dtype=np.int32)
    r = oracle.discounted_credit(c, cu, 1.0)
    g = oracle.output_error(r, K, sigma, seed, d, layer_id=2)
    exact = P.T @ G
    # per-draw terms X_i = -(1/sigma) r_i a_i: g is their mean; 5 standard errors per element
    X = -(r[:, :, None] * a) / sigma
    se = X.std(axis=0, ddof=1) / np.sqrt(K)
    assert np.all(np.abs(g - exact) <= 5 * se), np.max(np.abs(g - exact) / se)
    # a mis-signed reward or a scan in the wrong direction would land far away
    assert np.abs(g - exact).max() < 0.1 * np.abs(exact).max()
