"""Pins of the oracle's SPSA / MeZO weight-space probe (CPU), the contrast estimator.  For the
quadratic readout the two perturbed forwards differ by exact algebra:
    L_+ - L_- = 2 eps <z, G>,   L_+ + L_- - 2 L_0 = eps^2 sum_t |z x_t|^2,
with G = sum_t (W x_t - u_t) x_t^T the exact gradient, so p_j = <z_j, G> for every probe; and
the estimate (1/P) sum_j p_j z_j has expectation E[z z^T] G = s^2 G, s^2 the second moment of
the bf16-rounded normal (1 up to about 2^-16)."""
import numpy as np

import oracle
import workloads


def _layer(seed, N, d_in, d_out):
    L = workloads.custom_layer(seed, N, d_in, d_out, "bf16", 0.05)
    return L.x_f64, L.W_f64, L.u_f64


def test_directions_are_bf16_normals_in_their_own_counter_space():
    Z = oracle.spsa_directions(0x5EED0008, 3, 2, 16, 24, probe_offset=7)
    bits = (Z.astype(np.float32).view(np.uint32) & 0xFFFF)
    assert not bits.any()                                   # exactly representable in bf16
    # the same counters with the weight-space bit clear are the activation noise; rounding
    # that to bf16 must not give the directions (a separate stream)
    a = oracle.noise(0x5EED0008, 3, 16, 24, 9)[7:9]          # token = row o, draw = probe
    assert np.abs(Z - a).max() > 0.1
    n = oracle.noise(0x5EED0008, 3 | 0x80000000, 16, 24, 9)[7:9]
    np.testing.assert_allclose(Z, n, rtol=2.0**-8, atol=0)  # rounding of the same normals
    Z2 = oracle.spsa_directions(0x5EED0008, 3, 1, 16, 24, probe_offset=8)
    np.testing.assert_array_equal(Z2[0], Z[1])


def test_probe_equals_projection_on_the_exact_gradient():
    x, W, u = _layer(21, 40, 24, 16)
    P, eps, seed = 6, 1e-3, 0x5EED0009
    p, Lp, Lm = oracle.spsa_probe(x, W, u, P, eps, seed, layer_id=2, probe_offset=3)
    E = x @ W.T - u
    G = E.T @ x
    Z = oracle.spsa_directions(seed, 2, P, 16, 24, probe_offset=3)
    np.testing.assert_allclose(p, np.einsum("jok,ok->j", Z, G), rtol=1e-7,
                               atol=1e-9 * np.abs(G).sum())
    L0 = 0.5 * (E * E).sum()
    curv = np.array([(x @ Z[j].T) ** 2 for j in range(P)]).sum(axis=(1, 2))
    np.testing.assert_allclose(Lp + Lm - 2 * L0, eps * eps * curv, rtol=1e-5)


def test_estimate_is_unbiased_for_the_gradient():
    x, W, u = _layer(22, 16, 8, 6)
    P, eps, seed = 6000, 1e-2, 0x5EED000A
    p, _, _ = oracle.spsa_probe(x, W, u, P, eps, seed)
    g = oracle.spsa_estimate(p, P, 6, 8, seed)
    G = (x @ W.T - u).T @ x
    Z = oracle.spsa_directions(seed, 0, P, 6, 8)
    X = p[:, None, None] * Z                                 # per-probe terms
    se = X.std(axis=0, ddof=1) / np.sqrt(P)
    np.testing.assert_allclose(g, X.mean(axis=0), rtol=1e-10, atol=1e-12)
    assert np.all(np.abs(g - G) <= 5 * se + 1e-3 * np.abs(G)), np.max(np.abs(g - G) / se)
