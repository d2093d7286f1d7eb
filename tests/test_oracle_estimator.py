"""Pins of the oracle's estimator stages against facts the Dust page and mathematics fix (CPU).

Page: koala.ai.kr, "Dust: 역전파 없이 트랜스포머를 사전학습하다", section "신용 할당(credit
assignment): 보상에서 기울기까지" (noise, centred-loss, credit, output-error and
weight-estimate equations) and the remark after them that the signal grows linearly in the
number of draws while the noise grows as its square root; section "backprop과 닮은 기울기가
저절로 나타난다" for the two-parameter cosine law cos(K) = c_max / sqrt(1 + c/K).
Each check below reaches the oracle's value by a different route (an expansion, a library
routine, a special case or a statistical law) so that a dropped term, a wrong sign, index
or scale in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import workloads


def _layer(seed, N, d_in, d_out, w_std=None):
    L = workloads.custom_layer(seed, N, d_in, d_out, dtype="f32", w_std=w_std)
    return L.x_f64, L.W_f64, L.u_f64


# ----------------------------------------------------------------------------- loss
def test_loss_zero_sigma_equals_clean():
    x, W, u = _layer(1, 9, 12, 20)
    loss, clean = oracle.noisy_linear_loss(x, W, u, K=3, sigma=0.0, seed=11)
    assert np.array_equal(loss, np.broadcast_to(clean, loss.shape))
    np.testing.assert_allclose(clean, 0.5 * np.sum((x @ W.T - u) ** 2, axis=1), rtol=1e-12)


def test_loss_expansion_in_sigma():
    """l(s) - l(-s) = 2 s a.e  and  (l(s) + l(-s))/2 - clean = s^2 |a|^2 / 2  (exact algebra)."""
    x, W, u = _layer(2, 7, 16, 24)
    K, s, seed = 4, 0.03, 0x5EED0001
    lp, clean = oracle.noisy_linear_loss(x, W, u, K, s, seed, layer_id=3, draw_offset=5,
                                         token_offset=40)
    lm, _ = oracle.noisy_linear_loss(x, W, u, K, -s, seed, layer_id=3, draw_offset=5,
                                     token_offset=40)
    a = oracle.noise(seed, 3, 7, 24, K, draw_offset=5, token_offset=40)
    e = x @ W.T - u
    np.testing.assert_allclose((lp - lm) / (2 * s), np.einsum("ito,to->it", a, e),
                               rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose((lp + lm) / 2 - clean, 0.5 * s * s * np.sum(a * a, axis=2),
                               rtol=1e-7, atol=1e-12)


def test_loss_token_subset_matches_full():
    x, W, u = _layer(3, 11, 8, 8)
    full, cf = oracle.noisy_linear_loss(x, W, u, 5, 0.1, 77)
    tk = np.array([10, 0, 4])
    sub, cs = oracle.noisy_linear_loss(x, W, u, 5, 0.1, 77, tokens=tk)
    assert np.array_equal(sub, full[:, tk])
    assert np.array_equal(cs, cf[tk])


# ----------------------------------------------------------------------------- credit
def _rand_loss(seed, K, N):
    return np.random.default_rng(seed).standard_normal((K, N)) * 3.0 + 10.0


@pytest.mark.parametrize("gamma", [0.0, 0.5, 0.9, 0.99, 1.0])
def test_credit_double_sum_equals_recurrence(gamma):
    cu = workloads.random_segments(4, 300, 1, 70)
    loss = _rand_loss(5, 6, 300)
    a = oracle.credit(loss, cu, gamma)
    b = oracle.credit(loss, cu, gamma, route="recurrence")
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_credit_gamma_zero_is_centred_loss():
    cu = np.array([0, 50, 51, 120], dtype=np.int32)
    loss = _rand_loss(6, 7, 120)
    r = oracle.credit(loss, cu, 0.0)
    np.testing.assert_allclose(r, loss.mean(axis=0, keepdims=True) - loss, rtol=0, atol=1e-13)


def test_credit_gamma_one_is_segment_suffix_sum():
    cu = np.array([0, 1, 40, 41, 97, 128], dtype=np.int32)
    loss = _rand_loss(7, 4, 128)
    c = loss.mean(axis=0, keepdims=True) - loss
    r = oracle.credit(loss, cu, 1.0)
    for s in range(len(cu) - 1):
        lo, hi = cu[s], cu[s + 1]
        ref = np.flip(np.cumsum(np.flip(c[:, lo:hi], axis=1), axis=1), axis=1)
        np.testing.assert_allclose(r[:, lo:hi], ref, rtol=1e-12, atol=1e-12)


def test_credit_invariants():
    cu = workloads.random_segments(8, 500, 1, 90)
    loss = _rand_loss(9, 8, 500)
    r = oracle.credit(loss, cu, 0.9)
    # the centred losses sum to zero over draws, and the credit is linear in them
    np.testing.assert_allclose(r.sum(axis=0), 0.0, atol=1e-10)
    # the last token of a segment gets its own centred loss only (no credit crosses segments)
    c = loss.mean(axis=0, keepdims=True) - loss
    ends = cu[1:] - 1
    np.testing.assert_allclose(r[:, ends], c[:, ends], rtol=0, atol=1e-13)
    # a constant shift of one token's loss over all draws changes nothing
    loss2 = loss.copy()
    loss2[:, 17] += 123.0
    np.testing.assert_allclose(oracle.credit(loss2, cu, 0.9), r, atol=1e-10)


def test_credit_single_token_segments_and_whole_stream():
    loss = _rand_loss(10, 3, 64)
    cu_single = np.arange(65, dtype=np.int32)
    c = loss.mean(axis=0, keepdims=True) - loss
    np.testing.assert_allclose(oracle.credit(loss, cu_single, 0.99), c, atol=1e-13)
    cu_whole = np.array([0, 64], dtype=np.int32)
    r = oracle.credit(loss, cu_whole, 0.5)
    t = 10
    ref = sum(0.5 ** (s - t) * c[:, s] for s in range(t, 64))
    np.testing.assert_allclose(r[:, t], ref, rtol=1e-12)


# ----------------------------------------------------------------------------- g and G_W
def _closed_form_g(a, e, sigma, gamma, cu):
    """Expansion of the estimator for the quadratic readout l = 1/2 |e + sigma a|^2:
    g_t = sum_{s>=t, same segment} gamma^(s-t) (1/K) sum_i a_t^(i)
              [ (a_s^(i) - abar_s).e_s + sigma/2 (|a_s^(i)|^2 - m_s) ]."""
    K = a.shape[0]
    abar = a.mean(axis=0)
    m = np.sum(a * a, axis=2).mean(axis=0)
    term = np.einsum("ito,to->it", a - abar, e) + 0.5 * sigma * (np.sum(a * a, axis=2) - m)
    R = np.zeros_like(term)
    for s in range(len(cu) - 1):
        lo, hi = cu[s], cu[s + 1]
        acc = np.zeros(K)
        for t in range(hi - 1, lo - 1, -1):
            acc = term[:, t] + gamma * acc
            R[:, t] = acc
    return np.einsum("ito,it->to", a, R) / K


@pytest.mark.parametrize("gamma", [0.0, 0.9])
def test_output_error_matches_quadratic_expansion(gamma):
    N, d_in, d_out, K, sigma, seed = 24, 10, 12, 16, 1e-2, 0x5EED0001
    x, W, u = _layer(11, N, d_in, d_out)
    cu = np.array([0, 9, 10, 24], dtype=np.int32)
    out = oracle.dust_layer(x, W, u, K, sigma, gamma, cu, seed, layer_id=2)
    a = oracle.noise(seed, 2, N, d_out, K)
    g_ref = _closed_form_g(a, x @ W.T - u, sigma, gamma, cu)
    np.testing.assert_allclose(out["g"], g_ref, rtol=1e-8, atol=1e-10 * np.abs(g_ref).max())


def test_output_error_gamma_zero_sample_covariance():
    """gamma = 0: g_t = S_t e_t + sigma/(2K) sum_i (|a_t^(i)|^2 - m_t) a_t^(i), S_t the
    self-inclusive sample covariance of the draws (numpy's biased covariance)."""
    N, d, K, sigma, seed = 6, 8, 32, 1e-3, 0x5EED0003
    x, W, u = _layer(12, N, d, d)
    cu = np.array([0, N], dtype=np.int32)
    out = oracle.dust_layer(x, W, u, K, sigma, 0.0, cu, seed)
    a = oracle.noise(seed, 0, N, d, K)
    e = x @ W.T - u
    for t in range(N):
        S = np.cov(a[:, t, :].T, bias=True)
        n2 = np.sum(a[:, t, :] ** 2, axis=1)
        ref = S @ e[t] + sigma / (2 * K) * ((n2 - n2.mean()) @ a[:, t, :])
        np.testing.assert_allclose(out["g"][t], ref, rtol=1e-8, atol=1e-12)


def test_weight_grad_equals_library_matmul():
    rng = np.random.default_rng(13)
    g = rng.standard_normal((50, 7))
    x = rng.standard_normal((50, 5))
    np.testing.assert_allclose(oracle.weight_grad(g, x), g.T @ x, rtol=1e-12, atol=1e-12)


def test_output_error_chunks_add_up():
    """Draw chunks [0, K1) and [K1, K) with the global draw offset sum to the full estimate."""
    N, d, K, K1, sigma, seed = 10, 8, 12, 5, 1e-2, 0x5EED0004
    r = np.random.default_rng(14).standard_normal((K, N))
    full = oracle.output_error(r, K, sigma, seed, d, layer_id=1)
    p0 = oracle.output_error(r[:K1], K, sigma, seed, d, layer_id=1, draw_offset=0)
    p1 = oracle.output_error(r[K1:], K, sigma, seed, d, layer_id=1, draw_offset=K1)
    np.testing.assert_allclose(p0 + p1, full, rtol=1e-12, atol=1e-14)
    sub = oracle.output_error(r, K, sigma, seed, d, layer_id=1, tokens=[3, 7], chans=[0, 5, 7])
    np.testing.assert_array_equal(sub, full[np.ix_([3, 7], [0, 5, 7])])


def test_token_sharding_with_offsets_reproduces_whole_batch():
    """Splitting the batch at a segment boundary, each shard with its global token offset,
    gives the same r, g and (summed) G_W as the whole batch."""
    N, d_in, d_out, K, sigma, gamma, seed = 40, 6, 8, 6, 1e-2, 0.9, 0x5EED0006
    x, W, u = _layer(15, N, d_in, d_out)
    cu = np.array([0, 13, 25, 40], dtype=np.int32)
    whole = oracle.dust_layer(x, W, u, K, sigma, gamma, cu, seed)
    lo = oracle.dust_layer(x[:25], W, u[:25], K, sigma, gamma, cu[:3], seed)
    hi = oracle.dust_layer(x[25:], W, u[25:], K, sigma, gamma, cu[2:] - 25, seed,
                           token_offset=25)
    np.testing.assert_allclose(np.concatenate([lo["g"], hi["g"]]), whole["g"], rtol=1e-9,
                               atol=1e-12)
    np.testing.assert_allclose(lo["G_W"] + hi["G_W"], whole["G_W"], rtol=1e-9, atol=1e-11)


# ----------------------------------------------------------------------------- statistics
def _g_vs_gradient(K, N=8, d=32, sigma=1e-4, seed=0x5EED0010):
    x, W, u = _layer(16, N, d, d)
    cu = np.arange(N + 1, dtype=np.int32)  # gamma = 0 anyway
    out = oracle.dust_layer(x, W, u, K, sigma, 0.0, cu, seed)
    e = x @ W.T - u
    return out, e, x


def test_g_converges_to_gradient_at_half_power_of_draws():
    """gamma = 0, quadratic loss: E[g_t] = ((K-1)/K) e_t with e_t = W x_t - u_t, and the error
    shrinks as K^(-1/2) (signal linear in draws, noise as the square root)."""
    Ks = [64, 256, 1024, 4096]
    errs = []
    for K in Ks:
        out, e, x = _g_vs_gradient(K)
        errs.append(np.linalg.norm(out["g"] - e) / np.linalg.norm(e))
    slope = np.polyfit(np.log(Ks), np.log(errs), 1)[0]
    assert -0.62 < slope < -0.38, (slope, errs)
    d = 32
    for K, err in zip(Ks, errs):
        assert 0.5 * math.sqrt(d / K) < err < 2.0 * math.sqrt(d / K), (K, err)
    # G_W approaches the exact gradient of the summed quadratic loss, sum_t e_t x_t^T
    GW_true = e.T @ x
    rel = np.linalg.norm(out["G_W"] - GW_true) / np.linalg.norm(GW_true)
    assert rel < 2.0 * math.sqrt(d / Ks[-1])


def test_mean_of_g_is_biased_by_self_inclusive_centring():
    """Averaged over many independent seeds, g / e -> (K-1)/K for small K."""
    K, N, d = 4, 4, 8
    x, W, u = _layer(17, N, d, d)
    e = x @ W.T - u
    cu = np.arange(N + 1, dtype=np.int32)
    acc = np.zeros_like(e)
    n_rep = 400
    for rep in range(n_rep):
        out = oracle.dust_layer(x, W, u, K, 1e-4, 0.0, cu, seed=0x1000 + rep)
        acc += out["g"]
    ratio = np.sum(acc / n_rep * e) / np.sum(e * e)
    assert abs(ratio - (K - 1) / K) < 0.05, ratio


def test_cosine_law_fits():
    """cos(g, e) over K follows c_max / sqrt(1 + c/K) within the page's RMSE bar of 0.06."""
    from scipy.optimize import curve_fit
    Ks = np.array([4, 8, 16, 32, 64, 128, 256, 512])
    cos = []
    for K in Ks:
        out, e, _ = _g_vs_gradient(int(K), N=16, d=32, seed=0x5EED0020)
        g = out["g"]
        cos.append(np.mean(np.sum(g * e, 1) / np.linalg.norm(g, axis=1) / np.linalg.norm(e, axis=1)))
    cos = np.array(cos)
    f = lambda K, cmax, c: cmax / np.sqrt(1.0 + c / K)
    (cmax, c), _ = curve_fit(f, Ks, cos, p0=(1.0, 30.0))
    rmse = np.sqrt(np.mean((f(Ks, cmax, c) - cos) ** 2))
    assert rmse <= 0.06
    assert 0.85 < cmax < 1.1
    assert 10 < c < 80  # theory for isotropic noise: about d + 1 = 33
