"""Pins of the oracle's noise generator (CPU only).

The Dust page (koala.ai.kr, "Dust: 역전파 없이 트랜스포머를 사전학습하다", section "신용 할당")
only fixes a_t ~ N(0, I), independent per token and draw.  The generator is Philox4x32-10
(Salmon et al., SC'11) with Box-Muller.  Philox words are pinned by the published
known-answer vectors (tests/golden/philox_kat.json) and by cross-implementation against
PyTorch's header-only CPU engine (called, not copied).  Normals are pinned by exact invariants
of Box-Muller and by distribution tests.
"""
import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def torch_philox(tmp_path_factory):
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    exe = str(tmp_path_factory.mktemp("tp") / "torch_philox_probe")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-I", inc, "-o", exe,
                           os.path.join(HERE, "torch_philox_probe.cpp")])

    def run(ctr: np.ndarray, key: np.ndarray) -> np.ndarray:
        lines = "\n".join(" ".join(str(int(v)) for v in list(c) + list(k))
                          for c, k in zip(ctr, key)) + "\n"
        out = subprocess.run([exe], input=lines, capture_output=True, text=True, check=True)
        return np.array([[int(v) for v in ln.split()] for ln in out.stdout.strip().splitlines()],
                        dtype=np.uint64).astype(np.uint32)
    return run


def kat_vectors():
    """The published Philox4x32-10 known-answer vectors: [(ctr[4], key[2], out[4])]."""
    with open(os.path.join(HERE, "golden", "philox_kat.json")) as f:
        d = json.load(f)
    return [(np.array([int(v, 16) for v in e["ctr"]], dtype=np.uint32),
             np.array([int(v, 16) for v in e["key"]], dtype=np.uint32),
             np.array([int(v, 16) for v in e["out"]], dtype=np.uint32)) for e in d["vectors"]]


def test_philox_words_match_published_known_answers():
    vecs = kat_vectors()
    assert len(vecs) == 3
    for ctr, key, out in vecs:
        assert np.array_equal(oracle.philox4x32_10(ctr, key), out), (ctr, key)
        # the batch route under the 64-bit seed (key0 = low word, key1 = high word)
        seed = int(key[0]) | (int(key[1]) << 32)
        words, _ = oracle.philox_batch(ctr.reshape(1, 4), seed, want_normals=False)
        assert np.array_equal(words[0], out)


def test_philox_words_match_independent_implementation(torch_philox):
    rng = np.random.default_rng(7)
    n = 4000
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    ctr[:500] &= np.uint32(0xFFFF)          # small counters
    ctr[500:1000] |= np.uint32(0x80000000)  # all words >= 2^31
    key = rng.integers(0, 2**32, size=(n, 2), dtype=np.uint64).astype(np.uint32)
    key[:100] = 0
    ref = torch_philox(ctr, key)
    mine = np.stack([oracle.philox4x32_10(c, k) for c, k in zip(ctr, key)])
    assert np.array_equal(mine, ref)


def test_philox_batch_matches_single_blocks():
    rng = np.random.default_rng(8)
    ctr = rng.integers(0, 2**32, size=(257, 4), dtype=np.uint64).astype(np.uint32)
    seed = 0x123456789ABCDEF0
    words, _ = oracle.philox_batch(ctr, seed, want_normals=False)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for j in range(0, 257, 16):
        assert np.array_equal(words[j], oracle.philox4x32_10(ctr[j], key))


def test_uniform_conversion_exact():
    assert oracle.uniform(0) == 2.0**-24
    assert oracle.uniform(0xFFFFFFFF) == 1.0 - 2.0**-24
    assert oracle.uniform(0x1FF) == oracle.uniform(0)           # low 9 bits dropped
    assert oracle.uniform(0x200) == 3 * 2.0**-24
    assert oracle.uniform(0x80000000) == 0.5 + 2.0**-24
    # every value is exactly a float32 (24 significant bits) and strictly inside (0, 1)
    rng = np.random.default_rng(9)
    for w in rng.integers(0, 2**32, size=2000, dtype=np.uint64):
        u = oracle.uniform(int(w))
        assert 0.0 < u < 1.0
        assert float(np.float32(u)) == u


def test_box_muller_invariants():
    """rho^2 = -2 ln u(w0) and the angle is 2 pi u(w1), for both pairs of each block."""
    rng = np.random.default_rng(10)
    ctr = rng.integers(0, 2**32, size=(20000, 4), dtype=np.uint64).astype(np.uint32)
    words, z = oracle.philox_batch(ctr, 0x5EED0001)
    for p in range(2):
        u0 = ((words[:, 2 * p] >> 9).astype(np.float64) * 2 + 1) * 2.0**-24
        u1 = ((words[:, 2 * p + 1] >> 9).astype(np.float64) * 2 + 1) * 2.0**-24
        r2 = z[:, 2 * p] ** 2 + z[:, 2 * p + 1] ** 2
        np.testing.assert_allclose(r2, -2.0 * np.log(u0), rtol=1e-12, atol=1e-14)
        ang = np.mod(np.arctan2(z[:, 2 * p + 1], z[:, 2 * p]), 2 * np.pi)
        d = np.abs(ang - 2 * np.pi * u1)
        d = np.minimum(d, 2 * np.pi - d)
        big = r2 > 1e-6
        assert np.max(d[big]) < 1e-9


def test_normals_distribution():
    """mean, variance, KS against the standard normal CDF, and no cross-channel correlation."""
    from scipy import stats
    n_blocks = 1 << 20          # 2^22 normals
    q = np.arange(n_blocks, dtype=np.uint64)
    ctr = np.stack([(q % 997).astype(np.uint32), (q // 997).astype(np.uint32),
                    np.full(n_blocks, 3, np.uint32), np.full(n_blocks, 1, np.uint32)], axis=-1)
    _, z = oracle.philox_batch(ctr, 0x5EED0002)
    flat = z.reshape(-1)
    n = flat.size
    assert abs(flat.mean()) < 5.0 / math.sqrt(n)
    assert abs(flat.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    assert stats.kstest(flat, "norm").pvalue > 1e-3
    c = np.corrcoef(z.T)
    assert np.max(np.abs(c - np.eye(4))) < 5.0 / math.sqrt(n_blocks)
    assert np.max(np.abs(flat)) <= math.sqrt(2 * 24 * math.log(2)) + 1e-12


def test_normals_distribution_at_2_28():
    """2^28 normals, streamed: |mean| < 5/sqrt(n), variance within 5 standard errors of 1, and
    the Kolmogorov-Smirnov distance to the standard normal CDF, evaluated at the 2^16 + 1 edges
    of a histogram over [-6, 6) (a lower bound of the exact distance), below the 1e-3 critical
    value 1.9495/sqrt(n)."""
    from scipy import special
    n_blocks, n_bins, lo, hi = 1 << 26, 1 << 16, -6.0, 6.0
    sums, hist = oracle.normal_stats(0x5EED0002, 3, 1, n_blocks, n_bins, lo, hi)
    n = 4 * n_blocks
    assert int(hist.sum()) == n
    mean = sums[0] / n
    var = sums[1] / n - mean * mean
    assert abs(mean) < 5.0 / math.sqrt(n), mean
    assert abs(var - 1.0) < 5.0 * math.sqrt(2.0 / n), var
    edges = np.linspace(lo, hi, n_bins + 1)
    F = np.cumsum(hist)[: n_bins + 1] / n
    D = float(np.max(np.abs(F - special.ndtr(edges))))
    assert D < 1.9495 / math.sqrt(n), D
    assert hist[0] == 0 and hist[-1] == 0          # |z| <= sqrt(48 ln 2) = 5.77 < 6


def test_noise_mapping_channels_tokens_draws_layers():
    """noise[i, t, o] is normal o & 3 of the block with counter (o >> 2, t, i, layer)."""
    seed = 0x5EED0005
    a = oracle.noise(seed, layer_id=7, N=5, d_out=12, K=3, draw_offset=100, token_offset=2**31)
    for (i, t, o) in [(0, 0, 0), (2, 4, 11), (1, 3, 6), (0, 2, 9)]:
        z = np.zeros(4)
        words, zz = oracle.philox_batch(np.array([[o >> 2, 2**31 + t, 100 + i, 7]],
                                                 dtype=np.uint32), seed)
        assert a[i, t, o] == zz[0, o & 3]
    # different layers, draws, tokens give different noise
    b = oracle.noise(seed, layer_id=8, N=5, d_out=12, K=3, draw_offset=100, token_offset=2**31)
    assert not np.allclose(a, b)
