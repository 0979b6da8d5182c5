"""Pins of the oracle's Philox4x32-10 and of the draw transforms built on it."""
import math

import numpy as np
import pytest

from conftest import read_golden_table
from oracle import philox as P
from oracle import sampler as S


def test_known_answer_vectors():
    rows = read_golden_table("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for row in rows:
        vals = [int(x, 16) for x in row]
        ctr, key, want = vals[0:4], vals[4:6], vals[6:10]
        assert list(P.philox4x32_10(ctr, key)) == want


def test_vectorised_matches_scalar():
    rng = np.random.default_rng(5)
    for _ in range(20):
        ctr = rng.integers(0, 2**32, size=4, dtype=np.uint64)
        key = rng.integers(0, 2**32, size=2, dtype=np.uint64)
        want = P.philox4x32_10([int(c) for c in ctr], [int(k) for k in key])
        got = P.philox4x32_10_np(ctr[0], ctr[1], ctr[2], ctr[3], int(key[0]), int(key[1]))
        assert [int(g) for g in got] == list(want)
    # broadcasting over a vector of first counter words
    j = np.arange(37, dtype=np.uint64)
    got = P.philox4x32_10_np(j, 7, 3, 1, 11, 13)
    for i in range(37):
        assert [int(w[i]) for w in got] == list(P.philox4x32_10((i, 7, 3, 1), (11, 13)))


def test_vocab_words_layout():
    # word v of a row comes from counter block v >> 2, output word v & 3
    words = P.vocab_words(seed=9, b=2, block=3, step=4, pos=5, tag=P.TAG_GUMBEL, vocab=10)
    for v in range(10):
        blk = P.philox4x32_10((v >> 2, P.counter_word1(5, P.TAG_GUMBEL), 4, 3), (9, 2))
        assert int(words[v]) == blk[v & 3]


def test_uniform_open_interval_and_fp32_exact():
    r = np.array([0, 1, 511, 512, 2**31, 2**32 - 1], dtype=np.uint64)
    u = P.uniform_from_word(r)
    assert np.all(u > 0) and np.all(u < 1)
    assert u[0] == 2.0 ** -24 and u[-1] == 1.0 - 2.0 ** -24
    assert np.all(u.astype(np.float32).astype(np.float64) == u)
    assert np.all((1.0 - u).astype(np.float32).astype(np.float64) == 1.0 - u)


def _draws(n, tag=P.TAG_GUMBEL):
    j = np.arange(n // 4, dtype=np.uint64)
    w = P.philox4x32_10_np(j, P.counter_word1(0, tag), 0, 0, 1234, 0)
    return np.stack(w, axis=1).reshape(-1)


def test_uniform_moments_and_chi2():
    u = P.uniform_from_word(_draws(1 << 20))
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / u.size)
    counts, _ = np.histogram(u, bins=64, range=(0, 1))
    exp = u.size / 64
    chi2 = float(np.sum((counts - exp) ** 2 / exp))
    # 63 dof: mean 63, sd ~11.2; 120 is far in the tail
    assert chi2 < 120


def test_uniform_token_histogram():
    v = 512
    t = P.token_from_word(_draws(1 << 20, P.TAG_RENOISE), v)
    assert t.min() >= 0 and t.max() < v
    counts = np.bincount(t, minlength=v)
    exp = t.size / v
    chi2 = float(np.sum((counts - exp) ** 2 / exp))
    assert chi2 < 511 + 6 * math.sqrt(2 * 511)


def test_gumbel_moments():
    g = S.gumbel_noise(P.uniform_from_word(_draws(1 << 20)))
    euler_gamma = 0.5772156649015329
    assert abs(g.mean() - euler_gamma) < 0.01
    assert abs(g.var() - math.pi ** 2 / 6) < 0.02


def test_gumbel_transform_accuracy_near_one():
    # the largest u gives the largest noise; with w = 2^-24,
    # -ln(-ln(1 - w)) = -ln(w + w^2/2 + ...) = 24 ln 2 - w/2 + O(w^2)
    w = 2.0 ** -24
    u = np.array([1.0 - w])
    assert S.gumbel_noise(u)[0] == pytest.approx(24 * math.log(2) - w / 2, abs=1e-13)
