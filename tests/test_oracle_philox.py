"""Pins of the oracle's Philox4x32-10 and of the uniforms derived from it."""
import os

import numpy as np
from scipy import stats

from oracle import philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def test_known_answer_vectors():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = philox.philox4x32_10(*v[:6])
        assert [int(o) for o in out] == v[6:]


def test_vectorised_matches_scalar():
    c0 = np.arange(50, dtype=np.uint64)
    out = philox.philox4x32_10(c0, 7, 9, 3, 0x1234, 0xABCD)
    for i in (0, 17, 49):
        one = philox.philox4x32_10(i, 7, 9, 3, 0x1234, 0xABCD)
        assert [int(o[i]) for o in out] == [int(x) for x in one]


def test_accept_uniform_range_and_uniformity():
    u = philox.accept_uniform(seed=5, step=3, rows=np.arange(200_000))
    assert u.min() >= 0.0 and u.max() < 1.0
    # 24-bit grid: u * 2^24 is an integer
    assert np.all(np.floor(u * 2 ** 24) == u * 2 ** 24)
    counts, _ = np.histogram(u, bins=100, range=(0, 1))
    assert stats.chisquare(counts).pvalue > 1e-3


def test_float_uniform_exact_and_in_open_interval():
    x = np.array([1, 2, 3, 2 ** 40, 2 ** 63, 2 ** 64 - 1, 0xDEADBEEFCAFEBABE], dtype=np.uint64)
    V = philox._float_uniform(x)
    # known closed forms: x = 1 -> 2^-64, x = 2^63 -> 1/2, x = 2^64-1 -> 1 - 2^-24
    assert V[0] == 2.0 ** -64 and V[1] == 2.0 ** -63 and V[2] == 3 * 2.0 ** -64
    assert V[3] == 2.0 ** -24 and V[4] == 0.5 and V[5] == 1 - 2.0 ** -24
    # truncation to 24 significant bits
    xv = 0xDEADBEEFCAFEBABE
    assert V[6] == (xv >> 40) * 2.0 ** -24
    assert philox._float_uniform(np.array([0], np.uint64))[0] == 0.0
    # each value is float32-exact
    assert np.all(V.astype(np.float32).astype(np.float64) == V)


def test_token_uniform_rows_match_single_and_are_exponential():
    r = philox.token_uniform_rows(11, 2, [0, 5], 1, 4096)
    one = philox.token_uniform(11, 2, 5, 1, np.arange(4096))
    assert np.array_equal(r[1], one)
    assert not np.array_equal(r[0], r[1])
    # E = -ln(1 - V) ~ Exp(1)
    E = -np.log1p(-philox.token_uniform_rows(3, 0, np.arange(64), 2, 4096).ravel())
    assert abs(E.mean() - 1.0) < 0.01
    assert stats.kstest(E, "expon").pvalue > 1e-3


def test_purpose_and_step_separate_streams():
    a = philox.token_uniform(1, 0, 0, 1, np.arange(64))
    b = philox.token_uniform(1, 0, 0, 2, np.arange(64))
    c = philox.token_uniform(1, 1, 0, 1, np.arange(64))
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
