"""Pins of the oracle's candidate tables, random-number generator and noise transform.

None of these compare the oracle with itself: the candidate set is checked against the page's
listing and combinatorial counts, Philox against its published known answers, the bit
slicing against big-integer arithmetic, nlog's table against 50-digit logarithms, and the noise
against the Gumbel distribution's closed-form moments and the Gumbel-Max theorem.
"""
import math
from decimal import Decimal, getcontext
from itertools import combinations

import numpy as np
import pytest

from _golden import keyed, rows


# ---------------------------------------------------------------- candidate sets (Eq.2)

def test_candidates_2of4_match_page_listing(orc):
    expected = np.array([[int(v) for v in r] for r in rows("candidates_2of4.txt")], np.uint8)
    got = orc.candidates(2, 4)
    assert got.shape == (6, 4)
    np.testing.assert_array_equal(got, expected)
    # C(4,2) = 6 candidates, each keeping exactly N = 2 weights, all distinct
    assert math.comb(4, 2) == 6
    assert (got.sum(1) == 2).all()
    assert len({tuple(r) for r in got}) == 6


def test_candidates_4of8_lexicographic_subsets(orc):
    got = orc.candidates(4, 8)
    assert got.shape == (math.comb(8, 4), 8) == (70, 8)
    subsets = [tuple(np.flatnonzero(r)) for r in got]
    assert subsets == list(combinations(range(8), 4))
    # every position is kept by C(7,3) = 35 candidates
    assert (got.sum(0) == math.comb(7, 3)).all()


def test_unsupported_pattern_rejected(orc):
    assert orc.num_candidates(3, 4) == 0
    with pytest.raises(ValueError):
        orc.candidates(1, 4)


# ---------------------------------------------------------------- Philox4x32-10

def test_philox_known_answers(orc):
    for r in rows("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in r]
        out = orc.philox4x32_10(v[0:4], v[4:6])
        assert [int(x) for x in out] == v[6:10]


def test_fields21_are_bit_slices_of_the_128bit_word(orc):
    rng = np.random.default_rng(7)
    for _ in range(200):
        w = rng.integers(0, 2**32, size=4, dtype=np.uint64).astype(np.uint32)
        big = sum(int(w[i]) << (32 * i) for i in range(4))
        expect = [(big >> (21 * f)) & ((1 << 21) - 1) for f in range(6)]
        assert [int(x) for x in orc.fields21(w)] == expect


def test_noise_counter_layout(orc):
    """eps for candidate c of block gid at step s is field c%6 of Philox(counter =
    (gid lo, gid hi, s, c//6), key = (seed lo, seed hi))."""
    seed, step = 0x1234_5678_9ABC_DEF0, 17
    gids = np.array([0, 1, 2**32 + 5, 2**40 + 3], np.uint64)
    for n, m in [(2, 4), (4, 8)]:
        C = orc.num_candidates(n, m)
        eps, _ = orc.noise(n, m, seed, step, gids)
        for b, gid in enumerate(gids):
            gid = int(gid)
            for c in range(C):
                words = orc.philox4x32_10([gid & 0xFFFFFFFF, gid >> 32, step, c // 6],
                                          [seed & 0xFFFFFFFF, seed >> 32])
                big = sum(int(words[i]) << (32 * i) for i in range(4))
                k = (big >> (21 * (c % 6))) & ((1 << 21) - 1)
                assert eps[b, c] == np.float32((2 * k + 1) / 2.0**22)


def test_uniforms_open_interval_and_uniform(orc):
    gids = np.arange(200_000, dtype=np.uint64)
    eps, _ = orc.noise(2, 4, seed=3, step=0, gids=gids)
    e = eps.ravel().astype(np.float64)
    assert e.min() > 0.0 and e.max() < 1.0
    # every value sits on the (2k+1) 2^-22 grid
    k2 = e * 2.0**22
    assert np.all(k2 == np.round(k2)) and np.all(np.round(k2) % 2 == 1)
    # chi-square over 64 equal bins: 63 dof, mean 63, sd ~11.2 -> 6 sd bound
    counts, _ = np.histogram(e, bins=64, range=(0.0, 1.0))
    expected = e.size / 64
    chi2 = ((counts - expected) ** 2 / expected).sum()
    assert chi2 < 63 + 6 * math.sqrt(2 * 63)
    # no correlation between candidates of a block or neighbouring blocks
    c = np.corrcoef(eps[:, 0], eps[:, 5])[0, 1]
    assert abs(c) < 5 / math.sqrt(len(gids))
    c = np.corrcoef(eps[:-1, 2], eps[1:, 2])[0, 1]
    assert abs(c) < 5 / math.sqrt(len(gids))


# ---------------------------------------------------------------- nlog

def _ulp32(x):
    x = np.float32(abs(x))
    return float(np.spacing(x))


def test_nlog_table_correctly_rounded(orc):
    """c_j = fl32(1/F_j) and T[e][j] = fl32(e ln2 - ln c_j), checked with 50-digit
    logarithms; every T entry also lies far from an fp32 rounding boundary (more than 2^-20
    of an ulp), so any logarithm accurate to ~1e-15 rounds to the same fp32 value."""
    getcontext().prec = 50
    c, T, consts = orc.nlog_table()
    third, emin, emax = consts
    assert third == np.float32(1 / 3) and (emin, emax) == (-22, 4) and T.shape == (27, 128)
    ln2 = Decimal(2).ln()
    for j in range(128):
        F = (1 + j / 128) if j < 64 else (1 + j / 128) / 2
        assert c[j] == np.float32(1.0 / F)
        lnc = Decimal(float(c[j])).ln()
        for r, e in enumerate(range(-22, 5)):
            exact = e * ln2 - lnc
            f32 = np.float32(float(exact))
            assert T[r, j] == f32, (e, j)
            if exact != 0:
                ulp = Decimal(_ulp32(f32))
                dist = abs(exact - Decimal(float(f32)))
                assert dist < ulp / 2 - ulp * Decimal(2) ** -20, (e, j)   # not near a midpoint
            else:
                assert T[r, j] == 0.0


def test_nlog_accuracy_on_noise_domain(orc):
    """|nlog(x) - ln x| <= 2 ulp of the result (absolute 2^-30 near ln x = 0) over every
    uniform the generator can produce and a dense sweep of the second logarithm's inputs."""
    k = np.arange(2**21, dtype=np.float64)
    eps = ((2 * k + 1) / 2.0**22).astype(np.float32)
    t = np.concatenate([eps, np.geomspace(2.0**-22, 16.0, 400_000).astype(np.float32),
                        np.float32(1.0) + np.arange(-2000, 2000, dtype=np.float32) * np.float32(2**-23)])
    got = orc.nlog_array(t).astype(np.float64)
    ref = np.log(t.astype(np.float64))
    err = np.abs(got - ref)
    tol = np.maximum(2.0 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64), 2.0**-30)
    assert np.all(err <= tol), float(np.max(err / tol))


def test_noise_stays_in_nlog_domain(orc):
    """For every possible uniform, both logarithms of the noise transform take arguments in
    [2^-22, 16): eps >= 2^-22 and t = -nlog(eps) in [2^-22, 15.25]."""
    k = np.arange(2**21, dtype=np.float64)
    eps = ((2 * k + 1) / 2.0**22).astype(np.float32)
    t = -orc.nlog_array(eps)
    assert np.all(np.isfinite(t)) and t.min() >= np.float32(2.0**-22) and t.max() < 16.0
    g = -orc.nlog_array(t)
    assert np.all(np.isfinite(g))
    assert np.isnan(orc.nlog(2.0**-23)) and np.isnan(orc.nlog(32.0)) and np.isnan(orc.nlog(-1.0))


# ---------------------------------------------------------------- Gumbel noise (Eq.5)

def test_gumbel_moments(orc):
    """g = -log(-log eps) is standard Gumbel: mean = Euler's gamma, variance = pi^2/6."""
    gids = np.arange(250_000, dtype=np.uint64)
    _, g = orc.noise(2, 4, seed=11, step=5, gids=gids)
    g = g.ravel().astype(np.float64)
    n = g.size
    gamma = 0.5772156649015329
    var = math.pi**2 / 6
    assert abs(g.mean() - gamma) < 5 * math.sqrt(var / n)
    assert abs(g.var() - var) < 5 * math.sqrt(2.4 * var * var / n) + 5e-3
    # CDF exp(-exp(-x)) at a few quantiles
    for x in (-1.0, 0.0, 1.0, 3.0):
        p = math.exp(-math.exp(-x))
        assert abs((g <= x).mean() - p) < 5 * math.sqrt(p * (1 - p) / n)
    # the range allowed by the 21-bit uniforms
    assert g.min() >= -math.log(-math.log(2.0**-22)) - 1e-4
    assert g.max() <= -math.log(-math.log(1 - 2.0**-22)) + 1e-4


def test_gumbel_max_theorem(orc):
    """P(argmax_i(log p_i + g_i) = j) = p_j (Gumbel-Max trick, Eq.5): over many steps of one
    block, with tau -> 0 the soft index is one-hot at that argmax, and the frequencies follow
    softmax(kappa pi)."""
    kappa = 1.0
    pi = np.array([[0.3, -0.2, 1.1, 0.0, -1.0, 0.5]], np.float32)
    W = np.ones((1, 4))
    steps = 20_000
    counts = np.zeros(6)
    for s in range(steps):
        r = orc.sample_fwd(2, 4, W, pi, [123], kappa, 1e-4, seed=99, step=s)
        counts[np.argmax(r["y"][0])] += 1
    p = np.exp(kappa * pi[0].astype(np.float64))
    p /= p.sum()
    expected = p * steps
    chi2 = ((counts - expected) ** 2 / expected).sum()
    assert chi2 < 5 + 6 * math.sqrt(10)


def test_noise_distinct_per_step_and_seed(orc):
    gids = np.arange(1000, dtype=np.uint64)
    _, a = orc.noise(2, 4, 1, 0, gids)
    _, b = orc.noise(2, 4, 1, 1, gids)
    _, c = orc.noise(2, 4, 2, 0, gids)
    _, d = orc.noise(2, 4, 1, 0, gids)
    assert (a != b).mean() > 0.99 and (a != c).mean() > 0.99
    np.testing.assert_array_equal(a, d)
