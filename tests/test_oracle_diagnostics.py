"""Pins of the oracle's mask diagnostics and candidate-index codec (NEXT row f2).

Checked against closed forms and hand-built cases: a peaked or uniform distribution's
maximum probability, the magnitude mask's own L1 (ratio 1), explicit base-C digits, the
bits-per-weight figures (the page's 0.65 bits/param is the 2:4 entropy bound log2(6)/4)."""
import math

import numpy as np
import pytest

from _golden import keyed


def test_mask_diff_counts(orc):
    a = np.array([0, 1, 2, 3, 4, 5, 0], np.uint8)
    b = np.array([0, 1, 5, 3, 0, 5, 1], np.uint8)
    assert orc.mask_diff(a, b) == 3 and orc.mask_diff(a, a) == 0


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
def test_max_probability_limits(orc, n, m):
    C = orc.num_candidates(n, m)
    W = np.ones((3, m))
    pi = np.zeros((3, C), np.float32)
    pi[1, 0] = 100.0                          # one-hot
    pi[2, :2] = 1.0                           # two-way tie at the top
    s = orc.mask_stats(n, m, W, pi, kappa=1.0)
    expect = 1.0 / C + 1.0 + math.e / (2 * math.e + (C - 2))
    assert abs(s[0] - expect) < 1e-12


@pytest.mark.parametrize("n,m", [(2, 4), (4, 8)])
def test_kept_l1_and_agreement(orc, n, m):
    """Logits set to the magnitude prior (deterministic mode) keep exactly the magnitude
    mask: L1 ratio 1 and every block agrees; the opposite candidate keeps the smallest."""
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, size=(400, m))
    pi, pidx, _ = orc.prior_init(n, m, W, np.arange(400), 3.0, 0.0, 0)
    s = orc.mask_stats(n, m, W, pi.astype(np.float32), kappa=100.0)
    assert s[1] == s[2] and s[3] == 400
    topn = np.sort(np.abs(W), 1)[:, ::-1][:, :n].sum()
    assert abs(s[2] - topn) < 1e-12 * topn
    s2 = orc.mask_stats(n, m, W, -pi.astype(np.float32), kappa=100.0)
    assert s2[1] < s2[2] and s2[3] == 0


def test_codec_digits_and_rate(orc):
    idx = np.array([5, 0, 1] + [0] * 9 + [3], np.uint8)   # 13 indices -> 2 words
    w = orc.encode_candidates(2, 4, idx)
    assert list(w) == [5 + 0 * 6 + 1 * 36, 3]
    assert 6**12 < 2**32 and 70**5 < 2**32
    rng = np.random.default_rng(1)
    for n, m, C, D in [(2, 4, 6, 12), (4, 8, 70, 5)]:
        k = rng.integers(0, C, size=1001).astype(np.uint8)
        enc = orc.encode_candidates(n, m, k)
        assert enc.size == (1001 + D - 1) // D
        np.testing.assert_array_equal(orc.decode_candidates(n, m, enc, 1001), k)
    page = float(keyed("paper_figures.txt")["mask_bits_per_param_2of4"][0])
    assert 32 / (12 * 4) - page < 0.02 and round(math.log2(6) / 4, 2) == page
