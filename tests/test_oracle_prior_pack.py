"""Pins of the oracle's mask-prior initialisation (Eq.9, Eq.10) and hard-mask packing.

Checked against: the page's similarity values and mean inner product, combinatorial overlap
counts, a brute force over candidates for the magnitude prior, the moments of N(0, 0.01),
an independent unpacker of the packed format, and the page's 0.65 bits/param figure.
"""
import math
from itertools import combinations

import numpy as np
import pytest

from _golden import keyed, rows

NM = [(2, 4), (4, 8)]


def _energy_best(S, W):
    """Brute force: candidate that keeps the largest sum of squared weights."""
    energy = (W[:, None, :] ** 2 * S[None].astype(np.float64)).sum(-1)
    return np.argmax(energy, 1)


# ---------------------------------------------------------------- Eq.9 similarity

def test_similarity_values_2of4_match_page(orc):
    table = {int(r[0]): int(r[1]) for r in rows("prior_similarity_2of4.txt") if r[0] != "mean_inner_product"}
    mean_ip = float(keyed("prior_similarity_2of4.txt")["mean_inner_product"][0])
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, size=(500, 4))
    S = orc.candidates(2, 4)
    pi, pidx, sim = orc.prior_init(2, 4, W, np.arange(500), alpha=3.0, init_std=0.0, seed=0)
    for b in range(500):
        m0 = S[pidx[b]]
        ip = (S * m0).sum(1)
        assert ip.mean() == mean_ip            # mean inner product over the candidates
        for i in range(6):
            assert sim[b, i] == table[int(ip[i])]
        # counts of +1 / 0 / -1 are 1 / 4 / 1
        assert sorted(sim[b]) == [-1, 0, 0, 0, 0, 1]


def test_similarity_4of8_overlap_counts(orc):
    """For 4:8 the overlap of a candidate with the prior is 4,3,2,1,0 for 1,16,36,16,1
    candidates; the mean inner product is N^2/M = 2, so sim runs +2..-2 with mean 0."""
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, size=(50, 8))
    _, pidx, sim = orc.prior_init(4, 8, W, np.arange(50), 3.0, 0.0, 0)
    for b in range(50):
        vals, counts = np.unique(sim[b], return_counts=True)
        assert list(vals) == [-2, -1, 0, 1, 2]
        assert list(counts) == [1, 16, 36, 16, 1]
        assert sim[b].mean() == 0.0
        # the closed form of the mean: each kept position lies in C(M-1, N-1) candidates
        assert math.comb(7, 3) * 4 / math.comb(8, 4) == 2.0


# ---------------------------------------------------------------- magnitude prior

@pytest.mark.parametrize("n,m", NM)
def test_magnitude_prior_is_energy_maximiser(orc, n, m):
    rng = np.random.default_rng(2)
    S = orc.candidates(n, m)
    W = rng.normal(0, 0.02, size=(400, m))
    _, pidx, _ = orc.prior_init(n, m, W, np.arange(400), 3.0, 0.0, 0)
    np.testing.assert_array_equal(pidx, _energy_best(S, W))


def test_magnitude_prior_ties_and_nan(orc):
    S = orc.candidates(2, 4)
    W = np.array([[0.5, -0.5, 0.5, 0.1],       # tie among 0,1,2 -> keep 0,1
                  [np.nan, 0.1, 0.2, 0.3],     # NaN ranks last -> keep 2,3
                  [0.0, 0.0, 0.0, 0.0],        # all equal -> keep 0,1
                  [0.1, -0.3, 0.3, 0.05]])     # |.| tie between 1 and 2 -> keep 1,2
    _, pidx, _ = orc.prior_init(2, 4, W, np.arange(4), 3.0, 0.0, 0)
    kept = [tuple(np.flatnonzero(S[k])) for k in pidx]
    assert kept == [(0, 1), (2, 3), (0, 1), (1, 2)]


# ---------------------------------------------------------------- Eq.10 initialisation

@pytest.mark.parametrize("n,m", NM)
def test_deterministic_prior_argmax_reproduces_prior(orc, n, m):
    """init_std = 0: pi = alpha * sim, so argmax(kappa * pi) is the prior candidate in every
    block (and it is the unique maximum)."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, size=(1000, m))
    pi, pidx, sim = orc.prior_init(n, m, W, np.arange(1000), alpha=3.0, init_std=0.0, seed=0)
    np.testing.assert_array_equal(pi, 3.0 * sim)
    k = orc.argmax(np.float32(3.0) * pi.astype(np.float32), orc.num_candidates(n, m))
    np.testing.assert_array_equal(k, pidx)
    assert np.all((pi == pi.max(1, keepdims=True)).sum(1) == 1)


@pytest.mark.parametrize("n,m", NM)
def test_random_init_is_normal_with_std_001(orc, n, m):
    """alpha = 0 leaves the N(0, 0.01) draws (Table 7): zero mean, std 0.01, Box-Muller
    pairs with E[r^2] = 2, and independent of the weights."""
    C = orc.num_candidates(n, m)
    nb = 40_000 if m == 4 else 4000
    rng = np.random.default_rng(4)
    W = rng.normal(0, 0.02, size=(nb, m))
    pi, _, _ = orc.prior_init(n, m, W, np.arange(nb), alpha=0.0, init_std=0.01, seed=7)
    z = pi.ravel() / 0.01
    N = z.size
    assert abs(z.mean()) < 5 / math.sqrt(N)
    assert abs(z.var() - 1.0) < 5 * math.sqrt(2.0 / N)
    assert abs(((z - z.mean()) ** 4).mean() / z.var() ** 2 - 3.0) < 5 * math.sqrt(24.0 / N)
    pairs = pi[:, : (C // 2) * 2].reshape(nb, -1, 2) / 0.01
    r2 = (pairs ** 2).sum(-1).ravel()
    assert abs(r2.mean() - 2.0) < 5 * 2.0 / math.sqrt(r2.size)
    pi2, _, _ = orc.prior_init(n, m, W * 3.0, np.arange(nb), alpha=0.0, init_std=0.01, seed=7)
    np.testing.assert_array_equal(pi, pi2)


def _init_uniforms(orc, C, seed, gids):
    """u_c = (2k+1) 2^-22 of the reserved init step (0xFFFFFFFF), k the 21-bit field c%6 of
    Philox(counter (gid lo, gid hi, 0xFFFFFFFF, c//6), key (seed lo, seed hi)), computed
    here from the known-answer-pinned Philox and big-integer slicing of its 128 bits."""
    u = np.zeros((len(gids), C))
    for b, gid in enumerate(int(g) for g in gids):
        for grp in range((C + 5) // 6):
            words = orc.philox4x32_10([gid & 0xFFFFFFFF, gid >> 32, 0xFFFFFFFF, grp],
                                      [seed & 0xFFFFFFFF, seed >> 32])
            big = sum(int(words[i]) << (32 * i) for i in range(4))
            for f in range(6):
                c = 6 * grp + f
                if c < C:
                    u[b, c] = (2 * ((big >> (21 * f)) & ((1 << 21) - 1)) + 1) / 2.0 ** 22
    return u


@pytest.mark.parametrize("n,m", NM)
def test_box_muller_pairs_follow_their_uniforms(orc, n, m):
    """Each pair (2p, 2p+1) of the initial N(0,1) draws is one Box-Muller transform of the
    reserved-step uniforms: radius from u_2p, angle from u_2p+1, so
    n_2p^2 + n_2p+1^2 = -2 ln u_2p and atan2(n_2p+1, n_2p) = 2 pi u_2p+1 (mod 2 pi), to fp64
    rounding. A cosine taken for both members, a reused radius or angle, swapped roles of the
    two uniforms or a pair drawn from the wrong candidates all fail here, although they keep
    every one-dimensional moment; the two members of a pair are uncorrelated."""
    C = orc.num_candidates(n, m)
    nb = 1500 if m == 4 else 150
    seed = 0x5EED_0000_0000_0007
    gids = np.arange(nb, dtype=np.uint64) * np.uint64(7919) + np.uint64(2**33 + 12345)
    # no prior (index >= C) and init_std 1: the logits are the draws themselves
    z, _ = orc.prior_init_from_index(n, m, gids, np.full(nb, C, np.int32), 3.0, 1.0, seed)
    u = _init_uniforms(orc, C, seed, gids)
    P = C // 2
    a, b = z[:, 0:2 * P:2], z[:, 1:2 * P:2]
    u1, u2 = u[:, 0:2 * P:2], u[:, 1:2 * P:2]
    np.testing.assert_allclose(a * a + b * b, -2.0 * np.log(u1), rtol=1e-13, atol=0)
    ang = np.mod(np.arctan2(b, a), 2 * np.pi)
    d = np.abs(ang - 2 * np.pi * u2)
    d = np.minimum(d, 2 * np.pi - d)
    assert d.max() < 1e-12, d.max()
    # pair members uncorrelated (a mix-up like n_2p+1 = n_2p would give E = 1)
    prod = (a * b).ravel()
    assert abs(prod.mean()) < 5.0 / math.sqrt(prod.size)


@pytest.mark.parametrize("n,m", NM)
def test_prior_bias_scales_with_block_std(orc, n, m):
    """Eq.10: pi(alpha) - pi(0) = alpha * sigma(pi(0)) * sim, sigma the spread of the block's
    random logits."""
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, size=(300, m))
    p0, pidx, sim = orc.prior_init(n, m, W, np.arange(300), 0.0, 0.01, seed=9)
    p3, pidx3, _ = orc.prior_init(n, m, W, np.arange(300), 3.0, 0.01, seed=9)
    np.testing.assert_array_equal(pidx, pidx3)
    sigma = p0.std(1, keepdims=True)
    np.testing.assert_allclose(p3 - p0, 3.0 * sigma * sim, rtol=0, atol=1e-15)
    # with the bias the prior candidate's logit rises by alpha*sigma*max(sim) over its draw
    assert np.all(p3[np.arange(300), pidx] > p0[np.arange(300), pidx])


# ---------------------------------------------------------------- hard mask and packing

def _unpack(n, m, values, meta, rows_, cols, dtype):
    """Independent reading of the packed format back into a dense matrix."""
    dense = np.zeros((rows_, cols), dtype)
    bpr = cols // m
    for r in range(rows_):
        for q in range(bpr):
            if m == 4:
                nib = (int(meta[r, q // 8]) >> (4 * (q % 8))) & 0xF
                pos = [nib & 3, nib >> 2]
            else:
                code = int(meta[r, q])
                pos = [(code >> (3 * t)) & 7 for t in range(4)]
            assert pos == sorted(pos) and len(set(pos)) == n and max(pos) < m
            for t in range(n):
                dense[r, q * m + pos[t]] = values[r, q * n + t]
    return dense


@pytest.mark.parametrize("n,m", NM)
@pytest.mark.parametrize("wbits", [np.uint16, np.uint32])
def test_pack_roundtrip_is_masked_weight(orc, n, m, wbits):
    rng = np.random.default_rng(6)
    C = orc.num_candidates(n, m)
    S = orc.candidates(n, m)
    rows_, cols = 7, m * 21           # 21 blocks per row: a ragged last metadata word for 2:4
    Wraw = rng.integers(1, np.iinfo(wbits).max, size=(rows_, cols), dtype=wbits)
    pi = rng.normal(0, 1, size=(rows_ * cols // m, C)).astype(np.float32)
    values, meta, cand = orc.hard_pack(n, m, Wraw, pi)
    k = np.argmax(pi, 1)
    np.testing.assert_array_equal(cand, k)
    dense = _unpack(n, m, values, meta, rows_, cols, wbits)
    mask = S[k].reshape(rows_, cols)
    np.testing.assert_array_equal(dense, np.where(mask == 1, Wraw, 0))
    if m == 4:
        # unused nibbles of the last word are zero
        assert np.all((meta[:, -1] >> (4 * (21 % 8))) == 0)


def test_argmax_ties_and_nan(orc):
    pi = np.array([[1.0, 3.0, 3.0, 0.0, 3.0, 2.0],
                   [np.nan, 1.0, 2.0, np.nan, 2.0, 0.0],
                   [np.nan] * 6,
                   [-np.inf, -1.0, -np.inf, -1.0, -2.0, -3.0]], np.float32)
    np.testing.assert_array_equal(orc.argmax(pi, 6), [1, 2, 0, 1])


def test_mask_storage_bits_per_param(orc):
    """A 2:4 mask is one of C(4,2) = 6 candidates per 4 weights: log2(6)/4 = 0.646 bits per
    parameter, the page's 0.65 bits/param."""
    page = float(keyed("paper_figures.txt")["mask_bits_per_param_2of4"][0])
    C = orc.num_candidates(2, 4)
    assert C == int(keyed("paper_figures.txt")["logits_per_block_2of4"][0])
    assert round(math.log2(C) / 4, 2) == page


# ---------------------------------------------------------------- transfer prior (given M0)

@pytest.mark.parametrize("n,m", NM)
def test_prior_from_index_equals_magnitude_prior_when_given_it(orc, n, m):
    """Giving the magnitude prior's own candidate index reproduces prior_init exactly, in both
    the random and the deterministic mode."""
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, size=(300, m))
    gids = np.arange(300, dtype=np.uint64) + np.uint64(7)
    for init_std in (0.0, 0.01):
        pi, pidx, sim = orc.prior_init(n, m, W, gids, 3.0, init_std, 5)
        pi2, sim2 = orc.prior_init_from_index(n, m, gids, pidx, 3.0, init_std, 5)
        np.testing.assert_array_equal(pi, pi2)
        np.testing.assert_array_equal(sim, sim2)


@pytest.mark.parametrize("n,m", NM)
def test_prior_from_index_any_mask_and_no_prior(orc, n, m):
    """Any candidate can be the prior (deterministic mode: argmax = that candidate, sim takes
    the page's values); an index >= C leaves the random logits alone."""
    C = orc.num_candidates(n, m)
    rng = np.random.default_rng(13)
    k = rng.integers(0, C, size=500)
    pi, sim = orc.prior_init_from_index(n, m, np.arange(500), k, 3.0, 0.0, 0)
    np.testing.assert_array_equal(np.argmax(pi, 1), k)
    assert np.all(np.sort(np.unique(sim)) == (np.array([-1, 0, 1]) if m == 4 else np.array([-2, -1, 0, 1, 2])))
    none = np.full(500, C, np.int32)
    p0, _ = orc.prior_init_from_index(n, m, np.arange(500), none, 3.0, 0.01, 9)
    r0, _, _ = orc.prior_init(n, m, np.zeros((500, m)), np.arange(500), 0.0, 0.01, 9)
    np.testing.assert_array_equal(p0, r0)


@pytest.mark.parametrize("n,m", NM)
def test_eq10_argmax_is_prior_exactly_when_the_bias_covers_the_draws(orc, n, m):
    """Eq.10 with random draws: the prior candidate p is the argmax of pi = pi0 + alpha sigma
    sim exactly when, for every other candidate j, pi0_j - pi0_p < alpha sigma (sim_p - sim_j)
    (sigma the spread of the block's draws). Checked block by block against the oracle's own
    argmax; with alpha = 3 the prior wins in most blocks (~95 % at 2:4, ~85 % at 4:8, where 16
    candidates sit one similarity step below it), with alpha = 0 in about 1/C."""
    C = orc.num_candidates(n, m)
    nb = 4000
    rng = np.random.default_rng(21)
    W = rng.normal(0, 0.02, size=(nb, m))
    gids = np.arange(nb)
    p0, pidx, sim = orc.prior_init(n, m, W, gids, 0.0, 0.01, seed=3)
    for alpha, lo, hi in ((3.0, 0.75, 1.0), (0.0, 0.5 / C, 2.0 / C)):
        p, _, _ = orc.prior_init(n, m, W, gids, alpha, 0.01, seed=3)
        k = orc.argmax(p.astype(np.float32), C)
        sigma = p0.std(1)
        sp = sim[np.arange(nb), pidx]
        lhs = p0 - p0[np.arange(nb), pidx][:, None]
        rhs = alpha * sigma[:, None] * (sp[:, None] - sim)
        others = np.arange(C)[None, :] != pidx[:, None]
        predicate = np.all((lhs < rhs) | ~others, axis=1)
        np.testing.assert_array_equal(k == pidx, predicate)
        assert lo <= predicate.mean() <= hi, (alpha, predicate.mean())
