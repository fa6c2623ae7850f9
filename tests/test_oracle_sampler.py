"""Pins of the oracle's forward (Eq.6-Eq.8), backward and AdamW.

Each check ties the oracle to something other than itself: the page's worked example,
limits the page states (tau -> 0, large tau), invariants of the softmax, a brute force over
the candidates, central finite differences, torch autograd, 400-digit arithmetic, and
torch.optim.AdamW.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

from _golden import keyed


def _rand_blocks(rng, nb, m, C, pi_std=0.5):
    W = rng.normal(0, 0.02, size=(nb, m))
    pi = rng.normal(0, pi_std, size=(nb, C)).astype(np.float32)
    gids = rng.integers(0, 2**40, size=nb, dtype=np.uint64)
    return W, pi, gids


NM = [(2, 4), (4, 8)]


# ---------------------------------------------------------------- Eq.7 worked example

def test_soft_mask_worked_example(orc):
    g = keyed("soft_mask_worked_example.txt")
    y = np.array([float(v) for v in g["y"]])
    expected = np.array([float(v) for v in g["mask"]])
    got = orc.soft_mask(2, 4, y[None, :])[0]
    np.testing.assert_allclose(got, expected, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- softmax invariants

@pytest.mark.parametrize("n,m", NM)
def test_soft_index_is_a_distribution(orc, n, m):
    rng = np.random.default_rng(1)
    C = orc.num_candidates(n, m)
    W, pi, gids = _rand_blocks(rng, 500, m, C)
    for tau in (4.0, 1.0, 0.05):
        r = orc.sample_fwd(n, m, W, pi, gids, kappa=3.0, tau=tau, seed=5, step=2)
        y, ms, mc = r["y"], r["msoft"], r["mcomp"]
        assert np.all(y >= 0)
        np.testing.assert_allclose(y.sum(1), 1.0, rtol=0, atol=1e-12)
        # soft mask keeps N weights in total, each entry in [0, 1], complement sums to 1
        np.testing.assert_allclose(ms.sum(1), n, rtol=0, atol=1e-12)
        assert np.all(ms >= 0) and np.all(ms <= 1 + 1e-15)
        np.testing.assert_allclose(ms + mc, 1.0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["x"], W * ms, rtol=0, atol=0)
        np.testing.assert_allclose(r["reg"], (r["x"] ** 2).sum(), rtol=1e-12)


def test_shift_invariance(orc):
    """Adding a constant to every logit of a block leaves the soft index unchanged."""
    rng = np.random.default_rng(2)
    W, pi, gids = _rand_blocks(rng, 200, 4, 6)
    pi = (np.round(pi * 2**12) / 2**12).astype(np.float32)  # so that pi + 0.25 is exact
    a = orc.sample_fwd(2, 4, W, pi, gids, 1.0, 0.7, 9, 0, round_w=False)["y"]
    b = orc.sample_fwd(2, 4, W, pi + np.float32(0.25), gids, 1.0, 0.7, 9, 0, round_w=False)["y"]
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("n,m", NM)
def test_one_hot_as_tau_goes_to_zero(orc, n, m):
    """Noise off, tau = 1e-3 and logit gaps >= 0.1: the soft index is the one-hot argmax
    (s.3.4 Step 2: tau -> 0 approaches argmax), and the soft mask is that candidate."""
    rng = np.random.default_rng(3)
    C = orc.num_candidates(n, m)
    S = orc.candidates(n, m)
    nb = 300
    pi = np.zeros((nb, C), np.float32)
    for b in range(nb):
        pi[b] = rng.permutation(C).astype(np.float32) * np.float32(0.1)
    W = rng.normal(0, 0.02, size=(nb, m))
    r = orc.sample_fwd(n, m, W, pi, np.arange(nb), kappa=1.0, tau=1e-3, seed=0, step=0, noise_on=False)
    k = np.argmax(pi, 1)
    y = r["y"]
    others = y.copy()
    others[np.arange(nb), k] = 0.0
    assert np.all(others < 1e-40)                     # gaps of 0.1 / tau = 100 -> e^-100
    np.testing.assert_allclose(y[np.arange(nb), k], 1.0, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(r["msoft"].round(12), S[k].astype(np.float64))


@pytest.mark.parametrize("n,m", NM)
def test_uniform_as_tau_grows(orc, n, m):
    """Large tau makes the soft index uniform (s.3.4 Step 2), so every mask entry is N/M."""
    rng = np.random.default_rng(4)
    C = orc.num_candidates(n, m)
    W, pi, gids = _rand_blocks(rng, 100, m, C)
    r = orc.sample_fwd(n, m, W, pi, gids, kappa=1.0, tau=1e7, seed=1, step=0)
    np.testing.assert_allclose(r["y"], 1.0 / C, rtol=1e-5)
    np.testing.assert_allclose(r["msoft"], n / m, rtol=1e-5)


def test_regulariser_of_hard_masks(orc):
    """With a one-hot soft index, ||W . M||^2 is the sum of the kept weights' squares, and
    over all candidates the magnitude mask maximises it (s.3.4 regularisation rationale)."""
    rng = np.random.default_rng(5)
    S = orc.candidates(2, 4).astype(np.float64)
    nb = 400
    W = rng.normal(0, 0.02, size=(nb, 4))
    pi = np.zeros((nb, 6), np.float32)
    ks = rng.integers(0, 6, size=nb)
    pi[np.arange(nb), ks] = 1.0
    r = orc.sample_fwd(2, 4, W, pi, np.arange(nb), 1.0, 1e-4, 0, 0, noise_on=False)
    kept = (W**2 * S[ks]).sum()
    np.testing.assert_allclose(r["reg"], kept, rtol=1e-12)
    # brute force: the candidate keeping the most squared weight is the magnitude top-2
    energy = (W[:, None, :] ** 2 * S[None]).sum(-1)
    best = np.argmax(energy, 1)
    top2 = np.argsort(-np.abs(W), 1)[:, :2]
    for b in range(nb):
        assert set(np.flatnonzero(S[best[b]])) == set(top2[b])


# ---------------------------------------------------------------- backward

def _loss(orc, n, m, W, G, pi, gids, kappa, tau, lam, seed, step):
    r = orc.sample_fwd(n, m, W, pi, gids, kappa, tau, seed, step, round_w=False)
    return (G * r["x"]).sum() - lam * r["reg"]


@pytest.mark.parametrize("n,m", NM)
def test_gradient_matches_finite_differences(orc, n, m):
    """Central differences in double, noise held fixed, on the exact-w path."""
    rng = np.random.default_rng(6)
    C = orc.num_candidates(n, m)
    nb = 3
    W, _, gids = _rand_blocks(rng, nb, m, C)
    G = rng.normal(0, 1.0, size=(nb, m))
    lam = 1e-1  # large enough that the regulariser term is visible in the check
    kappa, tau = 1.5, 0.8
    base = rng.normal(0, 0.3, size=(nb, C))
    # finite differences need a logit that moves continuously; evaluate pi in float64 via a
    # float32 grid fine enough (h = 2^-10) that both neighbours are exactly representable
    pi = (np.round(base * 2**12) / 2**12).astype(np.float32)
    grad, _ = orc.sample_bwd(n, m, W, G, pi, gids, kappa, tau, lam, seed=4, step=3, round_w=False)
    h = np.float32(2.0**-10)
    for b in range(nb):
        for i in range(C):
            p1 = pi.copy(); p1[b, i] += h
            p0 = pi.copy(); p0[b, i] -= h
            fd = (_loss(orc, n, m, W, G, p1, gids, kappa, tau, lam, 4, 3)
                  - _loss(orc, n, m, W, G, p0, gids, kappa, tau, lam, 4, 3)) / (2 * float(h))
            # O(h^2) truncation: bound by the block's gradient scale
            scale = np.abs(grad[b]).max() + 1e-12
            assert abs(fd - grad[b, i]) <= 2e-5 * scale, (b, i, fd, grad[b, i])


@pytest.mark.parametrize("n,m", NM)
def test_gradient_matches_torch_autograd(orc, n, m):
    """The hand-derived backward agrees with torch autograd on the same noise (float64)."""
    rng = np.random.default_rng(7)
    C = orc.num_candidates(n, m)
    nb = 64
    W, pi, gids = _rand_blocks(rng, nb, m, C)
    G = rng.normal(0, 1e-3, size=(nb, m))
    kappa, tau, lam = 100.0, 2.0, 1e-5
    _, g = orc.noise(n, m, 21, 4, gids)
    S = torch.tensor(orc.candidates(n, m), dtype=torch.float64)
    P = torch.tensor(pi.astype(np.float64), requires_grad=True)
    y = torch.softmax((kappa * P + torch.tensor(g, dtype=torch.float64)) / tau, dim=1)
    X = torch.tensor(W) * (y @ S)
    L = (torch.tensor(G) * X).sum() - lam * (X**2).sum()
    L.backward()
    grad, scale = orc.sample_bwd(n, m, W, G, pi, gids, kappa, tau, lam, 21, 4, round_w=False)
    ref = P.grad.numpy()
    np.testing.assert_allclose(grad, ref, rtol=0, atol=1e-9 * np.abs(ref).max())
    # the softmax Jacobian annihilates constants: gradients of a block sum to zero
    np.testing.assert_allclose(grad.sum(1), 0.0, atol=1e-12 * scale.sum(1).max())


def test_gradient_accurate_when_soft_index_is_nearly_one_hot(orc):
    """At tau = 0.05, kappa = 500 most blocks are one-hot to within 1e-30; each gradient is
    still correct to 1e-12 of its own size, checked against 400-digit arithmetic of the
    textbook form y_i (a_i - sum_k y_k a_k), whose cancellation needs that many digits."""
    getcontext().prec = 400
    rng = np.random.default_rng(8)
    nb = 40
    W, pi, gids = _rand_blocks(rng, nb, 4, 6, pi_std=0.03)
    G = rng.normal(0, 1e-3, size=(nb, 4))
    kappa, tau, lam = 500.0, 0.05, 1e-5
    _, g = orc.noise(2, 4, 3, 77, gids)
    S = orc.candidates(2, 4)
    grad, _ = orc.sample_bwd(2, 4, W, G, pi, gids, kappa, tau, lam, 3, 77, round_w=True)
    tiny = 0
    for b in range(nb):
        # w is the specified fp32 perturbed logit fma(kappa, pi, g): one rounding of the
        # exact value, reproduced here with Decimal then rounded to fp32
        w = []
        for i in range(6):
            exact = Decimal(float(kappa)) * Decimal(float(pi[b, i])) + Decimal(float(g[b, i]))
            w.append(Decimal(float(np.float32(float(exact)))))
        wmax = max(w)
        e = [((wi - wmax) / Decimal(float(np.float32(tau)))).exp() for wi in w]
        tot = sum(e)
        y = [ei / tot for ei in e]
        ms = [sum(y[i] for i in range(6) if S[i, j]) for j in range(4)]
        u = [Decimal(G[b, j]) * Decimal(W[b, j]) - 2 * Decimal(float(np.float32(lam))) * Decimal(W[b, j]) ** 2 * ms[j]
             for j in range(4)]
        a = [sum(u[j] for j in range(4) if S[i, j]) for i in range(6)]
        abar = sum(y[i] * a[i] for i in range(6))
        c = Decimal(float(np.float32(kappa))) / Decimal(float(np.float32(tau)))
        for i in range(6):
            ref = c * y[i] * (a[i] - abar)
            if ref != 0 and abs(ref) < Decimal("1e-30"):
                tiny += 1
            assert abs(Decimal(grad[b, i]) - ref) <= abs(ref) * Decimal("1e-12") + Decimal("1e-300")
    assert tiny > 0  # the case the check is about did occur


# ---------------------------------------------------------------- AdamW

def test_adamw_matches_torch(orc):
    rng = np.random.default_rng(9)
    n = 3000
    p0 = rng.normal(0, 0.03, size=n)
    lr, b1, b2, eps, wd = 5e-4, 0.9, 0.999, 1e-8, 0.1
    P = torch.tensor(p0, requires_grad=True)
    opt = torch.optim.AdamW([P], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 8):
        g = rng.normal(0, 1.0, size=n) * 10.0 ** rng.integers(-12, 1, size=n)
        P.grad = torch.tensor(g)
        opt.step()
        p, m, v = orc.adamw(p, m, v, g, lr, b1, b2, eps, wd, t)
        st = opt.state[P]
        # torch forms m by lerp, the oracle as beta1 m + (1 - beta1) g: same value, rounding apart
        np.testing.assert_allclose(p, P.detach().numpy(), rtol=1e-12, atol=1e-18)
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-11, atol=1e-30)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-12, atol=1e-40)


def test_adamw_first_step_closed_form(orc):
    """t = 1 from zero state: p1 = p0 (1 - lr wd) - lr g / (|g| + eps)."""
    rng = np.random.default_rng(10)
    p0 = rng.normal(0, 0.03, size=500)
    g = rng.normal(0, 1e-6, size=500)
    lr, wd, eps = 1e-3, 0.1, 1e-8
    p1, m1, v1 = orc.adamw(p0, np.zeros(500), np.zeros(500), g, lr, 0.9, 0.999, eps, wd, 1)
    np.testing.assert_allclose(p1, p0 * (1 - lr * wd) - lr * g / (np.abs(g) + eps), rtol=1e-12)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-13)


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_values(orc):
    rng = np.random.default_rng(11)
    x = (rng.normal(0, 1, 100_000) * 10.0 ** rng.integers(-40, 30, 100_000)).astype(np.float32)
    x = np.concatenate([x, np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 2.0**-130, -3e-39], np.float32)])
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even(orc):
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even mantissa (1.0) wins;
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even (1 + 2^-6) wins
    got = orc.round_bf16(np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, 1 + 2.0**-8 + 2.0**-40]))
    vals = orc.bf16_bits_to_float(got)
    assert list(vals) == [1.0, 1 + 2.0**-6, 1 + 2.0**-7]
