"""Pins of the oracle's masked linear layer: the sampler inside the frozen network's linear
layer (MaskLLM summary s.3.2 "Frozen LLM Backbone": the network multiplies by W . M on its
forward pass and only the logits receive gradients).

The oracle composes the already pinned sampler forward/backward with a plain fp64 matrix
product. These tests pin the composition itself -- which operand is transposed, which
dimension is contracted, how the bf16 storage of X enters -- against facts that do not use
the composition: an identity activation returns X itself, a brute-force loop over the
definition, the trace identity <dY, A X^T> = <dY^T A, X>, and central finite differences of
the layer's loss <dY, A X^T> - lambda ||X||^2 with respect to the logits.
"""
import numpy as np
import pytest

NM = [(2, 4), (4, 8)]


def _case(n, m, rows, cols, T, seed=0):
    rng = np.random.default_rng(seed)
    C = {4: 6, 8: 70}[m]
    W = rng.normal(0, 0.02, size=(rows, cols)).astype(np.float32).astype(np.float64)
    pi = rng.normal(0, 0.02, size=(rows * cols // m, C)).astype(np.float32)
    A = rng.normal(0, 1, size=(T, cols)).astype(np.float32).astype(np.float64)
    dY = rng.normal(0, 1e-3, size=(T, rows)).astype(np.float32).astype(np.float64)
    gids = np.arange(rows * cols // m, dtype=np.uint64) + np.uint64(1000)
    return W, pi, A, dY, gids


@pytest.mark.parametrize("n,m", NM)
def test_identity_activations_return_the_stored_soft_masked_weights(orc, n, m):
    """A = I (T = cols): Y[t, r] = X[r, t], the bf16-stored soft-masked weight, exactly."""
    rows, cols = 5, 4 * m
    W, pi, _, _, gids = _case(n, m, rows, cols, cols, seed=1)
    out = orc.masked_linear_fwd(n, m, W, pi, gids, np.eye(cols), 100.0, 2.0, 7, 3)
    xr = orc.bf16_bits_to_float(out["x_bits"]).astype(np.float64)
    np.testing.assert_array_equal(out["y"], xr.T)
    f = orc.sample_fwd(n, m, W.reshape(-1, m), pi, gids, 100.0, 2.0, 7, 3)
    np.testing.assert_array_equal(out["x"].reshape(-1, m), f["x"])
    assert out["reg"] == f["reg"]


@pytest.mark.parametrize("n,m", NM)
def test_forward_matches_a_loop_over_the_definition(orc, n, m):
    """y[t][r] = sum over blocks q of row r and positions j of A[t, qM+j] * bf16(W * M)."""
    rows, cols, T = 3, 2 * m, 4
    W, pi, A, _, gids = _case(n, m, rows, cols, T, seed=2)
    out = orc.masked_linear_fwd(n, m, W, pi, gids, A, 300.0, 0.5, 11, 0)
    f = orc.sample_fwd(n, m, W.reshape(-1, m), pi, gids, 300.0, 0.5, 11, 0)
    xb = orc.bf16_bits_to_float(orc.round_bf16(f["x"])).astype(np.float64).reshape(rows, cols // m, m)
    for t in range(T):
        for r in range(rows):
            acc = 0.0
            for q in range(cols // m):
                for j in range(m):
                    acc += A[t, q * m + j] * xb[r, q, j]
            assert abs(out["y"][t, r] - acc) <= 1e-15 * np.abs(A[t]).sum() * np.abs(xb[r]).max()


@pytest.mark.parametrize("n,m", NM)
def test_weight_gradient_is_dy_transposed_times_a(orc, n, m):
    """The trace identity <dY, A X^T> = <dY^T A, X> fixes the orientation of G, and each
    entry is the brute-force sum over tokens."""
    rows, cols, T = 6, 3 * m, 7
    W, pi, A, dY, gids = _case(n, m, rows, cols, T, seed=3)
    out = orc.masked_linear_fwd(n, m, W, pi, gids, A, 100.0, 4.0, 1, 2)
    _, _, G = orc.masked_linear_bwd(n, m, W, pi, gids, A, dY, 100.0, 4.0, 1e-5, 1, 2)
    xr = orc.bf16_bits_to_float(out["x_bits"]).astype(np.float64)
    lhs = float((dY * out["y"]).sum())
    rhs = float((G * xr).sum())
    assert abs(lhs - rhs) <= 1e-12 * ((np.abs(dY).T @ np.abs(A)) * np.abs(xr)).sum()
    for r in range(rows):
        for k in range(cols):
            assert abs(G[r, k] - sum(dY[t, r] * A[t, k] for t in range(T))) <= 1e-15 * np.abs(dY[:, r] * A[:, k]).sum() + 1e-300


@pytest.mark.parametrize("n,m", NM)
def test_logit_gradient_by_central_differences(orc, n, m):
    """The logits' gradient of the layer's loss L(pi) = <dY, A X(pi)^T> - lambda ||X(pi)||^2
    (X unrounded, perturbed logits in double, the noise held fixed) by central differences."""
    rows, cols, T = 2, 2 * m, 3
    W, pi, A, dY, gids = _case(n, m, rows, cols, T, seed=4)
    W = W * 50.0  # weights large enough for the regulariser to matter
    lam, kappa, tau, seed, step = 1e-2, 3.0, 1.5, 5, 9
    pi64 = pi.astype(np.float64)
    g, _, _ = orc.masked_linear_bwd(n, m, W, pi, gids, A, dY, kappa, tau, lam, seed, step, round_w=False)

    def loss(p):
        f = orc.sample_fwd(n, m, W.reshape(-1, m), p, gids, kappa, tau, seed, step, round_w=False)
        x = f["x"].reshape(rows, cols)
        return float((dY * (A @ x.T)).sum()) - lam * f["reg"]

    C = pi.shape[1]
    for b in range(pi.shape[0]):
        for i in range(0, C, max(1, C // 6)):
            h = 1e-3 * max(1.0, abs(pi64[b, i]))
            hp, hm = pi64.copy(), pi64.copy()
            # the oracle takes fp32 logits: step by an fp32-representable amount
            hp[b, i] = np.float32(pi64[b, i] + h)
            hm[b, i] = np.float32(pi64[b, i] - h)
            fd = (loss(hp.astype(np.float32)) - loss(hm.astype(np.float32))) / (hp[b, i] - hm[b, i])
            assert abs(fd - g[b, i]) <= 1e-4 * np.abs(g[b]).max() + 1e-12, (b, i, fd, g[b, i])
