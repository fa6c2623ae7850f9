"""The sampler inside the frozen network's linear layer on the GPU (mllm_masked_linear_*),
through the C ABI, against the oracle's masked_linear_* (a plain fp64 product composed with
the pinned sampler).

Forward: Y = A X^T with X = W . M made tile by tile in shared memory. Checked three ways:
X itself (the optional inspection output) bit for bit against mllm_sample_fwd's X and
within 1 bf16 ulp of the oracle's; Y against the oracle's product within the bound derived in
_tol.assert_masked_linear_close; the regulariser against the oracle (1e-3) and against
mllm_sample_fwd's (1e-6: the same per-block arithmetic summed in another order).
Sizes span several row tiles and chunks, ragged row tiles, grouped launches, every MMA width
(tokens 1 .. 256) and the LLaMA-2-7B layer's shapes (rows sampled there).
"""
import numpy as np
import pytest
import torch

import _tol
from sparsity_mask_sampling_b200 import (Hparams, alloc_matrix, inputs, masked_linear_workspace,
                                         mllm_masked_linear_bwd_adam, mllm_masked_linear_fwd, mllm_sample_fwd,
                                         mllm_workspace_bytes)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def mlws():
    return masked_linear_workspace(DEV)


@pytest.fixture(scope="module")
def ws():
    return torch.zeros(mllm_workspace_bytes(), dtype=torch.uint8, device=DEV)


class Layer:
    """Matrices of one layer with logits, activations A and outputs."""

    def __init__(self, shapes, tokens, seed, outliers=0.0, x_out=True):
        self.shapes, self.tokens = shapes, tokens
        self.mats, self.ios, self.A = [], [], []
        off = 5 * 2**31 + 3
        for i, (r, c) in enumerate(shapes):
            W = inputs.weights(r, c, "bf16", 0.02, seed=seed + i, outlier_frac=outliers)
            mb = alloc_matrix(W.to(DEV), (2, 4), off, fwd=x_out, bwd=False, soft_mask=False)
            mb.logits.copy_(inputs.logits(r * c // 4, 6, 0.02, seed=seed + 40 + i).to(DEV))
            A = inputs.weights(tokens, c, "bf16", 1.0, seed=seed + 80 + i)
            y = torch.full((tokens, r), float("nan"), dtype=torch.float32, device=DEV)
            self.mats.append(mb)
            self.A.append(A)
            self.ios.append((A.to(DEV), y, None))
            off += r * c // 4


def _check(orc, layer, hp, reg, rows_sample=None):
    reg_ref = 0.0
    for (r, c), mb, A, (_, y, _) in zip(layer.shapes, layer.mats, layer.A, layer.ios):
        rows = np.arange(r) if rows_sample is None else rows_sample(r)
        Wrows = mb.W[torch.from_numpy(rows).to(DEV)].float().double().cpu().numpy()
        pi = mb.logits.view(r, c // 4, 6)[torch.from_numpy(rows).to(DEV)].cpu().numpy().reshape(-1, 6)
        gids = (np.uint64(mb.block_offset) + (rows[:, None] * (c // 4) + np.arange(c // 4)[None, :]).astype(np.uint64)).ravel()
        Av = A.float().double().numpy()
        out = orc.masked_linear_fwd(2, 4, Wrows, pi, gids, Av, hp.kappa, hp.tau, hp.seed, hp.step)
        y_gpu = y[:, torch.from_numpy(rows).to(DEV)].double().cpu().numpy()
        _tol.assert_masked_linear_close(y_gpu, out["y"], Av, out["x"], orc.round_bf16)
        if mb.X is not None:
            xg = mb.X[torch.from_numpy(rows).to(DEV)].float().double().cpu().numpy()
            _tol.assert_x_close(xg, out["x"], "bf16", Wrows)
        if rows_sample is None:
            reg_ref += out["reg"]
    if rows_sample is None:
        _tol.assert_reg_close(reg, reg_ref)


@pytest.mark.parametrize("tokens", [1, 17, 32, 40, 64, 100, 128, 200, 256])
def test_masked_linear_forward_parity(orc, mlws, ws, tokens):
    layer = Layer([(256, 128), (200, 192), (64, 64)], tokens, seed=10 + tokens)
    hp = Hparams(kappa=300.0, tau=0.5, step=4, seed=0xF00D)
    reg = torch.zeros(1, dtype=torch.float64, device=DEV)
    mllm_masked_linear_fwd(layer.mats, layer.ios, (2, 4), tokens, hp, mlws, reg)
    torch.cuda.synchronize()
    x_fused = [mb.X.clone() for mb in layer.mats]
    _check(orc, layer, hp, reg.item())
    # X is exactly the sampler forward's X; the regulariser is the same sum in another order
    reg2 = torch.zeros(1, dtype=torch.float64, device=DEV)
    mllm_sample_fwd(layer.mats, (2, 4), hp, reg2, ws)
    torch.cuda.synchronize()
    for a, mb in zip(x_fused, layer.mats):
        assert torch.equal(a, mb.X)
    assert abs(reg.item() - reg2.item()) <= 1e-6 * reg2.item()
    assert mlws[-16:].view(torch.int32)[0].item() == 0  # error word


def test_masked_linear_forward_many_matrices_and_no_inspection_outputs(orc, mlws):
    """20 matrices (two launches, the regulariser accumulated across them), X not written."""
    shapes = [(64 + 32 * (i % 5), 64 * (1 + i % 3)) for i in range(20)]
    layer = Layer(shapes, 48, seed=300, x_out=False)
    for mb in layer.mats:
        mb.X = None
    hp = Hparams(kappa=100.0, tau=4.0, step=0, seed=3)
    reg = torch.zeros(1, dtype=torch.float64, device=DEV)
    mllm_masked_linear_fwd(layer.mats, layer.ios, (2, 4), 48, hp, mlws, reg)
    torch.cuda.synchronize()
    _check(orc, layer, hp, reg.item())


def test_masked_linear_forward_llama2_7b_layer(orc, mlws):
    """The LLaMA-2-7B layer's seven matrices (50.6 M blocks, 1 % outlier channels) at 256
    tokens in one call; Y and X checked on sampled rows (first, last and random)."""
    from sparsity_mask_sampling_b200 import configs

    w = configs.WORKLOADS["llama2_7b_layer_2of4"]
    layer = Layer([(m.rows, m.cols) for m in w.matrices], 256, seed=500, outliers=0.01)
    hp = Hparams(kappa=420.0, tau=0.8, step=77, seed=12)
    reg = torch.zeros(1, dtype=torch.float64, device=DEV)
    mllm_masked_linear_fwd(layer.mats, layer.ios, (2, 4), 256, hp, mlws, reg)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    _check(orc, layer, hp, reg.item(),
           rows_sample=lambda r: np.unique(np.concatenate([[0, 127, 128, r - 1], rng.choice(r, 12, replace=False)])))
    r_x = sum(float((mb.X.double() ** 2).sum()) for mb in layer.mats)
    assert abs(reg.item() - r_x) <= 1e-3 * r_x


# ------------------------------------------------------------------------------ backward


def _bwd_check(orc, mb, A, dY, hp, pi0, m0, v0, rows_idx=None):
    """Logit gradient, AdamW-updated logits and moments of one matrix against the oracle
    (masked_linear_bwd, then AdamW). The GPU's G is the fp32 tensor-core sum of the T products
    dY[t, r] A[t, k] (each exact), off by at most (ceil(T/16) + 8) 2^-22 sum_t |dY A| per
    entry; that error reaches dpi_i through u_j = G_j W_j as
    (kappa/tau) y_i sum_j |S_ij - M_j| |W_j| dG_j, which is added to the 1e-4 bar."""
    r_all, c = mb.W.shape
    rows = np.arange(r_all) if rows_idx is None else rows_idx
    rt = torch.from_numpy(rows).to(DEV)
    Wv = mb.W[rt].float().double().cpu().numpy()
    Av = A.float().double().numpy()
    dYv = dY[:, rows].float().double().numpy()
    sel = (rows[:, None] * (c // 4) + np.arange(c // 4)[None, :]).ravel()
    gids = np.uint64(mb.block_offset) + sel.astype(np.uint64)
    pi, m, v = pi0[sel], m0[sel], v0[sel]
    g_ref, scale, G = orc.masked_linear_bwd(2, 4, Wv, pi, gids, Av, dYv, hp.kappa, hp.tau, hp.lambda_, hp.seed, hp.step)
    T = A.shape[0]
    dG = ((T + 15) // 16 + 8) * 2.0 ** -22 * (np.abs(dYv).T @ np.abs(Av))
    f = orc.sample_fwd(2, 4, Wv.reshape(-1, 4), pi, gids, hp.kappa, hp.tau, hp.seed, hp.step)
    S = orc.candidates(2, 4).astype(np.float64)
    wdg = (np.abs(Wv) * dG).reshape(-1, 4)
    # |d dpi_i / d u_j| / ((kappa/tau) y_i): the complement 1 - M_j for j in S_i, taken as the
    # oracle's sum of the soft-index weights of the candidates without j (1 - M_j in floating
    # point is 0 once M_j is within 2^-53 of 1, while that sum still carries the sensitivity),
    # and M_j otherwise
    sens = S[None, :, :] * f["mcomp"][:, None, :] + (1.0 - S[None, :, :]) * f["msoft"][:, None, :]
    prop = (hp.kappa / hp.tau) * f["y"] * (sens * wdg[:, None, :]).sum(-1)
    floor = _tol.grad_floor(Wv.reshape(-1, 4), G.reshape(-1, 4), hp.kappa, hp.tau, hp.lambda_)
    g_tol = 1e-4 * scale + prop + floor
    g_gpu = mb.grad_logits.view(r_all, c // 4, 6)[rt].cpu().numpy().reshape(-1, 6)
    err = np.abs(g_gpu - g_ref)
    assert (err <= g_tol).all(), f"{(~(err <= g_tol)).sum()} gradient mismatches, worst {np.max(err / g_tol):.3g} x tol"
    f32 = np.float32
    p_ref, m_ref, v_ref = orc.adamw(pi, m, v, g_ref, f32(hp.lr), f32(hp.beta1), f32(hp.beta2), f32(hp.eps),
                                    f32(hp.weight_decay), hp.adam_step)
    got = lambda t: t.view(r_all, c // 4, 6)[rt].cpu().numpy().reshape(-1, 6)
    _tol.assert_logits_close(got(mb.logits), p_ref)
    _tol.assert_moments_close(got(mb.adam_m), got(mb.adam_v), m_ref, v_ref, g_ref, g_tol, f32(hp.beta1), f32(hp.beta2))


def _bwd_layer(shapes, tokens, seed, outliers=0.0):
    mats, ios, As, dYs, state = [], [], [], [], []
    off = 7 * 2**31 + 5
    for i, (r, c) in enumerate(shapes):
        W = inputs.weights(r, c, "bf16", 0.02, seed=seed + i, outlier_frac=outliers)
        mb = alloc_matrix(W.to(DEV), (2, 4), off, fwd=False, bwd=True, grad_logits=True)
        mb.G = None
        B = r * c // 4
        pi = inputs.logits(B, 6, 0.02, seed=seed + 40 + i)
        m0, v0 = inputs.moments(B, 6, seed=seed + 60 + i)
        mb.logits.copy_(pi.to(DEV))
        mb.adam_m.copy_(m0.to(DEV))
        mb.adam_v.copy_(v0.to(DEV))
        A = inputs.weights(tokens, c, "bf16", 1.0, seed=seed + 80 + i)
        dY = inputs.upstream_grad(tokens, r, "bf16", 1e-3, seed=seed + 90 + i)
        mats.append(mb)
        ios.append((A.to(DEV), None, dY.to(DEV)))
        As.append(A)
        dYs.append(dY)
        state.append((pi.numpy(), m0.numpy(), v0.numpy()))
        off += B
    return mats, ios, As, dYs, state


@pytest.mark.parametrize("tokens", [1, 40, 64, 100, 256, 300, 1000])
def test_masked_linear_backward_adam_parity(orc, mlws, tokens):
    """Ragged tiles in both directions (200 rows, 192 = 1.5 column tiles), grouped matrices,
    token counts below, at and between the 64-token stages, and past the forward's 256 (the
    backward sums over the tokens in stages)."""
    shapes = [(256, 128), (200, 192), (64, 64)]
    mats, ios, As, dYs, state = _bwd_layer(shapes, tokens, seed=700 + tokens)
    hp = Hparams(kappa=250.0, tau=0.6, lambda_=1e-5, lr=5e-4, adam_step=3, step=2, seed=0xB0B)
    mllm_masked_linear_bwd_adam(mats, ios, (2, 4), tokens, hp, mlws)
    torch.cuda.synchronize()
    for mb, A, dY, (pi, m0, v0) in zip(mats, As, dYs, state):
        _bwd_check(orc, mb, A, dY, hp, pi, m0, v0)
    assert mlws[-16:].view(torch.int32)[0].item() == 0  # error word


@pytest.mark.parametrize("tokens", [256, 2048])
def test_masked_linear_backward_adam_llama2_7b_layer(orc, mlws, tokens):
    """The LLaMA-2-7B layer's seven matrices in one call (12,352 tiles of 128 x 128 over the
    persistent grid), at 256 tokens and at 2048 (past the forward's limit: the backward sums
    over the tokens in stages); sampled rows checked."""
    from sparsity_mask_sampling_b200 import configs

    w = configs.WORKLOADS["llama2_7b_layer_2of4"]
    mats, ios, As, dYs, state = _bwd_layer([(m.rows, m.cols) for m in w.matrices], tokens, seed=900, outliers=0.01)
    hp = Hparams(kappa=480.0, tau=0.1, lambda_=1e-5, lr=5e-4, adam_step=40, step=39, seed=5)
    mllm_masked_linear_bwd_adam(mats, ios, (2, 4), tokens, hp, mlws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    for mb, A, dY, (pi, m0, v0) in zip(mats, As, dYs, state):
        r = mb.W.shape[0]
        rows = np.unique(np.concatenate([[0, 127, 128, r - 1], rng.choice(r, 6, replace=False)]))
        _bwd_check(orc, mb, A, dY, hp, pi, m0, v0, rows_idx=rows)
