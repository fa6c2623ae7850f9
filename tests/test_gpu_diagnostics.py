"""Parity of the mask diagnostics and candidate-index codec (NEXT row f2) with the oracle."""
import numpy as np
import pytest
import torch

from sparsity_mask_sampling_b200 import (alloc_matrix, inputs, mllm_decode_candidates, mllm_encode_candidates,
                                         mllm_mask_diff, mllm_mask_stats, mllm_prior_init, mllm_workspace_bytes)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def orc():
    import oracle

    oracle.build()
    return oracle


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 1000, 1 << 20, (1 << 20) + 7])
def test_mask_diff(orc, n):
    rng = np.random.default_rng(n)
    a = rng.integers(0, 6, size=n).astype(np.uint8)
    b = a.copy()
    flip = rng.random(n) < 0.1
    b[flip] = (b[flip] + 1) % 6
    out = torch.full((1,), 12345, dtype=torch.int64, device=DEV)
    mllm_mask_diff(torch.from_numpy(a).to(DEV), torch.from_numpy(b).to(DEV), out)
    torch.cuda.synchronize()
    assert out.item() == orc.mask_diff(a, b) == int(flip.sum())


@pytest.mark.parametrize("nm,shapes", [((2, 4), [(64, 128), (7, 36), (300, 256)]),
                                       ((4, 8), [(64, 128), (7, 40), (130, 256)])])
def test_mask_stats(orc, nm, shapes):
    C = {(2, 4): 6, (4, 8): 70}[nm]
    mats, ref = [], np.zeros(4)
    for i, (r, c) in enumerate(shapes):
        W = inputs.weights(r, c, "bf16", 0.02, seed=i)
        mb = alloc_matrix(W.to(DEV), nm, 0, fwd=False, bwd=False)
        mllm_prior_init([mb], nm, 3.0, 0.01, seed=i)   # logits near the magnitude prior
        torch.cuda.synchronize()
        pi = mb.logits.cpu().numpy()
        ref += orc.mask_stats(*nm, W.float().double().numpy().reshape(-1, nm[1]), pi, kappa=100.0)
        mats.append(mb)
    ws = torch.zeros(mllm_workspace_bytes(), dtype=torch.uint8, device=DEV)
    out = torch.zeros(4, dtype=torch.float64, device=DEV)
    mllm_mask_stats(mats, nm, 100.0, out, ws)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert abs(got[0] - ref[0]) <= 1e-5 * ref[0]          # fp32 softmax sums per block
    assert abs(got[1] - ref[1]) <= 1e-9 * ref[1] and abs(got[2] - ref[2]) <= 1e-9 * ref[2]
    assert got[3] == ref[3]
    B = sum(r * c // nm[1] for r, c in shapes)
    assert 1.0 / C < got[0] / B <= 1.0 and got[1] <= got[2] + 1e-12


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
@pytest.mark.parametrize("n", [1, 11, 12, 13, 100_003])
def test_codec(orc, nm, n):
    C, D = {(2, 4): (6, 12), (4, 8): (70, 5)}[nm]
    k = np.random.default_rng(n).integers(0, C, size=n).astype(np.uint8)
    words = torch.zeros((n + D - 1) // D, dtype=torch.int32, device=DEV)
    mllm_encode_candidates(nm, torch.from_numpy(k).to(DEV), words)
    back = torch.zeros(n, dtype=torch.uint8, device=DEV)
    mllm_decode_candidates(nm, words, n, back)
    torch.cuda.synchronize()
    assert np.array_equal(words.cpu().numpy().view(np.uint32), orc.encode_candidates(*nm, k))
    assert np.array_equal(back.cpu().numpy(), k)
