"""mllm_sample_fwd_noalloc, the forward for callers that cannot allocate device memory.

Such callers (a plugin inside a framework that owns the whole device-memory budget and
forbids cudaMalloc/cudaFree once running, or a runtime that only passes the step's tensors)
cannot provide the workspace that mllm_sample_fwd needs for its regulariser reduction. The
no-alloc entry point keeps that scratch in a fixed array inside the library. Here it is
called through the C ABI twice in a row, and each call's outputs are compared with the
workspace-based entry point on the same inputs. Both entry points launch the same kernels
with the same grids and reduce in the same order, so the soft-masked weights and the
regulariser must be identical bit for bit (any wrong partial slot or stale ticket would
show); this is stricter than the oracle parity tolerances (1e-3 relative, 1 bf16 ulp). A
layer of more than 16 matrices is split into several launches, which exercises the paths
only the no-alloc call has between launches: the ticket cleared before each launch and the
later launches adding to the regulariser.

This file is named to be collected last, so a run that stops at the first failure has run
every other test before it. It needs nothing from the other test files and passes alone.
"""
import pytest
import torch

from sparsity_mask_sampling_b200 import (Hparams, MllmError, alloc_matrix, inputs, mllm_sample_fwd,
                                         mllm_sample_fwd_noalloc, mllm_workspace_bytes)
from sparsity_mask_sampling_b200.build import build

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def _layer(nm, shapes, seed):
    mats, off = [], 0
    for i, (r, c) in enumerate(shapes):
        W = inputs.weights(r, c, "bf16", 0.02, seed=seed + i).to(DEV)
        mb = alloc_matrix(W, nm, off, fwd=True, bwd=False)
        mb.logits.copy_(inputs.logits(r * c // nm[1], {(2, 4): 6, (4, 8): 70}[nm], 0.02, seed + 50 + i).to(DEV))
        mats.append(mb)
        off += r * c // nm[1]
    return mats


@pytest.mark.parametrize("nm,shapes", [((2, 4), [(512, 1024), (77, 36), (1, 4)]),
                                       ((4, 8), [(256, 512), (3, 16)]),
                                       ((2, 4), [(8, 16)] * 20),
                                       ((4, 8), [(8, 16), (5, 24)] * 9)])
def test_noalloc_forward_matches_workspace_forward_twice(nm, shapes):
    mats = _layer(nm, shapes, seed=7)
    ws = torch.zeros(mllm_workspace_bytes(), dtype=torch.uint8, device=DEV)
    for call in range(2):
        hp = Hparams(kappa=100.0 + 200.0 * call, tau=2.0 / (1 + 10 * call), step=call, seed=11)
        reg_ref = torch.zeros(1, dtype=torch.float64, device=DEV)
        mllm_sample_fwd(mats, nm, hp, reg_ref, ws)
        x_ref = [m.X.clone() for m in mats]
        for m in mats:
            m.X.zero_()
        reg = torch.full((1,), -1.0, dtype=torch.float64, device=DEV)
        mllm_sample_fwd_noalloc(mats, nm, hp, reg)
        torch.cuda.synchronize()
        assert reg.item() == reg_ref.item()
        for m, xr in zip(mats, x_ref):
            assert torch.equal(m.X, xr)


def test_noalloc_requires_regulariser_output():
    mats = _layer((2, 4), [(8, 16)], seed=3)
    with pytest.raises(MllmError):
        mllm_sample_fwd_noalloc(mats, (2, 4), Hparams(), None)
