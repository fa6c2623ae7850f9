"""Guard bands: no kernel writes outside its output buffers.

compute-sanitizer is not available on this machine, so out-of-bounds writes are checked with
canaries: every device buffer a call writes is a view into a larger allocation whose margins
(before and after, 16-byte aligned) hold a sentinel bit pattern, and after the call the
margins must be bit-identical. Ragged shapes put partial tiles, odd block counts and partial
metadata words at the buffers' ends; every entry point that writes device memory runs.
"""
import numpy as np
import pytest
import torch

from sparsity_mask_sampling_b200 import (Hparams, MatrixBuffers, inputs, mllm_hard_pack, mllm_mask_stats,
                                         mllm_prior_init, mllm_prior_init_from_mask, mllm_sample_bwd_adam,
                                         mllm_sample_bwd_adam_fwd, mllm_sample_fwd, mllm_sparse_linear,
                                         mllm_workspace_bytes, sparse_linear_workspace)
from sparsity_mask_sampling_b200.buffers import pack_shapes

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 256  # bytes of margin on each side
SENTINEL = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` inside a byte buffer with sentinel margins."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) if len(shape) else 1
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        body = (nbytes + 15) // 16 * 16
        self.raw = torch.full((GUARD + body + GUARD,), SENTINEL, dtype=torch.uint8, device=DEV)
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.t.numel() * self.t.element_size():]
        return bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())


SHAPES = {(2, 4): [(37, 84), (33, 256), (5, 4)], (4, 8): [(19, 72), (33, 256), (3, 8)]}


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_sampler_calls_write_only_their_buffers(nm):
    n, m = nm
    C = {(2, 4): 6, (4, 8): 70}[nm]
    mats, guards = [], []
    for i, (r, c) in enumerate(SHAPES[nm]):
        B = r * c // m
        W = inputs.weights(r, c, "bf16", 0.02, seed=60 + i).to(DEV)
        G = inputs.upstream_grad(r, c, "bf16", 1e-3, seed=70 + i).to(DEV)
        g = {k: Guarded(s, d) for k, (s, d) in {
            "X": ((r, c), torch.bfloat16), "soft": ((r, c), torch.float32), "grad": ((B, C), torch.float32),
            "pi": ((B, C), torch.float32), "m": ((B, C), torch.float32), "v": ((B, C), torch.float32),
            "cand": ((B,), torch.uint8)}.items()}
        (vs, (ms, mdt)) = pack_shapes(r, c, nm)
        g["vals"] = Guarded(vs, torch.bfloat16)
        g["meta"] = Guarded(ms, mdt)
        mb = MatrixBuffers(W=W, G=G, X=g["X"].t, soft_mask=g["soft"].t, grad_logits=g["grad"].t,
                           logits=g["pi"].t, adam_m=g["m"].t, adam_v=g["v"].t, pack_values=g["vals"].t,
                           pack_meta=g["meta"].t, cand_idx=g["cand"].t, block_offset=1000 * i)
        g["m"].t.zero_()
        g["v"].t.zero_()
        mats.append(mb)
        guards.append(g)
    ws = torch.zeros(mllm_workspace_bytes(), dtype=torch.uint8, device=DEV)
    reg1, reg2 = Guarded((1,), torch.float64), Guarded((1,), torch.float64)
    stats = Guarded((4,), torch.float64)
    hp = Hparams(kappa=100.0, tau=2.0, lambda_=1e-5, lr=1e-3, adam_step=1, step=0, seed=3)
    hp2 = Hparams(kappa=120.0, tau=1.5, lambda_=1e-5, lr=1e-3, adam_step=2, step=1, seed=3)
    mllm_prior_init(mats, nm, 3.0, 0.01, 5)
    mllm_sample_fwd(mats, nm, hp, reg1.t, ws)
    mllm_sample_bwd_adam(mats, nm, hp)
    mllm_sample_bwd_adam_fwd(mats, nm, hp, hp2, reg2.t, ws)
    mllm_hard_pack(mats, nm)
    mllm_mask_stats(mats, nm, 100.0, stats.t, ws)
    prior = [Guarded((mb.cand_idx.numel(),), torch.uint8, mb.cand_idx) for mb in mats]
    mllm_prior_init_from_mask(mats, nm, [p.t for p in prior], 3.0, 0.01, 6)
    torch.cuda.synchronize()
    for i, g in enumerate(guards):
        for k, gb in g.items():
            assert gb.intact(), (nm, SHAPES[nm][i], k)
    assert reg1.intact() and reg2.intact() and stats.intact() and all(p.intact() for p in prior)


@pytest.mark.parametrize("nm,tokens", [((2, 4), 8), ((2, 4), 16), ((2, 4), 40), ((4, 8), 8), ((4, 8), 24)])
def test_sparse_linear_writes_only_y(nm, tokens):
    n, m = nm
    ws = sparse_linear_workspace(DEV)
    ops, ys = [], []
    for i, (r, c) in enumerate([(37, 256), (33, 1024), (7, 96), (19, m * 9)]):
        vals, meta = inputs.packed_hard_mask(r, c, nm, seed=80 + i, device=DEV)
        x = inputs.weights(tokens, c, "bf16", 1.0, seed=90 + i, device=DEV)
        y = Guarded((tokens, r), torch.float32)
        ops.append((vals, meta, x, y.t))
        ys.append(y)
    mllm_sparse_linear(ops, nm, tokens, ws)
    torch.cuda.synchronize()
    for i, y in enumerate(ys):
        assert y.intact(), (nm, tokens, i)
        assert bool(torch.isfinite(y.t).all())
