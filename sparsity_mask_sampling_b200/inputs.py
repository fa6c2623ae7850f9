"""Seeded synthetic inputs (weights, upstream gradients, logits). No arithmetic of the method.

The pages evaluate on LLaMA-2 / GPT-3 checkpoints with language-modelling data; neither is
available, and the sampler's cost and arithmetic do not depend on the weights' values.
These generators stand in with normal weights of the workloads' shapes (std 0.02), a seeded
set of outlier input channels scaled up (the heavy-tailed channels of real LLM weights),
and normal upstream gradients dL/d(W.M) in place of the frozen network's backward pass.
Both the CUDA path and the oracle receive copies of the same bytes.
"""
from __future__ import annotations

import torch

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(rows: int, cols: int, dtype="bf16", std=0.02, seed=0, outlier_frac=0.0,
            outlier_scale=20.0, device="cpu") -> torch.Tensor:
    """W [rows, cols] ~ N(0, std^2); round(outlier_frac * cols) input channels (columns),
    chosen by a seeded permutation, are multiplied by outlier_scale."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    n_out = int(round(outlier_frac * cols))
    if n_out:
        idx = torch.randperm(cols, generator=g, device=device)[:n_out]
        w[:, idx] *= outlier_scale
    return w.to(_DT[dtype] if isinstance(dtype, str) else dtype)


def upstream_grad(rows: int, cols: int, dtype="bf16", std=1e-3, seed=1, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    return x.to(_DT[dtype] if isinstance(dtype, str) else dtype)


def logits(nblocks: int, C: int, std=0.02, seed=2, device="cpu") -> torch.Tensor:
    """Logits [nblocks, C] fp32 ~ N(0, std^2) (for exercising the forward on its own)."""
    g = _gen(seed, device)
    return torch.randn(nblocks, C, generator=g, device=device, dtype=torch.float32) * std


def moments(nblocks: int, C: int, seed=3, device="cpu"):
    """AdamW moments of a run in progress: m ~ N(0, 1e-4^2), v = |N(0, 1e-4^2)|^2-scale."""
    g = _gen(seed, device)
    m = torch.randn(nblocks, C, generator=g, device=device) * 1e-4
    v = torch.randn(nblocks, C, generator=g, device=device).abs() * 1e-8
    return m, v


def packed_hard_mask(rows: int, cols: int, nm, seed=0, device="cpu", std=0.02):
    """A hard-masked bf16 matrix already in mllm_hard_pack's compressed form: N(0, std^2)
    values and a uniformly drawn candidate per block, encoded as the pack encodes kept
    positions (2:4: nibble p0 | p1 << 2, 8 blocks per uint32 word of a row, unused nibbles
    zero; 4:8: uint16 p0 | p1 << 3 | p2 << 6 | p3 << 9). Returns (values [rows, cols*N/M]
    bf16, meta int32 [rows, ceil(cols/32)] or int16 [rows, cols/8]) -- a stand-in for a
    trained model's packed weights, whose serving cost does not depend on the values."""
    from itertools import combinations

    n, m = nm
    g = _gen(seed, device)
    bpr = cols // m
    vals = (torch.randn(rows, bpr * n, generator=g, device=device) * std).to(torch.bfloat16)
    combos = list(combinations(range(m), n))
    k = torch.randint(0, len(combos), (rows, bpr), generator=g, device=device)
    if m == 4:
        nib = torch.tensor([p[0] | p[1] << 2 for p in combos], device=device, dtype=torch.int64)[k]
        words = (bpr + 7) // 8
        pad = torch.zeros(rows, words * 8, device=device, dtype=torch.int64)
        pad[:, :bpr] = nib
        w = (pad.view(rows, words, 8) << (4 * torch.arange(8, device=device, dtype=torch.int64))).sum(-1)
        meta = torch.where(w >= 2 ** 31, w - 2 ** 32, w).to(torch.int32)
    else:
        codes = [p[0] | p[1] << 3 | p[2] << 6 | p[3] << 9 for p in combos]
        meta = torch.tensor(codes, device=device, dtype=torch.int16)[k]
    return vals, meta
