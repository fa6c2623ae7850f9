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
