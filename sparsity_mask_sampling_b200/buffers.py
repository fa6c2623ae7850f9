"""Allocation of the per-matrix device buffers with torch (plumbing only)."""
from __future__ import annotations

import torch

from ._mllm import MatrixBuffers


def pack_shapes(rows: int, cols: int, nm):
    """Shapes and dtypes of the packed outputs: values [rows, cols*N/M] (weight dtype) and
    metadata (2:4: uint32-words [rows, ceil(cols/32)]; 4:8: uint16 [rows, cols/8])."""
    n, m = nm
    if m == 4:
        meta = ((rows, (cols // 4 + 7) // 8), torch.int32)
    else:
        meta = ((rows, cols // 8), torch.int16)
    return (rows, cols // m * n), meta


def alloc_matrix(W: torch.Tensor, nm, block_offset: int = 0, *, fwd=True, bwd=True, pack=False,
                 g_dtype=None, soft_mask=False, grad_logits=False, logits=None) -> MatrixBuffers:
    """Buffers for one matrix W [rows, cols] on W's device. Logits and moments are fp32
    [B, C]; X matches W's dtype; G (when bwd) is g_dtype (default: W's dtype)."""
    n, m = nm
    C = {(2, 4): 6, (4, 8): 70}[(n, m)]
    rows, cols = W.shape
    B = rows * cols // m
    dev = W.device
    mb = MatrixBuffers(W=W, block_offset=block_offset)
    mb.logits = logits if logits is not None else torch.empty(B, C, device=dev, dtype=torch.float32)
    if bwd:
        mb.adam_m = torch.zeros(B, C, device=dev, dtype=torch.float32)
        mb.adam_v = torch.zeros(B, C, device=dev, dtype=torch.float32)
        mb.G = torch.empty(rows, cols, device=dev, dtype=g_dtype or W.dtype)
    if fwd:
        mb.X = torch.empty_like(W)
    if soft_mask:
        mb.soft_mask = torch.empty(rows, cols, device=dev, dtype=torch.float32)
    if grad_logits:
        mb.grad_logits = torch.empty(B, C, device=dev, dtype=torch.float32)
    if pack:
        (vshape, (mshape, mdt)) = pack_shapes(rows, cols, nm)
        mb.pack_values = torch.empty(vshape, device=dev, dtype=W.dtype)
        mb.pack_meta = torch.empty(mshape, device=dev, dtype=mdt)
        mb.cand_idx = torch.empty(B, device=dev, dtype=torch.uint8)
    return mb
