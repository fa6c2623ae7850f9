"""Workloads and host-side schedules of the sampler.

Hyper-parameters follow MaskLLM's Table 7 as restated in the paper-graph-ui summary
(s.3.4 "Complete Training Algorithm and Hyperparameter Configuration"): logits from
N(0, 0.01), prior strength alpha = 3, kappa 100 -> 500 and tau 4 -> 0.05 linearly,
lambda = 1e-5, AdamW lr 5e-4 (LLaMA-2) / 1e-3 (GPT-3), weight decay 0.1. Beta and epsilon
are not stated on the pages; PyTorch's defaults (0.9, 0.999, 1e-8) are used.

Matrix shapes are written in x out (as the workloads name them) and stored as PyTorch
nn.Linear weights, [out, in], so blocks of M weights run along the input dimension.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple


def linear_schedule(x0: float, x1: float, t: int, T: int) -> float:
    """x_t = x0 + (x1 - x0) t / (T - 1), endpoints included (t = 0 .. T-1); evaluated as
    x0 (1 - f) + x1 f, f = t / (T - 1), so that both endpoints are exact."""
    if T <= 1:
        return x0
    f = t / (T - 1)
    return x0 * (1.0 - f) + x1 * f


@dataclass(frozen=True)
class MatrixShape:
    name: str
    rows: int  # out features
    cols: int  # in features (blocks run along this axis)


@dataclass(frozen=True)
class Workload:
    name: str
    nm: Tuple[int, int]
    matrices: Tuple[MatrixShape, ...]   # one layer
    layers: int = 1
    w_dtype: str = "bf16"
    g_dtype: str = "bf16"
    w_std: float = 0.02
    g_std: float = 1e-3
    outlier_frac: float = 0.0
    outlier_scale: float = 20.0
    steps: int = 1
    tau: Tuple[float, float] = (4.0, 4.0)
    kappa: Tuple[float, float] = (100.0, 100.0)
    lr: float = 5e-4
    lam: float = 1e-5
    alpha: float = 3.0
    init_std: float = 0.01
    weight_decay: float = 0.1
    seeds: Tuple[int, ...] = (0,)

    @property
    def C(self) -> int:
        return {(2, 4): 6, (4, 8): 70}[self.nm]

    def blocks_per_layer(self) -> int:
        return sum(m.rows * m.cols // self.nm[1] for m in self.matrices)

    def total_blocks(self) -> int:
        return self.layers * self.blocks_per_layer()

    def tau_at(self, t: int) -> float:
        return linear_schedule(self.tau[0], self.tau[1], t, self.steps)

    def kappa_at(self, t: int) -> float:
        return linear_schedule(self.kappa[0], self.kappa[1], t, self.steps)


def _llama_layer():
    return (MatrixShape("q", 4096, 4096), MatrixShape("k", 4096, 4096),
            MatrixShape("v", 4096, 4096), MatrixShape("o", 4096, 4096),
            MatrixShape("gate", 11008, 4096), MatrixShape("up", 11008, 4096),
            MatrixShape("down", 4096, 11008))


WORKLOADS = {
    # one 64x128 fp32 matrix, one step, then pack
    "tiny_2of4": Workload(
        name="tiny_2of4", nm=(2, 4), matrices=(MatrixShape("w", 64, 128),),
        w_dtype="f32", g_dtype="f32", w_std=0.02, g_std=1.0, steps=1,
        tau=(4.0, 4.0), kappa=(100.0, 100.0), lr=1e-3, seeds=(0,)),
    # GPT-3 843M-shaped layer (hidden 1536): QKV 1536x4608, proj, FC1 1536x6144, FC2 6144x1536
    "gpt3_843m_layer_2of4": Workload(
        name="gpt3_843m_layer_2of4", nm=(2, 4),
        matrices=(MatrixShape("qkv", 4608, 1536), MatrixShape("proj", 1536, 1536),
                  MatrixShape("fc1", 6144, 1536), MatrixShape("fc2", 1536, 6144)),
        steps=10, tau=(4.0, 0.05), kappa=(100.0, 500.0), lr=1e-3, seeds=tuple(range(1, 11))),
    # LLaMA-2-7B decoder layer with 1% outlier input channels x20
    "llama2_7b_layer_2of4": Workload(
        name="llama2_7b_layer_2of4", nm=(2, 4), matrices=_llama_layer(),
        outlier_frac=0.01, steps=100, tau=(4.0, 0.05), kappa=(100.0, 500.0), lr=5e-4, seeds=(0,)),
    # the full 32-layer LLaMA-2-7B-shaped stack, logits and AdamW state resident
    "llama2_7b_stack_2of4": Workload(
        name="llama2_7b_stack_2of4", nm=(2, 4), matrices=_llama_layer(), layers=32,
        outlier_frac=0.01, steps=10, tau=(4.0, 0.05), kappa=(100.0, 500.0), lr=5e-4, seeds=(0,)),
    # general 4:8 on the two FFN-shaped matrices
    "general_4of8": Workload(
        name="general_4of8", nm=(4, 8),
        matrices=(MatrixShape("up", 11008, 4096), MatrixShape("down", 4096, 11008)),
        steps=50, tau=(2.0, 2.0), kappa=(100.0, 100.0), lr=5e-4, seeds=(0,)),
    # one 4096x4096 matrix at 4:8 (2.1M blocks, 0.6 GB of logits): a small case of the 4:8
    # kernels for profiler captures (inputs still larger than L2)
    "square_4096_4of8": Workload(
        name="square_4096_4of8", nm=(4, 8), matrices=(MatrixShape("w", 4096, 4096),),
        steps=50, tau=(2.0, 2.0), kappa=(100.0, 100.0), lr=5e-4, seeds=(0,)),
}


def layer_block_offsets(w: Workload) -> List[List[int]]:
    """Global block id of block 0 of every matrix: consecutive over layers and matrices."""
    out, acc = [], 0
    for _ in range(w.layers):
        row = []
        for m in w.matrices:
            row.append(acc)
            acc += m.rows * m.cols // w.nm[1]
        out.append(row)
    return out
