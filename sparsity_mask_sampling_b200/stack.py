"""A model's worth of sampler state on one GPU, driven layer by layer (host plumbing).

Holds, for every weight matrix of a workload, the resident buffers (frozen W, logits and
AdamW moments) and streams the per-step tensors (soft-masked weights X out, upstream
gradients G in) through a pool of two layers' worth of buffers, as a training loop would
hand them to and from the frozen network. One training step = the forward of every layer
(one grouped launch each) then the fused backward + AdamW in reverse layer order.

With x_per_layer=True every matrix keeps its own X, as a loop that runs the fused call
(step t's backward + AdamW and step t+1's forward in one launch per layer) needs: layer l's
next-step X is produced during this step's backward and read at the next step's forward.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import _mllm as M
from . import inputs, sharding
from .configs import Workload

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


class SamplerStack:
    def __init__(self, w: Workload, device, rank: int = 0, seed_base: int = 0, rng_seed: int = 0,
                 x_per_layer: bool = False):
        self.w = w
        self.x_per_layer = x_per_layer
        self.dev = torch.device(device)
        self.nm = w.nm
        self.C = w.C
        self.rng_seed = rng_seed
        self.offsets = sharding.weak_block_offsets(w, rank)
        wdt = _DT[w.w_dtype]
        # X and G pools: two layers' worth, alternating between consecutive layers
        self.pool = []
        for p in range(2):
            self.pool.append([(torch.empty(m.rows, m.cols, dtype=wdt, device=self.dev),
                               inputs.upstream_grad(m.rows, m.cols, w.g_dtype, w.g_std,
                                                    seed=seed_base + 1000 + 10 * p + i, device=self.dev))
                              for i, m in enumerate(w.matrices)])
        self.bufs: List[List[M.MatrixBuffers]] = []
        self._views = []
        self.own_x = []
        for l in range(w.layers):
            mats = []
            for i, m in enumerate(w.matrices):
                W = inputs.weights(m.rows, m.cols, w.w_dtype, w.w_std, seed=seed_base + 100 * l + i,
                                   outlier_frac=w.outlier_frac, outlier_scale=w.outlier_scale, device=self.dev)
                B = m.rows * m.cols // w.nm[1]
                mats.append(M.MatrixBuffers(
                    W=W, block_offset=self.offsets[l][i],
                    logits=torch.empty(B, w.C, dtype=torch.float32, device=self.dev),
                    adam_m=torch.zeros(B, w.C, dtype=torch.float32, device=self.dev),
                    adam_v=torch.zeros(B, w.C, dtype=torch.float32, device=self.dev)))
            self.bufs.append(mats)
            self._views.append(None)
            if x_per_layer:
                self.own_x.append([torch.empty(m.rows, m.cols, dtype=wdt, device=self.dev) for m in w.matrices])
        self.ws = torch.zeros(M.mllm_workspace_bytes(), dtype=torch.uint8, device=self.dev)
        self.reg = torch.zeros(w.layers, dtype=torch.float64, device=self.dev)
        self.blocks = w.total_blocks()
        self.rebuild_views()

    def rebuild_views(self):
        """(Re)build the C matrix arrays; call after replacing any buffer of self.bufs."""
        self._views = []
        for l, mats in enumerate(self.bufs):
            for i, (mb, (X, G)) in enumerate(zip(mats, self.pool[l % 2])):
                mb.X = self.own_x[l][i] if self.x_per_layer else X
                mb.G = G
            self._views.append(M.MatrixArray(mats))

    def view(self, l: int) -> M.MatrixArray:
        return self._views[l]

    def XG(self, l: int, i: int):
        """The (X, G) buffers layer l's matrix i uses."""
        X, G = self.pool[l % 2][i]
        return (self.own_x[l][i] if self.x_per_layer else X), G

    def prior_init(self, seed: int = 0, alpha: Optional[float] = None, init_std: Optional[float] = None):
        a = self.w.alpha if alpha is None else alpha
        s = self.w.init_std if init_std is None else init_std
        for l in range(self.w.layers):
            M.mllm_prior_init(self.view(l), self.nm, a, s, seed)

    def hparams(self, t: int) -> M.Hparams:
        T = max(self.w.steps, 1)
        return M.Hparams(kappa=self.w.kappa_at(t % T), tau=self.w.tau_at(t % T), lambda_=self.w.lam,
                         lr=self.w.lr, weight_decay=self.w.weight_decay, adam_step=t + 1, step=t,
                         seed=self.rng_seed)

    def forward(self, l: int, hp):
        M.mllm_sample_fwd(self.view(l), self.nm, hp, self.reg[l:l + 1], self.ws)

    def backward(self, l: int, hp):
        M.mllm_sample_bwd_adam(self.view(l), self.nm, hp)

    def backward_forward(self, l: int, hp, hp_next):
        M.mllm_sample_bwd_adam_fwd(self.view(l), self.nm, hp, hp_next, self.reg[l:l + 1], self.ws)

    def forward_all(self, t: int):
        """The forward of every layer for step t (the first step of a fused loop)."""
        hp = self.hparams(t).to_c()
        for l in range(self.w.layers):
            self.forward(l, hp)

    def step_fused(self, t: int, ev=None, copy_fn=None, g_free=None):
        """Enqueue step t of a fused loop: per layer in reverse order, step t's backward +
        AdamW and step t+1's forward in one launch (step t's forward ran before)."""
        hp, hpn = self.hparams(t).to_c(), self.hparams(t + 1).to_c()
        for l in reversed(range(self.w.layers)):
            if copy_fn is not None:
                copy_fn(l)
            if ev is not None:
                ev[l][0].record()
            self.backward_forward(l, hp, hpn)
            if ev is not None:
                ev[l][1].record()
            if g_free is not None:
                g_free[l % 2].record()

    def step(self, t: int, ev=None, copy_fn=None, g_free=None):
        """Enqueue one training step on the current stream. ev: optional {"fwd", "bwd"} lists of
        per-layer (start, end) CUDA events; copy_fn(l) enqueues layer l's G before its
        backward; g_free[p] is recorded after each backward that used pool p."""
        hp = self.hparams(t).to_c()
        L = self.w.layers
        for l in range(L):
            if ev is not None:
                ev["fwd"][l][0].record()
            self.forward(l, hp)
            if ev is not None:
                ev["fwd"][l][1].record()
        for l in reversed(range(L)):
            if copy_fn is not None:
                copy_fn(l)
            if ev is not None:
                ev["bwd"][l][0].record()
            self.backward(l, hp)
            if ev is not None:
                ev["bwd"][l][1].record()
            if g_free is not None:
                g_free[l % 2].record()

    # ------------------------------------------------------------------ checkpoint / resume

    def state_dict(self, step: int) -> dict:
        """The whole training state: logits and AdamW moments of every matrix (host copies)
        and the next step. The noise is a function of (seed, step, block), so this is all a
        resumed run needs to continue the same trajectory bit for bit."""
        return {"step": int(step), "rng_seed": self.rng_seed, "workload": self.w.name,
                "logits": [[mb.logits.cpu() for mb in mats] for mats in self.bufs],
                "adam_m": [[mb.adam_m.cpu() for mb in mats] for mats in self.bufs],
                "adam_v": [[mb.adam_v.cpu() for mb in mats] for mats in self.bufs]}

    def load_state_dict(self, sd: dict) -> int:
        """Restore a state saved by state_dict(); returns the step to continue from."""
        if sd["workload"] != self.w.name:
            raise ValueError("checkpoint of another workload")
        self.rng_seed = sd["rng_seed"]
        for l, mats in enumerate(self.bufs):
            for i, mb in enumerate(mats):
                mb.logits.copy_(sd["logits"][l][i])
                mb.adam_m.copy_(sd["adam_m"][l][i])
                mb.adam_v.copy_(sd["adam_v"][l][i])
        return int(sd["step"])
