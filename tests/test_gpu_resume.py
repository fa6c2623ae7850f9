"""Checkpoint and resume: the training state is the logits, the AdamW moments and the step
(the noise is a function of seed, step and block id), so a run saved after k steps and
resumed in a fresh stack continues the uninterrupted trajectory bit for bit."""
import os
import tempfile

import pytest
import torch

from sparsity_mask_sampling_b200 import configs
from sparsity_mask_sampling_b200.stack import SamplerStack

pytestmark = pytest.mark.gpu


def _run(stack, t0, t1):
    for t in range(t0, t1):
        stack.step(t)
    torch.cuda.synchronize()


def test_resume_is_bitwise_identical():
    w = configs.WORKLOADS["gpt3_843m_layer_2of4"]
    a = SamplerStack(w, "cuda", rng_seed=3)
    a.prior_init(seed=0)
    _run(a, 0, 6)
    final = [[(mb.logits.clone(), mb.adam_m.clone(), mb.adam_v.clone()) for mb in mats] for mats in a.bufs]
    del a

    b = SamplerStack(w, "cuda", rng_seed=3)
    b.prior_init(seed=0)
    _run(b, 0, 3)
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "ckpt.pt")
        torch.save(b.state_dict(step=3), path)
        del b
        c = SamplerStack(w, "cuda", rng_seed=999)       # a fresh stack, different seed until restored
        t = c.load_state_dict(torch.load(path))
    assert t == 3 and c.rng_seed == 3
    _run(c, t, 6)
    for mats, ref in zip(c.bufs, final):
        for mb, (pi, m, v) in zip(mats, ref):
            assert torch.equal(mb.logits, pi) and torch.equal(mb.adam_m, m) and torch.equal(mb.adam_v, v)
