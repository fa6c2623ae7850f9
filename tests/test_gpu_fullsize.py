"""Parity at the workloads' full sizes, in the launch configurations the benchmark times.

Each workload is built at its real shapes with SamplerStack (one grouped launch per layer,
global block ids as in the benchmark, up to 1.6e9 for the 32-layer stack) and driven
through its schedule (tau, kappa, AdamW step). The oracle cannot process 1.6e9 blocks, so
outputs are compared on a sample: whole rows (first, last and random ones, so that packed
metadata words are complete) plus random blocks, in the first, a middle and the last layer.

The oracle keeps its own state for the sampled blocks from its own prior initialisation,
and before each checked step that state (rounded to the fp32 storage) is written into the
sampled blocks on the GPU. Blocks are independent, so the sampled outputs of a full-size
step depend only on those inputs; every checked step is thus compared on identical
inputs, however far into the schedule (no input of the oracle ever comes from the GPU).
The regulariser of each checked layer is checked against a property that holds at any
size: the sum of squares of the layer's soft-masked weights.

The *_fused_loop tests drive the benchmark's timed loop itself (forward of step 0, then per
step one launch per layer of step t's backward + AdamW with step t+1's forward), so the
kernel the benchmark reports is checked at the benchmark's sizes and grid: its CTAs walk
many tiles each. There step t+1's soft-masked weights are compared with the oracle's
forward from the oracle's own updated logits.
"""
import numpy as np
import pytest
import torch

import _tol
from sparsity_mask_sampling_b200 import MatrixArray, buffers, configs, mllm_hard_pack
from sparsity_mask_sampling_b200.stack import SamplerStack

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def orc():
    import oracle

    oracle.build()
    return oracle


class Sample:
    """The sampled blocks of one matrix and the oracle's state for them."""

    def __init__(self, stack, l, i, rng, n_rows=3, n_rand=384):
        w = stack.w
        m = w.matrices[i]
        M = w.nm[1]
        self.l, self.i = l, i
        bpr = m.cols // M
        rows = sorted({0, m.rows - 1, *rng.choice(m.rows, size=n_rows - 2, replace=False).tolist()})
        self.rows = rows
        row_blocks = np.concatenate([np.arange(r * bpr, (r + 1) * bpr) for r in rows])
        B = m.rows * bpr
        rand = rng.choice(B, size=n_rand, replace=False)
        self.idx = np.unique(np.concatenate([row_blocks, rand, [0, B - 1]]))
        self.idx_t = torch.from_numpy(self.idx).to(DEV)
        mb = stack.bufs[l][i]
        self.mb = mb
        self.gids = np.uint64(mb.block_offset) + self.idx.astype(np.uint64)
        self.W = mb.W.view(-1, M)[self.idx_t].float().double().cpu().numpy()
        _, G = stack.XG(l, i)
        self.G = G.view(-1, M)[self.idx_t].float().double().cpu().numpy()
        self.Wraw_rows = mb.W[torch.tensor(rows, device=DEV)].cpu()

    def put_state(self, pi, m, v):
        """Write the oracle's state (fp32) into the sampled blocks on the GPU."""
        self.mb.logits[self.idx_t] = torch.from_numpy(np.asarray(pi, np.float32)).to(DEV)
        self.mb.adam_m[self.idx_t] = torch.from_numpy(np.asarray(m, np.float32)).to(DEV)
        self.mb.adam_v[self.idx_t] = torch.from_numpy(np.asarray(v, np.float32)).to(DEV)


def _check_prior(orc, stack, samples):
    w = stack.w
    for s in samples:
        pi_ref, _, _ = orc.prior_init(*w.nm, s.W, s.gids, w.alpha, w.init_std, 0)
        got = s.mb.logits[s.idx_t].cpu().numpy().astype(np.float64)
        err = np.abs(got - pi_ref)
        assert (err <= 1e-6 * np.abs(pi_ref).max(1, keepdims=True) + 1e-12).all()
        assert not s.mb.adam_m[s.idx_t].any() and not s.mb.adam_v[s.idx_t].any()
        s.pi, s.m, s.v = pi_ref.astype(np.float32), np.zeros_like(pi_ref, np.float32), np.zeros_like(pi_ref, np.float32)


def _checked_step(orc, stack, samples, t):
    """One full-size step on the GPU; sampled outputs against the oracle; oracle state advances."""
    w = stack.w
    n, M = w.nm
    hp = stack.hparams(t)
    hpc = hp.to_c()
    by_layer = {}
    for s in samples:
        s.put_state(s.pi, s.m, s.v)
        by_layer.setdefault(s.l, []).append(s)
    x_got = {}
    for l in range(w.layers):
        stack.forward(l, hpc)
        if l in by_layer:
            torch.cuda.synchronize()
            for s in by_layer[l]:
                X, _ = stack.XG(l, s.i)
                x_got[(l, s.i)] = X.view(-1, M)[s.idx_t].float().double().cpu().numpy()
            # regulariser of the layer: sum of squares of its soft-masked weights (rounded X)
            r_x = sum(float((stack.XG(l, i)[0].double() ** 2).sum()) for i in range(len(w.matrices)))
            r = float(stack.reg[l].item())
            assert abs(r - r_x) <= 1e-3 * r, (l, r, r_x)
    for l in reversed(range(w.layers)):
        stack.backward(l, hpc)
    torch.cuda.synchronize()
    for s in samples:
        fwd = orc.sample_fwd(n, M, s.W, s.pi, s.gids, hp.kappa, hp.tau, hp.seed, hp.step)
        _tol.assert_x_close(x_got[(s.l, s.i)], fwd["x"], w.w_dtype, s.W)
        g_ref, scale = orc.sample_bwd(n, M, s.W, s.G, s.pi, s.gids, hp.kappa, hp.tau, hp.lambda_, hp.seed, hp.step)
        f32 = np.float32
        p_ref, m_ref, v_ref = orc.adamw(s.pi, s.m, s.v, g_ref, f32(hp.lr), f32(hp.beta1), f32(hp.beta2),
                                        f32(hp.eps), f32(hp.weight_decay), hp.adam_step)
        floor = _tol.grad_floor(s.W, s.G, hp.kappa, hp.tau, hp.lambda_)
        _tol.assert_logits_close(s.mb.logits[s.idx_t].cpu().numpy(), p_ref)
        _tol.assert_moments_close(s.mb.adam_m[s.idx_t].cpu().numpy(), s.mb.adam_v[s.idx_t].cpu().numpy(),
                                  m_ref, v_ref, g_ref, 1e-4 * scale + floor, f32(hp.beta1), f32(hp.beta2))
        s.pi, s.m, s.v = p_ref.astype(np.float32), m_ref.astype(np.float32), v_ref.astype(np.float32)


def _advance(orc, stack, samples, t):
    """Oracle-only step for the sampled blocks (steps the GPU does not check)."""
    w = stack.w
    n, M = w.nm
    hp = stack.hparams(t)
    f32 = np.float32
    for s in samples:
        g_ref, _ = orc.sample_bwd(n, M, s.W, s.G, s.pi, s.gids, hp.kappa, hp.tau, hp.lambda_, hp.seed, hp.step)
        p, m, v = orc.adamw(s.pi, s.m, s.v, g_ref, f32(hp.lr), f32(hp.beta1), f32(hp.beta2), f32(hp.eps),
                            f32(hp.weight_decay), hp.adam_step)
        s.pi, s.m, s.v = p.astype(np.float32), m.astype(np.float32), v.astype(np.float32)


def _check_pack(orc, stack, samples):
    """Pack the checked layers (full matrices); the sampled rows match the oracle bit for bit."""
    w = stack.w
    n, M = w.nm
    layers = sorted({s.l for s in samples})
    for l in layers:
        mats = stack.bufs[l]
        for mb, m in zip(mats, w.matrices):
            (vs, (ms, mdt)) = buffers.pack_shapes(m.rows, m.cols, w.nm)
            mb.pack_values = torch.empty(vs, dtype=mb.W.dtype, device=DEV)
            mb.pack_meta = torch.empty(ms, dtype=mdt, device=DEV)
            mb.cand_idx = torch.empty(m.rows * m.cols // M, dtype=torch.uint8, device=DEV)
        for s in samples:
            if s.l == l:
                s.put_state(s.pi, s.m, s.v)
        mllm_hard_pack(MatrixArray(mats), w.nm)
    torch.cuda.synchronize()
    view = np.uint16 if w.w_dtype == "bf16" else np.uint32
    ity = torch.int16 if w.w_dtype == "bf16" else torch.int32
    for s in samples:
        m = w.matrices[s.i]
        bpr = m.cols // M
        rows_t = torch.tensor(s.rows, device=DEV)
        pos = {b: k for k, b in enumerate(s.idx)}
        raw = s.Wraw_rows.view(ity).numpy().view(view)
        pi_rows = np.stack([s.pi[pos[r * bpr + q]] for r in s.rows for q in range(bpr)])
        vals, meta, cand = orc.hard_pack(n, M, raw, pi_rows)
        got_v = s.mb.pack_values[rows_t].view(ity).cpu().numpy().view(view)
        got_m = s.mb.pack_meta[rows_t].cpu().numpy().view(meta.dtype)
        got_c = s.mb.cand_idx.view(m.rows, bpr)[rows_t].cpu().numpy().ravel()
        assert np.array_equal(got_v, vals) and np.array_equal(got_m, meta) and np.array_equal(got_c, cand)


def _run(orc, name, check_steps, layers=None, seed=0, rng_seed=0):
    w = configs.WORKLOADS[name]
    torch.cuda.empty_cache()
    stack = SamplerStack(w, DEV, rng_seed=rng_seed)
    stack.prior_init(seed=0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    layers = layers if layers is not None else sorted({0, w.layers // 2, w.layers - 1})
    samples = [Sample(stack, l, i, rng) for l in layers for i in range(len(w.matrices))]
    _check_prior(orc, stack, samples)
    last = max(check_steps)
    for t in range(last + 1):
        if t in check_steps:
            _checked_step(orc, stack, samples, t)
        else:
            _advance(orc, stack, samples, t)
    _check_pack(orc, stack, samples)
    del stack
    torch.cuda.empty_cache()


def _check_next_forward(orc, stack, samples, t_next):
    """X of step t_next (written by the previous launch) in the sampled blocks against the
    oracle's forward from the oracle's own state, and every checked layer's regulariser
    against the sum of squares of its soft-masked weights."""
    w = stack.w
    n, M = w.nm
    hp = stack.hparams(t_next)
    for s in samples:
        X, _ = stack.XG(s.l, s.i)
        got = X.view(-1, M)[s.idx_t].float().double().cpu().numpy()
        fwd = orc.sample_fwd(n, M, s.W, s.pi, s.gids, hp.kappa, hp.tau, hp.seed, hp.step)
        _tol.assert_x_close(got, fwd["x"], w.w_dtype, s.W)
    for l in sorted({s.l for s in samples}):
        r_x = sum(float((stack.XG(l, i)[0].double() ** 2).sum()) for i in range(len(w.matrices)))
        r = float(stack.reg[l].item())
        assert abs(r - r_x) <= 1e-3 * r, (l, r, r_x)


def _run_fused(orc, name, check_steps, layers=None, seed=0, rng_seed=0):
    """The benchmark's own loop (SamplerStack.forward_all, then one step_fused per step: per
    layer one launch of step t's backward + AdamW and step t+1's forward), at full size.
    Before a checked step the oracle's state is written into the sampled blocks; after it
    the sampled logits and moments are compared with the oracle's AdamW on the oracle's
    gradient, and the next step's soft-masked weights with the oracle's forward from the
    oracle's updated logits (no oracle input comes from the GPU)."""
    w = configs.WORKLOADS[name]
    n, M = w.nm
    torch.cuda.empty_cache()
    stack = SamplerStack(w, DEV, rng_seed=rng_seed, x_per_layer=True)
    stack.prior_init(seed=0)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    layers = layers if layers is not None else sorted({0, w.layers // 2, w.layers - 1})
    samples = [Sample(stack, l, i, rng) for l in layers for i in range(len(w.matrices))]
    _check_prior(orc, stack, samples)
    for s in samples:
        s.put_state(s.pi, s.m, s.v)
    stack.forward_all(0)
    torch.cuda.synchronize()
    _check_next_forward(orc, stack, samples, 0)
    f32 = np.float32
    for t in range(max(check_steps) + 1):
        if t not in check_steps:
            stack.step_fused(t)
            _advance(orc, stack, samples, t)
            continue
        for s in samples:
            s.put_state(s.pi, s.m, s.v)
        stack.step_fused(t)
        torch.cuda.synchronize()
        hp = stack.hparams(t)
        for s in samples:
            g_ref, scale = orc.sample_bwd(n, M, s.W, s.G, s.pi, s.gids, hp.kappa, hp.tau, hp.lambda_, hp.seed,
                                          hp.step)
            p_ref, m_ref, v_ref = orc.adamw(s.pi, s.m, s.v, g_ref, f32(hp.lr), f32(hp.beta1), f32(hp.beta2),
                                            f32(hp.eps), f32(hp.weight_decay), hp.adam_step)
            floor = _tol.grad_floor(s.W, s.G, hp.kappa, hp.tau, hp.lambda_)
            pe = _tol.assert_logits_close(s.mb.logits[s.idx_t].cpu().numpy(), p_ref)
            print(f"{name} step {t} layer {s.l} matrix {s.i}: worst per-element relative error of the "
                  f"updated logits {pe:.3g}")
            _tol.assert_moments_close(s.mb.adam_m[s.idx_t].cpu().numpy(), s.mb.adam_v[s.idx_t].cpu().numpy(),
                                      m_ref, v_ref, g_ref, 1e-4 * scale + floor, f32(hp.beta1), f32(hp.beta2))
            s.pi, s.m, s.v = p_ref.astype(np.float32), m_ref.astype(np.float32), v_ref.astype(np.float32)
        _check_next_forward(orc, stack, samples, t + 1)
    _check_pack(orc, stack, samples)
    del stack
    torch.cuda.empty_cache()


def test_gpt3_843m_layer_every_step_all_seeds(orc):
    """GPT-3-843M-shaped layer, tau 4 -> 0.05 and kappa 100 -> 500 over 10 steps, every step
    checked, for each of the workload's ten runs (noise seeds 1..10)."""
    for rs in configs.WORKLOADS["gpt3_843m_layer_2of4"].seeds:
        _run(orc, "gpt3_843m_layer_2of4", check_steps=set(range(10)), rng_seed=rs, seed=rs)


def test_gpt3_843m_layer_fused_loop(orc):
    """The GPT-3-843M-shaped layer through the benchmark's fused loop, every step checked."""
    _run_fused(orc, "gpt3_843m_layer_2of4", check_steps=set(range(10)), rng_seed=3, seed=3)


def test_llama2_7b_layer_fused_loop(orc):
    """One LLaMA-2-7B layer (50.6 M blocks) through the benchmark's fused loop: steps 0, 50
    and 99 of its 100-step schedule checked (logits, moments, next X, regulariser)."""
    _run_fused(orc, "llama2_7b_layer_2of4", check_steps={0, 50, 99})


def test_llama2_7b_full_stack_fused_loop(orc):
    """All 32 layers in the benchmark's fused loop (its exact launches: 1,619,001,344 blocks,
    logits, moments and every layer's next-step X resident): the first, a middle and the
    last layer checked at steps 0 and 9."""
    _run_fused(orc, "llama2_7b_stack_2of4", check_steps={0, 9})


def test_general_4of8_fused_loop(orc):
    """4:8 through the fused loop (the call runs its two kernels), steps 0 and 49 checked."""
    _run_fused(orc, "general_4of8", check_steps={0, 49})


def test_llama2_7b_layer(orc):
    """One LLaMA-2-7B layer (50.6 M blocks), steps 0, 50 and 99 of its 100-step schedule."""
    _run(orc, "llama2_7b_layer_2of4", check_steps={0, 50, 99})


def test_llama2_7b_full_stack(orc):
    """All 32 layers (1,619,001,344 blocks, ~130 GB resident): the first, a middle and the
    last layer checked at the first and last steps of the 10-step schedule."""
    _run(orc, "llama2_7b_stack_2of4", check_steps={0, 9})


def test_general_4of8(orc):
    """4:8 on the two FFN-shaped matrices (11.3 M blocks of 70 candidates), steps 0 and 49."""
    _run(orc, "general_4of8", check_steps={0, 49})


def test_tiny_fp32(orc):
    """The tiny fp32 workload, whole matrix sampled, its single step."""
    _run(orc, "tiny_2of4", check_steps={0})
