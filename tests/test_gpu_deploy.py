"""Parity of mllm_sparse_linear (y = x W*^T on the packed hard mask) with the oracle.

The packed operands come from the oracle's own hard_pack of seeded weights and logits (no
oracle input comes from the GPU); a second set of cases runs the whole chain on the GPU
(hard_pack then sparse_linear) from the same seeded inputs. Sizes cover several k-chunks and
row tiles, ragged tails (rows not a multiple of the 32-row task, columns not a multiple of
the 64-column chunk, columns not a multiple of 16: the element-wise loader), every token
count class (1, 8, 9, 16), grouped calls with empty operands, and the LLaMA-2-7B shapes at
full size on sampled rows.
"""
from itertools import combinations

import numpy as np
import pytest
import torch

import _tol
from sparsity_mask_sampling_b200 import (MatrixArray, MatrixBuffers, configs, inputs, mllm_hard_pack,
                                         mllm_sparse_linear, mllm_sparse_linear_check_timeout,
                                         mllm_sparse_linear_workspace_bytes, sparse_linear_workspace)

pytestmark = pytest.mark.gpu
DEV = "cuda"
C_OF = {(2, 4): 6, (4, 8): 70}


@pytest.fixture(scope="module")
def ws():
    return sparse_linear_workspace(DEV)


def _tickets_clear(ws):
    """The call leaves its completion counters and error word (the workspace's tail: 4096
    tickets, then the error word and padding) at zero."""
    return not ws[-(4 * 4096 + 16):].any()


def _bf16_bits(rng, shape, std):
    f = rng.normal(0.0, std, size=shape).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _val(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def _dev_meta(meta):
    meta = np.ascontiguousarray(meta)
    return torch.from_numpy(meta.view(np.int32 if meta.dtype == np.uint32 else np.int16)).to(DEV)


def _random_packed(rng, nm, rows, cols):
    """A packed operand drawn directly: random bf16 values and a random valid candidate per
    block, encoded as hard_pack encodes it (for full-size shapes, where [B, C] logits for the
    oracle's hard_pack would take gigabytes of host memory)."""
    n, m = nm
    bpr = cols // m
    values = _bf16_bits(rng, (rows, bpr * n), 0.02)
    combos = list(combinations(range(m), n))
    k = rng.integers(0, len(combos), size=(rows, bpr))
    if m == 4:
        nib = np.array([p[0] | p[1] << 2 for p in combos], np.uint64)[k]
        words = (bpr + 7) // 8
        pad = np.zeros((rows, words * 8), np.uint64)
        pad[:, :bpr] = nib
        meta = (pad.reshape(rows, words, 8) << (4 * np.arange(8, dtype=np.uint64))).sum(-1).astype(np.uint32)
    else:
        meta = np.array([p[0] | p[1] << 3 | p[2] << 6 | p[3] << 9 for p in combos], np.uint16)[k]
    return values, meta


class Operand:
    def __init__(self, orc, nm, rows, cols, tokens, seed, direct=False):
        rng = np.random.default_rng(seed)
        n, m = nm
        self.nm, self.rows, self.cols = nm, rows, cols
        if direct:
            self.values, self.meta = _random_packed(rng, nm, rows, cols)
        else:
            self.W = _bf16_bits(rng, (rows, cols), 0.02)
            self.pi = rng.normal(0, 1, size=(rows * cols // m, C_OF[nm])).astype(np.float32)
            self.values, self.meta, _ = orc.hard_pack(n, m, self.W, self.pi)
        self.x = _bf16_bits(rng, (tokens, cols), 1.0)
        self.d_values, self.d_meta = _dev16(self.values), _dev_meta(self.meta)
        self.d_x = _dev16(self.x)
        self.y = torch.full((tokens, rows), float("nan"), dtype=torch.float32, device=DEV)

    def op(self):
        return (self.d_values, self.d_meta, self.d_x, self.y)

    def check(self, orc, rows_sel=None):
        n, m = self.nm
        vals, meta = self.values, self.meta
        if rows_sel is not None:
            vals, meta = vals[rows_sel], meta[rows_sel]
        y_ref = orc.sparse_linear(n, m, vals, meta, self.x)
        # sum_k |x_k w_k| for the tolerance: the same product with the sign bits cleared
        absxw = orc.sparse_linear(n, m, vals & 0x7FFF, meta, self.x & 0x7FFF)
        got = self.y.cpu().numpy().astype(np.float64)
        if rows_sel is not None:
            got = got[:, rows_sel]
        return _tol.assert_spl_close(got, y_ref, absxw, self.cols)


SHAPES = [(48, 256), (37, 1040), (70, 1088), (33, 84), (16, 40), (5, 8)]


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
@pytest.mark.parametrize("tokens", [1, 8, 9, 16])
def test_sparse_linear_matches_oracle(orc, ws, nm, tokens):
    shapes = [(r, c) for r, c in SHAPES if c % nm[1] == 0]
    ops = [Operand(orc, nm, r, c, tokens, seed=10 * i + tokens) for i, (r, c) in enumerate(shapes)]
    mllm_sparse_linear([o.op() for o in ops[:3]], nm, tokens, ws)       # one grouped call (vector loads)
    for o in ops[3:]:
        mllm_sparse_linear([o.op()], nm, tokens, ws)                    # element-wise loads
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_grouped_call_with_empty_operands_and_determinism(orc, ws, nm):
    tokens = 5
    a = Operand(orc, nm, 40, 512, tokens, seed=1)
    b = Operand(orc, nm, 24, 128, tokens, seed=2)
    empty_rows = (a.d_values, a.d_meta, torch.empty(tokens, 0, device=DEV, dtype=torch.bfloat16),
                  torch.empty(tokens, 0, device=DEV))
    y0 = torch.full((tokens, 12), float("nan"), device=DEV)
    no_cols = (None, None, torch.empty(tokens, 0, device=DEV, dtype=torch.bfloat16), y0)
    mllm_sparse_linear([a.op(), empty_rows, no_cols, b.op()], nm, tokens, ws)
    torch.cuda.synchronize()
    a.check(orc)
    b.check(orc)
    assert torch.equal(y0, torch.zeros_like(y0))
    first = a.y.clone()
    for _ in range(3):
        mllm_sparse_linear([a.op()], nm, tokens, ws)
    torch.cuda.synchronize()
    assert torch.equal(first, a.y)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_gpu_chain_pack_then_linear(orc, ws, nm):
    """hard_pack on the GPU, then sparse_linear on its output, against the oracle chain."""
    n, m = nm
    rows, cols, tokens = 96, 768, 8
    o = Operand(orc, nm, rows, cols, tokens, seed=5)
    W = _dev16(o.W)
    mb = MatrixBuffers(W=W, logits=torch.from_numpy(o.pi).to(DEV))
    mb.pack_values = torch.empty(rows, cols // m * n, dtype=torch.bfloat16, device=DEV)
    mb.pack_meta = torch.empty(o.d_meta.shape, dtype=o.d_meta.dtype, device=DEV)
    mllm_hard_pack(MatrixArray([mb]), nm)
    mllm_sparse_linear([(mb.pack_values, mb.pack_meta, o.d_x, o.y)], nm, tokens, ws)
    torch.cuda.synchronize()
    assert torch.equal(mb.pack_meta, o.d_meta)
    o.check(orc)


@pytest.mark.parametrize("nm,tokens", [((2, 4), 8), ((2, 4), 16), ((4, 8), 8)])
def test_llama_shapes_full_size_sampled_rows(orc, ws, nm, tokens):
    """q/o [4096, 4096], gate [11008, 4096], down [4096, 11008] in one grouped call, the
    launch the benchmark times; the oracle checks 24 rows of each (first, last, random)."""
    shapes = [(4096, 4096), (11008, 4096), (4096, 11008)]
    ops = [Operand(orc, nm, r, c, tokens, seed=50 + i, direct=True) for i, (r, c) in enumerate(shapes)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    for o in ops:
        sel = np.unique(np.concatenate([[0, o.rows - 1], rng.choice(o.rows, 22, replace=False)]))
        o.check(orc, sel)
        assert torch.isfinite(o.y).all()
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
@pytest.mark.parametrize("tokens", [3, 16, 40])
def test_tiles_cut_into_many_pieces(orc, ws, nm, tokens):
    """Few rows and long rows: each tile is cut between hundreds of warps (32-row tiles) or,
    at 40 tokens and 2:4, between 128 CTAs (one 128-row tile of 128 chunks), whose partial
    tiles the last arriving warp or CTA adds; repeated calls reuse the workspace."""
    o = Operand(orc, nm, 40, 16384, tokens, seed=77, direct=True)
    for _ in range(2):
        mllm_sparse_linear([o.op()], nm, tokens, ws)
    torch.cuda.synchronize()
    o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("tokens", [2, 8, 13])
def test_2of4_tensor_core_path_ragged(orc, ws, tokens):
    """2:4 with whole metadata words (cols % 32 == 0) runs on the sparse tensor cores: rows
    not a multiple of the 32-row tile and a last 64-column chunk with only one 32-column
    window in the matrix."""
    nm = (2, 4)
    ops = [Operand(orc, nm, r, c, tokens, seed=90 + i) for i, (r, c) in enumerate([(45, 96), (33, 160), (7, 32)])]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


def test_full_stack_call_as_benchmarked(orc, ws):
    """The benchmark's serving call: the 224 matrices of the 32-layer LLaMA-2-7B stack as
    packed 2:4 hard masks (7.3 GB; inputs.packed_hard_mask with the benchmark's seeds), one
    call of 14 launches at 8 tokens; the oracle checks sampled rows of matrices in the first,
    middle and last layers (every shape), and every output is written."""
    w = configs.WORKLOADS["llama2_7b_stack_2of4"]
    T = 8
    shapes = [(m.rows, m.cols) for _ in range(w.layers) for m in w.matrices]
    packed = [inputs.packed_hard_mask(r, c, w.nm, seed=1000 + i, device=DEV) for i, (r, c) in enumerate(shapes)]
    xs = {c: inputs.weights(T, c, "bf16", 1.0, seed=c, device=DEV) for c in {c for _, c in shapes}}
    ys = [torch.full((T, r), float("nan"), device=DEV) for r, _ in shapes]
    mllm_sparse_linear([(v, mt, xs[c], y) for (v, mt), (r, c), y in zip(packed, shapes, ys)], w.nm, T, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    for i in [0, 4, 6, 7 * 15 + 1, 7 * 15 + 5, 7 * 31 + 3, len(shapes) - 1]:
        (v, mt), (r, c) = packed[i], shapes[i]
        sel = np.unique(np.concatenate([[0, r - 1], rng.choice(r, 14, replace=False)]))
        sel_t = torch.from_numpy(sel).to(DEV)
        vals = v[sel_t].view(torch.int16).cpu().numpy().view(np.uint16)
        meta = mt[sel_t].cpu().numpy().view(np.uint32)
        x = xs[c].view(torch.int16).cpu().numpy().view(np.uint16)
        y_ref = orc.sparse_linear(2, 4, vals, meta, x)
        absxw = orc.sparse_linear(2, 4, vals & 0x7FFF, meta, x & 0x7FFF)
        got = ys[i][:, sel_t].cpu().numpy().astype(np.float64)
        _tol.assert_spl_close(got, y_ref, absxw, c)
    assert all(bool(torch.isfinite(y).all()) for y in ys)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm,tokens", [((2, 4), 4), ((2, 4), 40), ((4, 8), 4), ((4, 8), 40)])
def test_bounded_wait_reports_error_and_context_survives(orc, nm, tokens):
    """Failure detection of the copy pipelines (per-warp kernels at 4 tokens, tensor-memory
    kernels at 40): a launch whose first stage is armed but never filled makes the bounded
    waits (1 s) run out; the call sets the workspace's error word, returns, and the next call
    on a re-zeroed workspace is exact."""
    import time

    ws = sparse_linear_workspace(DEV)
    o = Operand(orc, nm, 64, 256, tokens, seed=31)
    t0 = time.time()
    mllm_sparse_linear_check_timeout(o.op(), nm, tokens, ws)
    torch.cuda.synchronize()
    assert time.time() - t0 < 60
    assert int(ws[-16:-12].view(torch.int32).item()) != 0
    ws.zero_()
    mllm_sparse_linear([o.op()], nm, tokens, ws)
    torch.cuda.synchronize()
    o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm,tokens", [((2, 4), 6), ((4, 8), 6), ((2, 4), 40)])
def test_many_operands_of_mixed_widths_in_one_call(orc, ws, nm, tokens):
    """More than 16 operands whose widths take different kernels (multiples of 128, of 32, of
    16, and odd multiples of M) in one call: the call groups them per kernel and per 16 (at
    40 tokens: 2:4 widths that are multiples of 128 in two tensor-memory launches, the
    others in groups of 16 tokens)."""
    m = nm[1]
    widths = [256, 384, 96, 160, 48, 80, 4 * m * 3, 128, 1024, 32 * m, 16 * 3, 8 * m + m]
    widths = [c for c in widths if c % m == 0]
    n_ops = 22 if tokens <= 16 else 40
    ops = [Operand(orc, nm, 17 + 5 * i, widths[i % len(widths)], tokens, seed=200 + i) for i in range(n_ops)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("tokens", [17, 32, 33, 48, 49, 64])
def test_batched_decode_2of4(orc, ws, tokens):
    """17-64 tokens at 2:4: the tensor-memory kernel (128-row tiles, N = tokens rounded up to
    16, at least 32) for widths that are multiples of 128 (ragged rows, tiles cut between
    CTAs), token groups of 16 for the others, in one call."""
    nm = (2, 4)
    shapes = [(45, 256), (130, 1024), (7, 128), (64, 96), (33, 40)]
    ops = [Operand(orc, nm, r, c, tokens, seed=300 + i) for i, (r, c) in enumerate(shapes)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("tokens", [17, 24, 33, 48, 64])
def test_batched_decode_4of8(orc, ws, tokens):
    """17-64 tokens at 4:8: the tensor-memory kernel (blocks expanded to a dense tile in shared
    memory, dense tcgen05.mma) for widths that are multiples of 128 (ragged rows, tiles cut
    between CTAs), token groups of 16 for the others, in one call."""
    nm = (4, 8)
    shapes = [(40, 256), (130, 1024), (7, 128), (19, 72), (33, 40)]
    ops = [Operand(orc, nm, r, c, tokens, seed=320 + i) for i, (r, c) in enumerate(shapes)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
def test_batched_decode_full_size_64_tokens(orc, ws, nm):
    """q [4096, 4096], gate [11008, 4096], down [4096, 11008] at 64 tokens in one call."""
    tokens = 64
    ops = [Operand(orc, nm, r, c, tokens, seed=340 + i, direct=True)
           for i, (r, c) in enumerate([(4096, 4096), (11008, 4096), (4096, 11008)])]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    for o in ops:
        sel = np.unique(np.concatenate([[0, o.rows - 1], rng.choice(o.rows, 14, replace=False)]))
        o.check(orc, sel)
        assert torch.isfinite(o.y).all()
    assert _tickets_clear(ws)


@pytest.mark.parametrize("tokens", [8, 40])
def test_side_streams_and_concurrent_host_threads(orc, tokens):
    """The stream argument is honoured (work on a side stream, then that stream's sync) and
    two host threads can drive the library at once with their own workspaces and streams
    (the binding releases the GIL; the library keeps per-thread launch state). At 40 tokens
    the two streams' tensor-memory kernels share SMs (each CTA holds 128 TMEM columns)."""
    import threading

    nm = (2, 4)
    sets = [[Operand(orc, nm, r, c, tokens, seed=400 + 10 * k + i) for i, (r, c) in enumerate([(96, 512), (33, 256)])]
            for k in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    wss = [sparse_linear_workspace(DEV) for _ in range(2)]
    torch.cuda.synchronize()  # inputs were placed on the default stream
    errors = []

    def run(k):
        try:
            for _ in range(20):
                mllm_sparse_linear([o.op() for o in sets[k]], nm, tokens, wss[k], stream=streams[k].cuda_stream)
            streams[k].synchronize()
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors
    for k in range(2):
        for o in sets[k]:
            o.check(orc)
        assert _tickets_clear(wss[k])


# ------------------------------------------------------------------------------ prefill sizes

@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
@pytest.mark.parametrize("tokens", [65, 128, 200, 300, 512])
def test_prefill_sized_calls(orc, ws, nm, tokens):
    """More than 64 tokens: operands whose columns are whole 128-column stages run on the
    prefill kernels (2:4: units of two 128-row tiles x 128 tokens; 4:8: 128 rows x 256
    tokens, each stage expanded once), the others in groups of 16 tokens. Ragged rows and
    token chunks, several operands in one call."""
    shapes = [(300, 512), (128, 1024), (37, 1040), (200, 128)]
    ops = [Operand(orc, nm, r, c, tokens, seed=900 + 10 * i + tokens) for i, (r, c) in enumerate(shapes)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        o.check(orc)
    assert _tickets_clear(ws)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8)])
@pytest.mark.parametrize("tokens", [128, 512, 2048])
def test_prefill_llama_layer_sampled_rows(orc, ws, nm, tokens):
    """The LLaMA-2-7B layer's seven matrices at prefill sizes (the page's 128- and
    2048-token prompts), packed 2:4 (sparse MMA) or 4:8 (expanded once per stage for 256
    tokens), in one call; y checked on sampled rows, all tokens."""
    w = configs.WORKLOADS["llama2_7b_layer_2of4"]
    rng = np.random.default_rng(tokens)
    ops = [Operand(orc, nm, m.rows, m.cols, tokens, seed=950 + i, direct=True) for i, m in enumerate(w.matrices)]
    mllm_sparse_linear([o.op() for o in ops], nm, tokens, ws)
    torch.cuda.synchronize()
    for o in ops:
        # both tiles of the first units and the edges of every 128-row tile among them
        quarters = [0, 127, 128, 255, 256, 383, 384, 511, 512, 1023]
        rows = np.unique(np.concatenate([quarters, [o.rows - 1], rng.choice(o.rows, 5, replace=False)]))
        o.check(orc, rows_sel=rows)
    assert _tickets_clear(ws)
