"""Pins of the oracle's product with a hard-masked weight in the packed form (s.3.2,
"Information flow at inference": the learned mask is applied once, then the sparse network
serves).

Checked against: a dense fp64 matrix product with W (.) S_argmax(pi) built in the test from
the page's 2:4 candidate listing (and itertools for 4:8), without the packed form; one-hot
activations that must return single weights of an independent unpacking, bit for bit; and
the homogeneity of the product in x.
"""
from itertools import combinations

import numpy as np
import pytest

from _golden import rows

NM = [(2, 4), (4, 8)]


def _cands(n, m):
    if m == 4:
        return np.array([[int(v) for v in r] for r in rows("candidates_2of4.txt")], np.float64)
    return np.array([[1.0 if j in c else 0.0 for j in range(8)] for c in combinations(range(8), 4)])


def _bf16_bits(rng, shape, std):
    """Random bf16 bit patterns (truncation of fp32 normals: finite, both signs)."""
    f = rng.normal(0.0, std, size=shape).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _bf16_val(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _unpack(n, m, values, meta, rows_, cols):
    dense = np.zeros((rows_, cols), np.uint16)
    bpr = cols // m
    for r in range(rows_):
        for q in range(bpr):
            if m == 4:
                nib = (int(meta[r, q // 8]) >> (4 * (q % 8))) & 0xF
                pos = [nib & 3, nib >> 2]
            else:
                pos = [(int(meta[r, q]) >> (3 * t)) & 7 for t in range(4)]
            for t in range(n):
                dense[r, q * m + pos[t]] = values[r, q * n + t]
    return dense


@pytest.mark.parametrize("n,m", NM)
@pytest.mark.parametrize("rows_,bpr,tokens", [(7, 21, 3), (16, 16, 8), (5, 40, 16)])
def test_sparse_linear_equals_dense_masked_product(orc, n, m, rows_, bpr, tokens):
    rng = np.random.default_rng(100 + rows_ + m)
    cols = bpr * m
    C = orc.num_candidates(n, m)
    W = _bf16_bits(rng, (rows_, cols), 0.02)
    pi = rng.normal(0, 1, size=(rows_ * bpr, C)).astype(np.float32)
    x = _bf16_bits(rng, (tokens, cols), 1.0)
    values, meta, _ = orc.hard_pack(n, m, W, pi)
    y = orc.sparse_linear(n, m, values, meta, x)
    mask = _cands(n, m)[np.argmax(pi, 1)].reshape(rows_, cols)
    y_ref = _bf16_val(x) @ (_bf16_val(W) * mask).T
    scale = np.abs(_bf16_val(x)) @ np.abs(_bf16_val(W) * mask).T
    assert y.shape == (tokens, rows_)
    assert np.all(np.abs(y - y_ref) <= 1e-14 * scale)


@pytest.mark.parametrize("n,m", NM)
def test_one_hot_activations_return_kept_weights(orc, n, m):
    rng = np.random.default_rng(7)
    rows_, cols = 9, m * 12
    W = _bf16_bits(rng, (rows_, cols), 0.02)
    pi = rng.normal(0, 1, size=(rows_ * cols // m, orc.num_candidates(n, m))).astype(np.float32)
    values, meta, _ = orc.hard_pack(n, m, W, pi)
    dense = _bf16_val(_unpack(n, m, values, meta, rows_, cols))
    picks = rng.integers(0, cols, size=20)
    x = np.zeros((20, cols), np.uint16)
    x[np.arange(20), picks] = 0x3F80                       # bf16 1.0
    y = orc.sparse_linear(n, m, values, meta, x)
    np.testing.assert_array_equal(y, dense[:, picks].T)
    # a pruned position contributes nothing, a kept one its weight
    assert np.count_nonzero(dense) == rows_ * cols * n // m


@pytest.mark.parametrize("n,m", NM)
def test_sparse_linear_homogeneous_and_empty(orc, n, m):
    rng = np.random.default_rng(8)
    rows_, cols = 4, m * 8
    W = _bf16_bits(rng, (rows_, cols), 0.02)
    pi = rng.normal(0, 1, size=(rows_ * cols // m, orc.num_candidates(n, m))).astype(np.float32)
    values, meta, _ = orc.hard_pack(n, m, W, pi)
    x = _bf16_bits(rng, (2, cols), 1.0)
    x2 = ((x.astype(np.uint32) + (1 << 7)) & 0xFFFF).astype(np.uint16)   # x * 2: exponent + 1
    np.testing.assert_array_equal(orc.sparse_linear(n, m, values, meta, x2),
                                  2.0 * orc.sparse_linear(n, m, values, meta, x))
    assert orc.sparse_linear(n, m, values, meta, x[:0]).shape == (0, rows_)


@pytest.mark.parametrize("n,m", NM)
def test_packed_input_generator_is_valid_pack(orc, n, m):
    """inputs.packed_hard_mask (the serving benchmark's operands) encodes a valid candidate
    per block exactly as hard_pack does: decoding it through the oracle's product with
    one-hot activations keeps N nonzero positions per block, ascending, and round-trips
    through hard_pack of the decoded dense matrix with logits favouring those candidates."""
    import torch

    from sparsity_mask_sampling_b200 import inputs

    rows_, bpr = 6, 21
    cols = bpr * m
    v, mt = inputs.packed_hard_mask(rows_, cols, (n, m), seed=5)
    values = v.view(torch.int16).numpy().view(np.uint16)
    meta = mt.numpy().view(np.uint32 if m == 4 else np.uint16)
    eye = np.zeros((cols, cols), np.uint16)
    np.fill_diagonal(eye, 0x3F80)
    dense = orc.sparse_linear(n, m, values, meta, eye).T          # [rows, cols] = W*
    kept = (dense != 0).reshape(rows_, bpr, m)
    assert (kept.sum(-1) == n).all()
    S = _cands(n, m)
    k = np.array([np.flatnonzero((S == kb).all(1))[0] for kb in kept.reshape(-1, m).astype(np.float64)])
    pi = np.full((rows_ * bpr, orc.num_candidates(n, m)), -1.0, np.float32)
    pi[np.arange(rows_ * bpr), k] = 1.0
    W = np.zeros((rows_, cols), np.uint16)
    W[dense != 0] = _bits_of(dense[dense != 0])
    v2, m2, _ = orc.hard_pack(n, m, W, pi)
    np.testing.assert_array_equal(v2, values)
    np.testing.assert_array_equal(m2, meta)


def _bits_of(vals):
    return (np.asarray(vals, np.float32).view(np.uint32) >> 16).astype(np.uint16)
