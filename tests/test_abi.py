"""The C ABI library loads, exports every declared symbol, and rejects bad arguments on the
host before touching a device (these calls make no CUDA call and run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    from sparsity_mask_sampling_b200 import _mllm
    from sparsity_mask_sampling_b200.build import build

    build()
    _mllm.lib()
    return _mllm


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(mllm_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(M):
    names = _declared_functions()
    assert len(names) >= 12, names
    h = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(h, n), n


def test_abi_guards(M):
    L = M.lib()
    assert L.mllm_abi_version() == M.ABI_VERSION
    assert L.mllm_sizeof_matrix() == ctypes.sizeof(M.Matrix)
    assert L.mllm_sizeof_hparams() == ctypes.sizeof(M.HParams)
    assert L.mllm_sizeof_sparse_operand() == ctypes.sizeof(M.SparseOperand)
    assert M.mllm_workspace_bytes() >= 16 + 8 * 148


def test_num_candidates(M):
    assert M.mllm_num_candidates((2, 4)) == 6
    assert M.mllm_num_candidates((4, 8)) == 70
    assert M.mllm_num_candidates((1, 4)) == 0
    assert M.mllm_num_candidates((2, 8)) == 0


def test_status_strings(M):
    for s in range(6):
        assert M.mllm_status_string(s)


def _mat(M, **kw):
    base = dict(W=0x1000, X_out=0x2000, G=0x3000, w_dtype=0, g_dtype=0, rows=4, cols=8,
                logits=0x4000, adam_m=0x5000, adam_v=0x6000, block_offset=0,
                soft_mask_out=0, grad_logits_out=0, pack_values=0x7000, pack_meta=0x8000,
                cand_idx_out=0)
    base.update(kw)
    return M.Matrix(**base)


def _hp(M, **kw):
    base = dict(kappa=100.0, tau=4.0, lambda_=1e-5, lr=5e-4, beta1=0.9, beta2=0.999, eps=1e-8,
                weight_decay=0.1, adam_step=1, step=0, seed=0, noise_on=1, reserved=0)
    base.update(kw)
    return M.HParams(**base)


def _fwd(M, mats, hp, nm=(2, 4), reg=0, ws=0x9000, wsb=None):
    L = M.lib()
    arr = (M.Matrix * len(mats))(*mats)
    wsb = M.mllm_workspace_bytes() if wsb is None else wsb
    return L.mllm_sample_fwd(ctypes.cast(arr, ctypes.c_void_p), len(mats), M.NM(*nm),
                             ctypes.byref(hp), reg, ws, wsb, 0)


def _bwd(M, mats, hp, nm=(2, 4)):
    arr = (M.Matrix * len(mats))(*mats)
    return M.lib().mllm_sample_bwd_adam(ctypes.cast(arr, ctypes.c_void_p), len(mats), M.NM(*nm),
                                        ctypes.byref(hp), 0)


def test_invalid_arguments_rejected(M):
    L = M.lib()
    hp = _hp(M)
    # null matrix array / zero count
    assert L.mllm_sample_fwd(None, 1, M.NM(2, 4), ctypes.byref(hp), 0, 0, 0, 0) == M.MLLM_ERR_INVALID_ARG
    assert _fwd(M, [], hp) == M.MLLM_ERR_INVALID_ARG
    # unsupported pattern
    assert _fwd(M, [_mat(M)], hp, nm=(3, 4)) == M.MLLM_ERR_UNSUPPORTED
    # cols not a multiple of M
    assert _fwd(M, [_mat(M, cols=6)], hp) == M.MLLM_ERR_INVALID_ARG
    assert _fwd(M, [_mat(M, cols=12)], hp, nm=(4, 8)) == M.MLLM_ERR_INVALID_ARG
    assert _fwd(M, [_mat(M, rows=-1)], hp) == M.MLLM_ERR_INVALID_ARG
    # missing required buffers
    assert _fwd(M, [_mat(M, W=0)], hp) == M.MLLM_ERR_INVALID_ARG
    assert _fwd(M, [_mat(M, X_out=0)], hp) == M.MLLM_ERR_INVALID_ARG
    assert _fwd(M, [_mat(M, logits=0)], hp) == M.MLLM_ERR_INVALID_ARG
    assert _bwd(M, [_mat(M, G=0)], hp) == M.MLLM_ERR_INVALID_ARG
    assert _bwd(M, [_mat(M, adam_v=0)], hp) == M.MLLM_ERR_INVALID_ARG
    # unknown dtype, mixed dtypes in one call
    assert _fwd(M, [_mat(M, w_dtype=7)], hp) == M.MLLM_ERR_UNSUPPORTED
    assert _fwd(M, [_mat(M), _mat(M, w_dtype=1)], hp) == M.MLLM_ERR_UNSUPPORTED


def test_misaligned_pointers_rejected(M):
    hp = _hp(M)
    for field in ("W", "X_out", "logits", "soft_mask_out"):
        assert _fwd(M, [_mat(M, **{field: 0x1008})], hp) == M.MLLM_ERR_MISALIGNED, field
    for field in ("G", "adam_m", "adam_v", "grad_logits_out"):
        assert _bwd(M, [_mat(M, **{field: 0x1004})], hp) == M.MLLM_ERR_MISALIGNED, field
    assert _fwd(M, [_mat(M)], hp, reg=0x10004) == M.MLLM_ERR_MISALIGNED
    assert _fwd(M, [_mat(M)], hp, reg=0x10000, ws=0x9008) == M.MLLM_ERR_MISALIGNED


def test_workspace_checked(M):
    hp = _hp(M)
    assert _fwd(M, [_mat(M)], hp, reg=0x10000, ws=0) == M.MLLM_ERR_WORKSPACE
    assert _fwd(M, [_mat(M)], hp, reg=0x10000, wsb=M.mllm_workspace_bytes() - 8) == M.MLLM_ERR_WORKSPACE


@pytest.mark.parametrize("field,value", [
    ("tau", 0.0), ("tau", -1.0), ("tau", float("inf")), ("tau", float("nan")), ("tau", 1e-39),
    ("kappa", 0.0), ("kappa", float("nan")), ("step", 0xFFFFFFFF), ("reserved", 1)])
def test_bad_forward_scalars(M, field, value):
    assert _fwd(M, [_mat(M)], _hp(M, **{field: value})) == M.MLLM_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value", [
    ("lambda_", -1e-5), ("lr", float("nan")), ("beta1", 1.0), ("beta2", -0.1), ("eps", 0.0),
    ("weight_decay", -0.1), ("adam_step", 0)])
def test_bad_backward_scalars(M, field, value):
    assert _bwd(M, [_mat(M)], _hp(M, **{field: value})) == M.MLLM_ERR_INVALID_ARG


def test_prior_and_pack_validation(M):
    L = M.lib()
    arr = (M.Matrix * 1)(_mat(M))
    p = ctypes.cast(arr, ctypes.c_void_p)
    assert L.mllm_prior_init(p, 1, M.NM(2, 4), -1.0, 0.01, 0, 0) == M.MLLM_ERR_INVALID_ARG
    assert L.mllm_prior_init(p, 1, M.NM(2, 4), 3.0, float("nan"), 0, 0) == M.MLLM_ERR_INVALID_ARG
    bad = (M.Matrix * 1)(_mat(M, pack_meta=0))
    assert L.mllm_hard_pack(ctypes.cast(bad, ctypes.c_void_p), 1, M.NM(2, 4), 0) == M.MLLM_ERR_INVALID_ARG
    bad = (M.Matrix * 1)(_mat(M, pack_values=0x7004))
    assert L.mllm_hard_pack(ctypes.cast(bad, ctypes.c_void_p), 1, M.NM(2, 4), 0) == M.MLLM_ERR_MISALIGNED
    assert L.mllm_noise(M.NM(2, 4), 0, 0, 0x1000, -1, 0x2000, 0) == M.MLLM_ERR_INVALID_ARG
    assert L.mllm_noise(M.NM(2, 5), 0, 0, 0x1000, 1, 0x2000, 0) == M.MLLM_ERR_UNSUPPORTED
    assert L.mllm_noise(M.NM(2, 4), 0, 0, 0x1000, 0, 0x2000, 0) == M.MLLM_OK  # nothing to do


def test_compiled_noise_table_matches_oracle_table(M):
    """The kernels' compile-time logarithm table equals the oracle's, bit for bit (the
    oracle's is pinned to 50-digit logarithms)."""
    import numpy as np
    import oracle

    c, T = M.mllm_noise_table()
    oc, oT, _ = oracle.nlog_table()
    assert np.array_equal(c.view(np.uint32), oc.view(np.uint32))
    assert np.array_equal(T.view(np.uint32), oT.view(np.uint32))


def _spl(M, ops, nm=(2, 4), tokens=8, ws=0x100000, wsb=None):
    arr = (M.SparseOperand * max(len(ops), 1))(*ops)
    wsb = M.mllm_sparse_linear_workspace_bytes() if wsb is None else wsb
    return M.lib().mllm_sparse_linear(ctypes.cast(arr, ctypes.c_void_p) if ops else None, len(ops),
                                      M.NM(*nm), tokens, ws, wsb, 0)


def _op(M, **kw):
    base = dict(pack_values=0x1000, pack_meta=0x2000, x=0x3000, y=0x4000, rows=32, cols=64)
    base.update(kw)
    return M.SparseOperand(**base)


def test_sparse_linear_validation(M):
    assert _spl(M, []) == M.MLLM_ERR_INVALID_ARG
    assert _spl(M, [_op(M)], nm=(1, 4)) == M.MLLM_ERR_UNSUPPORTED
    for tokens in (0, -1, 16385):
        assert _spl(M, [_op(M)], tokens=tokens) == M.MLLM_ERR_INVALID_ARG, tokens
    assert _spl(M, [_op(M, cols=6)]) == M.MLLM_ERR_INVALID_ARG
    assert _spl(M, [_op(M, cols=12)], nm=(4, 8)) == M.MLLM_ERR_INVALID_ARG
    assert _spl(M, [_op(M, rows=-1)]) == M.MLLM_ERR_INVALID_ARG
    for field in ("pack_values", "pack_meta", "x", "y"):
        assert _spl(M, [_op(M, **{field: 0})]) == M.MLLM_ERR_INVALID_ARG, field
        assert _spl(M, [_op(M), _op(M, **{field: 0x5008})]) == M.MLLM_ERR_MISALIGNED, field
    # cols == 0 needs only y; rows == 0 needs nothing (these would launch, so only the
    # rejected variants are called here)
    assert _spl(M, [_op(M, cols=0, y=0)]) == M.MLLM_ERR_INVALID_ARG
    # workspace
    assert _spl(M, [_op(M)], ws=0) == M.MLLM_ERR_WORKSPACE
    assert _spl(M, [_op(M)], wsb=M.mllm_sparse_linear_workspace_bytes() - 4) == M.MLLM_ERR_WORKSPACE
    assert _spl(M, [_op(M)], ws=0x100008) == M.MLLM_ERR_MISALIGNED


def test_timeout_check_validation(M):
    L = M.lib()
    wsb = M.mllm_sparse_linear_workspace_bytes()

    def call(op, tokens=4, ws=0x100000, nm=(2, 4)):
        arr = (M.SparseOperand * 1)(op)
        return L.mllm_sparse_linear_check_timeout(ctypes.cast(arr, ctypes.c_void_p), M.NM(*nm), tokens, ws, wsb, 0)

    # shapes the tensor-copy pipelines do not take, rejected before any launch
    assert call(_op(M, cols=64)) == M.MLLM_ERR_UNSUPPORTED
    assert call(_op(M, cols=64), nm=(4, 8)) == M.MLLM_ERR_UNSUPPORTED
    assert call(_op(M, cols=128), nm=(3, 8)) == M.MLLM_ERR_UNSUPPORTED
    assert call(_op(M, cols=132), nm=(4, 8)) == M.MLLM_ERR_INVALID_ARG
    assert call(_op(M, cols=128), tokens=65) == M.MLLM_ERR_UNSUPPORTED  # prefill sizes: not this test
    assert call(_op(M, cols=128), tokens=16385) == M.MLLM_ERR_INVALID_ARG
    assert call(_op(M, cols=128, rows=0)) == M.MLLM_ERR_UNSUPPORTED
    assert call(_op(M, cols=128), ws=0) == M.MLLM_ERR_WORKSPACE
    assert call(_op(M, cols=128, x=0)) == M.MLLM_ERR_INVALID_ARG


def _mlin(M, mats, ios, tokens=32, nm=(2, 4), bwd=False, ws=0x9000, wsb=None, hp=None):
    L = M.lib()
    arr = (M.Matrix * max(1, len(mats)))(*mats)
    io = (M.LinearIO * max(1, len(ios)))(*ios)
    wsb = M.mllm_masked_linear_workspace_bytes() if wsb is None else wsb
    hp = _hp(M) if hp is None else hp
    if bwd:
        return L.mllm_masked_linear_bwd_adam(ctypes.cast(arr, ctypes.c_void_p), ctypes.cast(io, ctypes.c_void_p),
                                             len(mats), M.NM(*nm), tokens, ctypes.byref(hp), ws, wsb, 0)
    return L.mllm_masked_linear_fwd(ctypes.cast(arr, ctypes.c_void_p), ctypes.cast(io, ctypes.c_void_p), len(mats),
                                    M.NM(*nm), tokens, ctypes.byref(hp), 0, ws, wsb, 0)


def test_masked_linear_validation(M):
    """The masked linear layer's calls reject what they do not support before any launch."""
    assert ctypes.sizeof(M.LinearIO) == M.lib().mllm_sizeof_linear_io()
    mat = _mat(M, rows=128, cols=128)
    io = M.LinearIO(x=0xA000, y=0xB000, dy=0xC000)
    for bwd in (False, True):
        assert _mlin(M, [mat], [io], nm=(4, 8), bwd=bwd) == M.MLLM_ERR_UNSUPPORTED
        assert _mlin(M, [_mat(M, rows=128, cols=128, w_dtype=1)], [io], bwd=bwd) == M.MLLM_ERR_UNSUPPORTED
        assert _mlin(M, [_mat(M, rows=128, cols=96)], [io], bwd=bwd) == M.MLLM_ERR_UNSUPPORTED
        for tokens in (0, -1, 1048577 if bwd else 257):
            assert _mlin(M, [mat], [io], tokens=tokens, bwd=bwd) == M.MLLM_ERR_INVALID_ARG, tokens
        assert _mlin(M, [mat], [M.LinearIO(x=0, y=0xB000, dy=0xC000)], bwd=bwd) == M.MLLM_ERR_INVALID_ARG
        assert _mlin(M, [mat], [M.LinearIO(x=0xA008, y=0xB000, dy=0xC000)], bwd=bwd) == M.MLLM_ERR_MISALIGNED
        assert _mlin(M, [mat], [io], bwd=bwd, ws=0) == M.MLLM_ERR_WORKSPACE
        assert _mlin(M, [mat], [io], bwd=bwd, wsb=M.mllm_masked_linear_workspace_bytes() - 16) == M.MLLM_ERR_WORKSPACE
        assert _mlin(M, [mat], [io], bwd=bwd, ws=0x9008) == M.MLLM_ERR_MISALIGNED
    assert _mlin(M, [mat], [M.LinearIO(x=0xA000, y=0, dy=0xC000)]) == M.MLLM_ERR_INVALID_ARG
    assert _mlin(M, [mat], [M.LinearIO(x=0xA000, y=0xB000, dy=0)], bwd=True) == M.MLLM_ERR_INVALID_ARG
    assert _mlin(M, [_mat(M, rows=100, cols=128)], [io], bwd=True) == M.MLLM_ERR_UNSUPPORTED  # rows % 8
    assert _mlin(M, [_mat(M, rows=128, cols=128, adam_m=0)], [io], bwd=True) == M.MLLM_ERR_INVALID_ARG
    assert _mlin(M, [mat], [io], bwd=True, hp=_hp(M, adam_step=0)) == M.MLLM_ERR_INVALID_ARG
    assert _mlin(M, [mat], [io], hp=_hp(M, tau=0.0)) == M.MLLM_ERR_INVALID_ARG
