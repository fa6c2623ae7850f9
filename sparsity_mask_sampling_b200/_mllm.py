"""ctypes binding of libmllm (include/mllm.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but turn
torch tensors into device pointers, build the C structs and check the returned status. All
arithmetic of the sampler runs in the CUDA kernels of libmllm.so; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmllm.so")

ABI_VERSION = 1

MLLM_OK = 0
MLLM_ERR_INVALID_ARG = 1
MLLM_ERR_MISALIGNED = 2
MLLM_ERR_UNSUPPORTED = 3
MLLM_ERR_WORKSPACE = 4
MLLM_ERR_CUDA = 5

MLLM_BF16 = 0
MLLM_F32 = 1

INIT_STEP = 0xFFFFFFFF


class MllmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {mllm_status_string(status)} (status {status})")


class NM(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("m", ctypes.c_int32)]


class Matrix(ctypes.Structure):
    _fields_ = [
        ("W", ctypes.c_void_p),
        ("X_out", ctypes.c_void_p),
        ("G", ctypes.c_void_p),
        ("w_dtype", ctypes.c_int32),
        ("g_dtype", ctypes.c_int32),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("logits", ctypes.c_void_p),
        ("adam_m", ctypes.c_void_p),
        ("adam_v", ctypes.c_void_p),
        ("block_offset", ctypes.c_uint64),
        ("soft_mask_out", ctypes.c_void_p),
        ("grad_logits_out", ctypes.c_void_p),
        ("pack_values", ctypes.c_void_p),
        ("pack_meta", ctypes.c_void_p),
        ("cand_idx_out", ctypes.c_void_p),
    ]


class HParams(ctypes.Structure):
    _fields_ = [
        ("kappa", ctypes.c_float),
        ("tau", ctypes.c_float),
        ("lambda_", ctypes.c_float),
        ("lr", ctypes.c_float),
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("adam_step", ctypes.c_uint32),
        ("step", ctypes.c_uint32),
        ("seed", ctypes.c_uint64),
        ("noise_on", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class SparseOperand(ctypes.Structure):
    _fields_ = [
        ("pack_values", ctypes.c_void_p),
        ("pack_meta", ctypes.c_void_p),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
    ]


class LinearIO(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("dy", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_SIGS = {
    "mllm_num_candidates": (ctypes.c_int32, [NM]),
    "mllm_prior_init": (ctypes.c_int, [_P, ctypes.c_int32, NM, ctypes.c_float, ctypes.c_float, ctypes.c_uint64, _P]),
    "mllm_prior_init_from_mask": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P, ctypes.c_float, ctypes.c_float, ctypes.c_uint64, _P]),
    "mllm_sample_fwd": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P, _P, _P, ctypes.c_size_t, _P]),
    "mllm_sample_bwd_adam": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P, _P]),
    "mllm_sample_fwd_noalloc": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P, _P, _P]),
    "mllm_sample_bwd_adam_fwd": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "mllm_hard_pack": (ctypes.c_int, [_P, ctypes.c_int32, NM, _P]),
    "mllm_noise": (ctypes.c_int, [NM, ctypes.c_uint64, ctypes.c_uint32, _P, ctypes.c_int64, _P, _P]),
    "mllm_workspace_bytes": (ctypes.c_size_t, []),
    "mllm_mask_diff": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, _P]),
    "mllm_mask_stats": (ctypes.c_int, [_P, ctypes.c_int32, NM, ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "mllm_encode_candidates": (ctypes.c_int, [NM, _P, ctypes.c_int64, _P, _P]),
    "mllm_decode_candidates": (ctypes.c_int, [NM, _P, ctypes.c_int64, _P, _P]),
    "mllm_noise_table": (ctypes.c_int, [_P, _P]),
    "mllm_sparse_linear": (ctypes.c_int, [_P, ctypes.c_int32, NM, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "mllm_sparse_linear_workspace_bytes": (ctypes.c_size_t, []),
    "mllm_sparse_linear_check_timeout": (ctypes.c_int, [_P, NM, ctypes.c_int32, _P, ctypes.c_size_t, _P]),
    "mllm_sizeof_sparse_operand": (ctypes.c_size_t, []),
    "mllm_sizeof_linear_io": (ctypes.c_size_t, []),
    "mllm_masked_linear_fwd": (ctypes.c_int, [_P, _P, ctypes.c_int32, NM, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]),
    "mllm_masked_linear_workspace_bytes": (ctypes.c_size_t, []),
    "mllm_masked_linear_bwd_adam": (ctypes.c_int, [_P, _P, ctypes.c_int32, NM, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "mllm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mllm_last_cuda_error": (ctypes.c_int32, []),
    "mllm_abi_version": (ctypes.c_int32, []),
    "mllm_sizeof_matrix": (ctypes.c_size_t, []),
    "mllm_sizeof_hparams": (ctypes.c_size_t, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmllm.so from the package directory. Raises if it is missing or mismatched."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmllm.so not built ({LIB_PATH}); run __graft_entry__.build() "
                              "or python -m sparsity_mask_sampling_b200.build")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        if h.mllm_abi_version() != ABI_VERSION:
            raise ImportError("libmllm.so ABI version mismatch")
        if (h.mllm_sizeof_matrix() != ctypes.sizeof(Matrix) or h.mllm_sizeof_hparams() != ctypes.sizeof(HParams)
                or h.mllm_sizeof_sparse_operand() != ctypes.sizeof(SparseOperand)
                or h.mllm_sizeof_linear_io() != ctypes.sizeof(LinearIO)):
            raise ImportError("libmllm.so struct layout mismatch")
        _lib = h
    return _lib


def mllm_status_string(status: int) -> str:
    return lib().mllm_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != MLLM_OK:
        raise MllmError(status, what)


def _nm(nm) -> NM:
    n, m = nm
    return NM(int(n), int(m))


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.data_ptr()


def _dtype_code(t: Optional[torch.Tensor]) -> int:
    if t is None:
        return MLLM_BF16
    if t.dtype == torch.bfloat16:
        return MLLM_BF16
    if t.dtype == torch.float32:
        return MLLM_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclass
class MatrixBuffers:
    """Device buffers of one frozen weight matrix (layouts as in include/mllm.h)."""
    W: torch.Tensor
    logits: Optional[torch.Tensor] = None
    adam_m: Optional[torch.Tensor] = None
    adam_v: Optional[torch.Tensor] = None
    block_offset: int = 0
    X: Optional[torch.Tensor] = None
    G: Optional[torch.Tensor] = None
    soft_mask: Optional[torch.Tensor] = None
    grad_logits: Optional[torch.Tensor] = None
    pack_values: Optional[torch.Tensor] = None
    pack_meta: Optional[torch.Tensor] = None
    cand_idx: Optional[torch.Tensor] = None
    rows: Optional[int] = None
    cols: Optional[int] = None

    def to_c(self) -> Matrix:
        rows = self.W.shape[0] if self.rows is None else self.rows
        cols = self.W.shape[1] if self.cols is None else self.cols
        return Matrix(
            W=_ptr(self.W), X_out=_ptr(self.X), G=_ptr(self.G),
            w_dtype=_dtype_code(self.W), g_dtype=_dtype_code(self.G),
            rows=int(rows), cols=int(cols),
            logits=_ptr(self.logits), adam_m=_ptr(self.adam_m), adam_v=_ptr(self.adam_v),
            block_offset=int(self.block_offset),
            soft_mask_out=_ptr(self.soft_mask), grad_logits_out=_ptr(self.grad_logits),
            pack_values=_ptr(self.pack_values), pack_meta=_ptr(self.pack_meta),
            cand_idx_out=_ptr(self.cand_idx))


@dataclass
class Hparams:
    kappa: float = 100.0
    tau: float = 4.0
    lambda_: float = 1e-5
    lr: float = 5e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.1
    adam_step: int = 1
    step: int = 0
    seed: int = 0
    noise_on: bool = True

    def to_c(self) -> HParams:
        return HParams(kappa=self.kappa, tau=self.tau, lambda_=self.lambda_, lr=self.lr,
                       beta1=self.beta1, beta2=self.beta2, eps=self.eps,
                       weight_decay=self.weight_decay, adam_step=int(self.adam_step),
                       step=int(self.step), seed=int(self.seed), noise_on=int(bool(self.noise_on)),
                       reserved=0)


class MatrixArray:
    """A C array of mllm_matrix built once and reusable across calls (saves marshalling)."""

    def __init__(self, mats: Sequence[MatrixBuffers]):
        self.n = len(mats)
        self.arr = (Matrix * max(1, self.n))(*[m.to_c() for m in mats])

    @property
    def ptr(self):
        return ctypes.cast(self.arr, ctypes.c_void_p)


def _mats(mats) -> MatrixArray:
    return mats if isinstance(mats, MatrixArray) else MatrixArray(list(mats))


def mllm_num_candidates(nm) -> int:
    return lib().mllm_num_candidates(_nm(nm))


def mllm_workspace_bytes() -> int:
    return lib().mllm_workspace_bytes()


def mllm_prior_init(mats, nm, alpha: float, init_std: float, seed: int, stream=None):
    a = _mats(mats)
    _check(lib().mllm_prior_init(a.ptr, a.n, _nm(nm), float(alpha), float(init_std), int(seed),
                                 _stream(stream)), "mllm_prior_init")


def mllm_prior_init_from_mask(mats, nm, prior_idx, alpha: float, init_std: float, seed: int, stream=None):
    """Prior init with M0 = candidate prior_idx[i][b] (uint8 device tensors, one per matrix)."""
    a = _mats(mats)
    ptrs = (ctypes.c_void_p * max(1, a.n))(*[_ptr(t) for t in prior_idx])
    _check(lib().mllm_prior_init_from_mask(a.ptr, a.n, _nm(nm), ctypes.cast(ptrs, ctypes.c_void_p),
                                           float(alpha), float(init_std), int(seed), _stream(stream)),
           "mllm_prior_init_from_mask")


def mllm_sample_fwd(mats, nm, hp: Hparams, reg_sum_out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    a = _mats(mats)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mllm_sample_fwd(a.ptr, a.n, _nm(nm), ctypes.byref(h), _ptr(reg_sum_out),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "mllm_sample_fwd")


def mllm_sample_fwd_noalloc(mats, nm, hp: Hparams, reg_sum_out: torch.Tensor, stream=None):
    """mllm_sample_fwd for callers that cannot allocate: the reduction scratch is a fixed
    array inside libmllm (no workspace argument). Calls on one device must not overlap."""
    a = _mats(mats)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    _check(lib().mllm_sample_fwd_noalloc(a.ptr, a.n, _nm(nm), ctypes.byref(h), _ptr(reg_sum_out),
                                         _stream(stream)), "mllm_sample_fwd_noalloc")


def mllm_sample_bwd_adam(mats, nm, hp: Hparams, stream=None):
    a = _mats(mats)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    _check(lib().mllm_sample_bwd_adam(a.ptr, a.n, _nm(nm), ctypes.byref(h), _stream(stream)),
           "mllm_sample_bwd_adam")


def mllm_sample_bwd_adam_fwd(mats, nm, hp: Hparams, hp_next: Hparams,
                             reg_sum_out: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward + AdamW with hp, then the next step's forward with hp_next, in one pass."""
    a = _mats(mats)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    hn = hp_next.to_c() if isinstance(hp_next, Hparams) else hp_next
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mllm_sample_bwd_adam_fwd(a.ptr, a.n, _nm(nm), ctypes.byref(h), ctypes.byref(hn),
                                          _ptr(reg_sum_out), _ptr(workspace), ws_bytes,
                                          _stream(stream)), "mllm_sample_bwd_adam_fwd")


def mllm_hard_pack(mats, nm, stream=None):
    a = _mats(mats)
    _check(lib().mllm_hard_pack(a.ptr, a.n, _nm(nm), _stream(stream)), "mllm_hard_pack")


def mllm_noise(nm, seed: int, step: int, gids: torch.Tensor, g_out: torch.Tensor, stream=None):
    _check(lib().mllm_noise(_nm(nm), int(seed), int(step), _ptr(gids), int(gids.numel()),
                            _ptr(g_out), _stream(stream)), "mllm_noise")


def mllm_noise_table():
    """(c [128], T [27, 128]) of the noise logarithm as compiled into the kernels."""
    import numpy as np

    c = np.zeros(128, np.float32)
    T = np.zeros((27, 128), np.float32)
    _check(lib().mllm_noise_table(c.ctypes.data, T.ctypes.data), "mllm_noise_table")
    return c, T


def mllm_mask_diff(a: torch.Tensor, b: torch.Tensor, count_out: torch.Tensor, stream=None):
    _check(lib().mllm_mask_diff(_ptr(a), _ptr(b), int(a.numel()), _ptr(count_out), _stream(stream)),
           "mllm_mask_diff")


def mllm_mask_stats(mats, nm, kappa: float, out: torch.Tensor, workspace: torch.Tensor, stream=None):
    a = _mats(mats)
    _check(lib().mllm_mask_stats(a.ptr, a.n, _nm(nm), float(kappa), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "mllm_mask_stats")


def mllm_encode_candidates(nm, idx: torch.Tensor, words: torch.Tensor, stream=None):
    _check(lib().mllm_encode_candidates(_nm(nm), _ptr(idx), int(idx.numel()), _ptr(words), _stream(stream)),
           "mllm_encode_candidates")


def mllm_decode_candidates(nm, words: torch.Tensor, n: int, idx: torch.Tensor, stream=None):
    _check(lib().mllm_decode_candidates(_nm(nm), _ptr(words), int(n), _ptr(idx), _stream(stream)),
           "mllm_decode_candidates")


class SparseOperandArray:
    """C array of mllm_sparse_operand built from (pack_values, pack_meta, x, y) tensors:
    rows = y.shape[1], cols = x.shape[1]. Keeps the tensors alive with the array."""

    def __init__(self, ops: Sequence):
        self.ops = [tuple(o) for o in ops]
        self.arr = (SparseOperand * max(len(self.ops), 1))()
        for i, (vals, meta, x, y) in enumerate(self.ops):
            self.arr[i] = SparseOperand(_ptr(vals), _ptr(meta), _ptr(x), _ptr(y), int(y.shape[1]), int(x.shape[1]))
        self.n = len(self.ops)
        self.ptr = ctypes.cast(self.arr, ctypes.c_void_p)


def mllm_sparse_linear_workspace_bytes() -> int:
    return lib().mllm_sparse_linear_workspace_bytes()


def sparse_linear_workspace(device) -> torch.Tensor:
    """A zero-filled workspace for mllm_sparse_linear on `device`."""
    return torch.zeros(mllm_sparse_linear_workspace_bytes(), dtype=torch.uint8, device=device)


def mllm_sparse_linear(ops, nm, tokens: int, workspace: torch.Tensor, stream=None):
    """y = x W*^T for every (pack_values, pack_meta, x [tokens, cols], y [tokens, rows]) of ops
    (or a prepared SparseOperandArray); workspace from sparse_linear_workspace()."""
    a = ops if isinstance(ops, SparseOperandArray) else SparseOperandArray(ops)
    _check(lib().mllm_sparse_linear(a.ptr, a.n, _nm(nm), int(tokens), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "mllm_sparse_linear")


def mllm_sparse_linear_check_timeout(op, nm, tokens: int, workspace: torch.Tensor, stream=None):
    """One (pack_values, pack_meta, x, y) operand through the timeout test of the copy
    pipeline (see include/mllm.h): the call's error word ends nonzero."""
    a = SparseOperandArray([op])
    _check(lib().mllm_sparse_linear_check_timeout(a.ptr, _nm(nm), int(tokens), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "mllm_sparse_linear_check_timeout")


def mllm_last_cuda_error() -> int:
    return lib().mllm_last_cuda_error()


def mllm_masked_linear_workspace_bytes() -> int:
    return lib().mllm_masked_linear_workspace_bytes()


def masked_linear_workspace(device) -> torch.Tensor:
    """A zero-filled workspace for the mllm_masked_linear_* calls on `device`."""
    return torch.zeros(mllm_masked_linear_workspace_bytes(), dtype=torch.uint8, device=device)


def _linear_io(ios):
    """C array of mllm_linear_io from (x, y, dy) tuples (entries may be None)."""
    arr = (LinearIO * max(1, len(ios)))()
    for i, (x, y, dy) in enumerate(ios):
        arr[i] = LinearIO(_ptr(x), _ptr(y), _ptr(dy))
    return arr


def mllm_masked_linear_fwd(mats, ios, nm, tokens: int, hp: Hparams, workspace: torch.Tensor,
                           reg_sum_out: Optional[torch.Tensor] = None, stream=None):
    """Y = A (W . M)^T for every matrix, the soft-masked weight made on the fly: ios[i] =
    (x [tokens, cols] bf16, y [tokens, rows] fp32, None)."""
    a = _mats(mats)
    io = _linear_io(ios)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    _check(lib().mllm_masked_linear_fwd(a.ptr, ctypes.cast(io, ctypes.c_void_p), a.n, _nm(nm), int(tokens),
                                        ctypes.byref(h), _ptr(reg_sum_out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
           "mllm_masked_linear_fwd")


def mllm_masked_linear_bwd_adam(mats, ios, nm, tokens: int, hp: Hparams, workspace: torch.Tensor, stream=None):
    """G = dY^T A per matrix, then the logits' backward + AdamW from G (never stored):
    ios[i] = (x [tokens, cols] bf16, None, dy [tokens, rows] bf16)."""
    a = _mats(mats)
    io = _linear_io(ios)
    h = hp.to_c() if isinstance(hp, Hparams) else hp
    _check(lib().mllm_masked_linear_bwd_adam(a.ptr, ctypes.cast(io, ctypes.c_void_p), a.n, _nm(nm), int(tokens),
                                             ctypes.byref(h), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "mllm_masked_linear_bwd_adam")
