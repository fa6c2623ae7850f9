"""CPU oracle for the MaskLLM per-block N:M mask sampler -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The CUDA library never uses it and shares no code with it.

The arithmetic lives in ``mllm_oracle.c`` (plain C, IEEE double except the fp32 noise and
perturbed logit that the specification fixes bit for bit); this module only marshals numpy
arrays through ctypes. Each wrapper names the passage it follows; the pages are the text of
web pages summarising arXiv 2409.17481 ("MaskLLM: Learnable Semi-Structured Sparsity for
Large Language Models"), cited by section and equation.

Parity status per function (see the pins in tests/test_oracle_*.py):
  candidates, philox4x32_10, nlog, noise, soft_mask, sample_fwd, sample_bwd, adamw,
  prior_init (deterministic mode, similarity, magnitude prior), prior_init_from_index,
  hard_pack, round_bf16, mask_diff, mask_stats, encode/decode_candidates, sparse_linear,
  masked_linear_fwd, masked_linear_bwd: pinned.
  prior_init random mode: the N(0, 0.01) draws are pinned by their moments, each
  Box-Muller pair against its two uniforms (radius and angle identities at fp64 rounding,
  uniforms from the known-answer Philox), and the Eq.10 structure exactly. The GPU takes the
  logarithm, sine and cosine in fp32, so GPU parity there is by tolerance (1e-6).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mllm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmllm_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU code involved). Returns the library path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_U32 = ctypes.c_uint32
_U64 = ctypes.c_uint64
_F = ctypes.c_float
_D = ctypes.c_double

_SIGS = {
    "orc_num_candidates": (_I, [_I, _I]),
    "orc_candidates": (_I, [_I, _I, _P]),
    "orc_philox4x32_10": (None, [_P, _P, _P]),
    "orc_fields21": (None, [_P, _P]),
    "orc_nlog": (_F, [_F]),
    "orc_nlog_array": (None, [_I64, _P, _P]),
    "orc_nlog_table": (None, [_P, _P, _P]),
    "orc_noise": (_I, [_I, _I, _U64, _U32, _I64, _P, _P, _P]),
    "orc_soft_mask": (_I, [_I, _I, _I64, _P, _P]),
    "orc_sample_fwd": (_I, [_I, _I, _I64, _P, _P, _P, _F, _F, _U64, _U32, _I, _I, _P, _P, _P, _P, _P]),
    "orc_sample_bwd": (_I, [_I, _I, _I64, _P, _P, _P, _P, _F, _F, _F, _U64, _U32, _I, _I, _P, _P]),
    "orc_adamw": (None, [_I64, _P, _P, _P, _P, _D, _D, _D, _D, _D, _I64, _P, _P, _P]),
    "orc_prior_init": (_I, [_I, _I, _I64, _P, _P, _D, _D, _U64, _P, _P, _P]),
    "orc_prior_init_from_index": (_I, [_I, _I, _I64, _P, _P, _D, _D, _U64, _P, _P]),
    "orc_argmax": (_I, [_I64, _I, _P, _P]),
    "orc_hard_pack": (_I, [_I, _I, _I64, _I64, _I, _P, _P, _P, _P, _P]),
    "orc_round_bf16": (None, [_I64, _P, _P]),
    "orc_mask_diff": (_I64, [_I64, _P, _P]),
    "orc_mask_stats": (_I, [_I, _I, _I64, _P, _P, _D, _P]),
    "orc_encode_candidates": (_I, [_I, _I, _I64, _P, _P]),
    "orc_decode_candidates": (_I, [_I, _I, _I64, _P, _P]),
    "orc_sparse_linear": (_I, [_I, _I, _I64, _I64, _P, _P, _I64, _P, _P]),
}


def lib():
    global _lib
    with _lock:
        if _lib is None:
            handle = ctypes.CDLL(build())
            for name, (res, args) in _SIGS.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


# ---------------------------------------------------------------------------------------
# Tables and the random-number generator
# ---------------------------------------------------------------------------------------

def num_candidates(n: int, m: int) -> int:
    return lib().orc_num_candidates(n, m)


def candidates(n: int, m: int) -> np.ndarray:
    """Candidate set S_{N:M} as uint8 rows [C, M] (s.3.2 Eq.2 listing for 2:4)."""
    C = num_candidates(n, m)
    if C == 0:
        raise ValueError(f"unsupported N:M {n}:{m}")
    out = np.zeros((C, m), np.uint8)
    _check(lib().orc_candidates(n, m, _ptr(out)), "candidates")
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 block function (Salmon et al., SC'11) on one counter/key."""
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def fields21(words) -> np.ndarray:
    w = _c(words, np.uint32)
    out = np.zeros(6, np.uint32)
    lib().orc_fields21(_ptr(w), _ptr(out))
    return out


def nlog(x: float) -> np.float32:
    return np.float32(lib().orc_nlog(float(np.float32(x))))


def nlog_array(x) -> np.ndarray:
    a = _c(x, np.float32)
    out = np.zeros(a.shape, np.float32)
    lib().orc_nlog_array(a.size, _ptr(a), _ptr(out))
    return out


def nlog_table():
    """(c [128], T [27, 128] for exponents -22..4, (1/3, emin, emax)) of nlog."""
    c = np.zeros(128, np.float32)
    T = np.zeros((27, 128), np.float32)
    k = np.zeros(3, np.float32)
    lib().orc_nlog_table(_ptr(c), _ptr(T), _ptr(k))
    return c, T, k


def noise(n, m, seed, step, gids):
    """Uniforms eps and Gumbel noise g (Eq.5) [nb, C] for the given global block ids."""
    g_ids = _c(gids, np.uint64)
    C = num_candidates(n, m)
    eps = np.zeros((len(g_ids), C), np.float32)
    g = np.zeros((len(g_ids), C), np.float32)
    _check(lib().orc_noise(n, m, seed, step, len(g_ids), _ptr(g_ids), _ptr(eps), _ptr(g)), "noise")
    return eps, g


def soft_mask(n, m, y) -> np.ndarray:
    """Eq.7: M = y S for soft indices y [nb, C]."""
    y = _c(np.atleast_2d(y), np.float64)
    out = np.zeros((y.shape[0], m), np.float64)
    _check(lib().orc_soft_mask(n, m, y.shape[0], _ptr(y), _ptr(out)), "soft_mask")
    return out


# ---------------------------------------------------------------------------------------
# The sampler
# ---------------------------------------------------------------------------------------

def sample_fwd(n, m, W, pi, gids, kappa, tau, seed, step, noise_on=True, round_w=True):
    """Forward (Eq.5-Eq.8) for blocks W [nb, M] (float64 values), pi [nb, C] fp32.

    Returns dict with y [nb, C], msoft [nb, M], mcomp [nb, M] (1 - msoft formed as a sum),
    x [nb, M] (W * msoft, unrounded) and reg (sum of x^2)."""
    C = num_candidates(n, m)
    W = _c(W, np.float64).reshape(-1, m)
    nb = W.shape[0]
    pi = _c(pi, np.float32).reshape(nb, C)
    g_ids = _c(gids, np.uint64).reshape(nb)
    y = np.zeros((nb, C))
    ms = np.zeros((nb, m))
    mc = np.zeros((nb, m))
    x = np.zeros((nb, m))
    reg = ctypes.c_double(0.0)
    rc = lib().orc_sample_fwd(n, m, nb, _ptr(W), _ptr(pi), _ptr(g_ids), float(kappa), float(tau),
                              int(seed), int(step), int(bool(noise_on)), int(bool(round_w)),
                              _ptr(y), _ptr(ms), _ptr(mc), _ptr(x), ctypes.byref(reg))
    _check(rc, "sample_fwd")
    return {"y": y, "msoft": ms, "mcomp": mc, "x": x, "reg": reg.value}


def sample_bwd(n, m, W, G, pi, gids, kappa, tau, lam, seed, step, noise_on=True, round_w=True):
    """Gradient of <G, W.M> - lam ||W.M||^2 with respect to the logits.

    Returns (grad [nb, C], scale [nb, C]) where scale is the magnitude of each gradient's
    summands, (kappa/tau) y_i sum_j |S_ij - M_j| |u_j|."""
    C = num_candidates(n, m)
    W = _c(W, np.float64).reshape(-1, m)
    nb = W.shape[0]
    G = _c(G, np.float64).reshape(nb, m)
    pi = _c(pi, np.float32).reshape(nb, C)
    g_ids = _c(gids, np.uint64).reshape(nb)
    grad = np.zeros((nb, C))
    scale = np.zeros((nb, C))
    rc = lib().orc_sample_bwd(n, m, nb, _ptr(W), _ptr(G), _ptr(pi), _ptr(g_ids), float(kappa),
                              float(tau), float(lam), int(seed), int(step), int(bool(noise_on)),
                              int(bool(round_w)), _ptr(grad), _ptr(scale))
    _check(rc, "sample_bwd")
    return grad, scale


def adamw(param, m, v, grad, lr, beta1, beta2, eps, wd, t):
    """AdamW step (decoupled weight decay, PyTorch order); t is the 1-based step."""
    p = _c(param, np.float64).ravel()
    mm = _c(m, np.float64).ravel()
    vv = _c(v, np.float64).ravel()
    g = _c(grad, np.float64).ravel()
    po, mo, vo = np.zeros_like(p), np.zeros_like(p), np.zeros_like(p)
    lib().orc_adamw(p.size, _ptr(p), _ptr(mm), _ptr(vv), _ptr(g), float(lr), float(beta1),
                    float(beta2), float(eps), float(wd), int(t), _ptr(po), _ptr(mo), _ptr(vo))
    shape = np.shape(param)
    return po.reshape(shape), mo.reshape(shape), vo.reshape(shape)


def prior_init(n, m, W, gids, alpha, init_std, seed):
    """Eq.9-Eq.10 prior initialisation from the magnitude prior.

    Returns (pi [nb, C] float64, prior_idx [nb] int32, sim [nb, C])."""
    C = num_candidates(n, m)
    W = _c(W, np.float64).reshape(-1, m)
    nb = W.shape[0]
    g_ids = _c(gids, np.uint64).reshape(nb)
    pi = np.zeros((nb, C))
    pidx = np.zeros(nb, np.int32)
    sim = np.zeros((nb, C))
    rc = lib().orc_prior_init(n, m, nb, _ptr(W), _ptr(g_ids), float(alpha), float(init_std),
                              int(seed), _ptr(pi), _ptr(pidx), _ptr(sim))
    _check(rc, "prior_init")
    return pi, pidx, sim


def prior_init_from_index(n, m, gids, prior_idx, alpha, init_std, seed):
    """Eq.9-Eq.10 from a given prior candidate per block (index >= C: no prior).

    Returns (pi [nb, C] float64, sim [nb, C])."""
    C = num_candidates(n, m)
    g_ids = _c(gids, np.uint64).ravel()
    k = _c(prior_idx, np.int32).ravel()
    nb = g_ids.size
    pi = np.zeros((nb, C))
    sim = np.zeros((nb, C))
    rc = lib().orc_prior_init_from_index(n, m, nb, _ptr(g_ids), _ptr(k), float(alpha), float(init_std),
                                         int(seed), _ptr(pi), _ptr(sim))
    _check(rc, "prior_init_from_index")
    return pi, sim


def argmax(pi, C) -> np.ndarray:
    p = _c(pi, np.float32).reshape(-1, C)
    out = np.zeros(p.shape[0], np.int32)
    lib().orc_argmax(p.shape[0], C, _ptr(p), _ptr(out))
    return out


def hard_pack(n, m, W_raw, pi):
    """Hard mask and compressed export of one matrix.

    W_raw: [rows, cols] uint16 (bf16 bits) or uint32 (fp32 bits). Returns
    (values [rows, cols*N/M] same dtype, meta, cand_idx [rows*cols/M] uint8) where meta is
    uint32 [rows, ceil(cols/32)] for 2:4 and uint16 [rows, cols/8] for 4:8."""
    W_raw = np.ascontiguousarray(W_raw)
    rows, cols = W_raw.shape
    eb = W_raw.dtype.itemsize
    C = num_candidates(n, m)
    pi = _c(pi, np.float32).reshape(rows * cols // m, C)
    values = np.zeros((rows, cols // m * n), W_raw.dtype)
    if m == 4:
        meta = np.zeros((rows, (cols // 4 + 7) // 8), np.uint32)
    else:
        meta = np.zeros((rows, cols // 8), np.uint16)
    cand = np.zeros(rows * cols // m, np.uint8)
    rc = lib().orc_hard_pack(n, m, rows, cols, eb, _ptr(W_raw), _ptr(pi), _ptr(values), _ptr(meta),
                             _ptr(cand))
    _check(rc, "hard_pack")
    return values, meta, cand


def round_bf16(x) -> np.ndarray:
    """Round doubles to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = _c(x, np.float64)
    out = np.zeros(a.shape, np.uint16)
    lib().orc_round_bf16(a.size, _ptr(a), _ptr(out))
    return out


def bf16_bits_to_float(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns (a bit shift; no arithmetic of the method)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------------------
# The sampler inside the frozen network's linear layer
# ---------------------------------------------------------------------------------------

def masked_linear_fwd(n, m, W, pi, gids, A, kappa, tau, seed, step, noise_on=True, round_w=True):
    """Forward of one frozen linear layer whose weight is the soft-masked W (s.3.2 "Frozen
    LLM Backbone": every linear layer of the network multiplies by W . M on its forward
    pass): X = W . M from the sampler's forward (Eq.5-Eq.7), stored in bf16 (nearest, ties
    to even), then Y = A X^T for activations A [T, cols], as a plain fp64 matrix product.

    W [rows, cols] and A [T, cols] are float64 values; pi [rows*cols/M, C] fp32; gids the
    blocks' global ids. Returns a dict: y [T, rows]; x [rows, cols] (W . M unrounded);
    x_bits [rows, cols] uint16 (its bf16 storage); reg (sum of unrounded x^2, Eq.8)."""
    W = np.asarray(W, np.float64)
    rows, cols = W.shape
    f = sample_fwd(n, m, W.reshape(-1, m), pi, gids, kappa, tau, seed, step, noise_on=noise_on,
                   round_w=round_w)
    x = f["x"].reshape(rows, cols)
    bits = round_bf16(x)
    xr = bf16_bits_to_float(bits).astype(np.float64)
    y = np.asarray(A, np.float64) @ xr.T
    return {"y": y, "x": x, "x_bits": bits, "reg": f["reg"]}


def masked_linear_bwd(n, m, W, pi, gids, A, dY, kappa, tau, lam, seed, step, noise_on=True, round_w=True):
    """Weight side of the same layer's backward: the layer's weight X = W . M receives
    dL/dX = dY^T A (the gradient of Y = A X^T with respect to X), and the logits receive
    that gradient through Eq.7 and Eq.6 together with the regulariser's (sample_bwd); W
    stays frozen (s.3.2). dY [T, rows] and A [T, cols] float64 values.
    Returns (grad [B, C], scale [B, C] as sample_bwd gives it, G = dY^T A [rows, cols])."""
    W = np.asarray(W, np.float64)
    rows, cols = W.shape
    G = np.asarray(dY, np.float64).T @ np.asarray(A, np.float64)
    g, scale = sample_bwd(n, m, W.reshape(-1, m), G.reshape(-1, m), pi, gids, kappa, tau, lam, seed, step,
                          noise_on=noise_on, round_w=round_w)
    return g, scale, G


# ---------------------------------------------------------------------------------------
# Diagnostics and codec
# ---------------------------------------------------------------------------------------

def mask_diff(a, b) -> int:
    """Number of blocks whose candidate index differs (Fig. 5a / Fig. 8 mask difference)."""
    a = _c(a, np.uint8).ravel()
    b = _c(b, np.uint8).ravel()
    return int(lib().orc_mask_diff(a.size, _ptr(a), _ptr(b)))


def mask_stats(n, m, W, pi, kappa):
    """(sum of max softmax(kappa pi), L1 kept by argmax, L1 kept by magnitude, blocks where
    the two masks agree); see orc_mask_stats."""
    C = num_candidates(n, m)
    W = _c(W, np.float64).reshape(-1, m)
    pi = _c(pi, np.float32).reshape(-1, C)
    out = np.zeros(4)
    _check(lib().orc_mask_stats(n, m, W.shape[0], _ptr(W), _ptr(pi), float(kappa), _ptr(out)), "mask_stats")
    return out


def encode_candidates(n, m, idx) -> np.ndarray:
    idx = _c(idx, np.uint8).ravel()
    D = 12 if m == 4 else 5
    out = np.zeros((idx.size + D - 1) // D, np.uint32)
    _check(lib().orc_encode_candidates(n, m, idx.size, _ptr(idx), _ptr(out)), "encode")
    return out


def decode_candidates(n, m, words, nb) -> np.ndarray:
    words = _c(words, np.uint32).ravel()
    out = np.zeros(nb, np.uint8)
    _check(lib().orc_decode_candidates(n, m, nb, _ptr(words), _ptr(out)), "decode")
    return out


def sparse_linear(n, m, values, meta, x) -> np.ndarray:
    """Product with a hard-masked weight in hard_pack's compressed form (s.3.2, inference):
    values [rows, cols*N/M] uint16 (bf16 bits), meta as hard_pack returns it, x [tokens, cols]
    uint16 (bf16 bits). Returns y [tokens, rows] float64, y = x W*^T."""
    values = _c(values, np.uint16)
    rows = values.shape[0]
    x = _c(x, np.uint16)
    tokens, cols = x.shape
    meta = _c(meta, np.uint32 if m == 4 else np.uint16)
    y = np.zeros((tokens, rows))
    _check(lib().orc_sparse_linear(n, m, rows, cols, _ptr(values), _ptr(meta), tokens, _ptr(x), _ptr(y)),
           "sparse_linear")
    return y
