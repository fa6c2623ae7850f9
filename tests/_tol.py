"""Parity tolerances between the CUDA path and the oracle.

The bars are the stated ones: bit-exact for integer/index work (noise bits, hard masks,
packed values and metadata); soft masks 1e-5 relative; W.M within 1 bf16 ulp (1e-5 relative
when W is fp32); logit gradients and AdamW-updated logits 1e-4 relative; the regulariser
1e-3 relative. How "relative" is read:
  * soft mask: element-wise, |dM_j| <= 1e-5 M_ref_j (a sum of positive weights);
  * gradient: a signed sum of terms, so relative to the magnitude of its summands,
    |dg_i| <= 1e-4 (kappa/tau) y_i sum_j |S_ij - M_j| |u_j| (the oracle's `scale`);
  * updated logits: relative to the block, |dpi_i| <= 1e-4 max_k |pi_ref_k|. A block's
    logits enter the method only through softmax(kappa pi + g), which is invariant to a
    shift of all of them, so a single logit has no scale of its own (one that happens to sit
    near zero is not more precise for it); the block's largest magnitude is its scale. The
    worst per-element relative error is returned for reporting.
Every bound also admits an absolute floor 1e-30 times the block's natural scale: fp32 soft
index weights below 2^-126 flush to zero on the GPU (exp2 approximation with ftz) where the
fp64 oracle keeps them; such differences are representational, not arithmetic.
"""
import numpy as np

FLOOR = 1e-30


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significant bits, fp32 exponent range)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def assert_x_close(x_gpu, x_ref, w_dtype, W):
    """Soft-masked weights: 1 bf16 ulp (bf16) or 1e-5 relative (fp32), floor |W| 1e-30."""
    x_gpu = np.asarray(x_gpu, np.float64)
    x_ref = np.asarray(x_ref, np.float64)
    err = np.abs(x_gpu - x_ref)
    if w_dtype == "bf16":
        tol = bf16_ulp(x_ref)
    else:
        tol = 1e-5 * np.abs(x_ref)
    tol = tol + FLOOR * np.abs(W)
    bad = ~(err <= tol)  # NaN fails
    assert not bad.any(), f"{bad.sum()} X mismatches, worst {np.max(err / np.maximum(tol, 1e-300)):.3g} x tol"


def assert_soft_close(ms_gpu, ms_ref):
    err = np.abs(np.asarray(ms_gpu, np.float64) - ms_ref)
    tol = 1e-5 * ms_ref + FLOOR
    bad = ~(err <= tol)  # NaN fails
    assert not bad.any(), f"{bad.sum()} soft-mask mismatches, worst {np.max(err / tol):.3g} x tol"
    return float(np.max(err / np.maximum(ms_ref, 1e-300)))


def grad_floor(W, G, kappa, tau, lam):
    """Per-block floor: 1e-30 (kappa/tau) sum_j (|G_j W_j| + 2 lambda W_j^2)."""
    W = np.asarray(W, np.float64)
    G = np.asarray(G, np.float64)
    return FLOOR * (kappa / tau) * (np.abs(G * W) + 2 * lam * W * W).sum(1, keepdims=True)


def assert_grad_close(g_gpu, g_ref, scale, floor):
    err = np.abs(np.asarray(g_gpu, np.float64) - g_ref)
    tol = 1e-4 * scale + floor
    bad = ~(err <= tol)  # NaN fails
    assert not bad.any(), f"{bad.sum()} gradient mismatches, worst {np.max(err / tol):.3g} x tol"
    return float(np.max(err / np.maximum(scale, 1e-300)))


def assert_logits_close(p_gpu, p_ref):
    p_ref = np.asarray(p_ref, np.float64)
    err = np.abs(np.asarray(p_gpu, np.float64) - p_ref)
    tol = 1e-4 * np.abs(p_ref).max(1, keepdims=True) + FLOOR
    bad = ~(err <= tol)  # NaN fails
    assert not bad.any(), f"{bad.sum()} updated-logit mismatches, worst {np.max(err / tol):.3g} x tol"
    return float(np.max(err / np.maximum(np.abs(p_ref), FLOOR)))


def assert_moments_close(m_gpu, v_gpu, m_ref, v_ref, g_ref, g_tol, beta1, beta2):
    """AdamW moments carry the gradient's tolerance: dm <= (1-b1) dg, dv <= (1-b2)(2|g| dg + dg^2),
    plus fp32 rounding (2^-22 relative)."""
    m_err = np.abs(np.asarray(m_gpu, np.float64) - m_ref)
    v_err = np.abs(np.asarray(v_gpu, np.float64) - v_ref)
    m_tol = (1 - beta1) * g_tol + 2.0**-22 * np.abs(m_ref) + FLOOR
    v_tol = (1 - beta2) * (2 * np.abs(g_ref) * g_tol + g_tol**2) + 2.0**-22 * v_ref + 1e-45
    assert (m_err <= m_tol).all(), f"{(~(m_err <= m_tol)).sum()} first-moment mismatches"
    assert (v_err <= v_tol).all(), f"{(~(v_err <= v_tol)).sum()} second-moment mismatches"


def assert_reg_close(r_gpu, r_ref):
    assert abs(r_gpu - r_ref) <= 1e-3 * abs(r_ref), (r_gpu, r_ref)


def assert_spl_close(y_gpu, y_ref, absxw, cols):
    """Product with the packed hard-masked weight: every bf16 x bf16 product is exact in
    fp32; the tensor cores add them into an fp32 accumulator one k16 step after another
    (ceil(cols/16) steps) and the split-k partial tiles are added after (at most 8). Each
    of those additions errs by at most 2 ulp (2^-22) of a running sum bounded by
    sum_k |x_k w_k|, hence |dy| <= (ceil(cols/16) + 8) 2^-22 sum_k |x_k w_k|."""
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    tol = ((cols + 15) // 16 + 8) * 2.0 ** -22 * absxw
    bad = ~(err <= tol)  # NaN fails
    assert not bad.any(), f"{bad.sum()} y mismatches, worst {np.max(err / np.maximum(tol, 1e-300)):.3g} x tol"
    return float(np.max(err / np.maximum(absxw, 1e-300)))


def assert_masked_linear_close(y_gpu, y_ref, A, x_ref, round_bf16):
    """Y = A X^T with X = bf16(W * M) made inside the GEMM, against the oracle's fp64 product
    with its own bf16 X. Two sources of difference, each bounded:
      * an element of X may round to the neighbouring bf16 value when its unrounded value
        lies within the soft-mask tolerance (1e-5 relative) plus the fp32 product's rounding
        (2^-23) of a rounding midpoint; such elements are found by rounding both ends of that
        interval (round_bf16 of the oracle), and each may move Y by |A| times the gap;
      * the tensor cores add the exact bf16 x bf16 products into fp32, one k16 step after
        another (ceil(cols/16) steps) plus the partial tiles of rows split between CTAs (at
        most 8 more additions), each off by at most 2 ulp (2^-22) of a running sum bounded
        by sum_k |A_k X_k|.
    A [T, cols], x_ref [rows, cols] unrounded float64; y [T, rows]."""
    A = np.asarray(A, np.float64)
    x_ref = np.asarray(x_ref, np.float64)
    delta = 1e-5 + 2.0 ** -23
    lo = round_bf16(x_ref * (1 - delta)).astype(np.uint32) << 16
    hi = round_bf16(x_ref * (1 + delta)).astype(np.uint32) << 16
    lo_v = lo.view(np.float32).astype(np.float64)
    hi_v = hi.view(np.float32).astype(np.float64)
    gap = np.abs(hi_v - lo_v)  # 0 where the whole interval rounds to one value
    xb = (round_bf16(x_ref).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    cols = A.shape[1]
    bound = np.abs(A) @ gap.T + ((cols + 15) // 16 + 8) * 2.0 ** -22 * (np.abs(A) @ np.abs(xb).T)
    err = np.abs(np.asarray(y_gpu, np.float64) - y_ref)
    bad = ~(err <= bound + 1e-30)  # NaN fails
    assert not bad.any(), f"{bad.sum()} Y mismatches, worst {np.max(err / np.maximum(bound, 1e-300)):.3g} x tol"
    return float(np.max(err / np.maximum(np.abs(A) @ np.abs(xb).T, 1e-300)))
