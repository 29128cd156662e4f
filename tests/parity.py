"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the floating-point bar of the path):
  * corruption masks, replacement ids, t and p: bit-exact;
  * losses: relative 1e-5 (fp32 accumulation on the GPU vs double);
  * bf16 gradients: |gpu - exact| <= max(2e-3, one bf16 ulp of the exact
    value) -- 2e-3 absolute, except where a gradient is so large (w = 1/(pN)
    with small p and small N) that bf16 itself cannot hold 2e-3 -- and the
    GPU value is at most one ulp away from the exact value rounded to bf16
    (values below 2^-126, the smallest normal, count as zero in that last
    check: the kernels' exponentials flush subnormal results to zero, and
    2^-126 is far inside the 2e-3 absolute bar);
  * fused-head gradients dH = dZ W and dW = dZ^T H_M, element by element:
    each is a bf16 rounding of an fp32 sum of products a_k b_k in which a_k
    (dZ) was itself rounded to bf16, a relative error of at most u = 2^-8
    per product.  The bar is
        |gpu - exact| <= ulp(max(|gpu|, |exact|)) + 8 u s,
        s = sqrt(sum_k (a_k b_k)^2) over that element's products:
    the first term is the output's own rounding; u s bounds the standard
    deviation the sum can get from independent roundings of the a_k, and
    8 u s also covers their worst case u sum_k |a_k b_k| whenever at most 64
    products matter.  The fp32 accumulation (relative ~1e-6) is far below it.
"""
import numpy as np
import torch

LOSS_RTOL = 1e-5
GRAD_ATOL = 2e-3
BF16_U = 2.0 ** -8          # unit roundoff of bf16 (8 significant bits)
SUM_SIGMAS = 8.0


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 7), 2.0 ** -133)


def to_bf16_f64(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def gpu_bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_grad_close(gpu: np.ndarray, exact: np.ndarray, what: str = "dlogits"):
    gpu = np.asarray(gpu, np.float64)
    exact = np.asarray(exact, np.float64)
    assert gpu.shape == exact.shape
    err = np.abs(gpu - exact)
    tol = np.maximum(GRAD_ATOL, bf16_ulp(exact))
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max err {err.max():.3e}"
    # and within one ulp of the exactly rounded value (values below the
    # smallest normal bf16, 2^-126, are compared as zero: the kernels flush
    # exponentials that small)
    rnd = to_bf16_f64(exact)
    tiny = 2.0 ** -126
    rnd = np.where(np.abs(rnd) < tiny, 0.0, rnd)
    g = np.where(np.abs(gpu) < tiny, 0.0, gpu)
    ulps = np.abs(g - rnd) / bf16_ulp(np.maximum(np.abs(rnd), np.abs(g)))
    assert ulps.max() <= 1.0 + 1e-9, f"{what}: {ulps.max()} bf16 ulps from the rounded exact value"
    # exact zeros stay exact zeros
    assert (gpu[exact == 0] == 0).all(), f"{what}: nonzero where the exact gradient is 0"


def assert_loss_close(gpu: float, exact: float, what: str = "loss"):
    assert abs(gpu - exact) <= LOSS_RTOL * max(abs(exact), 1e-30), \
        f"{what}: gpu {gpu!r} vs oracle {exact!r} (rel {abs(gpu - exact) / max(abs(exact), 1e-30):.2e})"


def assert_units_close(gpu: np.ndarray, exact: np.ndarray, total: float):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - exact)
    tol = LOSS_RTOL * np.abs(exact) + 1e-7 * abs(total)
    assert (err <= tol).all(), f"unit_loss: max err {err.max():.3e}"


def product_rms_scale(a: np.ndarray, b: np.ndarray, transpose_a: bool = False,
                      chunk: int = 16384) -> np.ndarray:
    """s = sqrt((a*a) @ (b*b)) (or sqrt((a*a)^T @ (b*b))) in float32: for
    C = a @ b the root of the sum of squared products of each element of C.
    Streams the shared dimension in chunks to bound host memory."""
    n = a.shape[0] if transpose_a else a.shape[1]
    out = None
    for k0 in range(0, n, chunk):
        ak = (a[k0:k0 + chunk] if transpose_a else a[:, k0:k0 + chunk]).astype(np.float32)
        ak *= ak
        bk = b[k0:k0 + chunk].astype(np.float32)
        bk *= bk
        part = (ak.T @ bk) if transpose_a else (ak @ bk)
        out = part if out is None else out + part
    return np.sqrt(out)


def assert_bf16_sum_close(gpu: np.ndarray, exact: np.ndarray, scale: np.ndarray, what: str,
                          block_rows: int = 8192):
    """Element-wise bar for a bf16 sum of products whose one operand was
    rounded to bf16 (see the module docstring); `scale` = product_rms_scale
    of that sum.  Compared in blocks of rows (full-size gradients are
    gigabytes).  Returns the relative Frobenius error, for reports."""
    assert gpu.shape == exact.shape == scale.shape, (gpu.shape, exact.shape, scale.shape)
    n_bad = 0
    worst = None
    d2 = e2 = 0.0
    for r0 in range(0, gpu.shape[0], block_rows):
        g = np.asarray(gpu[r0:r0 + block_rows], np.float64)
        e = np.asarray(exact[r0:r0 + block_rows], np.float64)
        err = np.abs(g - e)
        tol = bf16_ulp(np.maximum(np.abs(g), np.abs(e))) + SUM_SIGMAS * BF16_U * scale[r0:r0 + block_rows]
        bad = err > tol
        d2 += float(np.square(err).sum())
        e2 += float(np.square(e).sum())
        if bad.any():
            n_bad += int(bad.sum())
            i = np.unravel_index(int(np.argmax(err - tol)), err.shape)
            cand = (float((err - tol)[i]), (i[0] + r0,) + tuple(i[1:]), g[i], e[i], float(tol[i]))
            worst = cand if worst is None or cand[0] > worst[0] else worst
    if n_bad:
        _, i, gv, ev, tv = worst
        raise AssertionError(f"{what}: {n_bad} of {gpu.size} elements out of tolerance; worst at {i}: "
                             f"gpu {gv!r} exact {ev!r} tol {tv:.3e}")
    return float(np.sqrt(d2) / max(np.sqrt(e2), 1e-300))
