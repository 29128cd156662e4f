"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the floating-point bar of the path):
  * corruption masks, replacement ids, t and p: bit-exact;
  * losses: relative 1e-5 (fp32 accumulation on the GPU vs double);
  * bf16 gradients: |gpu - exact| <= max(2e-3, one bf16 ulp of the exact
    value) -- 2e-3 absolute, except where a gradient is so large (w = 1/(pN)
    with small p and small N) that bf16 itself cannot hold 2e-3 -- and the
    GPU value is at most one ulp away from the exact value rounded to bf16.
"""
import numpy as np
import torch

LOSS_RTOL = 1e-5
GRAD_ATOL = 2e-3


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
