"""The GPU-vs-oracle comparison helpers accept what the bar allows and refuse
what it does not (CPU only): bf16 ulps, the gradient bar (2e-3 absolute or
one bf16 ulp, and within one ulp of the exactly rounded value), exact zeros,
the 1e-5 relative loss bar and the per-unit bar."""
import numpy as np
import pytest

from parity import (assert_bf16_sum_close, assert_grad_close, assert_loss_close, assert_units_close, bf16_ulp,
                    product_rms_scale, to_bf16_f64)


def test_bf16_ulp_of_powers_of_two_and_between():
    x = np.array([1.0, 1.5, 0.75, 2.0 ** -20, 3.0e4, -6.0])
    assert np.array_equal(bf16_ulp(x), np.array([2.0 ** -7, 2.0 ** -7, 2.0 ** -8, 2.0 ** -27, 2.0 ** 7, 2.0 ** -5]))


def _exact(seed=0, n=4096):
    rng = np.random.default_rng(seed)
    g = rng.standard_normal(n) * 1e-3
    g[::7] = 0.0
    return g


def test_gradient_rounded_exactly_passes():
    e = _exact()
    assert_grad_close(to_bf16_f64(e), e)


def test_gradient_one_ulp_off_passes_two_ulps_off_fails():
    e = _exact(1)
    r = to_bf16_f64(e)
    k = 11
    one = r.copy()
    one[k] = r[k] + bf16_ulp(r[k])
    assert_grad_close(one, e)
    two = r.copy()
    two[k] = r[k] + 2 * bf16_ulp(np.array([r[k]]))[0] * 1.01
    with pytest.raises(AssertionError, match="ulps"):
        assert_grad_close(two, e)


def test_gradient_absolute_bar():
    e = np.array([0.5, 0.25, 1.0e-3])
    g = to_bf16_f64(e)
    g[2] += 2.5e-3                                   # beyond 2e-3 absolute where bf16 could hold it
    with pytest.raises(AssertionError):
        assert_grad_close(g, e)


def test_large_gradients_get_one_ulp_not_2e3():
    """Where bf16 cannot hold 2e-3 (spacing 2^-5 at 7.8), a value one ulp
    from the rounded exact value and within one ulp of the exact value
    passes although it is ~0.019 away; one more ulp does not."""
    e = np.array([7.8, -7.8])
    g = to_bf16_f64(e)                               # 7.8125: the nearest bf16
    g[0] = g[0] - bf16_ulp(np.array([g[0]]))[0]      # 7.78125
    assert abs(g[0] - e[0]) > 2e-3
    assert_grad_close(g, e)
    g[0] = g[0] - bf16_ulp(np.array([g[0]]))[0]
    with pytest.raises(AssertionError):
        assert_grad_close(g, e)


def test_nonzero_where_exact_is_zero_fails():
    e = _exact(2)
    g = to_bf16_f64(e)
    z = int(np.nonzero(e == 0)[0][0])
    g[z] = 1e-6
    with pytest.raises(AssertionError):
        assert_grad_close(g, e)


def test_loss_bar():
    assert_loss_close(1.0 + 9e-6, 1.0)
    with pytest.raises(AssertionError):
        assert_loss_close(1.0 + 1.1e-5, 1.0)
    with pytest.raises(AssertionError):
        assert_loss_close(-2.0 * (1 + 2e-5), -2.0)


def test_unit_bar():
    exact = np.array([1.0, 0.0, 3.0])
    assert_units_close(exact * (1 + 5e-6), exact, 4.0)
    with pytest.raises(AssertionError):
        assert_units_close(exact + np.array([0.0, 1e-5, 0.0]), exact, 4.0)


def _rounded_product_sum(a, b, rng_flip=None):
    """bf16(sum_k bf16(a_k) b_k), the way the fused head forms dH and dW."""
    ar = to_bf16_f64(a)
    return to_bf16_f64(ar @ b)


def test_sum_bar_accepts_bf16_rounded_operand_and_output():
    """A sum whose one operand and result are rounded to bf16 passes the
    element-wise fused-head bar -- many small products (the softmax part)
    and one dominant product (the target) alike."""
    rng = np.random.default_rng(3)
    a = rng.random((64, 3000)) * 1e-4          # softmax-like: many small positive terms
    a[np.arange(64), rng.integers(0, 3000, 64)] = -0.9   # one dominant target per row
    b = rng.standard_normal((3000, 96)) * 0.02
    exact = a @ b
    gpu = _rounded_product_sum(a, b)
    s = product_rms_scale(a, b)
    assert_bf16_sum_close(gpu, exact, s, "dH-like")
    # the transposed form (dW = a^T H)
    h = rng.standard_normal((64, 96))
    exact_t = a.T @ h
    gpu_t = to_bf16_f64(to_bf16_f64(a).T @ h)
    assert_bf16_sum_close(gpu_t, exact_t, product_rms_scale(a, h, transpose_a=True), "dW-like")


def test_sum_bar_refuses_a_wrong_tile_a_scaled_row_and_a_dropped_target():
    rng = np.random.default_rng(4)
    a = rng.random((64, 3000)) * 1e-4
    tgt = rng.integers(0, 3000, 64)
    a[np.arange(64), tgt] = -0.9
    b = rng.standard_normal((3000, 96)) * 0.02
    exact = a @ b
    s = product_rms_scale(a, b)
    good = _rounded_product_sum(a, b)
    tile = good.copy()
    tile[32:48, 64:96] = 0.0                   # one output tile never written
    with pytest.raises(AssertionError):
        assert_bf16_sum_close(tile, exact, s, "tile")
    scaled = good.copy()
    scaled[5] *= 1.05                          # one row 5% off
    with pytest.raises(AssertionError):
        assert_bf16_sum_close(scaled, exact, s, "row")
    dropped = a.copy()
    dropped[7, tgt[7]] = 0.0                   # a row's target term lost
    with pytest.raises(AssertionError):
        assert_bf16_sum_close(_rounded_product_sum(dropped, b), exact, s, "target")
    # many small products: a 5% error of a whole column of dW is caught
    h = rng.standard_normal((64, 96))
    a2 = rng.random((4000, 3000)) * 1e-4
    h2 = rng.standard_normal((4000, 96))
    exact_t = a2.T @ h2
    gpu_t = to_bf16_f64(to_bf16_f64(a2).T @ h2)
    s_t = product_rms_scale(a2, h2, transpose_a=True)
    assert_bf16_sum_close(gpu_t, exact_t, s_t, "dW-like")
    bad = gpu_t.copy()
    bad[:, 10] *= 1.05
    with pytest.raises(AssertionError):
        assert_bf16_sum_close(bad, exact_t, s_t, "dW column")
    del h
