"""Pins of the oracle's per-token corrections around the activation prune
(D-PTS shift, VAR rescale; Flexible (N:M) Activation Sparsity, technical
summary §2.B) against closed forms, exact integer arithmetic, exact
summation and library variance -- never against the oracle itself."""
import math

import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs


def _ints(shape, lo, hi, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi, size=shape).astype(np.float64)


def test_no_correction_is_the_plain_product():
    x = inputs.student_t_bf16((24, 256), 4.0, 1)
    w = inputs.normal_bf16((40, 256), 0.02, 2)
    for N, M in [(2, 4), (8, 16), (16, 32)]:
        np.testing.assert_array_equal(oracle.act_sparse_linear_xf(x, w, N, M, False, False),
                                      oracle.act_sparse_linear(x, w, N, M))


@pytest.mark.parametrize("K,dist", [(4096, "student_t4"), (4096, "normal"), (14336, "normal_outliers"),
                                    (256, "normal")])
def test_mean_is_the_exactly_rounded_mean(K, dist):
    """The fp64 sum of bf16 tokens is exact here, so the mean equals
    math.fsum's correctly rounded sum divided by K, whatever the order."""
    if dist == "student_t4":
        x = inputs.student_t_bf16((16, K), 4.0, 3)
    elif dist == "normal_outliers":
        x = inputs.normal_with_outlier_channels_bf16((16, K), 0.001, 20.0, 3)
    else:
        x = inputs.normal_bf16((16, K), 1.0, 3)
    mu64, mu32 = oracle.row_mean(x)
    xf = inputs.bf16_to_f64(x)
    for r in range(x.shape[0]):
        assert mu64[r] == math.fsum(xf[r]) / K
        assert mu64[r] == math.fsum(xf[r][::-1]) / K
    np.testing.assert_array_equal(mu32, mu64.astype(np.float32))


def test_shift_of_integer_tokens_is_exact():
    """Integer tokens whose mean is an integer c: the shifted token is x - c
    exactly (small integers are bf16 values)."""
    base = _ints((12, 64), -20, 21, 4)
    base -= np.round(base.mean(axis=1, keepdims=True))
    c = _ints((12, 1), -5, 6, 5)
    base[:, -1] -= base.sum(axis=1)                  # every row sums to 0 ...
    x = inputs.bf16_from_f64(base + c)               # ... so its mean is c exactly
    mu64, mu32 = oracle.row_mean(x)
    np.testing.assert_array_equal(mu64, c[:, 0])
    xs = oracle.shift_bf16(x, mu32)
    np.testing.assert_array_equal(inputs.bf16_to_f64(xs), base)


@pytest.mark.parametrize("var", [False, True])
def test_unpruned_shift_returns_the_dense_product(var):
    """With N = M nothing is pruned: the shift and its add-back cancel, and
    VAR's factor is exactly 1, so on integers the result is X . W^T exactly."""
    base = _ints((10, 64), -8, 9, 6)
    base[:, -1] -= base.sum(axis=1) - 64 * _ints((10,), -3, 4, 7)   # integer means
    x = inputs.bf16_from_f64(base)
    w = inputs.bf16_from_f64(_ints((20, 64), -4, 5, 8))
    exact = inputs.bf16_to_f64(x) @ inputs.bf16_to_f64(w).T          # integers < 2^24: exact
    t = oracle.act_transform(x, 4, 4, True, var)
    np.testing.assert_array_equal(t["alpha"], np.ones(10))
    np.testing.assert_array_equal(oracle.act_sparse_linear_xf(x, w, 4, 4, True, var), exact)


def test_constant_tokens():
    """A constant token c shifts to zero, so the product is c times the row
    sums of W, which for a constant token is also the unpruned product."""
    c = np.array([[3.0], [-0.5], [0.0], [1.25]])
    x = inputs.bf16_from_f64(np.repeat(c, 32, axis=1))
    w = inputs.bf16_from_f64(_ints((8, 32), -4, 5, 9))
    exact = inputs.bf16_to_f64(x) @ inputs.bf16_to_f64(w).T
    for var in (False, True):
        y = oracle.act_sparse_linear_xf(x, w, 2, 4, True, var)
        np.testing.assert_array_equal(y, exact)


def test_worked_example():
    """x = [4, -1, 3, 2], 2:4, W = I.  Without the shift the prune keeps 4 and
    3: the token's variance is 7.5 - 2^2 = 3.5, the pruned token's
    6.25 - 1.75^2 = 3.1875.  With the shift (mean 2) the token is
    [2, -3, 1, 0], the prune keeps 2 and -3, and the variances are 3.5 and
    3.25 - 0.25^2 = 3.1875 again; the output is alpha * [2, -3, 0, 0] + 2."""
    x = inputs.bf16_from_f64(np.array([[4.0, -1.0, 3.0, 2.0]]))
    eye = inputs.bf16_from_f64(np.eye(4))
    a = math.sqrt(3.5 / 3.1875)
    t = oracle.act_transform(x, 2, 4, False, True)
    np.testing.assert_array_equal(t["keep"], [[1, 0, 1, 0]])
    assert t["alpha"][0] == pytest.approx(a, rel=1e-15)
    np.testing.assert_allclose(oracle.act_sparse_linear_xf(x, eye, 2, 4, False, True), [[4 * a, 0, 3 * a, 0]],
                               rtol=1e-15)
    t = oracle.act_transform(x, 2, 4, True, True)
    np.testing.assert_array_equal(inputs.bf16_to_f64(t["xs"]), [[2.0, -3.0, 1.0, 0.0]])
    np.testing.assert_array_equal(t["keep"], [[1, 1, 0, 0]])
    assert t["alpha"][0] == pytest.approx(a, rel=1e-15)
    np.testing.assert_allclose(oracle.act_sparse_linear_xf(x, eye, 2, 4, True, True),
                               [[2 * a + 2, -3 * a + 2, 2, 2]], rtol=1e-15)
    np.testing.assert_allclose(oracle.act_sparse_linear_xf(x, eye, 2, 4, True, False), [[4, -1, 2, 2]],
                               rtol=0)


@pytest.mark.parametrize("N,M", [(2, 4), (8, 16), (16, 32)])
def test_var_factor_matches_library_variance(N, M):
    x = inputs.student_t_bf16((32, 512), 4.0, 10)
    keep = oracle.prune(x, N, M)
    alpha = oracle.var_scale(x, x, keep)
    xf = inputs.bf16_to_f64(x)
    ref = np.sqrt(np.var(xf, axis=1) / np.var(xf * keep, axis=1))
    np.testing.assert_allclose(alpha, ref, rtol=1e-12)
    # the rescaled survivors have the variance of the token they came from
    np.testing.assert_allclose(np.var(alpha[:, None] * xf * keep, axis=1), np.var(xf, axis=1), rtol=1e-12)
    # nothing pruned: factor 1; a token whose survivors are all zero: factor 1
    np.testing.assert_array_equal(oracle.var_scale(x, x, np.ones_like(keep)), np.ones(32))
    np.testing.assert_array_equal(oracle.var_scale(x, x, np.zeros_like(keep)), np.ones(32))


def test_var_with_the_shift_restores_the_dense_token_variance():
    """With the shift, the kept entries are those of the shifted token and
    the target variance is the incoming token's."""
    x = inputs.bf16_from_f64(inputs.bf16_to_f64(inputs.student_t_bf16((16, 512), 4.0, 16)) + 2.0)
    t = oracle.act_transform(x, 8, 16, True, True)
    xf, xs = inputs.bf16_to_f64(x), inputs.bf16_to_f64(t["xs"])
    ref = np.sqrt(np.var(xf, axis=1) / np.var(xs * t["keep"], axis=1))
    np.testing.assert_allclose(t["alpha"], ref, rtol=1e-12)
    # the shifted token has the same variance up to its bf16 rounding
    np.testing.assert_allclose(np.var(xs, axis=1), np.var(xf, axis=1), rtol=1e-2)


def test_shift_error_is_the_bf16_rounding_of_the_shifted_token():
    """Unpruned, the shifted product differs from X . W^T only by the bf16
    rounding of x - mu (at most 2^-9 relative per entry)."""
    x = inputs.student_t_bf16((16, 256), 4.0, 11)
    x = inputs.bf16_from_f64(inputs.bf16_to_f64(x) + 3.0)          # tokens off centre
    w = inputs.normal_bf16((24, 256), 0.02, 12)
    y = oracle.act_sparse_linear_xf(x, w, 4, 4, True, False)
    xf, wf = inputs.bf16_to_f64(x), inputs.bf16_to_f64(w)
    _, mu32 = oracle.row_mean(x)
    d = np.abs(xf - mu32.astype(np.float64)[:, None])
    bound = (2.0 ** -9) * d @ np.abs(wf).T + 1e-12
    assert (np.abs(y - xf @ wf.T) <= bound).all()


def test_shift_recentres_the_token():
    x = inputs.bf16_from_f64(inputs.bf16_to_f64(inputs.student_t_bf16((8, 1024), 4.0, 13)) + 5.0)
    _, mu32 = oracle.row_mean(x)
    xs = inputs.bf16_to_f64(oracle.shift_bf16(x, mu32))
    assert (np.abs(xs.mean(axis=1)) < 1e-2).all()
    assert (np.abs(mu32 - 5.0) < 0.2).all()


def test_row_sums():
    w = inputs.bf16_from_f64(_ints((6, 100), -7, 8, 14))
    np.testing.assert_array_equal(oracle.rowsum_f64(w), inputs.bf16_to_f64(w).sum(axis=1))
    w = inputs.normal_bf16((6, 4096), 0.02, 15)
    wf = inputs.bf16_to_f64(w)
    for o in range(6):
        assert oracle.rowsum_f64(w)[o] == math.fsum(wf[o])
