"""Pins for the hybrid dense + 2:4 weight (column energy, dense selection,
permutation, input-split accumulation)."""
import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs


def _int_bf16(rng, shape, lo=-8, hi=9):
    return inputs.bf16_from_f64(rng.integers(lo, hi, size=shape).astype(np.float64))


def test_colnorm_exact_on_integers():
    rng = np.random.default_rng(0)
    w = _int_bf16(rng, (33, 20))
    wi = inputs.bf16_to_f64(w).astype(np.int64)
    np.testing.assert_array_equal(oracle.colnorm_f64(w), (wi * wi).sum(axis=0).astype(np.float64))


def test_dense_count():
    assert oracle.hybrid_dense_count(4096, 0.25) == 1024
    assert oracle.hybrid_dense_count(4096, 0.0) == 0
    assert oracle.hybrid_dense_count(4096, 1.0) == 4096
    assert oracle.hybrid_dense_count(100, 0.3) == 28   # whole 2:4 groups remain


@pytest.mark.parametrize("D", [0, 4, 8, 32, 64])
def test_perm_selects_top_columns(D):
    rng = np.random.default_rng(D)
    w = _int_bf16(rng, (16, 64), -3, 4)          # many equal column energies
    cn = oracle.colnorm_f64(w)
    perm, dense = oracle.hybrid_perm(cn, D)
    assert sorted(perm.tolist()) == list(range(64))
    s, d = perm[:64 - D], perm[64 - D:]
    assert (np.diff(s) > 0).all() and (np.diff(d) > 0).all()
    # stable sort by energy descending: ties go to the lower column
    expect = np.sort(np.argsort(-cn, kind="stable")[:D])
    np.testing.assert_array_equal(d, expect)
    np.testing.assert_array_equal(np.flatnonzero(dense), expect)


def test_input_split_equals_unsplit_exactly_on_integers():
    """Y = X[:, pi_s] W_s^T + X[:, pi_d] W_d^T equals X Wp^T (SpenseGPT,
    technical summary 2.A, input-split with accumulation)."""
    rng = np.random.default_rng(5)
    x = _int_bf16(rng, (7, 64))
    w = _int_bf16(rng, (12, 64))
    hw = oracle.hybrid_weight(w, 0.25)
    Ks = hw["Ks"]
    perm = hw["perm"]
    xs = oracle.gather_cols(x, perm)
    y_s = oracle.linear_f64(oracle.to_f64(xs[:, :Ks].copy()),
                            oracle.expand_lifted(hw["vals_s"], hw["nib_s"]))
    y_d = oracle.linear_f64(oracle.to_f64(xs[:, Ks:].copy()), oracle.to_f64(hw["W_d"]))
    np.testing.assert_array_equal(y_s + y_d, oracle.hybrid_linear(x, w, 0.25))
    # and X Wp^T itself, from the keep mask in the original order
    xi = inputs.bf16_to_f64(x).astype(np.int64)
    wi = inputs.bf16_to_f64(w).astype(np.int64) * hw["keep_full"]
    np.testing.assert_array_equal(oracle.hybrid_linear(x, w, 0.25), (xi @ wi.T).astype(np.float64))


def test_dense_region_is_fully_kept_and_sparse_region_is_2_of_4():
    w = inputs.normal_bf16((9, 128), 0.02, seed=3)
    hw = oracle.hybrid_weight(w, 0.25)
    kf = hw["keep_full"]
    d = hw["perm"][hw["Ks"]:]
    s = hw["perm"][:hw["Ks"]]
    assert kf[:, d].all()
    assert (kf[:, s].reshape(9, -1, 4).sum(axis=2) == 2).all()


def test_dense_frac_limits():
    x = inputs.normal_bf16((3, 64), 1.0, seed=1)
    w = inputs.normal_bf16((5, 64), 0.02, seed=2)
    np.testing.assert_array_equal(oracle.hybrid_linear(x, w, 1.0),
                                  oracle.linear_f64(oracle.to_f64(x), oracle.to_f64(w)))
    np.testing.assert_array_equal(oracle.hybrid_linear(x, w, 0.0),
                                  oracle.weight_sparse_linear(x, w, 2, 4))
