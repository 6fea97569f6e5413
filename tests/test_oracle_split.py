"""The split window order (every group's even windows, then its odd ones):
pins of the oracle's reordering against the sliding-window definition and
the pruned product (SlideSparse page, technical summary §2.A-§2.C)."""
import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs


@pytest.mark.parametrize("K,M", [(64, 8), (384, 8), (256, 16), (1024, 32), (96, 8)])
def test_split_order_is_a_permutation_of_the_windows(K, M):
    perm = oracle.split_window_order(K, M)
    assert perm.size == oracle.lifted_k(K, M) // 4
    assert np.array_equal(np.sort(perm), np.arange(perm.size))


@pytest.mark.parametrize("rows,K,M", [(5, 64, 8), (3, 384, 8), (4, 256, 16), (2, 1024, 32)])
def test_even_windows_are_the_raw_row(rows, K, M):
    """Windows 2e of a group cover positions 4e .. 4e + 3 of it: in the split
    order the first K lifted columns are X itself."""
    x = inputs.normal_bf16((rows, K), 1.0, rows + K)
    ls = oracle.lift_split(x, M)
    assert ls.shape == (rows, oracle.lifted_k(K, M))
    np.testing.assert_array_equal(ls[:, :K], x)


@pytest.mark.parametrize("rows,K,M", [(3, 64, 8), (2, 256, 16), (2, 1024, 32)])
def test_odd_windows_straddle_the_even_ones(rows, K, M):
    """Odd window 2o + 1 of group g starts two elements into even window 2o:
    positions g M + 4o + 2 .. + 5, read here by brute force from X."""
    x = np.arange(rows * K, dtype=np.uint16).reshape(rows, K)
    ls = oracle.lift_split(x, M)
    NO = M // 4 - 1
    odd = ls[:, K:].reshape(rows, K // M, NO, 4)
    for g in range(K // M):
        for o in range(NO):
            np.testing.assert_array_equal(odd[:, g, o, :], x[:, g * M + 4 * o + 2: g * M + 4 * o + 6])


@pytest.mark.parametrize("N,M", [(6, 8), (4, 8), (14, 16), (10, 16), (30, 32)])
def test_split_operand_gives_the_pruned_product(N, M):
    """Both operands in the split order give the pruned product exactly on
    integers, as the natural order does: the reordering moves values and
    their index pairs together."""
    rng = np.random.default_rng(N * 100 + M)
    K = 4 * M * 3
    w = inputs.bf16_from_f64(rng.integers(-4, 5, size=(7, K)).astype(np.float64))
    x = inputs.bf16_from_f64(rng.integers(-3, 4, size=(5, K)).astype(np.float64))
    sp = oracle.sparse_operand_split(w, N, M)
    W_lift = oracle.expand_lifted(sp["vals"], sp["nib"])          # [7, K'] sparse, split order
    X_lift = oracle.to_f64(oracle.lift_split(x, M))
    y = oracle.linear_f64(X_lift, W_lift)
    np.testing.assert_array_equal(y, oracle.weight_sparse_linear(x, w, N, M))
    # and the natural order agrees element for element
    nat = oracle.sparse_operand(w, N, M)
    y_nat = oracle.linear_f64(oracle.to_f64(oracle.lift(x, M)), oracle.expand_lifted(nat["vals"], nat["nib"]))
    np.testing.assert_array_equal(y, y_nat)
    # the image is the natural one's blocks rebuilt from the moved index pairs
    assert sp["meta"].size == nat["meta"].size
