"""Pins for the oracle's fp64 linear step, the lifted-GEMM equivalence and the
hardware metadata image."""
import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs


def test_linear_exact_on_integers():
    rng = np.random.default_rng(1)
    A = rng.integers(-50, 51, size=(13, 70))
    B = rng.integers(-50, 51, size=(9, 70))
    Y = oracle.linear_f64(A.astype(np.float64), B.astype(np.float64))
    np.testing.assert_array_equal(Y, (A @ B.T).astype(np.float64))


def test_linear_matches_library_matmul():
    rng = np.random.default_rng(2)
    A = rng.standard_normal((17, 300))
    B = rng.standard_normal((23, 300))
    Y = oracle.linear_f64(A, B)
    np.testing.assert_allclose(Y, A @ B.T, rtol=1e-12, atol=1e-12)
    # transposed operands are not the same product
    assert not np.allclose(oracle.linear_f64(A[:, ::-1].copy(), B), Y)


def test_linear_row_selection():
    rng = np.random.default_rng(3)
    A = rng.standard_normal((11, 40))
    B = rng.standard_normal((5, 40))
    full = oracle.linear_f64(A, B)
    sel = [10, 0, 7]
    np.testing.assert_array_equal(oracle.linear_f64(A, B, rows=sel), full[sel])


def test_to_f64_widening():
    x = inputs.normal_bf16((4, 8), 3.0, seed=1)
    np.testing.assert_array_equal(oracle.to_f64(x), inputs.bf16_to_f64(x))
    f = np.random.default_rng(0).standard_normal((3, 5)).astype(np.float32)
    np.testing.assert_array_equal(oracle.to_f64(f), f.astype(np.float64))
    keep = np.zeros((4, 8), np.uint8)
    keep[1, 2] = 1
    z = oracle.to_f64(x, keep)
    assert np.count_nonzero(z) <= 1 and z[1, 2] == inputs.bf16_to_f64(x[1, 2])


@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (6, 8), (4, 8), (8, 16), (16, 32)])
def test_lifted_gemm_equals_pruned_gemm_bitwise(N, M):
    """The windows keep the kept terms in ascending order and add exact zeros,
    so the lifted fp64 product equals the pruned dense fp64 product bit for bit
    (SlideSparse, technical summary 2.B: the lifted product is the original)."""
    x = inputs.student_t_bf16((6, M * 8), 4.0, seed=N * 31 + M)
    w = inputs.normal_bf16((10, M * 8), 0.02, seed=4)
    keep = oracle.prune(x, N, M)
    vals, nib = oracle.compress(x, keep, M)
    A_lift = oracle.expand_lifted(vals, nib)
    B_lift = oracle.to_f64(oracle.lift(w, M))
    y_lift = oracle.linear_f64(A_lift, B_lift)
    y_ref = oracle.linear_f64(oracle.to_f64(x, keep), oracle.to_f64(w))
    assert np.array_equal(y_lift, y_ref)
    np.testing.assert_array_equal(y_ref, oracle.act_sparse_linear(x, w, N, M))


def test_weight_side_is_the_transpose_problem():
    x = inputs.normal_bf16((5, 64), 1.0, seed=8)
    w = inputs.normal_bf16((7, 64), 0.02, seed=9)
    y = oracle.weight_sparse_linear(x, w, 6, 8)
    yt = oracle.act_sparse_linear(w, x, 6, 8)
    np.testing.assert_array_equal(y, yt.T)


@pytest.mark.parametrize("M", [4, 8, 16, 32])
def test_n_equals_m_reproduces_dense(M):
    x = inputs.normal_bf16((4, M * 4), 1.0, seed=2)
    w = inputs.normal_bf16((6, M * 4), 0.02, seed=3)
    np.testing.assert_array_equal(oracle.act_sparse_linear(x, w, M, M),
                                  oracle.linear_f64(oracle.to_f64(x), oracle.to_f64(w)))


# ---------------------------------------------------------- hardware metadata


def _decode_meta_image(meta, rows, Kl):
    """Independent reading of the 16-bit sparse-MMA metadata image: inside one
    128-row x 128-lifted-K block, the logical coordinate (m, k) with
    m = m0 + 8 m1 + 16 m2 and k = k0 + 16 k1 + 32 k2 sits at eighth-byte offset
    128 m0 + 16 m1 + 2048 m2 + k0 + 1024 k1 + 32 k2; a nibble covers the 4
    eighth-bytes of one group of 4 k."""
    RB, KB = -(-rows // 128), -(-Kl // 128)
    out = np.zeros((RB * 128, KB * 32), np.uint8)
    m = np.arange(128)
    m0, m1, m2 = m % 8, (m // 8) % 2, m // 16
    for kq in range(32):                       # group of 4 lifted k in the block
        k = kq * 4
        k0, k1, k2 = k % 16, (k // 16) % 2, k // 32
        off8 = 128 * m0 + 16 * m1 + 2048 * m2 + k0 + 1024 * k1 + 32 * k2
        byte, half = off8 // 8, (off8 // 4) % 2
        for rb in range(RB):
            for kb in range(KB):
                blk = meta[(rb * KB + kb) * 2048:(rb * KB + kb + 1) * 2048]
                out[rb * 128:(rb + 1) * 128, kb * 32 + kq] = (blk[byte] >> (4 * half)) & 0xF
    return out


@pytest.mark.parametrize("rows,N,M,K", [(128, 2, 4, 128), (200, 8, 16, 512), (37, 6, 8, 96), (5, 16, 32, 64)])
def test_meta_image_decodes_to_nibbles(rows, N, M, K):
    x = inputs.normal_bf16((rows, K), 1.0, seed=rows)
    keep = oracle.prune(x, N, M)
    vals, nib = oracle.compress(x, keep, M)
    Kl = oracle.lifted_k(K, M)
    meta = oracle.meta_hw(nib, Kl)
    assert meta.size == -(-rows // 128) * -(-Kl // 128) * 2048
    dec = _decode_meta_image(meta, rows, Kl)
    np.testing.assert_array_equal(dec[:rows, :Kl // 4], nib)
    # padding rows and windows carry the valid nibble 0x4
    assert (dec[rows:, :] == 0x4).all()
    assert (dec[:, Kl // 4:] == 0x4).all()
