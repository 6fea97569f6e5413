"""Seeded random shapes through every product of the library against the
oracle: row counts, reduction lengths and output widths drawn off the tile
grid (ragged tails, single rows, split-K and SM-pair paths), each N:M family,
both sides, the hybrid format, the 8-bit path and the per-token corrections.
Compressed operands bit-exact, products within tolerance."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu

PATTERNS = [(2, 4), (1, 4), (4, 8), (6, 8), (8, 16), (14, 16), (16, 32), (30, 32)]


def _draw(i):
    """Shape i of the sweep: (T, K, O, N, M), K a multiple of M with a lifted
    width that is a multiple of 16."""
    rng = np.random.default_rng(1000 + i)
    N, M = PATTERNS[i % len(PATTERNS)]
    T = int(rng.choice([1, 3, 16, 40, 127, 129, 256, 300, 512]))
    O = int(rng.choice([16, 72, 128, 200, 256, 384, 520]))
    while True:
        K = int(M * rng.integers(2, 2048 // M + 1))
        if nm.lifted_k(K, M) % 16 == 0:
            return T, K, O, N, M


@pytest.mark.parametrize("i", range(24))
def test_activation_side(i):
    T, K, O, N, M = _draw(i)
    x = inputs.student_t_bf16((T, K), 4.0, i)
    w = inputs.normal_bf16((O, K), 0.02, i + 1)
    comp = nm.prune_compress(dev(x), N, M)
    y = nm.sparse_gemm(comp, nm.lift(dev(w), M), nm.NM_ACT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.sparse_operand(x, N, M)
    np.testing.assert_array_equal(host_bits(comp.vals), ref["vals"])
    np.testing.assert_array_equal(host_bits(comp.meta)[:ref["meta"].size], ref["meta"])
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, N, M), f"act {T}x{K}x{O} {N}:{M}")


@pytest.mark.parametrize("i", range(24))
def test_weight_side(i):
    T, K, O, N, M = _draw(i + 100)
    x = inputs.normal_bf16((T, K), 1.0, i)
    w = inputs.normal_bf16((O, K), 0.02, i + 1)
    comp = nm.slide_decompose(dev(w), N, M) if N == M - 2 or (N, M) == (2, 4) else nm.prune_compress(dev(w), N, M)
    xl = nm.lift(dev(x), M)
    y = nm.sparse_gemm(comp, xl, nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.weight_sparse_linear(x, w, N, M), f"weight {T}x{K}x{O} {N}:{M}")


@pytest.mark.parametrize("i", range(12))
def test_hybrid(i):
    rng = np.random.default_rng(2000 + i)
    B = int(rng.choice([1, 5, 16, 33, 64, 100, 130]))
    K = int(512 * rng.integers(1, 5))                 # the 2:4 part a whole number of 128-K blocks
    O = int(rng.choice([64, 128, 200, 256, 512]))
    f = float(rng.choice([0.0, 0.25, 0.5, 1.0]))
    x = inputs.normal_bf16((B, K), 1.0, i)
    w = inputs.normal_bf16((O, K), 0.02, i + 1)
    h = nm.hybrid_prepare(dev(w), f)
    y = nm.hybrid_gemm(dev(x), h, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.hybrid_linear(x, w, f), f"hybrid B={B} K={K} O={O} f={f}")


@pytest.mark.parametrize("i", range(12))
def test_corrections(i):
    T, K, O, N, M = _draw(i + 200)
    flags = [nm.NM_XF_SHIFT, nm.NM_XF_VAR, nm.NM_XF_SHIFT | nm.NM_XF_VAR][i % 3]
    x = inputs.bf16_from_f64(inputs.bf16_to_f64(inputs.student_t_bf16((T, K), 4.0, i)) + 0.5)
    w = inputs.normal_bf16((O, K), 0.02, i + 1)
    W = dev(w)
    Wl, s = nm.lift(W, M), nm.row_sums(W)
    torch.cuda.synchronize()
    X = nm.prune_compress_xf(dev(x), N, M, flags)
    y = nm.sparse_gemm_xf(X, Wl, s, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.act_transform(x, N, M, bool(flags & nm.NM_XF_SHIFT), bool(flags & nm.NM_XF_VAR))
    np.testing.assert_array_equal(host_bits(X.comp.vals), ref["vals"])
    check_close(host_f64(y), oracle.act_sparse_linear_xf(x, w, N, M, bool(flags & nm.NM_XF_SHIFT),
                                                         bool(flags & nm.NM_XF_VAR)), f"xf {T}x{K}x{O} {N}:{M}")


@pytest.mark.parametrize("i", range(12))
def test_fp8_weight_side(i):
    T, K, O, N, M = _draw(i + 300)
    N = M - 2 if M > 4 else 2                          # the 8-bit packer is the (2N-2):2N one
    if nm.lifted_k(K, M) % 128 != 0:
        K = K * 8                                      # K' a multiple of 128
    if T > 64:
        O = 256 * max(1, O // 256)                     # SM-pair shapes need whole 256-row blocks
    x = inputs.student_t_bf16((T, K), 4.0, i)
    w = inputs.normal_bf16((O, K), 0.02, i + 1)
    P = nm.slide_decompose_fp8(dev(w), N, M)
    q = nm.quant_lift_fp8(dev(x), M)
    y = nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, N, M), f"fp8 {T}x{K}x{O} {N}:{M}")


@pytest.mark.parametrize("T,K,O,N,M,side", [
    (40, 131072, 300, 8, 16, "act"),       # 114688 lifted K: 896 k-blocks, split-K on single CTAs
    (256, 65536, 512, 16, 32, "act"),      # 122880 lifted K on SM pairs
    (16, 98304, 256, 6, 8, "weight"),      # 147456 lifted K, decode shape
])
def test_long_reductions(T, K, O, N, M, side):
    """Reductions far beyond the workloads' (up to 147456 lifted K): the
    operand stays bit-exact and the product within tolerance, so no index
    or k-block count overflows on the way."""
    x = inputs.student_t_bf16((T, K), 4.0, T + K)
    w = inputs.normal_bf16((O, K), 0.02, O + K)
    if side == "act":
        comp = nm.prune_compress(dev(x), N, M, with_mask=True)
        y = nm.sparse_gemm(comp, nm.lift(dev(w), M), nm.NM_ACT, torch.float32)
        ref_op, y_ref = oracle.sparse_operand(x, N, M), oracle.act_sparse_linear(x, w, N, M)
    else:
        comp = nm.slide_decompose(dev(w), N, M, with_mask=True)
        y = nm.sparse_gemm(comp, nm.lift(dev(x), M), nm.NM_WEIGHT, torch.float32)
        ref_op, y_ref = oracle.sparse_operand(w, N, M), oracle.weight_sparse_linear(x, w, N, M)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    np.testing.assert_array_equal(host_bits(comp.mask), ref_op["mask"], err_msg="mask")
    np.testing.assert_array_equal(host_bits(comp.vals), ref_op["vals"], err_msg="values")
    np.testing.assert_array_equal(host_bits(comp.meta)[:ref_op["meta"].size], ref_op["meta"], err_msg="metadata")
    check_close(host_f64(y), y_ref, f"K={K} {N}:{M} {side}")
