"""The 8-bit (E4M3) path on the GPU against the oracle: quantise + lift and
the weight packing bit-exact (codes, scales, 8-bit metadata image), the
rescaled sparse product within tolerance, exactly on integer grids."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _x(rows, K, kind, seed):
    if kind == "fp32":
        return np.random.default_rng(seed).standard_normal((rows, K)).astype(np.float32) * 3
    if kind == "student_t":
        return inputs.student_t_bf16((rows, K), 4.0, seed)
    if kind == "outliers":
        return inputs.normal_with_outlier_channels_bf16((rows, K), 0.01, 20.0, seed)
    if kind == "zero_rows":
        x = inputs.normal_bf16((rows, K), 1.0, seed)
        x[::3] = 0
        return x
    vals = np.array([-448.0, -2.0, -1e-3, -0.0, 0.0, 3e-6, 1.0, 2.0, 300.0])     # ties and extremes
    return inputs.bf16_from_f64(vals[np.random.default_rng(seed).integers(0, vals.size, size=(rows, K))])


@pytest.mark.parametrize("rows,K,M,kind", [
    (17, 256, 8, "student_t"), (64, 1024, 8, "outliers"), (5, 512, 16, "zero_rows"), (33, 640, 4, "ties"),
    (9, 2048, 32, "student_t"), (12, 768, 8, "fp32"), (130, 4096, 8, "student_t"),
    # group counts that leave lanes partly or wholly idle, and more rows than
    # one pass of the grid (one warp per row, at most eight CTAs per SM)
    (11, 800, 8, "student_t"), (6, 2112, 16, "ties"), (5, 1152, 32, "outliers"), (70, 528, 4, "student_t"),
    (10000, 256, 8, "student_t"), (3, 14336, 16, "fp32"),
])
def test_quant_lift_bit_exact(rows, K, M, kind):
    x = _x(rows, K, kind, rows + K)
    q = nm.quant_lift_fp8(dev(x), M)
    torch.cuda.synchronize()
    ref = oracle.fp8_activation(x, M)
    np.testing.assert_array_equal(host_bits(q.scale), oracle._as_bits(ref["scale"]), err_msg="scales")
    np.testing.assert_array_equal(q.codes.cpu().numpy(), ref["lifted"], err_msg="lifted codes")


@pytest.mark.parametrize("rows,K,N,M", [(256, 1024, 6, 8), (130, 512, 2, 4), (40, 768, 14, 16), (9, 2048, 30, 32)])
def test_weight_packing_bit_exact(rows, K, N, M):
    w = inputs.normal_bf16((rows, K), 0.02, rows + 1)
    P = nm.slide_decompose_fp8(dev(w), N, M)
    torch.cuda.synchronize()
    ref = oracle.fp8_weight(w, N, M)
    np.testing.assert_array_equal(host_bits(P.scale), oracle._as_bits(ref["scale"]), err_msg="scales")
    np.testing.assert_array_equal(P.codes.cpu().numpy(), ref["vals"], err_msg="codes")
    np.testing.assert_array_equal(P.meta.cpu().numpy()[:ref["meta"].size], ref["meta"], err_msg="8-bit metadata")


@pytest.mark.parametrize("T,O,K,N,M", [
    (300, 512, 1024, 6, 8),     # 256-K blocks only
    (40, 256, 768, 6, 8),       # K' = 1152: the last block holds 128 K
    (16, 256, 640, 2, 4),       # 2:4, half last block, a decode-sized T
    (129, 768, 512, 14, 16),
])
def test_fp8_weight_sparse_product(T, O, K, N, M):
    x = inputs.student_t_bf16((T, K), 4.0, seed=T)
    w = inputs.normal_bf16((O, K), 0.02, seed=O)
    P = nm.slide_decompose_fp8(dev(w), N, M)
    q = nm.quant_lift_fp8(dev(x), M)
    y = nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, N, M), f"fp8 {T}x{O}x{K} {N}:{M}")


def test_fp8_product_exact_on_integer_grid():
    """Integer values on the E4M3 grid with every row maximum at 448: both
    scales are 1 and every product and fp32 partial sum is an exact integer."""
    rng = np.random.default_rng(9)
    def make(rows, K):
        v = rng.integers(-16, 17, size=(rows, K)).astype(np.float64)
        v[:, 0] = 448.0
        return inputs.bf16_from_f64(v)
    x, w = make(48, 512), make(256, 512)
    P = nm.slide_decompose_fp8(dev(w), 6, 8)
    q = nm.quant_lift_fp8(dev(x), 8)
    y = nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, 6, 8))


@pytest.mark.parametrize("variant", ["2cta224", "2cta160", "2cta192x2", "2cta160x2", "2cta128x2"])
def test_fp8_tile_variants_exact_on_integer_grid(monkeypatch, variant):
    """Every 8-bit tile variant of the SM-pair kernel, 512-row tiles included,
    on E4M3-grid integers with row maxima 448 (both scales 1): exact, with a
    partial last column tile and more tiles than one round of SM pairs."""
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    rng = np.random.default_rng(17)

    def make(rows, K):
        v = rng.integers(-16, 17, size=(rows, K)).astype(np.float64)
        v[:, 0] = 448.0
        return inputs.bf16_from_f64(v)
    x, w = make(1000, 768), make(1024, 768)
    P = nm.slide_decompose_fp8(dev(w), 6, 8)
    y = nm.sparse_gemm_fp8(P, nm.quant_lift_fp8(dev(x), 8), nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    np.testing.assert_array_equal(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, 6, 8))


def test_fp8_full_size():
    """The 6:8 weight-sparse prefill workload in 8 bits: the packed weight and
    the quantised, lifted activations bit-exact, every output row within
    tolerance."""
    wl, x, w = inputs.make_workload("slide_6of8_wt_prefill")
    P = nm.slide_decompose_fp8(dev(w), wl.N, wl.M)
    q = nm.quant_lift_fp8(dev(x), wl.M)
    y = nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    wref = oracle.fp8_weight(w, wl.N, wl.M)
    np.testing.assert_array_equal(P.codes.cpu().numpy(), wref["vals"], err_msg="weight codes")
    np.testing.assert_array_equal(host_bits(P.scale), oracle._as_bits(wref["scale"]), err_msg="weight scales")
    np.testing.assert_array_equal(P.meta.cpu().numpy()[:wref["meta"].size], wref["meta"], err_msg="8-bit metadata")
    xref = oracle.fp8_activation(x, wl.M)
    np.testing.assert_array_equal(q.codes.cpu().numpy(), xref["lifted"], err_msg="lifted activation codes")
    np.testing.assert_array_equal(host_bits(q.scale), oracle._as_bits(xref["scale"]), err_msg="activation scales")
    y = host_f64(y)
    y_ref = oracle.fp8_weight_sparse_linear(x, w, wl.N, wl.M)
    for r0 in range(0, wl.T, 512):
        check_close(y[r0:r0 + 512], y_ref[r0:r0 + 512], f"fp8 full size, rows {r0}..")


def test_fp8_unsupported_shapes_launch_nothing():
    w_np = inputs.normal_bf16((130, 512), 0.02, 1)
    P = nm.slide_decompose_fp8(dev(w_np), 6, 8)              # packing works for any row count
    q = nm.quant_lift_fp8(dev(inputs.normal_bf16((100, 512), 1.0, 2)), 8)
    with pytest.raises(nm.NmError) as e:
        nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT)                # 100 tokens: SM pairs, whole 256-row blocks
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    # a decode shape (8 tokens) runs on single CTAs, which take the 130 rows
    x8 = inputs.normal_bf16((8, 512), 1.0, 2)
    y = nm.sparse_gemm_fp8(P, nm.quant_lift_fp8(dev(x8), 8), nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.fp8_weight_sparse_linear(x8, w_np, 6, 8), "fp8 130 rows, 8 tokens")
    with pytest.raises(nm.NmError) as e:
        nm.quant_lift_fp8(dev(inputs.normal_bf16((4, 40), 1.0, 3)), 8)   # K' = 60: not a multiple of 16
    assert e.value.status == nm.NM_ERR_UNSUPPORTED


# ------------------------------------------------ activation side (quantise + prune)


@pytest.mark.parametrize("rows,K,N,M,kind", [
    (130, 1024, 8, 16, "student_t"), (40, 640, 2, 4, "ties"), (64, 2048, 16, 32, "outliers"),
    (33, 512, 4, 8, "zero_rows"), (256, 4096, 8, 16, "student_t"),
])
def test_prune_compress_fp8_bit_exact(rows, K, N, M, kind):
    x = _x(rows, K, kind, rows + K)
    P = nm.prune_compress_fp8(dev(x), N, M, with_mask=True)
    torch.cuda.synchronize()
    ref = oracle.fp8_act_operand(x, N, M)
    np.testing.assert_array_equal(host_bits(P.scale), oracle._as_bits(ref["scale"]), err_msg="scales")
    np.testing.assert_array_equal(host_bits(P.mask), ref["mask"], err_msg="mask")
    np.testing.assert_array_equal(P.codes.cpu().numpy(), ref["vals"], err_msg="codes")
    np.testing.assert_array_equal(P.meta.cpu().numpy()[:ref["meta"].size], ref["meta"], err_msg="8-bit metadata")


@pytest.mark.parametrize("T,O,K,N,M", [(256, 384, 1024, 8, 16), (512, 136, 512, 2, 4), (256, 200, 2048, 16, 32)])
def test_fp8_act_sparse_product(T, O, K, N, M):
    x = inputs.student_t_bf16((T, K), 4.0, seed=T + 3)
    w = inputs.normal_bf16((O, K), 0.02, seed=O + 3)
    P = nm.prune_compress_fp8(dev(x), N, M)
    Wq = nm.quant_lift_fp8(dev(w), M)                       # per output channel, lifted
    y = nm.sparse_gemm_fp8(P, Wq, nm.NM_ACT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.fp8_act_sparse_linear(x, w, N, M), f"fp8 act {T}x{O}x{K} {N}:{M}")


def test_fp8_act_full_size():
    """The 8:16 up_proj workload in 8 bits: the quantised, pruned activation
    operand bit-exact, every output row within tolerance."""
    wl, x, w = inputs.make_workload("up_proj_8of16_act")
    P = nm.prune_compress_fp8(dev(x), wl.N, wl.M)
    Wq = nm.quant_lift_fp8(dev(w), wl.M)
    y = nm.sparse_gemm_fp8(P, Wq, nm.NM_ACT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.fp8_act_operand(x, wl.N, wl.M)
    np.testing.assert_array_equal(host_bits(P.scale), oracle._as_bits(ref["scale"]), err_msg="scales")
    np.testing.assert_array_equal(P.codes.cpu().numpy(), ref["vals"], err_msg="codes")
    np.testing.assert_array_equal(P.meta.cpu().numpy()[:ref["meta"].size], ref["meta"], err_msg="8-bit metadata")
    y = host_f64(y)
    y_ref = oracle.fp8_act_sparse_linear(x, w, wl.N, wl.M)
    for r0 in range(0, wl.T, 512):
        check_close(y[r0:r0 + 512], y_ref[r0:r0 + 512], f"fp8 act full size, rows {r0}..")


# ------------------------------------------------ decode shapes (single-CTA kernel)


@pytest.mark.parametrize("variant", ["auto", "1cta"])
@pytest.mark.parametrize("T,O,K,N,M", [
    (1, 256, 1024, 6, 8),       # one token
    (16, 512, 768, 6, 8),       # K' = 1152: the last block holds 128 K
    (33, 384, 2048, 14, 16),
    (64, 256, 640, 2, 4),       # 2:4, half last block
    (200, 256, 1024, 30, 32),   # wider than a decode tile: 1cta only when forced
])
def test_fp8_weight_sparse_single_cta(monkeypatch, variant, T, O, K, N, M):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    x = inputs.student_t_bf16((T, K), 4.0, seed=T + 11)
    w = inputs.normal_bf16((O, K), 0.02, seed=O + 11)
    P = nm.slide_decompose_fp8(dev(w), N, M)
    q = nm.quant_lift_fp8(dev(x), M)
    for out_dt in (torch.float32, torch.bfloat16):
        y = nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, out_dt)
        torch.cuda.synchronize()
        assert nm.device_error() == nm.NM_OK
        check_close(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, N, M), f"fp8 1cta {T}x{O}x{K} {N}:{M}")


def test_fp8_act_sparse_single_cta(monkeypatch):
    monkeypatch.setenv("NMSPARSE_GEMM", "1cta")
    T, O, K, N, M = 256, 200, 1024, 8, 16
    x = inputs.student_t_bf16((T, K), 4.0, seed=5)
    w = inputs.normal_bf16((O, K), 0.02, seed=6)
    P = nm.prune_compress_fp8(dev(x), N, M)
    y = nm.sparse_gemm_fp8(P, nm.quant_lift_fp8(dev(w), M), nm.NM_ACT, torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.fp8_act_sparse_linear(x, w, N, M), "fp8 act 1cta")


def test_fp8_single_cta_exact_on_integer_grid():
    rng = np.random.default_rng(19)

    def make(rows, K):
        v = rng.integers(-16, 17, size=(rows, K)).astype(np.float64)
        v[:, 0] = 448.0
        return inputs.bf16_from_f64(v)
    x, w = make(16, 1536), make(512, 1536)
    P = nm.slide_decompose_fp8(dev(w), 6, 8)
    y = nm.sparse_gemm_fp8(P, nm.quant_lift_fp8(dev(x), 8), nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, 6, 8))


def test_fp8_decode_full_size():
    """The 6:8 weight-sparse decode workload (T = 16, K = O = 4096) in 8 bits,
    every output against the oracle."""
    wl, x, w = inputs.make_workload("slide_6of8_wt_decode")
    P = nm.slide_decompose_fp8(dev(w), wl.N, wl.M)
    y = nm.sparse_gemm_fp8(P, nm.quant_lift_fp8(dev(x), wl.M), nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.fp8_weight_sparse_linear(x, w, wl.N, wl.M), "fp8 decode full size")
