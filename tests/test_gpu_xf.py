"""The per-token corrections around the activation prune (D-PTS shift, VAR
rescale) on the GPU against the oracle: shift bit-exact, the shifted
operand's mask, values and metadata bit-exact, the VAR factor within 2 ulp,
the weight's row sums bit-exact, products within tolerance (exact on
integers)."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu

SHIFT, VAR = nm.NM_XF_SHIFT, nm.NM_XF_VAR
FLAGS = [SHIFT, VAR, SHIFT | VAR]


def _x(rows, K, seed, offset=0.75):
    """Student-t tokens moved off centre, so that the shift matters."""
    x = inputs.bf16_to_f64(inputs.student_t_bf16((rows, K), 4.0, seed))
    return inputs.bf16_from_f64(x + offset * np.sign(np.sin(np.arange(rows) + seed))[:, None])


def _check_operand(X, x, N, M, flags):
    ref = oracle.act_transform(x, N, M, bool(flags & SHIFT), bool(flags & VAR))
    np.testing.assert_array_equal(host_bits(X.row_shift), ref["mu32"].view(np.uint32), err_msg="shift")
    np.testing.assert_array_equal(host_bits(X.comp.mask), ref["mask"], err_msg="mask")
    np.testing.assert_array_equal(host_bits(X.comp.vals), ref["vals"], err_msg="values")
    np.testing.assert_array_equal(host_bits(X.comp.meta)[:ref["meta"].size], ref["meta"], err_msg="metadata")
    a = X.row_scale.cpu().numpy()
    ulp = np.spacing(ref["alpha32"])
    assert (np.abs(a - ref["alpha32"]) <= 2 * ulp).all(), "VAR factor"
    return ref


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("rows,K,N,M", [(200, 512, 2, 4), (37, 256, 4, 8), (130, 1024, 8, 16), (64, 4096, 8, 16),
                                        (48, 1024, 16, 32), (20, 96, 2, 8), (16, 160, 6, 8)])
def test_operand_bit_exact(flags, rows, K, N, M):
    x = _x(rows, K, rows + K)
    X = nm.prune_compress_xf(dev(x), N, M, flags, with_mask=True)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    _check_operand(X, x, N, M, flags)


def test_row_sums_bit_exact():
    # (rows, K, row stride): the last case ends every row in half a 16-byte word
    for O, K, ld in [(300, 4096, 4096), (64, 14336, 14336), (7, 100, 104)]:
        w = inputs.normal_bf16((O, ld), 0.02, O + K)
        s = nm.row_sums(dev(w)[:, :K])
        torch.cuda.synchronize()
        ref = oracle.rowsum_f64(np.ascontiguousarray(w[:, :K])).astype(np.float32)
        np.testing.assert_array_equal(host_bits(s), ref.view(np.uint32))


@pytest.mark.parametrize("variant", ["auto", "1cta", "2cta224", "2cta128"])
@pytest.mark.parametrize("T,K,O,N,M", [(40, 512, 256, 2, 4), (512, 1024, 512, 8, 16), (16, 4096, 128, 8, 16),
                                       (256, 2048, 1024, 16, 32)])
def test_product_matches_the_oracle(monkeypatch, variant, T, K, O, N, M):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    x = _x(T, K, T + O)
    w = inputs.normal_bf16((O, K), 0.02, K + 1)
    W = dev(w)
    for flags in FLAGS:
        X = nm.prune_compress_xf(dev(x), N, M, flags)
        y = nm.sparse_gemm_xf(X, nm.lift(W, M), nm.row_sums(W))
        torch.cuda.synchronize()
        assert nm.device_error() == nm.NM_OK
        ref = oracle.act_sparse_linear_xf(x, w, N, M, bool(flags & SHIFT), bool(flags & VAR))
        check_close(host_f64(y), ref, f"{variant} T={T} K={K} O={O} {N}:{M} flags={flags}")


@pytest.mark.parametrize("variant", ["1cta", "2cta224"])
def test_shift_exact_on_integers(monkeypatch, variant):
    """Integer tokens with integer means and integer weights: the shifted
    token, the products and the add-back are all exact, so the fp32 output
    equals the oracle exactly."""
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    T, K, O = 256, 512, 512
    rng = np.random.default_rng(5)
    v = rng.integers(-6, 7, size=(T, K // 2)).astype(np.float64)
    base = np.concatenate([v, -v], axis=1)[:, rng.permutation(K)]          # every row sums to 0
    x = inputs.bf16_from_f64(base + rng.integers(-3, 4, size=(T, 1)))      # integer means, |x| <= 9
    w = inputs.bf16_from_f64(rng.integers(-3, 4, size=(O, K)).astype(np.float64))
    W = dev(w)
    X = nm.prune_compress_xf(dev(x), 8, 16, SHIFT)
    y = nm.sparse_gemm_xf(X, nm.lift(W, 16), nm.row_sums(W), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.act_sparse_linear_xf(x, w, 8, 16, True, False)
    np.testing.assert_array_equal(host_f64(y), ref)


def test_empty_and_unshifted_calls():
    x = _x(32, 256, 9)
    X = nm.prune_compress_xf(dev(x), 2, 4, VAR)
    torch.cuda.synchronize()
    assert (X.row_shift.cpu().numpy() == 0).all()
    X = nm.prune_compress_xf(dev(x), 2, 4, SHIFT)
    torch.cuda.synchronize()
    assert (X.row_scale.cpu().numpy() == 1).all()
    e = nm.prune_compress_xf(dev(x)[:0], 2, 4, SHIFT | VAR)
    torch.cuda.synchronize()
    assert e.comp.rows == 0


def test_full_size_up_proj():
    """The 8:16 up_proj workload (T = 2048, K = 4096, O = 14336) with both
    corrections, in the launch configuration bench.py times: first and last
    the whole operand bit-exact, every shift and VAR factor, every output
    row within tolerance."""
    wl, x, w = inputs.make_workload("up_proj_8of16_act")
    flags = SHIFT | VAR
    W = dev(w)
    X = nm.prune_compress_xf(dev(x), wl.N, wl.M, flags)
    y = nm.sparse_gemm_xf(X, nm.lift(W, wl.M), nm.row_sums(W))
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.act_transform(x, wl.N, wl.M, True, True)
    np.testing.assert_array_equal(host_bits(X.row_shift), ref["mu32"].view(np.uint32))
    assert (np.abs(X.row_scale.cpu().numpy() - ref["alpha32"]) <= 2 * np.spacing(ref["alpha32"])).all()
    Kl = ref["K_lift"]
    vals = host_bits(X.comp.vals)
    meta = host_bits(X.comp.meta)
    KB = -(-Kl // 128)
    for rb in range(wl.T // 128):
        np.testing.assert_array_equal(vals[128 * rb:128 * rb + 128], ref["vals"][128 * rb:128 * rb + 128],
                                      err_msg=f"values, row block {rb}")
        np.testing.assert_array_equal(meta[rb * KB * 2048:(rb + 1) * KB * 2048],
                                      ref["meta"][rb * KB * 2048:(rb + 1) * KB * 2048],
                                      err_msg=f"metadata, row block {rb}")
    y = host_f64(y)
    y_ref = oracle.act_sparse_linear_xf(x, w, wl.N, wl.M, True, True)
    for r0 in range(0, wl.T, 512):
        check_close(y[r0:r0 + 512], y_ref[r0:r0 + 512], f"up_proj xf, rows {r0}..")
