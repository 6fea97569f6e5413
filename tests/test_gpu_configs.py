"""Every workload at its full size, through the same calls and launch
configuration bench.py times, checked against the oracle over the whole
result: the compressed operand (values and metadata image, every 128-row
block) bit-exact, and every output element within the stated tolerance."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def check_operand(comp, ref):
    """The whole compressed operand against the oracle's, one 128-row block at
    a time (values, then that block's metadata blocks), so that a mismatch
    names its block."""
    vals = host_bits(comp.vals)
    meta = host_bits(comp.meta)
    rows = vals.shape[0]
    KB = -(-ref["K_lift"] // 128)
    assert meta.size >= ref["meta"].size
    for rb in range(-(-rows // 128)):
        r0, r1 = 128 * rb, min(128 * rb + 128, rows)
        np.testing.assert_array_equal(vals[r0:r1], ref["vals"][r0:r1], err_msg=f"values, row block {rb}")
        b0, b1 = rb * KB * 2048, (rb + 1) * KB * 2048
        np.testing.assert_array_equal(meta[b0:b1], ref["meta"][b0:b1], err_msg=f"metadata image, row block {rb}")


def check_rows(y, y_ref, what, chunk=512):
    """Every output row within tolerance, in row chunks (a failure names its rows)."""
    y = host_f64(y)
    assert y.shape == y_ref.shape
    for r0 in range(0, y.shape[0], chunk):
        check_close(y[r0:r0 + chunk], y_ref[r0:r0 + chunk], f"{what}, rows {r0}..{min(r0 + chunk, y.shape[0]) - 1}")


@pytest.mark.parametrize("name", ["up_proj_8of16_act", "up_proj_2of4_act", "down_proj_16of32_act"])
def test_activation_sparse_full_size(name):
    wl, x, w = inputs.make_workload(name)
    comp = nm.prune_compress(dev(x), wl.N, wl.M)
    y = nm.sparse_gemm(comp, nm.lift(dev(w), wl.M), nm.NM_ACT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.sparse_operand(x, wl.N, wl.M)
    check_operand(comp, ref)
    y_ref = oracle.linear_f64(oracle.to_f64(x, ref["keep"]), oracle.to_f64(w))
    check_rows(y, y_ref, name)


@pytest.mark.parametrize("name", ["slide_6of8_wt_prefill", "slide_6of8_wt_decode"])
def test_weight_sparse_full_size(name):
    wl, x, w = inputs.make_workload(name)
    comp = nm.slide_decompose(dev(w), wl.N, wl.M)
    xd = dev(x)
    y = nm.sparse_gemm(comp, nm.lift(xd, wl.M), nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.sparse_operand(w, wl.N, wl.M)
    check_operand(comp, ref)
    y_ref = oracle.linear_f64(oracle.to_f64(x), oracle.to_f64(w, ref["keep"]))
    check_rows(y, y_ref, name)
    if name.endswith("decode"):
        # the step's one-launch form (the lift inside the GEMM) on the same inputs
        y1 = nm.slide_gemm(comp, xd, torch.bfloat16)
        torch.cuda.synchronize()
        assert nm.device_error() == nm.NM_OK
        check_rows(y1, y_ref, name + " (slide_gemm)")


@pytest.mark.parametrize("B", [1, 8, 32, 128])
def test_hybrid_decode_full_size(B):
    wl, x, w = inputs.make_workload(f"hybrid_decode_b{B}")
    h = nm.hybrid_prepare(dev(w), wl.dense_frac)
    y = nm.hybrid_gemm(dev(x), h, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.hybrid_weight(w, wl.dense_frac)
    np.testing.assert_array_equal(h.perm.cpu().numpy(), ref["perm"])
    np.testing.assert_array_equal(host_bits(h.W_d), ref["W_d"])
    np.testing.assert_array_equal(host_bits(h.vals_s), ref["vals_s"])
    np.testing.assert_array_equal(host_bits(h.meta_s)[:ref["meta_s"].size], ref["meta_s"])
    check_close(host_f64(y), oracle.linear_f64(oracle.to_f64(x), oracle.to_f64(w, ref["keep_full"])),
                f"hybrid b{B}")


def test_tiny_fp32_full_size():
    wl, x, w = inputs.make_workload("tiny_2of4_act_fp32")
    comp = nm.prune_compress(dev(x), wl.N, wl.M, with_mask=True)
    y = nm.sparse_gemm(comp, nm.lift(dev(w), wl.M), nm.NM_ACT, torch.float32)
    torch.cuda.synchronize()
    ref = oracle.sparse_operand(x, wl.N, wl.M)
    np.testing.assert_array_equal(host_bits(comp.mask), ref["mask"])
    np.testing.assert_array_equal(host_bits(comp.vals), ref["vals"])
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, wl.N, wl.M), "tiny")


@pytest.mark.parametrize("B", [1, 128])
def test_spense_mlp_decode_full_size(B):
    """The GLU-MLP decode workloads (d = 4096, I = 14336, a quarter of the
    intermediate indices dense) through the calls bench.py times: the packed
    weights bit-exact, every output row within tolerance."""
    wl, x, wu = inputs.make_workload(f"spense_mlp_decode_b{B}")
    _, wg, wd = inputs.make_mlp_weights(wl)
    W = nm.spense_mlp_prepare(dev(wu), dev(wg), dev(wd), wl.dense_frac)
    ws = torch.empty(max(16, nm.spense_mlp_workspace_size(W, wl.T)), dtype=torch.uint8, device="cuda")
    y = nm.spense_mlp(dev(x), W, ws=ws)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.spense_mlp_weights(wu, wg, wd, wl.dense_frac)
    np.testing.assert_array_equal(W.perm.cpu().numpy(), ref["perm"])
    np.testing.assert_array_equal(host_bits(W.ug_vals), ref["ug_vals"])
    np.testing.assert_array_equal(host_bits(W.ug_dense), ref["ug_dense"])
    np.testing.assert_array_equal(host_bits(W.down_vals), ref["down_vals"])
    np.testing.assert_array_equal(host_bits(W.down_dense), ref["down_dense"])
    check_close(host_f64(y), oracle.spense_mlp(x, wu, wg, wd, wl.dense_frac), f"spense mlp b{B}")
