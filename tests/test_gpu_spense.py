"""The GLU-MLP mapping of the hybrid format on the GPU against the oracle:
the prepared weights bit-exact (permutation, packed up/gate rows, packed down
columns, dense blocks), the MLP output within tolerance."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _weights(I, d, seed):
    wu = inputs.normal_bf16((I, d), 0.02, seed)
    wg = inputs.normal_bf16((I, d), 0.02, seed + 1)
    wd = inputs.normal_bf16((d, I), 0.02, seed + 2)
    return wu, wg, wd


@pytest.mark.parametrize("I,d,frac", [(1024, 256, 0.25), (512, 384, 0.5), (768, 128, 0.0), (512, 256, 1.0)])
def test_prepare_bit_exact(I, d, frac):
    wu, wg, wd = _weights(I, d, I + d)
    W = nm.spense_mlp_prepare(dev(wu), dev(wg), dev(wd), frac)
    torch.cuda.synchronize()
    ref = oracle.spense_mlp_weights(wu, wg, wd, frac)
    assert W.D == ref["D"]
    np.testing.assert_array_equal(W.perm.cpu().numpy(), ref["perm"])
    if ref["Is"] > 0:
        np.testing.assert_array_equal(host_bits(W.ug_vals), ref["ug_vals"], err_msg="up/gate values")
        np.testing.assert_array_equal(host_bits(W.ug_meta)[:ref["ug_meta"].size], ref["ug_meta"])
        np.testing.assert_array_equal(host_bits(W.down_vals), ref["down_vals"], err_msg="down values")
        np.testing.assert_array_equal(host_bits(W.down_meta)[:ref["down_meta"].size], ref["down_meta"])
    if ref["D"] > 0:
        np.testing.assert_array_equal(host_bits(W.ug_dense), ref["ug_dense"], err_msg="up/gate dense rows")
        np.testing.assert_array_equal(host_bits(W.down_dense), ref["down_dense"], err_msg="down dense columns")


@pytest.mark.parametrize("B,I,d,frac", [(1, 1024, 256, 0.25), (8, 1024, 256, 0.25), (40, 512, 384, 0.5),
                                        (130, 768, 256, 0.0), (16, 512, 256, 1.0)])
def test_mlp_matches_the_oracle(B, I, d, frac):
    wu, wg, wd = _weights(I, d, 7 * I + d)
    x = inputs.normal_bf16((B, d), 1.0, B)
    W = nm.spense_mlp_prepare(dev(wu), dev(wg), dev(wd), frac)
    y = nm.spense_mlp(dev(x), W)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.spense_mlp(x, wu, wg, wd, frac), f"mlp B={B} I={I} d={d} f={frac}")


def test_mlp_full_size_decode():
    """Llama-8B MLP shape (d = 4096, I = 14336), a quarter of the intermediate
    indices dense, batch 8."""
    I, d = 14336, 4096
    wu, wg, wd = _weights(I, d, 3)
    x = inputs.normal_bf16((8, d), 1.0, 4)
    W = nm.spense_mlp_prepare(dev(wu), dev(wg), dev(wd), 0.25)
    y = nm.spense_mlp(dev(x), W)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK and W.D == 3584
    check_close(host_f64(y), oracle.spense_mlp(x, wu, wg, wd, 0.25), "mlp full size")


@pytest.mark.parametrize("variant", ["1cta", "2cta128", "2cta224"])
@pytest.mark.parametrize("B,I,d,frac", [(40, 1024, 256, 0.25), (130, 1024, 384, 0.5), (72, 768, 256, 0.0),
                                        (96, 512, 256, 1.0)])
def test_mlp_every_gemm_variant(monkeypatch, variant, B, I, d, frac):
    """The output-split up/gate product and the input-split down product on
    each GEMM kernel: single CTAs (128-row tiles, split-K) and SM pairs
    (256-row tiles; dense tiles scheduled first)."""
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    wu, wg, wd = _weights(I, d, 5 * I + d + B)
    x = inputs.normal_bf16((B, d), 1.0, B + 1)
    W = nm.spense_mlp_prepare(dev(wu), dev(wg), dev(wd), frac)
    y = nm.spense_mlp(dev(x), W)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(y), oracle.spense_mlp(x, wu, wg, wd, frac), f"mlp {variant} B={B} I={I} d={d} f={frac}")
