"""The split window order on the GPU: slide_decompose_split() and
nm_lift_odd() bit-exact against the oracle's reordering, and the product of
the two through nm_sparse_gemm() against the pruned product (exact on
integers, within tolerance on random data, equal to the natural order on
integers), on SM-pair and single-CTA shapes."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,K,N,M", [
    (260, 1024, 6, 8),      # whole 512-element chunks
    (130, 768, 6, 8),       # a last chunk of 32 of 64 groups: its even blocks stop at K/128
    (5, 1152, 6, 8),
    (200, 1280, 14, 16),
    (64, 3072, 30, 32),
    (4096, 4096, 6, 8),     # the 6:8 prefill weight
])
def test_decompose_split_bit_exact(rows, K, N, M):
    w = inputs.normal_bf16((rows, K), 0.02, rows + K)
    comp = nm.slide_decompose_split(dev(w), N, M, with_mask=True)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.sparse_operand_split(w, N, M)
    np.testing.assert_array_equal(host_bits(comp.mask), ref["mask"], err_msg="mask")
    np.testing.assert_array_equal(host_bits(comp.vals), ref["vals"], err_msg="values")
    np.testing.assert_array_equal(host_bits(comp.meta)[:ref["meta"].size], ref["meta"], err_msg="metadata image")


@pytest.mark.parametrize("rows,K,M,extra", [(37, 1024, 8, 0), (16, 4096, 8, 0), (300, 1280, 16, 8), (9, 2048, 32, 24)])
def test_lift_odd_in_place(rows, K, M, extra):
    x = inputs.normal_bf16((rows, K), 1.0, rows + K + M)
    Kl = nm.lifted_k(K, M)
    wide = torch.full((rows, Kl + extra), -7.0, dtype=torch.bfloat16, device="cuda")
    wide[:, :K] = dev(x)
    out = nm.lift_odd(wide, K, M)
    torch.cuda.synchronize()
    assert out.shape == (rows, Kl)
    np.testing.assert_array_equal(host_bits(wide[:, :Kl]), oracle.lift_split(x, M))
    if extra:
        assert torch.all(wide[:, Kl:] == -7.0), "columns past K' untouched"


def _split_product(w, x, N, M, out_dtype):
    Wc = nm.slide_decompose_split(dev(w), N, M)
    T, K = x.shape
    wide = torch.empty((T, nm.lifted_k(K, M)), dtype=torch.bfloat16, device="cuda")
    wide[:, :K] = dev(x)
    D = nm.lift_odd(wide, K, M)
    return nm.sparse_gemm(Wc, D, nm.NM_WEIGHT, out_dtype)


@pytest.mark.parametrize("T,K,O,N,M", [(512, 1024, 512, 6, 8), (16, 4096, 256, 6, 8), (256, 1280, 768, 14, 16),
                                       (40, 2048, 384, 30, 32)])
def test_split_product_exact_on_integers(T, K, O, N, M):
    rng = np.random.default_rng(T + K + O)
    w = inputs.bf16_from_f64(rng.integers(-4, 5, size=(O, K)).astype(np.float64))
    x = inputs.bf16_from_f64(rng.integers(-3, 4, size=(T, K)).astype(np.float64))
    y = _split_product(w, x, N, M, torch.float32)
    y_nat = nm.sparse_gemm(nm.slide_decompose(dev(w), N, M), nm.lift(dev(x), M), nm.NM_WEIGHT, torch.float32)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.weight_sparse_linear(x, w, N, M)
    np.testing.assert_array_equal(host_f64(y), ref)
    assert torch.equal(y, y_nat)


@pytest.mark.parametrize("T,K,O,N,M", [(4096, 4096, 4096, 6, 8), (16, 4096, 4096, 6, 8), (300, 2048, 1000, 14, 16)])
def test_split_product_random(T, K, O, N, M):
    x = inputs.normal_bf16((T, K), 1.0, T + 1)
    w = inputs.normal_bf16((O, K), 0.02, O + 2)
    y = _split_product(w, x, N, M, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    rows = np.unique(np.linspace(0, T - 1, min(T, 64)).astype(np.int64))
    y_ref = oracle.weight_sparse_linear(x, w, N, M, rows=rows)
    check_close(inputs.bf16_to_f64(host_bits(y)[rows]), y_ref, f"split {N}:{M} T={T}")
