"""Hybrid dense + 2:4 weight on the GPU vs the oracle: selection and packing
bit-exact, the input-split product within tolerance (exact on integers)."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("O,K,frac", [(300, 512, 0.25), (128, 1024, 0.5), (64, 256, 0.0), (200, 384, 1.0),
                                      (257, 640, 0.2)])
def test_prepare_bit_exact(O, K, frac):
    w = inputs.normal_bf16((O, K), 0.02, seed=O)
    D = oracle.hybrid_dense_count(K, frac)
    if (K - D) % 128 != 0:
        pytest.skip("sparse share not a whole number of 128-column blocks")
    h = nm.hybrid_prepare(dev(w), frac)
    ref = oracle.hybrid_weight(w, frac)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h.perm.cpu().numpy(), ref["perm"])
    if D:
        np.testing.assert_array_equal(host_bits(h.W_d), ref["W_d"])
    if K - D:
        np.testing.assert_array_equal(host_bits(h.vals_s), ref["vals_s"])
        np.testing.assert_array_equal(host_bits(h.meta_s)[:ref["meta_s"].size], ref["meta_s"])


def test_prepare_ties_go_to_lower_column():
    rng = np.random.default_rng(2)
    w = inputs.bf16_from_f64(rng.integers(-2, 3, size=(64, 512)).astype(np.float64))
    h = nm.hybrid_prepare(dev(w), 0.25)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h.perm.cpu().numpy(), oracle.hybrid_weight(w, 0.25)["perm"])


@pytest.mark.parametrize("B", [1, 8, 32, 128, 3])
def test_hybrid_gemm_random(B):
    O, K = 640, 1024
    w = inputs.normal_bf16((O, K), 0.02, seed=1)
    x = inputs.normal_bf16((B, K), 1.0, seed=B)
    h = nm.hybrid_prepare(dev(w), 0.25)
    y = nm.hybrid_gemm(dev(x), h, torch.bfloat16)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.hybrid_linear(x, w, 0.25), f"hybrid B={B}")


@pytest.mark.parametrize("frac", [0.0, 0.25, 1.0])
def test_hybrid_gemm_integers_exact(frac):
    rng = np.random.default_rng(7)
    O, K, B = 256, 512, 16
    w = inputs.bf16_from_f64(rng.integers(-4, 5, size=(O, K)).astype(np.float64))
    x = inputs.bf16_from_f64(rng.integers(-4, 5, size=(B, K)).astype(np.float64))
    h = nm.hybrid_prepare(dev(w), frac)
    y = nm.hybrid_gemm(dev(x), h, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.hybrid_linear(x, w, frac))
