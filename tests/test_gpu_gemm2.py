"""The persistent 2-CTA sparse GEMM (256-row tiles on SM pairs) vs the fp64
oracle, each tile variant pinned through NMSPARSE_GEMM: exact on integers and
one-hot weights, within tolerance on random data; more tiles than clusters so
that the accumulator buffers and barrier phases are reused."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_f64

pytestmark = pytest.mark.gpu

VARIANTS = ["2cta224", "2cta192", "2cta256", "2cta128", "2cta224x2", "2cta192x2", "2cta160x2", "2cta128x2"]


def _int_bf16(rng, shape, lo=-4, hi=5):
    return inputs.bf16_from_f64(rng.integers(lo, hi, size=shape).astype(np.float64))


def _act(x, w, N, M, out_dtype):
    comp = nm.prune_compress(dev(x), N, M)
    return nm.sparse_gemm(comp, nm.lift(dev(w), M), nm.NM_ACT, out_dtype)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("N,M", [(2, 4), (8, 16)])
def test_integers_exact(variant, N, M, monkeypatch):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    rng = np.random.default_rng(11)
    T, O, K = 512, 1000, 1024          # partial last column tile for every variant
    x = _int_bf16(rng, (T, K))
    w = _int_bf16(rng, (O, K))
    y = _act(x, w, N, M, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.act_sparse_linear(x, w, N, M))
    assert nm.device_error() == nm.NM_OK


@pytest.mark.parametrize("variant", VARIANTS)
def test_one_hot(variant, monkeypatch):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    K = 512
    x = inputs.normal_bf16((256, K), 1.0, seed=3)
    w = inputs.bf16_from_f64(np.eye(K))
    y = _act(x, w, 6, 8, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.to_f64(x, oracle.prune(x, 6, 8)))


@pytest.mark.parametrize("variant", VARIANTS + ["auto"])
def test_many_tiles_per_cluster(variant, monkeypatch):
    """2048 x 4096 output: more tiles than SM pairs, every row checked."""
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    T, O, K = 2048, 4096, 512
    x = inputs.student_t_bf16((T, K), 4.0, seed=5)
    w = inputs.normal_bf16((O, K), 0.02, seed=6)
    y = _act(x, w, 2, 4, torch.bfloat16)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, 2, 4), variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_weight_side_transposed(variant, monkeypatch):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    T, O, K = 600, 512, 1024
    x = inputs.normal_bf16((T, K), 1.0, seed=8)
    w = inputs.normal_bf16((O, K), 0.02, seed=9)
    comp = nm.prune_compress(dev(w), 6, 8)
    y = nm.sparse_gemm(comp, nm.lift(dev(x), 8), nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.weight_sparse_linear(x, w, 6, 8), variant)


def test_partial_last_k_block(monkeypatch):
    monkeypatch.setenv("NMSPARSE_GEMM", "2cta224")
    T, O, K = 256, 700, 192              # 6:8 -> K' = 288: 2.25 k-blocks
    rng = np.random.default_rng(3)
    x = _int_bf16(rng, (T, K))
    w = _int_bf16(rng, (O, K))
    y = _act(x, w, 6, 8, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.act_sparse_linear(x, w, 6, 8))


@pytest.mark.parametrize("B", [64, 128, 200])
def test_hybrid_on_sm_pairs(B):
    """Hybrid input-split with sparse and dense k-blocks in the 2-CTA kernel
    (weight rows a multiple of 256, 64 or more tokens): exact on integers."""
    rng = np.random.default_rng(B)
    O, K = 512, 1024
    w = _int_bf16(rng, (O, K))
    x = _int_bf16(rng, (B, K))
    h = nm.hybrid_prepare(dev(w), 0.25)
    y = nm.hybrid_gemm(dev(x), h, torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.hybrid_linear(x, w, 0.25))


def test_hybrid_on_sm_pairs_random_bf16():
    O, K, B = 1024, 2048, 128
    w = inputs.normal_bf16((O, K), 0.02, seed=3)
    x = inputs.normal_bf16((B, K), 1.0, seed=4)
    h = nm.hybrid_prepare(dev(w), 0.25)
    y = nm.hybrid_gemm(dev(x), h, torch.bfloat16)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.hybrid_linear(x, w, 0.25), "hybrid pairs")


@pytest.mark.parametrize("rows_b", [96, 700])
def test_dense_comparator_on_sm_pairs(rows_b):
    rng = np.random.default_rng(rows_b)
    a = _int_bf16(rng, (512, 640))
    b = _int_bf16(rng, (rows_b, 640))
    y = nm.dense_gemm(dev(a), dev(b), torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.linear_f64(oracle.to_f64(a), oracle.to_f64(b)))
