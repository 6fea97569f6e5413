"""Sparse GEMM on the GPU (tcgen05.mma.sp through the C ABI) vs the fp64 oracle.

Exactness cases first (one-hot and small integers, where fp32 accumulation is
exact and any metadata / layout error shows as a wrong value), then random
data within the stated tolerance, over ragged shapes that span several tiles.
"""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_f64

pytestmark = pytest.mark.gpu


def _int_bf16(rng, shape, lo=-4, hi=5):
    return inputs.bf16_from_f64(rng.integers(lo, hi, size=shape).astype(np.float64))


def act_path(x, w, N, M, out_dtype=torch.float32):
    comp = nm.prune_compress(dev(x), N, M)
    wl = nm.lift(dev(w), M)
    return nm.sparse_gemm(comp, wl, nm.NM_ACT, out_dtype)


def weight_path(x, w, N, M, out_dtype=torch.float32):
    comp = nm.prune_compress(dev(w), N, M)
    xl = nm.lift(dev(x), M)
    return nm.sparse_gemm(comp, xl, nm.NM_WEIGHT, out_dtype)


@pytest.mark.parametrize("N,M", [(2, 4), (1, 4), (6, 8), (8, 16), (16, 32)])
def test_one_hot_weight_gathers_pruned_x(N, M):
    """W = identity: Y must equal X (.) mask exactly, position by position."""
    K = 256
    x = inputs.normal_bf16((200, K), 1.0, seed=M)
    w = inputs.bf16_from_f64(np.eye(K))
    y = act_path(x, w, N, M)
    torch.cuda.synchronize()
    expect = oracle.to_f64(x, oracle.prune(x, N, M))
    np.testing.assert_array_equal(host_f64(y), expect)


@pytest.mark.parametrize("N,M", [(2, 4), (6, 8), (8, 16), (16, 32), (3, 8)])
@pytest.mark.parametrize("side", ["act", "weight"])
def test_integer_inputs_exact(N, M, side):
    rng = np.random.default_rng(N * 100 + M)
    T, O, K = 150, 200, 1024
    x = _int_bf16(rng, (T, K))
    w = _int_bf16(rng, (O, K))
    if side == "act":
        y = act_path(x, w, N, M)
        ref = oracle.act_sparse_linear(x, w, N, M)
    else:
        y = weight_path(x, w, N, M)
        ref = oracle.weight_sparse_linear(x, w, N, M)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), ref)


ACT_SHAPES = [
    # (T, O, K, N, M)
    (1, 64, 256, 2, 4),
    (3, 16, 512, 8, 16),
    (127, 300, 512, 2, 4),
    (129, 136, 640, 8, 16),
    (256, 512, 1024, 16, 32),
    (300, 40, 192, 6, 8),      # K' = 288: a partial last k-block
    (64, 24, 256, 2, 4),       # O below one column tile
    (128, 32, 4096, 2, 4),     # one 128 x 32 tile, split-K over a cluster of 8
    (200, 16, 1024, 8, 16),    # split-K of 2 with a ragged row tile
]


@pytest.mark.parametrize("T,O,K,N,M", ACT_SHAPES)
@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_act_sparse_random(T, O, K, N, M, out):
    x = inputs.student_t_bf16((T, K), 4.0, seed=T)
    w = inputs.normal_bf16((O, K), 0.02, seed=O)
    y = act_path(x, w, N, M, torch.bfloat16 if out == "bf16" else torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, N, M), f"act {T}x{O}x{K} {N}:{M}")


WEIGHT_SHAPES = [
    # (T, O, K, N, M) -- T is the MMA N dimension; small T takes the split-K path
    (16, 512, 1024, 6, 8),
    (1, 384, 2048, 6, 8),
    (8, 256, 4096, 2, 4),
    (40, 130, 512, 14, 16),
    (300, 256, 512, 6, 8),
    (32, 256, 2048, 6, 8),     # 32-column tiles, split-K of 4
    (16, 1024, 4096, 6, 8),    # split-K of 8
]


@pytest.mark.parametrize("T,O,K,N,M", WEIGHT_SHAPES)
def test_weight_sparse_random(T, O, K, N, M):
    x = inputs.normal_bf16((T, K), 1.0, seed=T + 7)
    w = inputs.normal_bf16((O, K), 0.02, seed=O + 7)
    y = weight_path(x, w, N, M, torch.bfloat16)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.weight_sparse_linear(x, w, N, M), f"weight {T}x{O}x{K} {N}:{M}")


def test_fp32_tiny_workload():
    """The tiny 2:4 fp32 workload: X fp32 [16 x 256] pruned on fp32 keys,
    survivors and W rounded to bf16 for the tensor cores, fp32 output."""
    wl, x, w = inputs.make_workload("tiny_2of4_act_fp32")
    y = act_path(x, w, wl.N, wl.M, torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, wl.N, wl.M), "tiny fp32")


@pytest.mark.parametrize("A_rows,B_rows,K", [(256, 256, 512), (100, 72, 1024), (16, 300, 64)])
def test_dense_comparator(A_rows, B_rows, K):
    a = inputs.normal_bf16((A_rows, K), 1.0, 1)
    b = inputs.normal_bf16((B_rows, K), 0.02, 2)
    y = nm.dense_gemm(dev(a), dev(b), torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.linear_f64(oracle.to_f64(a), oracle.to_f64(b)), "dense")


def test_dense_comparator_integers_exact():
    rng = np.random.default_rng(4)
    a = _int_bf16(rng, (130, 512))
    b = _int_bf16(rng, (70, 512))
    y = nm.dense_gemm(dev(a), dev(b), torch.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_f64(y), oracle.linear_f64(oracle.to_f64(a), oracle.to_f64(b)))


def test_repeat_calls_are_deterministic():
    x = inputs.normal_bf16((16, 2048), 1.0, 5)
    w = inputs.normal_bf16((512, 2048), 0.02, 6)
    y1 = weight_path(x, w, 6, 8)
    y2 = weight_path(x, w, 6, 8)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert nm.device_error() == nm.NM_OK
