"""Prune + window-compress and lift on the GPU vs the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import dev, host_bits

pytestmark = pytest.mark.gpu

CASES = [
    # (rows, K, N, M, dist)
    (16, 256, 2, 4, "normal"),
    (37, 512, 1, 4, "ties"),
    (300, 384, 6, 8, "normal"),
    (129, 1024, 8, 16, "student_t"),
    (64, 448, 8, 16, "ties"),
    (200, 1024, 16, 32, "outliers"),
    (5, 64, 30, 32, "ties"),
    (128, 2048, 14, 16, "normal"),
    (3, 96, 0, 8, "normal"),
    # rows whose group count is not a multiple of the groups one lane takes
    (19, 72, 2, 4, "ties"),
    (130, 520, 2, 4, "student_t"),
    (21, 40, 4, 8, "ties"),
    (9, 40, 6, 8, "normal"),
    (50, 1048, 4, 8, "ties"),
    (40, 640, 16, 32, "ties"),
]


def _make(rows, K, dist, seed):
    if dist == "normal":
        return inputs.normal_bf16((rows, K), 1.0, seed)
    if dist == "student_t":
        return inputs.student_t_bf16((rows, K), 4.0, seed)
    if dist == "outliers":
        return inputs.normal_with_outlier_channels_bf16((rows, K), 0.01, 20.0, seed)
    vals = np.array([-2.0, -1.0, -0.0, 0.0, 1.0, 2.0])
    return inputs.bf16_from_f64(vals[np.random.default_rng(seed).integers(0, 6, size=(rows, K))])


def _check_operand(x, N, M, comp):
    ref = oracle.sparse_operand(x, N, M)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(comp.mask), ref["mask"], err_msg="mask")
    np.testing.assert_array_equal(host_bits(comp.vals), ref["vals"], err_msg="values")
    meta = host_bits(comp.meta)[:ref["meta"].size]
    np.testing.assert_array_equal(meta, ref["meta"], err_msg="metadata image")


@pytest.mark.parametrize("rows,K,N,M,dist", CASES)
def test_prune_compress_bit_exact(rows, K, N, M, dist):
    x = _make(rows, K, dist, seed=rows + K)
    comp = nm.prune_compress(dev(x), N, M, with_mask=True)
    _check_operand(x, N, M, comp)


@pytest.mark.parametrize("rows,K,N,M,dist", [
    # several tasks per CTA (persistent grid), a ragged last row group, and a
    # last chunk of each row group that holds 2 of 32 groups, so that whole
    # and partial task rows (bulk-copied and element-copied values) alternate
    # in one CTA's sequence of tasks
    (4100, 14400, 16, 32, "outliers"),
    (2051, 4128, 8, 16, "student_t"),
    (1030, 2112, 3, 8, "ties"),
    # about eleven whole tasks per CTA, each row one bulk-copied chunk
    (100003, 512, 4, 8, "student_t"),
])
def test_prune_many_tasks_ragged(rows, K, N, M, dist):
    x = _make(rows, K, dist, seed=rows + K)
    comp = nm.prune_compress(dev(x), N, M, with_mask=True)
    _check_operand(x, N, M, comp)


def test_prune_fp32_input():
    x = np.random.default_rng(0).standard_normal((16, 256)).astype(np.float32)
    comp = nm.prune_compress(dev(x), 2, 4, with_mask=True)
    _check_operand(x, 2, 4, comp)


def test_prune_strided_rows():
    x = inputs.normal_bf16((70, 512), 1.0, 3)
    xt = dev(x)[:, :256]                       # row stride 512, K = 256
    comp = nm.prune_compress(xt, 8, 16, with_mask=True)
    _check_operand(np.ascontiguousarray(x[:, :256]), 8, 16, comp)


@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (14, 16), (30, 32)])
def test_slide_decompose(N, M):
    w = inputs.normal_bf16((260, 4 * M * 4), 0.02, 9)
    comp = nm.slide_decompose(dev(w), N, M, with_mask=True)
    _check_operand(w, N, M, comp)


@pytest.mark.parametrize("rows,K,M,dt", [(33, 256, 4, "fp32"), (100, 512, 8, "bf16"), (7, 1024, 16, "bf16"),
                                         (64, 1024, 32, "bf16"),
                                         # rows of several 2048-element segments with a partial last one
                                         (5, 4624, 8, "bf16"), (3, 6144, 16, "fp32"), (9, 2112, 32, "bf16"),
                                         # more rows than one grid dimension holds
                                         (70000, 16, 4, "bf16")])
def test_lift_bit_exact(rows, K, M, dt):
    if dt == "fp32":
        x = np.random.default_rng(1).standard_normal((rows, K)).astype(np.float32)
    else:
        x = inputs.normal_bf16((rows, K), 1.0, 2)
    out = nm.lift(dev(x), M)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(out), oracle.lift(x, M))


def test_empty_rows_is_a_no_op():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    comp = nm.prune_compress(x, 2, 4)
    assert comp.vals.shape[0] == 0
