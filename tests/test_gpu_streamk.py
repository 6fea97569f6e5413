"""The split last round of the SM-pair GEMM (stream-K tail): with the
workspace nm_sparse_gemm_workspace_size() reports, a last persistent round
that would leave most SM pairs idle is split along K across them and a second
kernel adds the parts.  Exact on integer inputs (any summation order is exact
there), equal to the unsplit schedule on them, within tolerance of the oracle
on random data, deterministic from call to call."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _int_bf16(rng, shape, lo=-4, hi=5):
    return inputs.bf16_from_f64(rng.integers(lo, hi, size=shape).astype(np.float64))


# (rows of the sparse operand, rows of the dense one, K, N, M, side): tile
# counts a little above one round of 74 SM pairs, so that a short last round
# is split; the weight side stores Y transposed
# (each part keeps at least 16 k-blocks of 128 lifted K)
SHAPES = [
    (2560, 1792, 4096, 2, 4, "act"),        # 10 x 8 tiles of 256 x 224, 2 parts
    (2560, 1800, 4096, 8, 16, "act"),       # a partial last column tile, 3 parts
    (4096, 4480, 4096, 6, 8, "weight"),     # 16 x 20 tiles of 256 x 224 (whole columns), 3 parts
]


def test_no_split_when_the_last_round_is_the_partial_last_column():
    """The 6:8 prefill workload's tiles (16 x 19 of 256 x 224, 4096 rows of X):
    the eight tiles of the last round are the last column, which holds 64 of
    224 rows, so the round is short already and runs whole."""
    w = inputs.normal_bf16((4096, 4096), 0.02, seed=1)
    x = inputs.normal_bf16((4096, 4096), 1.0, seed=2)
    Wc = nm.slide_decompose(dev(w), 6, 8)
    nm.sparse_gemm(Wc, nm.lift(dev(x), 8), nm.NM_WEIGHT, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.last_gemm_kernel() == "k_nm_gemm_2cta<224,2,1>", nm.last_gemm_kernel()


@pytest.mark.parametrize("ra,rb,K,N,M,side", SHAPES)
def test_split_round_exact_on_integers(ra, rb, K, N, M, side):
    rng = np.random.default_rng(ra + rb + K)
    a = _int_bf16(rng, (ra, K))
    b = _int_bf16(rng, (rb, K), -3, 4)
    S = nm.prune_compress(dev(a), N, M)
    D = nm.lift(dev(b), M)
    sd = nm.NM_ACT if side == "act" else nm.NM_WEIGHT
    y = nm.sparse_gemm(S, D, sd, torch.float32)
    kname = nm.last_gemm_kernel()
    assert "+split" in kname, kname
    y_plain = torch.empty_like(y)
    st = S.struct()
    import ctypes
    nm._check("nm_sparse_gemm", nm.lib().nm_sparse_gemm(ctypes.byref(st), nm._p(D), rb, sd, nm._p(y_plain),
                                                          nm.NM_FP32, None, 0, nm._stream(D)))
    assert "+split" not in nm.last_gemm_kernel()
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.act_sparse_linear(a, b, N, M) if side == "act" else oracle.act_sparse_linear(a, b, N, M).T
    np.testing.assert_array_equal(host_f64(y), ref)
    np.testing.assert_array_equal(host_f64(y_plain), ref)


@pytest.mark.parametrize("ra,rb,K,N,M,side", SHAPES)
def test_split_round_random_within_tolerance_and_deterministic(ra, rb, K, N, M, side):
    a = inputs.student_t_bf16((ra, K), 4.0, seed=ra)
    b = inputs.normal_bf16((rb, K), 0.02, seed=rb)
    S = nm.prune_compress(dev(a), N, M)
    D = nm.lift(dev(b), M)
    sd = nm.NM_ACT if side == "act" else nm.NM_WEIGHT
    y1 = nm.sparse_gemm(S, D, sd, torch.bfloat16)
    y2 = nm.sparse_gemm(S, D, sd, torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    ref = oracle.act_sparse_linear(a, b, N, M)
    y = host_f64(y1)
    if side == "weight":
        y = y.T
    for r0 in range(0, ra, 512):
        check_close(y[r0:r0 + 512], ref[r0:r0 + 512], f"split round {ra}x{rb}x{K}, rows {r0}..")


# 512-row tiles (two M = 256 MMAs per B stage), pinned by NMSPARSE_GEMM:
# (sparse rows, dense rows, K, N, M, side, variant), one round of 74 pairs
# and a few tiles more
SHAPES_512 = [
    (4096, 2240, 4096, 2, 4, "act", "2cta224x2"),      # 8 x 10 tiles of 512 x 224, 2 parts
    (4096, 1280, 4096, 6, 8, "weight", "2cta128x2"),   # 8 x 10 tiles of 512 x 128, 3 parts
]


@pytest.mark.parametrize("ra,rb,K,N,M,side,variant", SHAPES_512)
def test_split_round_on_512_row_tiles(monkeypatch, ra, rb, K, N, M, side, variant):
    monkeypatch.setenv("NMSPARSE_GEMM", variant)
    rng = np.random.default_rng(ra + rb + K + 1)
    a = _int_bf16(rng, (ra, K))
    b = _int_bf16(rng, (rb, K), -3, 4)
    S = nm.prune_compress(dev(a), N, M)
    D = nm.lift(dev(b), M)
    sd = nm.NM_ACT if side == "act" else nm.NM_WEIGHT
    y = nm.sparse_gemm(S, D, sd, torch.float32)
    kname = nm.last_gemm_kernel()
    assert ",1,2>" in kname and "+split" in kname, kname
    # random data: within tolerance of the oracle and deterministic
    ar = inputs.student_t_bf16((ra, K), 4.0, seed=ra + 7)
    br = inputs.normal_bf16((rb, K), 0.02, seed=rb + 7)
    Sr = nm.prune_compress(dev(ar), N, M)
    Dr = nm.lift(dev(br), M)
    y1 = nm.sparse_gemm(Sr, Dr, sd, torch.bfloat16)
    y2 = nm.sparse_gemm(Sr, Dr, sd, torch.bfloat16)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    ref = oracle.act_sparse_linear(a, b, N, M)
    np.testing.assert_array_equal(host_f64(y), ref if side == "act" else ref.T)
    assert torch.equal(y1, y2)
    ref_r = oracle.act_sparse_linear(ar, br, N, M)
    check_close(host_f64(y1), ref_r if side == "act" else ref_r.T, f"512-row tiles {variant}")

