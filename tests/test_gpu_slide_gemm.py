"""slide_gemm: the activation lift and the weight-sparse product in one call
(SlideSparse, technical summary §2.B-§2.C).  Decode shapes run as one kernel
that forms the lifted activation panel in shared memory; the results must
equal the two-call path (nm_lift + nm_sparse_gemm) bit for bit, and the CPU
oracle within the output tolerance."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits, host_f64

pytestmark = pytest.mark.gpu


def two_call(Wc, xd, out_dtype):
    return nm.sparse_gemm(Wc, nm.lift(xd, Wc.M), nm.NM_WEIGHT, out_dtype)


# (T, K, O, N, M): the 6:8 decode workload; ragged O and a partial last
# k-block (K' = 1440); 14:16, 30:32 and 2:4; one to 32 token rows; a shape that
# takes the workspace path (40 rows)
SHAPES = [
    (16, 4096, 4096, 6, 8),
    (1, 512, 256, 6, 8),
    (5, 1024, 384, 6, 8),
    (16, 960, 200, 6, 8),
    (9, 2048, 256, 14, 16),
    (16, 4096, 256, 30, 32),
    (16, 1024, 256, 2, 4),
    (24, 1024, 512, 6, 8),
    (32, 1024, 4096, 6, 8),
    (40, 1024, 256, 6, 8),
]


@pytest.mark.parametrize("T,K,O,N,M", SHAPES)
def test_equals_the_two_call_path(T, K, O, N, M):
    x = inputs.normal_bf16((T, K), 1.0, seed=T + K)
    w = inputs.normal_bf16((O, K), 0.02, seed=O + 3)
    Wc = nm.slide_decompose(dev(w), N, M)
    xd = dev(x)
    fused = nm.slide_gemm_workspace_size(Wc, T) == 0
    assert fused == (T <= 32 and not (T > 16 and K >= 4096)), (T, K)
    for out_dtype in (torch.bfloat16, torch.float32):
        y = nm.slide_gemm(Wc, xd, out_dtype)
        ref = two_call(Wc, xd, out_dtype)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(y), host_bits(ref)), f"{T}x{K}x{O} {N}:{M} {out_dtype}"
    check_close(host_f64(y), oracle.weight_sparse_linear(x, w, N, M), f"slide {T}x{K}x{O} {N}:{M}")
    assert nm.device_error() == nm.NM_OK


def test_strided_activation_rows():
    """X as a column slice of a wider tensor (row stride K + 64)."""
    T, K, O = 16, 2048, 512
    big = inputs.normal_bf16((T, K + 64), 1.0, seed=5)
    w = inputs.normal_bf16((O, K), 0.02, seed=6)
    Wc = nm.slide_decompose(dev(w), 6, 8)
    xd = dev(big)[:, 32:32 + K]
    assert xd.stride(0) == K + 64
    y = nm.slide_gemm(Wc, xd, torch.float32)
    ref = two_call(Wc, xd.contiguous(), torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(y), host_bits(ref))
    check_close(host_f64(y), oracle.weight_sparse_linear(np.ascontiguousarray(big[:, 32:32 + K]), w, 6, 8),
                "strided")


def test_integer_inputs_exact():
    """Integer-valued bf16 operands with |sums| < 2^24: the fp32 result equals
    the fp64 oracle exactly, so a misplaced lifted column cannot hide."""
    rng = np.random.default_rng(11)
    T, K, O = 16, 1024, 384
    x = inputs.bf16_from_f64(rng.integers(-8, 9, size=(T, K)).astype(np.float64))
    w = inputs.bf16_from_f64(rng.integers(-8, 9, size=(O, K)).astype(np.float64))
    Wc = nm.slide_decompose(dev(w), 6, 8)
    y = nm.slide_gemm(Wc, dev(x), torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host_f64(y), oracle.weight_sparse_linear(x, w, 6, 8))


def test_one_hot_weight_gathers_lifted_x():
    """Each weight row keeps one entry (a one-hot row is its own 6:8 pruning):
    the output column is that column of X, exactly."""
    T, K, O = 16, 512, 128
    rng = np.random.default_rng(3)
    x = inputs.normal_bf16((T, K), 1.0, seed=9)
    wf = np.zeros((O, K), np.float64)
    cols = rng.integers(0, K, size=O)
    wf[np.arange(O), cols] = 1.0
    w = inputs.bf16_from_f64(wf)
    Wc = nm.slide_decompose(dev(w), 6, 8)
    y = nm.slide_gemm(Wc, dev(x), torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host_f64(y), oracle.to_f64(x)[:, cols])


def test_consecutive_calls_with_new_activations():
    """Back-to-back calls on one stream, each with its own X: every call must
    see its own activations (the panel is formed after the preceding kernel)."""
    T, K, O = 16, 4096, 1024
    w = inputs.normal_bf16((O, K), 0.02, seed=1)
    Wc = nm.slide_decompose(dev(w), 6, 8)
    xs = [inputs.normal_bf16((T, K), 1.0, seed=40 + i) for i in range(4)]
    xd = dev(xs[0])
    outs = []
    for i in range(4):
        xd.copy_(dev(xs[i]))                       # rewritten in place between the calls
        outs.append(nm.slide_gemm(Wc, xd, torch.float32))
    torch.cuda.synchronize()
    for i in range(4):
        check_close(host_f64(outs[i]), oracle.weight_sparse_linear(xs[i], w, 6, 8), f"call {i}")


# ----------------------------------------------- prefill shapes (SM pairs)
# slide_gemm with at least 64 activation rows and the weight in whole 256-row
# tiles runs the SM-pair kernel whose lift warps write the lifted B stages
# from X; the two-call reference runs the same tile variant.
# (T, K, O, N, M, variant of the reference)
PAIR_SHAPES = [
    (4096, 4096, 4096, 6, 8, "auto"),      # the 6:8 prefill workload
    (600, 1024, 512, 6, 8, "auto"),        # ragged last column tile
    (1000, 2048, 768, 14, 16, "auto"),
    (512, 4096, 256, 30, 32, "auto"),
    (520, 1024, 512, 2, 4, "auto"),        # 2:4: the lift is the identity
    (200, 1024, 512, 6, 8, "2cta128"),     # 128-wide tiles below 512 rows
    (64, 960, 256, 6, 8, "2cta128"),       # K' = 1440: a partial last k-block
    (2048, 16384, 256, 6, 8, "auto"),      # K' >= 16384: the 256-wide tile
    (1792, 4096, 2560, 6, 8, "auto"),      # 10 x 8 tiles: the last round split in 3 (lift warps and parts)
]


@pytest.mark.parametrize("T,K,O,N,M,variant", PAIR_SHAPES)
def test_prefill_equals_the_two_call_path(monkeypatch, T, K, O, N, M, variant):
    x = inputs.normal_bf16((T, K), 1.0, seed=T + 7 * K)
    w = inputs.normal_bf16((O, K), 0.02, seed=O + 11)
    Wc = nm.slide_decompose(dev(w), N, M)
    xd = dev(x)
    assert nm.slide_gemm_workspace_size(Wc, T) == (0 if T < 512 else nm.sparse_gemm_workspace_size(Wc, T, nm.NM_WEIGHT))
    for out_dtype in (torch.bfloat16, torch.float32):
        y = nm.slide_gemm(Wc, xd, out_dtype)
        assert ",lift>" in nm.last_gemm_kernel(), nm.last_gemm_kernel()
        if (T, O) == (1792, 2560):
            assert nm.last_gemm_kernel().endswith("+split3"), nm.last_gemm_kernel()
        monkeypatch.setenv("NMSPARSE_GEMM", variant)
        ref = two_call(Wc, xd, out_dtype)
        monkeypatch.delenv("NMSPARSE_GEMM")
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(y), host_bits(ref)), f"{T}x{K}x{O} {N}:{M} {out_dtype}"
    assert nm.device_error() == nm.NM_OK
    y = host_f64(y)
    y_ref = oracle.weight_sparse_linear(x, w, N, M)
    for r0 in range(0, T, 512):
        check_close(y[r0:r0 + 512], y_ref[r0:r0 + 512], f"slide prefill {T}x{K}x{O} {N}:{M}, rows {r0}..")


def test_prefill_integer_inputs_exact():
    rng = np.random.default_rng(13)
    T, K, O = 700, 1024, 768
    x = inputs.bf16_from_f64(rng.integers(-8, 9, size=(T, K)).astype(np.float64))
    w = inputs.bf16_from_f64(rng.integers(-8, 9, size=(O, K)).astype(np.float64))
    for N, M in ((6, 8), (14, 16)):
        Wc = nm.slide_decompose(dev(w), N, M)
        y = nm.slide_gemm(Wc, dev(x), torch.float32)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_f64(y), oracle.weight_sparse_linear(x, w, N, M))


def test_prefill_strided_activation_rows():
    """X as a column slice of a wider tensor (row stride K + 64) on the
    SM-pair path."""
    T, K, O = 640, 2048, 512
    big = inputs.normal_bf16((T, K + 64), 1.0, seed=15)
    w = inputs.normal_bf16((O, K), 0.02, seed=16)
    Wc = nm.slide_decompose(dev(w), 6, 8)
    xd = dev(big)[:, 32:32 + K]
    y = nm.slide_gemm(Wc, xd, torch.float32)
    ref = two_call(Wc, xd.contiguous(), torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(y), host_bits(ref))
    check_close(host_f64(y), oracle.weight_sparse_linear(np.ascontiguousarray(big[:, 32:32 + K]), w, 6, 8),
                "strided prefill")
