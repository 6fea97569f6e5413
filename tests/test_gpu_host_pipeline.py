"""The chunked host-buffer pipeline (nm_act_sparse_linear_host): results
equal the device-buffer calls on every chunk, and the oracle within
tolerance; exact on integers."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_bits

pytestmark = pytest.mark.gpu


def _host(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).pin_memory()


def _chunks(T, O, chunk):
    """The pipeline's chunks as (first row, rows).  The default chunk is 256
    rows, or more when a chunk's product would leave more than half the SM
    pairs idle, and its last chunk of F >= 256 rows goes as F - 128 and 128."""
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    Tc = chunk or min(T, 256 * max(1, -(-pairs // (2 * -(-O // 224)))))
    out = [(r0, min(Tc, T - r0)) for r0 in range(0, T, Tc)]
    r0, last = out[-1]
    if chunk == 0 and last >= 256:
        out[-1:] = [(r0, last - 128), (T - 128, 128)]
    return out


@pytest.mark.parametrize("chunk", [0, 128, 384])
@pytest.mark.parametrize("T,K,O,N,M", [(600, 1024, 768, 8, 16), (256, 512, 1024, 2, 4), (130, 2048, 512, 16, 32),
                                       (1000, 1024, 4096, 8, 16)])
def test_host_pipeline_matches_device_calls(chunk, T, K, O, N, M):
    x = inputs.student_t_bf16((T, K), 4.0, T + K)
    w = inputs.normal_bf16((O, K), 0.02, O)
    Wl = nm.lift(dev(w), M)
    xh = _host(x)
    yh = torch.empty((T, O), dtype=torch.bfloat16).pin_memory()
    nm.act_sparse_linear_host(xh, Wl, N, M, yh, chunk_rows=chunk)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    # the same kernels, called chunk by chunk on device buffers
    ref = []
    for r0, rows in _chunks(T, O, chunk):
        c = nm.prune_compress(dev(x[r0:r0 + rows]), N, M)
        ref.append(host_bits(nm.sparse_gemm(c, Wl, nm.NM_ACT, torch.bfloat16)))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(yh), np.concatenate(ref))
    check_close(inputs.bf16_to_f64(host_bits(yh)), oracle.act_sparse_linear(x, w, N, M), f"host T={T}")


def test_host_pipeline_exact_on_integers():
    T, K, O = 520, 512, 640
    rng = np.random.default_rng(3)
    x = inputs.bf16_from_f64(rng.integers(-8, 9, size=(T, K)).astype(np.float64))
    w = inputs.bf16_from_f64(rng.integers(-3, 4, size=(O, K)).astype(np.float64))
    yh = torch.empty((T, O), dtype=torch.bfloat16).pin_memory()
    xh = _host(x)
    nm.act_sparse_linear_host(xh, nm.lift(dev(w), 8), 4, 8, yh)
    torch.cuda.synchronize()
    ref = oracle.act_sparse_linear(x, w, 4, 8)
    np.testing.assert_array_equal(inputs.bf16_to_f64(host_bits(yh)), inputs.bf16_to_f64(inputs.bf16_from_f64(ref)))


def test_host_pipeline_back_to_back_calls_reuse_buffers():
    """Two calls in a row on the same stream with one workspace: the second
    call's first chunks wait for the first call's copies out."""
    T, K, O = 700, 1024, 512
    x1 = inputs.student_t_bf16((T, K), 4.0, 1)
    x2 = inputs.student_t_bf16((T, K), 4.0, 2)
    w = inputs.normal_bf16((O, K), 0.02, 3)
    Wl = nm.lift(dev(w), 16)
    ws = nm.act_sparse_linear_host_workspace(T, K, 8, 16, O, Wl.device)
    y1 = torch.empty((T, O), dtype=torch.bfloat16).pin_memory()
    y2 = torch.empty((T, O), dtype=torch.bfloat16).pin_memory()
    h1, h2 = _host(x1), _host(x2)          # host inputs stay alive until the copies have run
    nm.act_sparse_linear_host(h1, Wl, 8, 16, y1, ws=ws)
    nm.act_sparse_linear_host(h2, Wl, 8, 16, y2, ws=ws)
    torch.cuda.synchronize()
    check_close(inputs.bf16_to_f64(host_bits(y1)), oracle.act_sparse_linear(x1, w, 8, 16), "first call")
    check_close(inputs.bf16_to_f64(host_bits(y2)), oracle.act_sparse_linear(x2, w, 8, 16), "second call")


def test_host_pipeline_many_chunks():
    """Sixteen chunks through the two slots: every copy in must land before
    its prune, and no slot may be overwritten while a copy still reads it."""
    T, K, O, N, M = 2048, 4096, 1024, 8, 16
    x = inputs.student_t_bf16((T, K), 4.0, 31)
    w = inputs.normal_bf16((O, K), 0.02, 32)
    Wl = nm.lift(dev(w), M)
    xh = _host(x)
    yh = torch.empty((T, O), dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        yh.zero_()
        nm.act_sparse_linear_host(xh, Wl, N, M, yh, chunk_rows=128)
        torch.cuda.synchronize()
        assert nm.device_error() == nm.NM_OK
        ref = []
        for r0 in range(0, T, 128):                  # the same kernels, chunk by chunk
            c = nm.prune_compress(dev(x[r0:r0 + 128]), N, M)
            ref.append(host_bits(nm.sparse_gemm(c, Wl, nm.NM_ACT, torch.bfloat16)))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_bits(yh), np.concatenate(ref))
