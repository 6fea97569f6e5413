"""Bounded waits, error reporting and the tensor-core rate probe on the GPU.
Nothing here faults, traps or hangs the device: the expired wait is a barrier
nobody arrives on, with a 1 ms limit, and the kernel returns normally after
recording the status."""
import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_f64

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    assert nm.device_error() == nm.NM_OK
    nm.debug_expire_wait(1000)
    assert nm.device_error() == nm.NM_ERR_DEVICE_TIMEOUT
    # the status word was cleared and the context still works
    assert nm.device_error() == nm.NM_OK
    x = inputs.normal_bf16((32, 256), 1.0, 1)
    w = inputs.normal_bf16((64, 256), 0.02, 2)
    comp = nm.prune_compress(dev(x), 2, 4)
    y = nm.sparse_gemm(comp, nm.lift(dev(w), 4), nm.NM_ACT, torch.float32)
    torch.cuda.synchronize()
    check_close(host_f64(y), oracle.act_sparse_linear(x, w, 2, 4))
    assert nm.device_error() == nm.NM_OK


def test_errors_launch_nothing():
    x = dev(inputs.normal_bf16((8, 256), 1.0, 1))
    comp = nm.alloc_compressed(8, 256, 2, 4, x.device)
    comp.vals.zero_()
    before = comp.vals.clone()
    with pytest.raises(nm.NmError) as e:
        nm.prune_compress(x, 3, 4, out=comp)          # 3:4 is not a supported pattern
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    with pytest.raises(nm.NmError) as e:
        nm.prune_compress(x[:, 4:], 2, 4)             # rows start 8 bytes off a 16-byte boundary
    assert e.value.status == nm.NM_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.equal(comp.vals.view(torch.int16), before.view(torch.int16))


def test_mma_rate_probe():
    """The tensor-core probe runs on every SM pair and reports sane rates: the
    2:4 modes execute twice the logical K per MMA, the 8-bit one four times."""
    dense = nm.mma_rate_probe(0, iters=2000, reps=3)
    sp16 = nm.mma_rate_probe(1, iters=2000, reps=3)
    sp8 = nm.mma_rate_probe(2, iters=2000, reps=3)
    assert nm.device_error() == nm.NM_OK
    assert 500.0 < dense < 2600.0, dense
    assert 1.5 * dense < sp16 < 2.2 * dense, (dense, sp16)
    assert 1.5 * sp16 < sp8 < 2.2 * sp16, (sp16, sp8)


def test_injected_launch_error_launches_nothing():
    """A launch that fails (injected on the host) makes the call return
    NM_ERR_CUDA with the error code; nothing runs, the outputs keep their
    contents, and the next call works."""
    x = inputs.normal_bf16((48, 512), 1.0, 3)
    w = inputs.normal_bf16((96, 512), 0.02, 4)
    comp = nm.alloc_compressed(48, 512, 8, 16, "cuda")
    comp.vals.fill_(7.0)
    before = comp.vals.clone()
    nm.debug_fail_next_launch(701)
    with pytest.raises(nm.NmError) as e:
        nm.prune_compress(dev(x), 8, 16, out=comp)
    assert e.value.status == nm.NM_ERR_CUDA and nm.last_cuda_error() == 701
    torch.cuda.synchronize()
    assert torch.equal(comp.vals, before)
    # the GEMM path (its own launcher) and a call made of several launches
    Wl = nm.lift(dev(w), 16)
    nm.prune_compress(dev(x), 8, 16, out=comp)
    Y = torch.full((48, 96), 3.0, dtype=torch.float32, device="cuda")
    nm.debug_fail_next_launch(719)
    with pytest.raises(nm.NmError) as e:
        nm.sparse_gemm(comp, Wl, nm.NM_ACT, torch.float32, out=Y)
    assert e.value.status == nm.NM_ERR_CUDA and nm.last_cuda_error() == 719
    torch.cuda.synchronize()
    assert bool((Y == 3.0).all())
    nm.sparse_gemm(comp, Wl, nm.NM_ACT, torch.float32, out=Y)
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    check_close(host_f64(Y), oracle.act_sparse_linear(x, w, 8, 16))
