"""hybrid_gemm_noalloc: the hybrid dense + 2:4 product for callers that must
not allocate device memory (for instance a plugin whose host engine owns and
pre-plans all device memory).  Its scratch is an array compiled into the
library, so the test checks it against the ordinary entry point, which takes
a caller-provided workspace, on two calls in a row (the second call sees
the previous call's leftovers in the shared array).  This file is collected
last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import check_close, dev, host_f64


def test_rejects_sizes_beyond_the_builtin_scratch():
    # validated before any device work: B * K * 2 bytes must fit in 2 MiB
    L = nm.lib()
    H = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, 256, 8192, 2048)
    fake = ctypes.c_void_p(0x10000)
    assert L.hybrid_gemm_noalloc(fake, 129, ctypes.byref(H), fake, nm.NM_BF16, None) == nm.NM_ERR_WORKSPACE
    assert L.hybrid_gemm_noalloc(fake, 4, None, fake, nm.NM_BF16, None) == nm.NM_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("B", [8, 128])
def test_matches_the_workspace_entry_point(B):
    O, K = 640, 4096
    w = inputs.normal_bf16((O, K), 0.02, seed=21)
    h = nm.hybrid_prepare(dev(w), 0.25)
    for call in range(2):
        x = dev(inputs.normal_bf16((B, K), 1.0, seed=100 + 10 * B + call))
        ref = nm.hybrid_gemm(x, h, torch.bfloat16)
        got = nm.hybrid_gemm_noalloc(x, h, torch.bfloat16)
        torch.cuda.synchronize()
        check_close(host_f64(got), host_f64(ref), f"no-alloc call {call}, B={B}")
    assert nm.device_error() == nm.NM_OK
