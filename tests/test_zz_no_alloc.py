"""hybrid_gemm_noalloc: the hybrid dense + 2:4 product for callers that must
not allocate device memory (for instance a plugin whose host engine owns and
pre-plans all device memory).  Its scratch is an array compiled into the
library, so the test checks it against the ordinary entry point, which takes
a caller-provided workspace: on two calls in a row, each synchronised, and on
two calls queued back to back on one stream before a single synchronisation
(the second call's gather rewrites the shared array right after the first
call's GEMM has read it).  The same kernels run on the same inputs, so the
outputs must be equal bit for bit.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import dev


def test_rejects_sizes_beyond_the_builtin_scratch():
    # validated before any device work: with a column permutation, B * K * 2
    # bytes must fit in 2 MiB
    L = nm.lib()
    H = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, 256, 8192, 2048)
    fake = ctypes.c_void_p(0x10000)
    assert L.hybrid_gemm_noalloc(fake, 129, ctypes.byref(H), fake, nm.NM_BF16, None) == nm.NM_ERR_WORKSPACE
    assert L.hybrid_gemm_noalloc(fake, 4, None, fake, nm.NM_BF16, None) == nm.NM_ERR_INVALID_ARG


def test_malformed_weight_is_an_argument_error_before_the_size_check():
    L = nm.lib()
    fake = ctypes.c_void_p(0x10000)
    for O, K, D in [(256, 0, 0), (256, -8, 0), (0, 4096, 1024), (256, 4096, 5000), (256, 4096, -4)]:
        H = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, O, K, D)
        assert L.hybrid_gemm_noalloc(fake, 1 << 40, ctypes.byref(H), fake, nm.NM_BF16, None) == nm.NM_ERR_INVALID_ARG


def test_no_permutation_needs_no_scratch():
    # without a column permutation nothing is gathered, so the size limit does
    # not apply; this call then fails hybrid_gemm's own check (K % 8 != 0)
    # before launching anything
    L = nm.lib()
    fake = ctypes.c_void_p(0x10000)
    H = nm.HybridWeight(None, 0x10000, 0x10000, 0x10000, 256, 8196, 2052)
    assert L.hybrid_gemm_noalloc(fake, 1 << 20, ctypes.byref(H), fake, nm.NM_BF16, None) == nm.NM_ERR_INVALID_ARG


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
        assert torch.equal(got, ref), f"no-alloc call {call}, B={B}"
    assert nm.device_error() == nm.NM_OK


@pytest.mark.gpu
def test_two_calls_queued_on_one_stream():
    O, K, B = 640, 4096, 128
    w = inputs.normal_bf16((O, K), 0.02, seed=23)
    h = nm.hybrid_prepare(dev(w), 0.25)
    xs = [dev(inputs.normal_bf16((B, K), 1.0, seed=300 + i)) for i in range(2)]
    refs = [nm.hybrid_gemm(x, h, torch.bfloat16) for x in xs]
    torch.cuda.synchronize()
    got = [nm.hybrid_gemm_noalloc(x, h, torch.bfloat16) for x in xs]      # no synchronisation in between
    torch.cuda.synchronize()
    assert nm.device_error() == nm.NM_OK
    for i in range(2):
        assert torch.equal(got[i], refs[i]), f"queued call {i}"
    assert not torch.equal(got[0], got[1])
