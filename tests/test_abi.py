"""The C ABI without a GPU: the library loads, exports every function that
include/nmsparse.h declares, sizes match the documented formulas, and argument
validation rejects bad calls before anything touches the device."""
import ctypes
import os
import re

import pytest

import oracle
from semi_structured_sparse_nm_b200 import build as nmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    path = nmbuild.build()
    from semi_structured_sparse_nm_b200 import _lib
    assert _lib.LIB_PATH == path
    return _lib.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nmsparse.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 18, names
    for n in ["nm_prune_compress", "slide_decompose", "nm_sparse_gemm", "hybrid_gemm", "nm_lift",
              "hybrid_prepare", "nm_get_device_error"]:
        assert n in names
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_sizes_match_the_oracle(L):
    for K, M in [(4096, 4), (4096, 8), (4096, 16), (14336, 32), (96, 8), (64, 32)]:
        assert L.nm_lifted_k(K, M) == oracle.lifted_k(K, M)
        for rows in (1, 16, 128, 129, 2048):
            assert L.nm_meta_bytes(rows, K, M) == oracle._load().or_meta_hw_bytes(rows, oracle.lifted_k(K, M))
    assert L.nm_lifted_k(100, 8) == -1 and L.nm_lifted_k(12, 3) == -1
    for K, f in [(4096, 0.25), (4096, 0.0), (4096, 1.0), (100, 0.3), (640, 0.2)]:
        assert L.hybrid_dense_count(K, f) == oracle.hybrid_dense_count(K, f)


def test_validation_before_launch(L):
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10001)
    null = ctypes.c_void_p(0)
    s = null
    # invalid arguments
    assert L.nm_prune_compress(null, 0, 4, 256, 256, 2, 4, null, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(fake, 0, 4, 250, 256, 2, 4, null, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(fake, 7, 4, 256, 256, 2, 4, null, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(fake, 0, 4, 256, 128, 2, 4, null, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    # unsupported patterns
    assert L.nm_prune_compress(fake, 0, 4, 256, 256, 3, 4, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.nm_prune_compress(fake, 0, 4, 240, 240, 2, 6, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.nm_prune_compress(fake, 0, 4, 256, 256, 16, 16, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.slide_decompose(fake, 0, 4, 256, 4, 8, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    # alignment
    assert L.nm_prune_compress(odd, 0, 4, 256, 256, 2, 4, null, fake, fake, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_prune_compress(fake, 0, 4, 256, 260, 2, 4, null, fake, fake, s) == nm.NM_ERR_ALIGNMENT
    # empty operands are a no-op
    assert L.nm_prune_compress(null, 0, 0, 256, 256, 2, 4, null, null, null, s) == nm.NM_OK
    assert L.nm_lift(null, 0, 0, 256, 256, 8, null, s) == nm.NM_OK
    # the split window order: 6:8, 14:16, 30:32 with K % 128 == 0 only
    assert L.slide_decompose_split(fake, 4, 192, 6, 8, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.slide_decompose_split(fake, 4, 256, 2, 4, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.slide_decompose_split(fake, 4, 256, 4, 8, null, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.slide_decompose_split(null, 4, 256, 6, 8, null, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.slide_decompose_split(null, 0, 256, 6, 8, null, null, null, s) == nm.NM_OK
    assert L.nm_lift_odd(fake, 4, 192, 288, 8, s) == nm.NM_ERR_UNSUPPORTED      # K % 128
    assert L.nm_lift_odd(fake, 4, 256, 256, 8, s) == nm.NM_ERR_INVALID_ARG      # ld < K' = 384
    assert L.nm_lift_odd(fake, 4, 256, 384, 4, s) == nm.NM_ERR_UNSUPPORTED      # 2:4 has no odd windows
    assert L.nm_lift_odd(odd, 4, 256, 384, 8, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_lift_odd(fake, 4, 256, 388, 8, s) == nm.NM_ERR_ALIGNMENT        # 776-byte rows
    assert L.nm_lift_odd(null, 0, 256, 384, 8, s) == nm.NM_OK
    # GEMM
    S = nm.SparseOperand(0x10000, 0x10000, 128, 256, 2, 4, 256)
    assert L.nm_sparse_gemm(ctypes.byref(S), null, 64, 0, fake, 0, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_sparse_gemm(ctypes.byref(S), fake, 64, 5, fake, 0, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_sparse_gemm(ctypes.byref(S), odd, 64, 0, fake, 0, null, 0, s) == nm.NM_ERR_ALIGNMENT
    bad = nm.SparseOperand(0x10000, 0x10000, 128, 256, 2, 4, 300)
    assert L.nm_sparse_gemm(ctypes.byref(bad), fake, 64, 0, fake, 0, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_dense_gemm(fake, 16, fake, 16, 40, fake, 0, s) == nm.NM_ERR_UNSUPPORTED
    # hybrid
    H = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, 64, 512, 128)
    assert L.hybrid_gemm(fake, 4, ctypes.byref(H), fake, 0, null, 0, s) == nm.NM_ERR_WORKSPACE
    H2 = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, 64, 512, 100)
    assert L.hybrid_gemm(fake, 4, ctypes.byref(H2), fake, 0, fake, 1 << 20, s) == nm.NM_ERR_UNSUPPORTED
    assert L.hybrid_prepare(fake, 64, 512, 0.25, ctypes.byref(H), null, 0, s) == nm.NM_ERR_WORKSPACE
    assert L.nm_debug_expire_wait(0, s) == nm.NM_ERR_INVALID_ARG
    for code in range(7):
        assert L.nm_status_string(code)


def test_correction_calls_validate_before_launch(L):
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    odd4 = ctypes.c_void_p(0x10002)
    null = ctypes.c_void_p(0)
    s = null
    both = nm.NM_XF_SHIFT | nm.NM_XF_VAR
    # workspace: the token moments (two fp64 per row, padded to 256 bytes) and
    # two fp64 per (row, chunk of 32 G groups)
    assert L.nm_prune_compress_xf_workspace_size(16, 4096, 16) == 256 + 16 * (256 // 32) * 16
    assert L.nm_prune_compress_xf_workspace_size(100, 4096, 4) == 1792 + 100 * (1024 // 128) * 16
    assert L.nm_prune_compress_xf_workspace_size(0, 4096, 16) == 0
    # bad flags, missing scale outputs, missing workspace with VAR, misaligned scales
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 2, 4, 4, null, fake, fake, fake, fake, fake, 4096, s) \
        == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 2, 4, both, null, fake, fake, null, fake, fake, 4096, s) \
        == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 2, 4, both, null, fake, fake, fake, fake, null, 0, s) \
        == nm.NM_ERR_WORKSPACE
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 2, 4, both, null, fake, fake, fake, fake, fake, 16, s) \
        == nm.NM_ERR_WORKSPACE
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 2, 4, nm.NM_XF_SHIFT, null, fake, fake, odd4, fake,
                                  null, 0, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_prune_compress_xf(fake, 16, 256, 256, 3, 4, both, null, fake, fake, fake, fake, fake, 4096, s) \
        == nm.NM_ERR_UNSUPPORTED
    assert L.nm_prune_compress_xf(null, 0, 256, 256, 2, 4, both, null, null, null, null, null, null, 0, s) \
        == nm.NM_OK
    # row sums
    assert L.nm_row_sums(null, 4, 256, 256, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_row_sums(fake, 4, 256, 252, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_row_sums(fake, 4, 252, 260, fake, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_row_sums(fake, 4, 256, 256, odd4, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_row_sums(null, 0, 256, 256, null, s) == nm.NM_OK
    # the corrected GEMM
    S = nm.SparseOperand(0x10000, 0x10000, 128, 256, 2, 4, 256)
    assert L.nm_sparse_gemm_xf(ctypes.byref(S), fake, 64, null, fake, fake, fake, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_sparse_gemm_xf(ctypes.byref(S), fake, 64, fake, fake, odd4, fake, 0, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_sparse_gemm_xf(ctypes.byref(S), fake, 0, null, null, null, fake, 0, s) == nm.NM_OK


def test_host_pipeline_validates_before_launch(L):
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10001)
    null = ctypes.c_void_p(0)
    s = null
    ws = L.nm_act_sparse_linear_host_workspace_size(600, 1024, 8, 16, 768, 256)
    Kl = 1024 * 7 // 4                                                 # K' = 1.75 K for 8:16
    slot = (256 * 1024 * 2) + (256 * Kl) + L.nm_meta_bytes(256, 1024, 16) + (256 * 768 * 2)
    assert ws == 2 * slot
    assert L.nm_act_sparse_linear_host_workspace_size(100, 1024, 8, 16, 768, 0) == \
        2 * ((100 * 2048 + 255) // 256 * 256 + (100 * Kl + 255) // 256 * 256 + L.nm_meta_bytes(100, 1024, 16)
             + (100 * 1536 + 255) // 256 * 256)
    assert L.nm_act_sparse_linear_host(fake, 600, 1024, 8, 16, fake, 768, fake, 100, fake, ws, s) \
        == nm.NM_ERR_INVALID_ARG                                           # chunk not a multiple of 128
    assert L.nm_act_sparse_linear_host(fake, 600, 1024, 15, 16, fake, 768, fake, 0, fake, ws, s) \
        == nm.NM_ERR_UNSUPPORTED
    assert L.nm_act_sparse_linear_host(null, 600, 1024, 8, 16, fake, 768, fake, 0, fake, ws, s) \
        == nm.NM_ERR_INVALID_ARG
    assert L.nm_act_sparse_linear_host(fake, 600, 1024, 8, 16, odd, 768, fake, 0, fake, ws, s) \
        == nm.NM_ERR_ALIGNMENT
    assert L.nm_act_sparse_linear_host(fake, 600, 1024, 8, 16, fake, 768, fake, 0, fake, ws - 1, s) \
        == nm.NM_ERR_WORKSPACE
    assert L.nm_act_sparse_linear_host(null, 0, 1024, 8, 16, null, 768, null, 0, null, 0, s) == nm.NM_OK


def test_slide_gemm_sizes_and_validation(L):
    """slide_gemm runs fused (no workspace) on decode shapes whose lifted panel
    fits a CTA's shared memory, else it needs rows x K' bf16 of workspace for
    the separate lift; arguments are checked before any launch."""
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    null = ctypes.c_void_p(0)
    s = null
    W68 = nm.SparseOperand(0x10000, 0x10000, 4096, 4096, 6, 8, 6144)       # the 6:8 decode weight
    for rows_x in (1, 16):
        assert L.slide_gemm_workspace_size(ctypes.byref(W68), rows_x) == 0
    # 17..32 rows double the panel and the raw boxes: no room left for 4 ring stages
    for rows_x in (17, 32, 33):
        assert L.slide_gemm_workspace_size(ctypes.byref(W68), rows_x) == rows_x * 6144 * 2
    W68s = nm.SparseOperand(0x10000, 0x10000, 4096, 1024, 6, 8, 1536)    # shorter K: 32 rows fit
    assert L.slide_gemm_workspace_size(ctypes.byref(W68s), 32) == 0
    # a long reduction on one row tile: 96 k-blocks per CTA cannot be held as a panel
    Wlong = nm.SparseOperand(0x10000, 0x10000, 128, 65536, 6, 8, 98304)
    assert L.slide_gemm_workspace_size(ctypes.byref(Wlong), 8) == 8 * 98304 * 2
    W24 = nm.SparseOperand(0x10000, 0x10000, 256, 512, 2, 4, 512)
    assert L.slide_gemm_workspace_size(ctypes.byref(W24), 16) == 0
    # prefill shapes on SM pairs (whole 256-row weight tiles, >= 64 rows of X):
    # the lift warps write B from X; from 512 rows on, optional scratch for a
    # split last round (the sparse product's own bound)
    for rows_x in (64, 511):
        assert L.slide_gemm_workspace_size(ctypes.byref(W68), rows_x) == 0
    for rows_x in (512, 4096):
        assert L.slide_gemm_workspace_size(ctypes.byref(W68), rows_x) == \
            L.nm_sparse_gemm_workspace_size(ctypes.byref(W68), rows_x, 1)
    W200 = nm.SparseOperand(0x10000, 0x10000, 200, 4096, 6, 8, 6144)     # not whole 256-row tiles
    assert L.slide_gemm_workspace_size(ctypes.byref(W200), 4096) == 4096 * 6144 * 2
    assert L.slide_gemm(ctypes.byref(W68), fake, 16, 4000, fake, 0, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.slide_gemm(ctypes.byref(W68), null, 16, 4096, fake, 0, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.slide_gemm(ctypes.byref(W68), odd, 16, 4096, fake, 0, null, 0, s) == nm.NM_ERR_ALIGNMENT
    assert L.slide_gemm(ctypes.byref(W68), fake, 16, 4100, fake, 0, null, 0, s) == nm.NM_ERR_ALIGNMENT
    assert L.slide_gemm(ctypes.byref(W68), fake, 16, 4096, fake, 7, null, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.slide_gemm(ctypes.byref(W68), fake, 40, 4096, fake, 0, null, 0, s) == nm.NM_ERR_WORKSPACE
    assert L.slide_gemm(ctypes.byref(W68), null, 0, 4096, null, 0, null, 0, s) == nm.NM_OK


def _ceil256(n):
    return (n + 255) // 256 * 256


def test_fp8_calls_size_and_validate_before_launch(L):
    """The 8-bit (E4M3) entry points: documented workspace size, and every
    bad call rejected before anything reaches the device."""
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    odd4 = ctypes.c_void_p(0x10002)
    null = ctypes.c_void_p(0)
    s = null
    # scratch of the 8-bit packer: the 16-bit windows, then the 16-bit metadata image
    for rows, K, M in [(4096, 4096, 8), (100, 1024, 16), (256, 512, 4)]:
        Kl = L.nm_lifted_k(K, M)
        assert L.slide_decompose_fp8_workspace_size(rows, K, M) == \
            _ceil256(rows * (Kl // 2) * 2) + L.nm_meta_bytes(rows, K, M)
    assert L.slide_decompose_fp8_workspace_size(16, 100, 8) == 0
    # quantise + lift
    assert L.nm_quant_lift_fp8(fake, 7, 16, 4096, 4096, 8, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_quant_lift_fp8(fake, nm.NM_BF16, 16, 4100, 4100, 8, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_quant_lift_fp8(fake, nm.NM_BF16, 16, 4092, 4096, 6, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.nm_quant_lift_fp8(fake, nm.NM_BF16, 16, 8, 8, 8, fake, fake, s) == nm.NM_ERR_UNSUPPORTED  # K' = 12
    assert L.nm_quant_lift_fp8(null, nm.NM_BF16, 16, 4096, 4096, 8, fake, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_quant_lift_fp8(fake, nm.NM_BF16, 16, 4096, 4096, 8, fake, odd4, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_quant_lift_fp8(fake, nm.NM_BF16, 16, 4096, 4100, 8, fake, fake, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_quant_lift_fp8(null, nm.NM_BF16, 0, 4096, 4096, 8, null, null, s) == nm.NM_OK
    # quantise + prune (activation side)
    assert L.nm_prune_compress_fp8(fake, 16, 4096, 4096, 3, 4, null, fake, fake, fake, s) == nm.NM_ERR_UNSUPPORTED
    assert L.nm_prune_compress_fp8(fake, 16, 4096, 4096, 8, 16, null, fake, null, fake, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress_fp8(fake, 16, 4096, 4096, 8, 16, null, fake, odd4, fake, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_prune_compress_fp8(null, 0, 4096, 4096, 8, 16, null, null, null, null, s) == nm.NM_OK
    # offline 8-bit packer
    ws = L.slide_decompose_fp8_workspace_size(256, 4096, 8)
    assert L.slide_decompose_fp8(fake, 256, 4096, 6, 8, fake, fake, fake, null, ws, s) == nm.NM_ERR_INVALID_ARG
    assert L.slide_decompose_fp8(fake, 256, 4096, 6, 8, fake, fake, fake, fake, ws - 1, s) == nm.NM_ERR_WORKSPACE
    assert L.slide_decompose_fp8(fake, 256, 4096, 6, 8, fake, odd4, fake, fake, ws, s) == nm.NM_ERR_ALIGNMENT
    # 8-bit product
    S = nm.SparseOperand(0x10000, 0x10000, 4096, 4096, 6, 8, 6144)
    P = ctypes.byref(S)
    assert L.nm_sparse_gemm_fp8(P, fake, fake, fake, 16, 5, fake, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_sparse_gemm_fp8(P, fake, fake, fake, 16, 0, fake, 7, s) == nm.NM_ERR_INVALID_ARG
    S2 = nm.SparseOperand(0x10000, 0x10000, 4096, 1040, 2, 4, 1040)       # K' % 128 != 0
    assert L.nm_sparse_gemm_fp8(ctypes.byref(S2), fake, fake, fake, 16, 0, fake, 0, s) == nm.NM_ERR_UNSUPPORTED
    S3 = nm.SparseOperand(0x10000, 0x10000, 300, 4096, 6, 8, 6144)        # SM pairs need 256-row blocks
    assert L.nm_sparse_gemm_fp8(ctypes.byref(S3), fake, fake, fake, 512, 0, fake, 0, s) == nm.NM_ERR_UNSUPPORTED
    assert L.nm_sparse_gemm_fp8(P, null, fake, fake, 16, 1, fake, 0, s) == nm.NM_ERR_INVALID_ARG
    assert L.nm_sparse_gemm_fp8(P, odd4, fake, fake, 16, 1, fake, 0, s) == nm.NM_ERR_ALIGNMENT
    assert L.nm_sparse_gemm_fp8(P, null, null, null, 0, 1, null, 0, s) == nm.NM_OK


def test_hybrid_and_mlp_sizes_and_validation(L):
    """Workspace sizes of the hybrid and GLU-MLP calls match their documented
    layouts, the MLP's dense count matches the oracle's, and incomplete or
    misaligned weights are rejected before the first launch."""
    from semi_structured_sparse_nm_b200 import _lib as nm
    fake = ctypes.c_void_p(0x10000)
    null = ctypes.c_void_p(0)
    s = null
    for O, K in [(14336, 4096), (640, 4096), (128, 512)]:
        assert L.hybrid_prepare_workspace_size(O, K) == _ceil256(K * 8) + _ceil256(K) + O * K * 2
        H = nm.HybridWeight(0x10000, 0x10000, 0x10000, 0x10000, O, K, L.hybrid_dense_count(K, 0.25))
        for B in (1, 8, 128):
            assert L.hybrid_gemm_workspace_size(ctypes.byref(H), B) == _ceil256(B * K * 2)
    assert L.hybrid_prepare_workspace_size(0, 4096) == 0
    for I, f in [(14336, 0.25), (14336, 0.0), (14336, 1.0), (1024, 0.3), (512, 0.2)]:
        assert L.spense_dense_count(I, f) == oracle.spense_dense_count(I, f)
    for d, I in [(4096, 14336), (256, 512)]:
        assert L.spense_mlp_prepare_workspace_size(d, I) == \
            4 * _ceil256(I * 8) + _ceil256(I) + _ceil256(2 * I * d * 2) + _ceil256(d * I * 2)
    # a complete weight: the Llama-8B shape with a quarter of the intermediate indices dense
    d, I = 4096, 14336
    D = L.spense_dense_count(I, 0.25)
    full = [0x10000] * 7
    Wm = nm.SpenseMlpStruct(*full, d, I, D)
    for B in (1, 32):
        assert L.spense_mlp_workspace_size(ctypes.byref(Wm), B) == _ceil256(B * 2 * I * 2) + _ceil256(B * I * 2)
    ws = L.spense_mlp_workspace_size(ctypes.byref(Wm), 8)
    assert L.spense_mlp(fake, 8, ctypes.byref(Wm), fake, null, 0, s) == nm.NM_ERR_WORKSPACE
    assert L.spense_mlp(fake, 0, ctypes.byref(Wm), fake, null, 0, s) == nm.NM_OK
    bad_d = nm.SpenseMlpStruct(*full, d, I, 1000)                            # D not whole 256-blocks
    assert L.spense_mlp(fake, 8, ctypes.byref(bad_d), fake, fake, ws, s) == nm.NM_ERR_UNSUPPORTED
    # missing or misaligned packed weights: perm, ug_vals, ug_meta, ug_dense, down_vals, down_meta, down_dense
    for i in range(1, 7):
        parts = list(full)
        parts[i] = 0
        assert L.spense_mlp(fake, 8, ctypes.byref(nm.SpenseMlpStruct(*parts, d, I, D)), fake, fake, ws, s) \
            == nm.NM_ERR_INVALID_ARG, i
        parts[i] = 0x10008
        assert L.spense_mlp(fake, 8, ctypes.byref(nm.SpenseMlpStruct(*parts, d, I, D)), fake, fake, ws, s) \
            == nm.NM_ERR_ALIGNMENT, i
    # all-sparse and all-dense weights need only their own parts
    sparse_only = nm.SpenseMlpStruct(0x10000, 0x10000, 0x10000, 0, 0x10000, 0x10000, 0, d, I, 0)
    assert L.spense_mlp(fake, 0, ctypes.byref(sparse_only), fake, null, 0, s) == nm.NM_OK
    dense_only = nm.SpenseMlpStruct(0x10000, 0, 0, 0x10000, 0, 0, 0x10000, d, I, I)
    assert L.spense_mlp(fake, 0, ctypes.byref(dense_only), fake, null, 0, s) == nm.NM_OK
    # preparation
    pws = L.spense_mlp_prepare_workspace_size(d, I)
    assert L.spense_mlp_prepare(fake, fake, fake, 0.25, ctypes.byref(nm.SpenseMlpStruct(*full, d, I, D + 256)),
                                fake, pws, s) == nm.NM_ERR_INVALID_ARG             # D disagrees with the share
    assert L.spense_mlp_prepare(fake, fake, fake, 0.25, ctypes.byref(Wm), fake, pws - 1, s) == nm.NM_ERR_WORKSPACE
    odd_d = nm.SpenseMlpStruct(*full, 4000, I, D)
    assert L.spense_mlp_prepare(fake, fake, fake, 0.25, ctypes.byref(odd_d), fake, pws, s) == nm.NM_ERR_UNSUPPORTED


def test_misc_entry_points(L):
    from semi_structured_sparse_nm_b200 import _lib as nm
    assert b"sm_100a" in L.nm_version()
    S = nm.SparseOperand(0x10000, 0x10000, 4096, 4096, 8, 16, 7168)
    # SM-pair products: optional scratch for a split last round, at most one
    # 256 x 256 fp32 tile per SM pair; single-CTA products need none (their
    # split-K stays in the cluster)
    bound = L.nm_sparse_gemm_workspace_size(ctypes.byref(S), 2048, 0)
    assert bound > 0 and bound % (256 * 256 * 4) == 0
    assert L.nm_sparse_gemm_workspace_size(ctypes.byref(S), 16, 0) == 0
    S200 = nm.SparseOperand(0x10000, 0x10000, 200, 4096, 8, 16, 7168)
    assert L.nm_sparse_gemm_workspace_size(ctypes.byref(S200), 2048, 0) == 0
    out = ctypes.c_double(0.0)
    null = ctypes.c_void_p(0)
    assert L.nm_mma_rate_probe(3, 10, ctypes.byref(out), null) == nm.NM_ERR_INVALID_ARG
    assert L.nm_mma_rate_probe(0, 0, ctypes.byref(out), null) == nm.NM_ERR_INVALID_ARG
    assert L.nm_mma_rate_probe(0, 10, None, null) == nm.NM_ERR_INVALID_ARG
