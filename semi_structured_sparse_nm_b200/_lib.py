"""ctypes binding of libnmsparse.so (include/nmsparse.h).

Argument marshalling only: every step of the sparse path runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  If the
shared library is missing the import fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnmsparse.so")

NM_BF16, NM_FP32 = 0, 1
NM_ACT, NM_WEIGHT = 0, 1
NM_OK, NM_ERR_INVALID_ARG, NM_ERR_UNSUPPORTED, NM_ERR_ALIGNMENT = 0, 1, 2, 3
NM_ERR_CUDA, NM_ERR_DEVICE_TIMEOUT, NM_ERR_WORKSPACE = 4, 5, 6


class NmError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({lib().nm_status_string(status).decode()})"
                         + (f", cudaError {lib().nm_last_cuda_error()}" if status == NM_ERR_CUDA else ""))


class SparseOperand(ctypes.Structure):
    _fields_ = [("vals", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("K", ctypes.c_int64), ("N", ctypes.c_int32), ("M", ctypes.c_int32),
                ("K_lift", ctypes.c_int64)]


class SpenseMlpStruct(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("ug_vals", ctypes.c_void_p), ("ug_meta", ctypes.c_void_p),
                ("ug_dense", ctypes.c_void_p), ("down_vals", ctypes.c_void_p), ("down_meta", ctypes.c_void_p),
                ("down_dense", ctypes.c_void_p), ("d", ctypes.c_int64), ("I", ctypes.c_int64), ("D", ctypes.c_int64)]


class HybridWeight(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("vals_s", ctypes.c_void_p), ("meta_s", ctypes.c_void_p),
                ("W_d", ctypes.c_void_p), ("O", ctypes.c_int64), ("K", ctypes.c_int64),
                ("K_dense", ctypes.c_int64)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m semi_structured_sparse_nm_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
        sigs = {
            "nm_lifted_k": (I64, [I64, I]),
            "nm_meta_bytes": (SZ, [I64, I64, I]),
            "nm_prune_compress": (I, [P, I, I64, I64, I64, I, I, P, P, P, P]),
            "slide_decompose": (I, [P, I, I64, I64, I, I, P, P, P, P]),
            "nm_lift": (I, [P, I, I64, I64, I64, I, P, P]),
            "slide_decompose_split": (I, [P, I64, I64, I, I, P, P, P, P]),
            "nm_lift_odd": (I, [P, I64, I64, I64, I, P]),
            "nm_sparse_gemm_workspace_size": (SZ, [ctypes.POINTER(SparseOperand), I64, I]),
            "nm_sparse_gemm": (I, [ctypes.POINTER(SparseOperand), P, I64, I, P, I, P, SZ, P]),
            "slide_gemm_workspace_size": (SZ, [ctypes.POINTER(SparseOperand), I64]),
            "slide_gemm": (I, [ctypes.POINTER(SparseOperand), P, I64, I64, P, I, P, SZ, P]),
            "nm_dense_gemm": (I, [P, I64, P, I64, I64, P, I, P]),
            "nm_quant_lift_fp8": (I, [P, I, I64, I64, I64, I, P, P, P]),
            "nm_prune_compress_fp8": (I, [P, I64, I64, I64, I, I, P, P, P, P, P]),
            "slide_decompose_fp8_workspace_size": (SZ, [I64, I64, I]),
            "slide_decompose_fp8": (I, [P, I64, I64, I, I, P, P, P, P, SZ, P]),
            "nm_sparse_gemm_fp8": (I, [ctypes.POINTER(SparseOperand), P, P, P, I64, I, P, I, P]),
            "hybrid_dense_count": (I64, [I64, D]),
            "hybrid_prepare_workspace_size": (SZ, [I64, I64]),
            "hybrid_prepare": (I, [P, I64, I64, D, ctypes.POINTER(HybridWeight), P, SZ, P]),
            "hybrid_gemm_workspace_size": (SZ, [ctypes.POINTER(HybridWeight), I64]),
            "hybrid_gemm": (I, [P, I64, ctypes.POINTER(HybridWeight), P, I, P, SZ, P]),
            "hybrid_gemm_noalloc": (I, [P, I64, ctypes.POINTER(HybridWeight), P, I, P]),
            "spense_dense_count": (I64, [I64, D]),
            "spense_mlp_prepare_workspace_size": (SZ, [I64, I64]),
            "spense_mlp_prepare": (I, [P, P, P, D, ctypes.POINTER(SpenseMlpStruct), P, SZ, P]),
            "spense_mlp_workspace_size": (SZ, [ctypes.POINTER(SpenseMlpStruct), I64]),
            "spense_mlp": (I, [P, I64, ctypes.POINTER(SpenseMlpStruct), P, P, SZ, P]),
            "nm_prune_compress_xf_workspace_size": (SZ, [I64, I64, I]),
            "nm_prune_compress_xf": (I, [P, I64, I64, I64, I, I, ctypes.c_uint, P, P, P, P, P, P, SZ, P]),
            "nm_row_sums": (I, [P, I64, I64, I64, P, P]),
            "nm_sparse_gemm_xf": (I, [ctypes.POINTER(SparseOperand), P, I64, P, P, P, P, I, P]),
            "nm_act_sparse_linear_host_workspace_size": (SZ, [I64, I64, I, I, I64, I64]),
            "nm_act_sparse_linear_host": (I, [P, I64, I64, I, I, P, I64, P, I64, P, SZ, P]),
            "nm_mma_rate_probe": (I, [I, I, ctypes.POINTER(ctypes.c_double), P]),
            "nm_status_string": (ctypes.c_char_p, [I]),
            "nm_last_cuda_error": (I, []),
            "nm_last_gemm_kernel": (ctypes.c_char_p, []),
            "nm_get_device_error": (I, [P]),
            "nm_debug_expire_wait": (I, [ctypes.c_uint, P]),
            "nm_debug_fail_next_launch": (I, [I]),
            "nm_version": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sigs.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != NM_OK:
        raise NmError(fn, status)


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else None
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return NM_BF16
    if t.dtype == torch.float32:
        return NM_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")


# ------------------------------------------------------------------ sizes


def lifted_k(K: int, M: int) -> int:
    return int(lib().nm_lifted_k(K, M))


def meta_bytes(rows: int, K: int, M: int) -> int:
    return int(lib().nm_meta_bytes(rows, K, M))


def hybrid_dense_count(K: int, dense_frac: float) -> int:
    return int(lib().hybrid_dense_count(K, dense_frac))


# ---------------------------------------------------------------- prune


class Compressed:
    """A window-compressed sparse operand living on the device."""

    def __init__(self, vals, meta, rows, K, N, M, mask=None):
        self.vals, self.meta, self.mask = vals, meta, mask
        self.rows, self.K, self.N, self.M = rows, K, N, M
        self.K_lift = lifted_k(K, M)

    def struct(self) -> SparseOperand:
        return SparseOperand(self.vals.data_ptr(), self.meta.data_ptr(), self.rows, self.K,
                             self.N, self.M, self.K_lift)


def alloc_compressed(rows: int, K: int, N: int, M: int, device, with_mask=False) -> Compressed:
    Kl = lifted_k(K, M)
    if Kl < 0:
        raise ValueError(f"M={M} does not divide K={K}")
    vals = torch.empty((rows, Kl // 2), dtype=torch.bfloat16, device=device)
    meta = torch.empty(max(meta_bytes(rows, K, M), 16), dtype=torch.uint8, device=device)
    mask = torch.empty((rows, (K + 31) // 32), dtype=torch.int32, device=device) if with_mask else None
    return Compressed(vals, meta, rows, K, N, M, mask)


def prune_compress(x: torch.Tensor, N: int, M: int, out: Compressed | None = None,
                   with_mask: bool = False) -> Compressed:
    _need_cuda(x)
    rows, K = x.shape
    if out is None:
        out = alloc_compressed(rows, K, N, M, x.device, with_mask)
    _check("nm_prune_compress", lib().nm_prune_compress(
        _p(x), _dt(x), rows, K, x.stride(0), N, M, _p(out.mask), _p(out.vals), _p(out.meta), _stream(x)))
    return out


def slide_decompose(w: torch.Tensor, N: int, M: int, with_mask: bool = False) -> Compressed:
    _need_cuda(w)
    rows, K = w.shape
    out = alloc_compressed(rows, K, N, M, w.device, with_mask)
    if w.stride(0) != K:
        raise ValueError("slide_decompose expects a contiguous weight")
    _check("slide_decompose", lib().slide_decompose(
        _p(w), _dt(w), rows, K, N, M, _p(out.mask), _p(out.vals), _p(out.meta), _stream(w)))
    return out


def slide_decompose_split(w: torch.Tensor, N: int, M: int, with_mask: bool = False) -> Compressed:
    """slide_decompose() with every row's windows in the split order (each
    group's even windows, then its odd ones); multiply it by lifted
    activations in the same order (lift_odd())."""
    _need_cuda(w)
    rows, K = w.shape
    if w.stride(0) != K or w.dtype != torch.bfloat16:
        raise ValueError("slide_decompose_split expects a contiguous bf16 weight")
    out = alloc_compressed(rows, K, N, M, w.device, with_mask)
    _check("slide_decompose_split", lib().slide_decompose_split(
        _p(w), rows, K, N, M, _p(out.mask), _p(out.vals), _p(out.meta), _stream(w)))
    return out


def lift_odd(x_wide: torch.Tensor, K: int, M: int) -> torch.Tensor:
    """In place: x_wide bf16 [rows, >= K'] holds X in its first K columns;
    columns [K, K') receive X's odd windows (the split order).  Returns
    x_wide[:, :K'], the dense operand for a slide_decompose_split() weight."""
    _need_cuda(x_wide)
    rows = x_wide.shape[0]
    Kl = lifted_k(K, M)
    _check("nm_lift_odd", lib().nm_lift_odd(_p(x_wide), rows, K, x_wide.stride(0), M, _stream(x_wide)))
    return x_wide[:, :Kl]


def lift(src: torch.Tensor, M: int, out: torch.Tensor | None = None) -> torch.Tensor:
    _need_cuda(src)
    rows, K = src.shape
    Kl = lifted_k(K, M)
    if out is None:
        out = torch.empty((rows, Kl), dtype=torch.bfloat16, device=src.device)
    _check("nm_lift", lib().nm_lift(_p(src), _dt(src), rows, K, src.stride(0), M, _p(out), _stream(src)))
    return out


# ----------------------------------------------------------------- GEMM


def sparse_gemm_workspace_size(S: Compressed, rows_d: int, side: int) -> int:
    st = S.struct()
    return int(lib().nm_sparse_gemm_workspace_size(ctypes.byref(st), rows_d, side))


def sparse_gemm(S: Compressed, D: torch.Tensor, side: int, out_dtype=torch.bfloat16,
                out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """side NM_ACT: Y [S.rows, D.rows]; NM_WEIGHT: Y [D.rows, S.rows]."""
    _need_cuda(D)
    rows_d = D.shape[0]
    if D.dtype != torch.bfloat16 or D.shape[1] != S.K_lift or not D.is_contiguous():
        raise ValueError("dense operand must be contiguous bf16 [rows, K_lift]")
    shape = (S.rows, rows_d) if side == NM_ACT else (rows_d, S.rows)
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=D.device)
    st = S.struct()
    ws_bytes = int(lib().nm_sparse_gemm_workspace_size(ctypes.byref(st), rows_d, side))
    if ws_bytes and (ws is None or ws.numel() < ws_bytes):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=D.device)
    _check("nm_sparse_gemm", lib().nm_sparse_gemm(
        ctypes.byref(st), _p(D), rows_d, side, _p(out), _dt(out), _p(ws if ws_bytes else None), ws_bytes,
        _stream(D)))
    return out


def slide_gemm_workspace_size(W: Compressed, rows_x: int) -> int:
    st = W.struct()
    return int(lib().slide_gemm_workspace_size(ctypes.byref(st), rows_x))


def slide_gemm(W: Compressed, X: torch.Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
               ws: torch.Tensor | None = None) -> torch.Tensor:
    """Y [X.rows, W.rows] = lift(X) . W_c^T from the raw (unlifted) bf16 X."""
    _need_cuda(X)
    rows_x = X.shape[0]
    if X.dtype != torch.bfloat16 or X.shape[1] != W.K or X.stride(1) != 1:
        raise ValueError("X must be bf16 [rows, K] with unit column stride")
    if out is None:
        out = torch.empty((rows_x, W.rows), dtype=out_dtype, device=X.device)
    st = W.struct()
    ws_bytes = int(lib().slide_gemm_workspace_size(ctypes.byref(st), rows_x))
    if ws_bytes and (ws is None or ws.numel() < ws_bytes):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=X.device)
    _check("slide_gemm", lib().slide_gemm(ctypes.byref(st), _p(X), rows_x, X.stride(0), _p(out), _dt(out),
                                          _p(ws if ws_bytes else None), ws_bytes, _stream(X)))
    return out


def dense_gemm(A: torch.Tensor, B: torch.Tensor, out_dtype=torch.bfloat16, out=None) -> torch.Tensor:
    _need_cuda(A, B)
    if not (A.is_contiguous() and B.is_contiguous()):
        raise ValueError("contiguous operands expected")
    if out is None:
        out = torch.empty((A.shape[0], B.shape[0]), dtype=out_dtype, device=A.device)
    _check("nm_dense_gemm", lib().nm_dense_gemm(_p(A), A.shape[0], _p(B), B.shape[0], A.shape[1], _p(out),
                                                _dt(out), _stream(A)))
    return out


# ------------------------------------------ per-token activation corrections

NM_XF_SHIFT, NM_XF_VAR = 1, 2


class XfOperand:
    """An activation operand pruned with the per-token corrections: the
    compressed shifted token plus its VAR factor and shift (fp32 per row)."""

    def __init__(self, comp: Compressed, row_scale: torch.Tensor, row_shift: torch.Tensor, flags: int,
                 ws: torch.Tensor | None):
        self.comp, self.row_scale, self.row_shift, self.flags, self.ws = comp, row_scale, row_shift, flags, ws


def alloc_xf(rows: int, K: int, N: int, M: int, flags: int, device, with_mask=False) -> XfOperand:
    comp = alloc_compressed(rows, K, N, M, device, with_mask)
    ws_bytes = int(lib().nm_prune_compress_xf_workspace_size(rows, K, M)) if flags & NM_XF_VAR else 0
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device) if ws_bytes else None
    f = lambda: torch.empty(rows, dtype=torch.float32, device=device)
    return XfOperand(comp, f(), f(), flags, ws)


def prune_compress_xf(x: torch.Tensor, N: int, M: int, flags: int, out: XfOperand | None = None,
                      with_mask: bool = False) -> XfOperand:
    """Prune + compress of the bf16 activation with NM_XF_SHIFT (D-PTS) and/or
    NM_XF_VAR applied."""
    _need_cuda(x)
    rows, K = x.shape
    if out is None:
        out = alloc_xf(rows, K, N, M, flags, x.device, with_mask)
    c = out.comp
    ws_bytes = out.ws.numel() if out.ws is not None else 0
    _check("nm_prune_compress_xf", lib().nm_prune_compress_xf(
        _p(x), rows, K, x.stride(0), N, M, flags, _p(c.mask), _p(c.vals), _p(c.meta), _p(out.row_scale),
        _p(out.row_shift), _p(out.ws), ws_bytes, _stream(x)))
    return out


def row_sums(w: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 row sums of a bf16 matrix (fp64 accumulation)."""
    _need_cuda(w)
    rows, K = w.shape
    if out is None:
        out = torch.empty(rows, dtype=torch.float32, device=w.device)
    _check("nm_row_sums", lib().nm_row_sums(_p(w), rows, K, w.stride(0), _p(out), _stream(w)))
    return out


def sparse_gemm_xf(X: XfOperand, W_lift: torch.Tensor, w_row_sums: torch.Tensor, out_dtype=torch.bfloat16,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = (X_c . W'^T) * row_scale + row_shift * w_row_sums (activation side)."""
    _need_cuda(W_lift, w_row_sums)
    S = X.comp
    rows_w = W_lift.shape[0]
    if W_lift.dtype != torch.bfloat16 or W_lift.shape[1] != S.K_lift or not W_lift.is_contiguous():
        raise ValueError("lifted weight must be contiguous bf16 [rows, K_lift]")
    if w_row_sums.dtype != torch.float32 or w_row_sums.numel() != rows_w:
        raise ValueError("w_row_sums must be fp32 [rows of W]")
    if out is None:
        out = torch.empty((S.rows, rows_w), dtype=out_dtype, device=W_lift.device)
    st = S.struct()
    _check("nm_sparse_gemm_xf", lib().nm_sparse_gemm_xf(
        ctypes.byref(st), _p(W_lift), rows_w, _p(X.row_scale), _p(X.row_shift), _p(w_row_sums), _p(out),
        _dt(out), _stream(W_lift)))
    return out


# ------------------------------------------------- host-buffer pipeline


def act_sparse_linear_host_workspace(T: int, K: int, N: int, M: int, O: int, device, chunk_rows: int = 0):
    n = int(lib().nm_act_sparse_linear_host_workspace_size(T, K, N, M, O, chunk_rows))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def act_sparse_linear_host(x_host: torch.Tensor, W_lift: torch.Tensor, N: int, M: int, y_host: torch.Tensor,
                           ws: torch.Tensor | None = None, chunk_rows: int = 0) -> torch.Tensor:
    """y_host = prune_{N:M}(x_host) . W^T with x_host, y_host bf16 tensors in
    (page-locked) host memory and the lifted weight on the device; chunked
    copies in and out overlap the math.  Asynchronous on the current stream:
    keep x_host and y_host alive until the stream has passed the call."""
    _need_cuda(W_lift)
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host live in host memory")
    for t in (x_host, y_host):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("contiguous bf16 host tensors expected")
    T, K = x_host.shape
    O = W_lift.shape[0]
    if tuple(y_host.shape) != (T, O):
        raise ValueError("y_host must be [T, O]")
    if ws is None:
        ws = act_sparse_linear_host_workspace(T, K, N, M, O, W_lift.device, chunk_rows)
    _check("nm_act_sparse_linear_host", lib().nm_act_sparse_linear_host(
        ctypes.c_void_p(x_host.data_ptr()), T, K, N, M, _p(W_lift), O, ctypes.c_void_p(y_host.data_ptr()),
        chunk_rows, _p(ws), ws.numel(), _stream(W_lift)))
    return y_host


# ---------------------------------------------------------- 8-bit (E4M3)


class Fp8Operand:
    """Per-row E4M3 codes with their fp32 scales; `lifted` codes for the
    dense side, window-compressed codes + 8-bit metadata for the sparse side."""

    def __init__(self, codes, scale, rows, K, N, M, meta=None):
        self.codes, self.scale, self.meta = codes, scale, meta
        self.rows, self.K, self.N, self.M = rows, K, N, M
        self.K_lift = lifted_k(K, M)

    def struct(self) -> SparseOperand:
        return SparseOperand(self.codes.data_ptr(), self.meta.data_ptr(), self.rows, self.K,
                             self.N, self.M, self.K_lift)


def quant_lift_fp8(x: torch.Tensor, M: int, out: Fp8Operand | None = None) -> Fp8Operand:
    """Per-token E4M3 quantisation fused with the lift: codes [rows, K'] and
    scales [rows]."""
    _need_cuda(x)
    rows, K = x.shape
    Kl = lifted_k(K, M)
    if out is None:
        out = Fp8Operand(torch.empty((rows, Kl), dtype=torch.uint8, device=x.device),
                         torch.empty(rows, dtype=torch.float32, device=x.device), rows, K, 0, M)
    _check("nm_quant_lift_fp8", lib().nm_quant_lift_fp8(
        _p(x), _dt(x), rows, K, x.stride(0), M, _p(out.codes), _p(out.scale), _stream(x)))
    return out


def prune_compress_fp8(x: torch.Tensor, N: int, M: int, out: Fp8Operand | None = None,
                       with_mask: bool = False) -> Fp8Operand:
    """Per-token scales, then N:M prune + window compress with the kept values
    as E4M3 codes and the 8-bit metadata image (bf16 input)."""
    _need_cuda(x)
    rows, K = x.shape
    if x.dtype != torch.bfloat16:
        raise ValueError("prune_compress_fp8 expects bf16 input")
    if out is None:
        Kl = lifted_k(K, M)
        out = Fp8Operand(torch.empty((rows, Kl // 2), dtype=torch.uint8, device=x.device),
                         torch.empty(rows, dtype=torch.float32, device=x.device), rows, K, N, M,
                         torch.empty(max(meta_bytes(rows, K, M), 16), dtype=torch.uint8, device=x.device))
    mask = torch.empty((rows, (K + 31) // 32), dtype=torch.int32, device=x.device) if with_mask else None
    out.mask = mask
    _check("nm_prune_compress_fp8", lib().nm_prune_compress_fp8(
        _p(x), rows, K, x.stride(0), N, M, _p(mask), _p(out.codes), _p(out.scale), _p(out.meta), _stream(x)))
    return out


def slide_decompose_fp8(w: torch.Tensor, N: int, M: int) -> Fp8Operand:
    """Offline 8-bit weight packing: window-compressed codes, per-row scales,
    8-bit metadata image."""
    _need_cuda(w)
    rows, K = w.shape
    if w.dtype != torch.bfloat16 or w.stride(0) != K:
        raise ValueError("slide_decompose_fp8 expects a contiguous bf16 weight")
    Kl = lifted_k(K, M)
    codes = torch.empty((rows, Kl // 2), dtype=torch.uint8, device=w.device)
    scale = torch.empty(rows, dtype=torch.float32, device=w.device)
    meta = torch.empty(max(meta_bytes(rows, K, M), 16), dtype=torch.uint8, device=w.device)
    ws_bytes = int(lib().slide_decompose_fp8_workspace_size(rows, K, M))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=w.device)
    _check("slide_decompose_fp8", lib().slide_decompose_fp8(
        _p(w), rows, K, N, M, _p(codes), _p(scale), _p(meta), _p(ws), ws_bytes, _stream(w)))
    return Fp8Operand(codes, scale, rows, K, N, M, meta)


def sparse_gemm_fp8(S: Fp8Operand, D: Fp8Operand, side: int, out_dtype=torch.bfloat16,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """8-bit sparse product rescaled by both operands' row scales;
    side NM_ACT: Y [S.rows, D.rows]; NM_WEIGHT: Y [D.rows, S.rows]."""
    _need_cuda(D.codes)
    rows_d = D.rows
    if D.codes.shape[1] != S.K_lift or not D.codes.is_contiguous():
        raise ValueError("dense operand must be contiguous codes [rows, K_lift]")
    shape = (S.rows, rows_d) if side == NM_ACT else (rows_d, S.rows)
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=D.codes.device)
    st = S.struct()
    _check("nm_sparse_gemm_fp8", lib().nm_sparse_gemm_fp8(
        ctypes.byref(st), _p(S.scale), _p(D.codes), _p(D.scale), rows_d, side, _p(out), _dt(out),
        _stream(D.codes)))
    return out


# --------------------------------------------------------------- hybrid


class Hybrid:
    def __init__(self, perm, vals_s, meta_s, W_d, O, K, K_dense):
        self.perm, self.vals_s, self.meta_s, self.W_d = perm, vals_s, meta_s, W_d
        self.O, self.K, self.K_dense = O, K, K_dense

    def struct(self) -> HybridWeight:
        return HybridWeight(self.perm.data_ptr(), _p(self.vals_s).value or 0, _p(self.meta_s).value or 0,
                            _p(self.W_d).value or 0, self.O, self.K, self.K_dense)


def hybrid_prepare(w: torch.Tensor, dense_frac: float) -> Hybrid:
    _need_cuda(w)
    O, K = w.shape
    D = hybrid_dense_count(K, dense_frac)
    Ks = K - D
    dev = w.device
    h = Hybrid(torch.empty(K, dtype=torch.int32, device=dev),
               torch.empty((O, Ks // 2), dtype=torch.bfloat16, device=dev) if Ks else None,
               torch.empty(max(meta_bytes(O, Ks, 4), 16), dtype=torch.uint8, device=dev) if Ks else None,
               torch.empty((O, D), dtype=torch.bfloat16, device=dev) if D else None, O, K, D)
    ws_bytes = int(lib().hybrid_prepare_workspace_size(O, K))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = h.struct()
    _check("hybrid_prepare", lib().hybrid_prepare(_p(w), O, K, dense_frac, ctypes.byref(st), _p(ws), ws_bytes,
                                                  _stream(w)))
    return h


def hybrid_gemm(x: torch.Tensor, h: Hybrid, out_dtype=torch.bfloat16, out=None, ws=None) -> torch.Tensor:
    _need_cuda(x)
    B = x.shape[0]
    if out is None:
        out = torch.empty((B, h.O), dtype=out_dtype, device=x.device)
    st = h.struct()
    ws_bytes = int(lib().hybrid_gemm_workspace_size(ctypes.byref(st), B))
    if ws is None:
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    _check("hybrid_gemm", lib().hybrid_gemm(_p(x), B, ctypes.byref(st), _p(out), _dt(out), _p(ws), ws.numel(),
                                            _stream(x)))
    return out


NOALLOC_SCRATCH_BYTES = 2 * 1024 * 1024


def hybrid_gemm_noalloc(x: torch.Tensor, h: Hybrid, out_dtype=torch.bfloat16, out=None) -> torch.Tensor:
    """hybrid_gemm() through the entry point that allocates nothing: its scratch
    is the library's built-in array (B * K * 2 bytes at most 2 MiB)."""
    _need_cuda(x)
    B = x.shape[0]
    if out is None:
        out = torch.empty((B, h.O), dtype=out_dtype, device=x.device)
    st = h.struct()
    _check("hybrid_gemm_noalloc", lib().hybrid_gemm_noalloc(_p(x), B, ctypes.byref(st), _p(out), _dt(out),
                                                            _stream(x)))
    return out


# ----------------------------------------------------------- diagnostics


def device_error(stream=None) -> int:
    s = stream if stream is not None else _stream()
    return int(lib().nm_get_device_error(s))


def mma_rate_probe(mode: int, iters: int = 4000, reps: int = 5) -> float:
    """Tensor-core rate in TFLOP/s (dense-equivalent) of back-to-back MMAs from
    shared memory on every SM pair: mode 0 bf16 dense, 1 bf16 2:4 sparse,
    2 E4M3 2:4 sparse.  Best of `reps` timed launches after one warm-up."""
    st = _stream()
    flops = ctypes.c_double(0.0)
    _check("nm_mma_rate_probe", lib().nm_mma_rate_probe(mode, iters, ctypes.byref(flops), st))
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        _check("nm_mma_rate_probe", lib().nm_mma_rate_probe(mode, iters, ctypes.byref(flops), st))
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return flops.value / (best * 1e-3) / 1e12


def debug_fail_next_launch(cuda_error: int):
    _check("nm_debug_fail_next_launch", lib().nm_debug_fail_next_launch(cuda_error))


def last_cuda_error() -> int:
    return int(lib().nm_last_cuda_error())


def last_gemm_kernel() -> str:
    """The GEMM kernel instantiation the latest GEMM call on this thread launched."""
    return lib().nm_last_gemm_kernel().decode()


def debug_expire_wait(timeout_us: int):
    _check("nm_debug_expire_wait", lib().nm_debug_expire_wait(timeout_us, _stream()))


# ------------------------------------------------------- hybrid GLU MLP


class SpenseMlp:
    """A GLU MLP in the hybrid format (device buffers)."""

    def __init__(self, perm, ug_vals, ug_meta, ug_dense, down_vals, down_meta, down_dense, d, I, D):
        self.perm, self.ug_vals, self.ug_meta, self.ug_dense = perm, ug_vals, ug_meta, ug_dense
        self.down_vals, self.down_meta, self.down_dense = down_vals, down_meta, down_dense
        self.d, self.I, self.D = d, I, D

    def struct(self) -> SpenseMlpStruct:
        return SpenseMlpStruct(_p(self.perm), _p(self.ug_vals), _p(self.ug_meta), _p(self.ug_dense),
                               _p(self.down_vals), _p(self.down_meta), _p(self.down_dense), self.d, self.I, self.D)


def spense_dense_count(I: int, dense_frac: float) -> int:
    return int(lib().spense_dense_count(I, dense_frac))


def spense_mlp_prepare(w_up: torch.Tensor, w_gate: torch.Tensor, w_down: torch.Tensor,
                       dense_frac: float) -> SpenseMlp:
    """Offline: dense intermediate set, permutation, packed up/gate (output
    split) and down (input split)."""
    _need_cuda(w_up, w_gate, w_down)
    I, d = w_up.shape
    if w_gate.shape != (I, d) or w_down.shape != (d, I):
        raise ValueError("expected W_up, W_gate [I, d] and W_down [d, I]")
    for t in (w_up, w_gate, w_down):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("contiguous bf16 weights expected")
    D = spense_dense_count(I, dense_frac)
    Is = I - D
    dev = w_up.device
    e = lambda *shape, dt=torch.bfloat16: torch.empty(shape, dtype=dt, device=dev)
    W = SpenseMlp(e(I, dt=torch.int32),
                  e(2 * Is, d // 2) if Is else None, e(max(meta_bytes(2 * Is, d, 4), 16), dt=torch.uint8) if Is else None,
                  e(2 * D, d) if D else None,
                  e(d, Is // 2) if Is else None, e(max(meta_bytes(d, Is, 4), 16), dt=torch.uint8) if Is else None,
                  e(d, D) if D else None, d, I, D)
    ws_bytes = int(lib().spense_mlp_prepare_workspace_size(d, I))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = W.struct()
    _check("spense_mlp_prepare", lib().spense_mlp_prepare(_p(w_up), _p(w_gate), _p(w_down), dense_frac,
                                                          ctypes.byref(st), _p(ws), ws_bytes, _stream(w_up)))
    return W


def spense_mlp_workspace_size(W: SpenseMlp, B: int) -> int:
    """Bytes of scratch spense_mlp() needs for a batch of B tokens."""
    return int(lib().spense_mlp_workspace_size(ctypes.byref(W.struct()), B))


def spense_mlp(x: torch.Tensor, W: SpenseMlp, out: torch.Tensor | None = None, ws=None) -> torch.Tensor:
    """y = (silu(x . W_gate^T) * (x . W_up^T)) . W_down^T through the packed weights."""
    _need_cuda(x)
    B = x.shape[0]
    if x.dtype != torch.bfloat16 or x.shape[1] != W.d or not x.is_contiguous():
        raise ValueError("x must be contiguous bf16 [B, d]")
    if out is None:
        out = torch.empty((B, W.d), dtype=torch.bfloat16, device=x.device)
    st = W.struct()
    ws_bytes = spense_mlp_workspace_size(W, B)
    if ws is None:
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    _check("spense_mlp", lib().spense_mlp(_p(x), B, ctypes.byref(st), _p(out), _p(ws), ws_bytes, _stream(x)))
    return out
