"""CPU oracle for N:M semi-structured sparse linear layers (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA path shares no code with it and
never calls it.

The arithmetic lives in ``nm_oracle.c`` (plain loops, fp64 sums); this module
compiles it with gcc on first use and marshals numpy arrays through ctypes.
Every function states the step of the method it follows; the pages are cited
in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16, FP32 = 0, 1


def build(force: bool = False) -> str:
    """Compile nm_oracle.c into liboracle.so (gcc -O2 -fopenmp)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call([
                "gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                "-Wall", "-Wextra", "-Wno-unused-parameter", _SRC, "-o", tmp, "-lm",
            ])
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "or_prune": (I, [P, I, I64, I64, I, I, P]),
            "or_mask_pack": (None, [P, I64, I64, P]),
            "or_window_assign_batch": (None, [P, I64, I, P, P, P]),
            "or_lifted_k": (I64, [I64, I]),
            "or_compress": (I, [P, I, I64, I64, I, P, P, P]),
            "or_expand_lifted": (None, [P, P, I64, I64, P]),
            "or_decompress": (None, [P, P, I64, I64, I, P]),
            "or_meta_hw_bytes": (I64, [I64, I64]),
            "or_meta_hw": (None, [P, I64, I64, P]),
            "or_lift": (I, [P, I, I64, I64, I, P]),
            "or_to_f64": (None, [P, I, I64, P, P]),
            "or_linear_f64": (None, [P, P, I64, I64, I64, P, I64, P]),
            "or_colnorm_f64": (None, [P, I, I64, I64, P]),
            "or_rownorm_f64": (None, [P, I, I64, I64, P]),
            "or_silu_f64": (None, [P, I64, P]),
            "or_hybrid_dense_count": (I64, [I64, ctypes.c_double]),
            "or_hybrid_perm": (None, [P, I64, I64, P, P]),
            "or_gather_cols_bf16": (None, [P, I64, I64, P, P]),
            "or_num_threads": (I, []),
            "or_e4m3_to_f64": (ctypes.c_double, [ctypes.c_uint8]),
            "or_e4m3_from_f32": (ctypes.c_uint8, [ctypes.c_float]),
            "or_quant_rows_e4m3": (None, [P, I, I64, I64, P, P]),
            "or_quant_vals_e4m3": (None, [P, I64, I64, P, P]),
            "or_lift_u8": (I, [P, I64, I64, I, P]),
            "or_meta8": (None, [P, I64, I64, P]),
            "or_row_mean": (None, [P, I, I64, I64, P, P]),
            "or_shift_bf16": (None, [P, I, I64, I64, P, P]),
            "or_var_scale": (None, [P, I, P, P, I64, I64, P]),
            "or_rowsum_f64": (None, [P, I, I64, I64, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype, f.argtypes = res, args
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle expects C-contiguous arrays"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dt(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return FP32
    raise TypeError(f"oracle inputs are bf16 bits (uint16) or float32, got {x.dtype}")


def _as_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    return x.view(np.uint32) if x.dtype == np.float32 else x


def num_threads() -> int:
    return int(_load().or_num_threads())


# ------------------------------------------------------------------ prune


def prune(x: np.ndarray, N: int, M: int) -> np.ndarray:
    """Keep mask (uint8 0/1, same shape as x): top-N |x| per aligned group of M
    along the last axis, ties to the lower index."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    keep = np.zeros((rows, K), np.uint8)
    rc = _load().or_prune(_ptr(_as_bits(x)), _dt(x), rows, K, N, M, _ptr(keep))
    if rc != 0:
        raise ValueError(f"or_prune rejected N={N} M={M} K={K}")
    return keep


def mask_pack(keep: np.ndarray) -> np.ndarray:
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    rows, K = keep.shape
    out = np.zeros((rows, (K + 31) // 32), np.uint32)
    _load().or_mask_pack(_ptr(keep), rows, K, _ptr(out))
    return out


# ---------------------------------------------------------------- windows


def window_assign_batch(masks: np.ndarray, M: int):
    """Greedy window assignment for many single-group masks (bit i = position i).
    Returns (win[count, M], slot[count, M], status[count])."""
    masks = np.ascontiguousarray(masks, dtype=np.uint64)
    cnt = masks.shape[0]
    win = np.zeros((cnt, M), np.int8)
    slot = np.zeros((cnt, M), np.int8)
    st = np.zeros(cnt, np.int8)
    _load().or_window_assign_batch(_ptr(masks), cnt, M, _ptr(win), _ptr(slot), _ptr(st))
    return win, slot, st


def lifted_k(K: int, M: int) -> int:
    return int(_load().or_lifted_k(K, M))


def compress(x: np.ndarray, keep: np.ndarray, M: int):
    """Window-compressed values (bf16 bits [rows, K'/2]) and canonical nibbles
    ([rows, K'/4], one per byte)."""
    x = np.ascontiguousarray(x)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    rows, K = x.shape
    Kl = lifted_k(K, M)
    vals = np.zeros((rows, Kl // 2), np.uint16)
    nib = np.zeros((rows, Kl // 4), np.uint8)
    rc = _load().or_compress(_ptr(_as_bits(x)), _dt(x), rows, K, M, _ptr(keep), _ptr(vals), _ptr(nib))
    if rc != 0:
        raise ValueError(f"or_compress failed ({rc})")
    return vals, nib


def expand_lifted(vals: np.ndarray, nib: np.ndarray) -> np.ndarray:
    rows, half = vals.shape
    Kl = half * 2
    out = np.zeros((rows, Kl), np.float64)
    _load().or_expand_lifted(_ptr(np.ascontiguousarray(vals)), _ptr(np.ascontiguousarray(nib)),
                             rows, Kl, _ptr(out))
    return out


def decompress(vals: np.ndarray, nib: np.ndarray, K: int, M: int) -> np.ndarray:
    rows = vals.shape[0]
    out = np.zeros((rows, K), np.uint16)
    _load().or_decompress(_ptr(np.ascontiguousarray(vals)), _ptr(np.ascontiguousarray(nib)),
                          rows, K, M, _ptr(out))
    return out


def meta_hw(nib: np.ndarray, Kl: int) -> np.ndarray:
    nib = np.ascontiguousarray(nib, dtype=np.uint8)
    rows = nib.shape[0]
    nbytes = int(_load().or_meta_hw_bytes(rows, Kl))
    out = np.zeros(nbytes, np.uint8)
    _load().or_meta_hw(_ptr(nib), rows, Kl, _ptr(out))
    return out


def lift(src: np.ndarray, M: int) -> np.ndarray:
    src = np.ascontiguousarray(src)
    rows, K = src.shape
    Kl = lifted_k(K, M)
    out = np.zeros((rows, Kl), np.uint16)
    rc = _load().or_lift(_ptr(_as_bits(src)), _dt(src), rows, K, M, _ptr(out))
    if rc != 0:
        raise ValueError("or_lift rejected the shape")
    return out


# ----------------------------------------------------------------- linear


def to_f64(x: np.ndarray, keep: np.ndarray | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x)
    out = np.zeros(x.shape, np.float64)
    kp = _ptr(np.ascontiguousarray(keep, dtype=np.uint8)) if keep is not None else None
    _load().or_to_f64(_ptr(_as_bits(x)), _dt(x), x.size, kp, _ptr(out))
    return out


def linear_f64(A: np.ndarray, B: np.ndarray, rows=None) -> np.ndarray:
    """Y[t, o] = sum_k A[t, k] * B[o, k], k ascending, fp64.  ``rows`` selects
    a subset of t (the result then has len(rows) rows)."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    T, K = A.shape
    O = B.shape[0]
    assert B.shape[1] == K
    if rows is None:
        Y = np.zeros((T, O), np.float64)
        _load().or_linear_f64(_ptr(A), _ptr(B), T, O, K, None, 0, _ptr(Y))
    else:
        sel = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        Y = np.zeros((sel.size, O), np.float64)
        _load().or_linear_f64(_ptr(A), _ptr(B), T, O, K, _ptr(sel), sel.size, _ptr(Y))
    return Y


# ----------------------------------------------------------------- hybrid


def colnorm_f64(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w)
    O, K = w.shape
    out = np.zeros(K, np.float64)
    _load().or_colnorm_f64(_ptr(_as_bits(w)), _dt(w), O, K, _ptr(out))
    return out


def hybrid_dense_count(K: int, dense_frac: float) -> int:
    return int(_load().or_hybrid_dense_count(K, float(dense_frac)))


def hybrid_perm(colnorm: np.ndarray, D: int):
    colnorm = np.ascontiguousarray(colnorm, dtype=np.float64)
    K = colnorm.size
    perm = np.zeros(K, np.int32)
    dense = np.zeros(K, np.uint8)
    _load().or_hybrid_perm(_ptr(colnorm), K, D, _ptr(perm), _ptr(dense))
    return perm, dense


def gather_cols(w: np.ndarray, perm: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, K = w.shape
    out = np.zeros_like(w)
    _load().or_gather_cols_bf16(_ptr(w), rows, K, _ptr(np.ascontiguousarray(perm, dtype=np.int32)),
                                _ptr(out))
    return out


# ------------------------------------------------------ composite references


def sparse_operand(x: np.ndarray, N: int, M: int):
    """Everything the prune + compress step produces for one operand:
    keep mask, packed bit mask, values, canonical nibbles, hardware metadata."""
    keep = prune(x, N, M)
    vals, nib = compress(x, keep, M)
    Kl = lifted_k(x.shape[1], M)
    return dict(keep=keep, mask=mask_pack(keep), vals=vals, nib=nib, meta=meta_hw(nib, Kl), K_lift=Kl)


def split_window_order(K: int, M: int) -> np.ndarray:
    """The split window order of a row of K = G M elements (M = 2n, n even):
    window w of group g covers positions g M + 2w .. g M + 2w + 3 (SlideSparse
    page, technical summary §2.A), so the even windows 0, 2, ..., n - 2 of a
    group tile it exactly and the odd ones overlap them.  The split order
    lists every group's even windows, group by group, then every group's odd
    windows: entry j is the natural (group-major) index of the window placed
    j-th.  Lifting in this order gives [X | the odd windows of X]."""
    assert M % 4 == 0 and K % M == 0
    NW, NE = M // 2 - 1, M // 4
    G = K // M
    even = [g * NW + 2 * e for g in range(G) for e in range(NE)]
    odd = [g * NW + 2 * o + 1 for g in range(G) for o in range(NE - 1)]
    return np.array(even + odd, dtype=np.int64)


def lift_split(x: np.ndarray, M: int) -> np.ndarray:
    """The lifted operand with its windows in the split order (bf16 bits)."""
    rows, K = x.shape
    nat = lift(x, M)
    perm = split_window_order(K, M)
    return np.ascontiguousarray(nat.reshape(rows, -1, 4)[:, perm, :].reshape(rows, -1))


def sparse_operand_split(x: np.ndarray, N: int, M: int):
    """sparse_operand() with the windows in the split order: values and
    index pairs moved window by window, the metadata image built from them."""
    ref = sparse_operand(x, N, M)
    rows, K = x.shape
    perm = split_window_order(K, M)
    vals = np.ascontiguousarray(ref["vals"].reshape(rows, -1, 2)[:, perm, :].reshape(rows, -1))
    nib = np.ascontiguousarray(ref["nib"][:, perm])
    return dict(keep=ref["keep"], mask=ref["mask"], vals=vals, nib=nib, meta=meta_hw(nib, ref["K_lift"]),
                K_lift=ref["K_lift"])


def act_sparse_linear(x: np.ndarray, w: np.ndarray, N: int, M: int, rows=None) -> np.ndarray:
    """Y = prune_{N:M}(X) . W^T in fp64 (activation sparsity)."""
    keep = prune(x, N, M)
    return linear_f64(to_f64(x, keep), to_f64(w), rows)


def weight_sparse_linear(x: np.ndarray, w: np.ndarray, N: int, M: int, rows=None) -> np.ndarray:
    """Y = X . prune_{N:M}(W)^T in fp64 (weight sparsity)."""
    keep = prune(w, N, M)
    return linear_f64(to_f64(x), to_f64(w, keep), rows)


def hybrid_weight(w: np.ndarray, dense_frac: float):
    """Hybrid dense + 2:4 weight: permutation, dense block, compressed 2:4 block,
    and the pruned weight in the original column order."""
    O, K = w.shape
    D = hybrid_dense_count(K, dense_frac)
    cn = colnorm_f64(w)
    perm, is_dense = hybrid_perm(cn, D)
    wp = gather_cols(w, perm)
    Ks = K - D
    ws = np.ascontiguousarray(wp[:, :Ks])
    wd = np.ascontiguousarray(wp[:, Ks:])
    out = dict(D=D, Ks=Ks, colnorm=cn, perm=perm, is_dense=is_dense, W_d=wd)
    keep_full = np.ones((O, K), np.uint8)
    if Ks > 0:
        keep_s = prune(ws, 2, 4)
        vals, nib = compress(ws, keep_s, 4)
        out.update(keep_s=keep_s, vals_s=vals, nib_s=nib, meta_s=meta_hw(nib, Ks))
        keep_full[:, perm[:Ks]] = keep_s
    out["keep_full"] = keep_full
    return out


def hybrid_linear(x: np.ndarray, w: np.ndarray, dense_frac: float, rows=None) -> np.ndarray:
    """Y = X . Wp^T where Wp is W with the pruned entries of the 2:4 region
    zeroed, in the original column order (fp64)."""
    hw = hybrid_weight(w, dense_frac)
    return linear_f64(to_f64(x), to_f64(w, hw["keep_full"]), rows)


# -------------------------------------------------------------------- fp8


def e4m3_to_f64(codes) -> np.ndarray:
    """Values of E4M3 codes (NaN for the two NaN codes)."""
    L = _load()
    table = np.array([L.or_e4m3_to_f64(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_from_f32(x) -> np.ndarray:
    """E4M3 codes of fp32 values: nearest, ties to even, saturated to +-448."""
    L = _load()
    x = np.asarray(x, dtype=np.float32)
    return np.array([L.or_e4m3_from_f32(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def quant_rows(x: np.ndarray):
    """Per-row E4M3 codes and fp32 scales (scale = row amax / 448)."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    codes = np.zeros((rows, K), np.uint8)
    scale = np.zeros(rows, np.float32)
    _load().or_quant_rows_e4m3(_ptr(_as_bits(x)), _dt(x), rows, K, _ptr(codes), _ptr(scale))
    return codes, scale


def quant_vals(vals: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Codes of compressed bf16 values, row r divided by scale[r]."""
    vals = np.ascontiguousarray(vals, dtype=np.uint16)
    rows, nv = vals.shape
    codes = np.zeros((rows, nv), np.uint8)
    _load().or_quant_vals_e4m3(_ptr(vals), rows, nv, _ptr(np.ascontiguousarray(scale, dtype=np.float32)),
                               _ptr(codes))
    return codes


def lift_u8(codes: np.ndarray, M: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    out = np.zeros((rows, lifted_k(K, M)), np.uint8)
    if _load().or_lift_u8(_ptr(codes), rows, K, M, _ptr(out)) != 0:
        raise ValueError("or_lift_u8 rejected the shape")
    return out


def meta8(nib: np.ndarray, Kl: int) -> np.ndarray:
    nib = np.ascontiguousarray(nib, dtype=np.uint8)
    rows = nib.shape[0]
    out = np.zeros(int(_load().or_meta_hw_bytes(rows, Kl)), np.uint8)
    _load().or_meta8(_ptr(nib), rows, Kl, _ptr(out))
    return out


def fp8_activation(x: np.ndarray, M: int):
    """The quantise + lift step: per-token codes lifted for windows of M, and
    the per-token scales."""
    codes, scale = quant_rows(x)
    return dict(codes=codes, lifted=lift_u8(codes, M), scale=scale)


def fp8_weight(w: np.ndarray, N: int, M: int):
    """The offline weight packing in 8 bits: prune, windows, per-row scale of
    the dense row, codes of the compressed values, 8-bit metadata image."""
    keep = prune(w, N, M)
    vals, nib = compress(w, keep, M)
    _, scale = quant_rows(w)
    Kl = lifted_k(w.shape[1], M)
    return dict(keep=keep, vals=quant_vals(vals, scale), nib=nib, meta=meta8(nib, Kl), scale=scale, K_lift=Kl)


def fp8_weight_sparse_linear(x: np.ndarray, w: np.ndarray, N: int, M: int, rows=None) -> np.ndarray:
    """Y[t, o] = sx[t] * sw[o] * sum_k e4m3(X)[t, k] * e4m3(prune(W))[o, k] in fp64."""
    qx, sx = quant_rows(x)
    qw, sw = quant_rows(w)
    keep = prune(w, N, M)
    xd = e4m3_to_f64(qx)
    wd = np.where(keep.astype(bool), e4m3_to_f64(qw), 0.0)
    Y = linear_f64(xd, wd, rows)
    sxs = sx.astype(np.float64) if rows is None else sx.astype(np.float64)[np.asarray(rows)]
    return Y * sxs[:, None] * sw.astype(np.float64)[None, :]


def fp8_act_operand(x: np.ndarray, N: int, M: int):
    """The 8-bit prune + compress step: keep mask, per-token scales (amax of
    the dense row), codes of the window-compressed kept values, 8-bit image."""
    keep = prune(x, N, M)
    vals, nib = compress(x, keep, M)
    _, scale = quant_rows(x)
    Kl = lifted_k(x.shape[1], M)
    return dict(keep=keep, mask=mask_pack(keep), vals=quant_vals(vals, scale), nib=nib, meta=meta8(nib, Kl),
                scale=scale, K_lift=Kl)


def fp8_act_sparse_linear(x: np.ndarray, w: np.ndarray, N: int, M: int, rows=None) -> np.ndarray:
    """Y[t, o] = sx[t] * sw[o] * sum_k e4m3(prune(X))[t, k] * e4m3(W)[o, k] in fp64."""
    qx, sx = quant_rows(x)
    qw, sw = quant_rows(w)
    keep = prune(x, N, M)
    xd = np.where(keep.astype(bool), e4m3_to_f64(qx), 0.0)
    Y = linear_f64(xd, e4m3_to_f64(qw), rows)
    sxs = sx.astype(np.float64) if rows is None else sx.astype(np.float64)[np.asarray(rows)]
    return Y * sxs[:, None] * sw.astype(np.float64)[None, :]


# ------------------------------------------------------- GLU MLP (hybrid)


def rownorm_f64(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w)
    O, K = w.shape
    out = np.zeros(O, np.float64)
    _load().or_rownorm_f64(_ptr(_as_bits(w)), _dt(w), O, K, _ptr(out))
    return out


def silu_f64(z: np.ndarray) -> np.ndarray:
    z = np.ascontiguousarray(z, dtype=np.float64)
    out = np.zeros_like(z)
    _load().or_silu_f64(_ptr(z), z.size, _ptr(out))
    return out


def spense_dense_count(I: int, dense_frac: float) -> int:
    """Dense intermediate indices: whole blocks of 256, 256 * floor(f * I / 256)."""
    if dense_frac <= 0.0:
        return 0
    if dense_frac >= 1.0:
        return I
    return 256 * int((dense_frac * I) / 256.0)


def spense_mlp_weights(w_up: np.ndarray, w_gate: np.ndarray, w_down: np.ndarray, dense_frac: float):
    """The GLU-MLP packing: score = rownorm(up) + rownorm(gate) + colnorm(down)
    (fp64, summed in that order), the top D intermediate indices dense (ties to
    the lower index), perm = [sparse asc | dense asc]; keep masks of the
    pruned weights in the original index order."""
    I, d = w_up.shape
    D = spense_dense_count(I, dense_frac)
    score = (rownorm_f64(w_up) + rownorm_f64(w_gate)) + colnorm_f64(w_down)
    perm, is_dense = hybrid_perm(score, D)
    Is = I - D
    keep_up = np.ones((I, d), np.uint8)
    keep_gate = np.ones((I, d), np.uint8)
    keep_down = np.ones(w_down.shape, np.uint8)
    out = dict(D=D, Is=Is, score=score, perm=perm, is_dense=is_dense)
    if Is > 0:
        sp = perm[:Is]
        up_s = np.ascontiguousarray(w_up[sp])
        gate_s = np.ascontiguousarray(w_gate[sp])
        ku, kg = prune(up_s, 2, 4), prune(gate_s, 2, 4)
        keep_up[sp] = ku
        keep_gate[sp] = kg
        ug = np.ascontiguousarray(np.concatenate([up_s, gate_s]))
        vals, nib = compress(ug, np.concatenate([ku, kg]), 4)
        out.update(ug_vals=vals, ug_meta=meta_hw(nib, d))
        dp = gather_cols(w_down, perm)
        ds = np.ascontiguousarray(dp[:, :Is])
        kd = prune(ds, 2, 4)
        keep_down[:, sp] = kd
        vals_d, nib_d = compress(ds, kd, 4)
        out.update(down_vals=vals_d, down_meta=meta_hw(nib_d, Is))
    if D > 0:
        dn = perm[Is:]
        out["ug_dense"] = np.ascontiguousarray(np.concatenate([w_up[dn], w_gate[dn]]))
        out["down_dense"] = np.ascontiguousarray(gather_cols(w_down, perm)[:, Is:])
    out.update(keep_up=keep_up, keep_gate=keep_gate, keep_down=keep_down)
    return out


def spense_mlp(x: np.ndarray, w_up: np.ndarray, w_gate: np.ndarray, w_down: np.ndarray, dense_frac: float,
               rows=None) -> np.ndarray:
    """y = (silu(x . Gp^T) * (x . Up^T)) . Dp^T in fp64, with Up, Gp, Dp the
    pruned weights in the original index order."""
    p = spense_mlp_weights(w_up, w_gate, w_down, dense_frac)
    xd = to_f64(x)
    u = linear_f64(xd, to_f64(w_up, p["keep_up"]), rows)
    g = linear_f64(xd, to_f64(w_gate, p["keep_gate"]), rows)
    h = silu_f64(g) * u
    return linear_f64(h, to_f64(w_down, p["keep_down"]))


# ------------------------------------------------- shift and variance (step 9)


def row_mean(x: np.ndarray):
    """Step 9a: the per-token mean in fp64 and rounded to fp32."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    mu64 = np.empty(rows, np.float64)
    mu32 = np.empty(rows, np.float32)
    _load().or_row_mean(_ptr(_as_bits(x)), _dt(x), rows, K, _ptr(mu64), _ptr(mu32))
    return mu64, mu32


def shift_bf16(x: np.ndarray, mu32: np.ndarray) -> np.ndarray:
    """Step 9b: bf16(fl32(x - mu32)) per token (bf16 bits)."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    mu32 = np.ascontiguousarray(mu32, np.float32)
    out = np.empty((rows, K), np.uint16)
    _load().or_shift_bf16(_ptr(_as_bits(x)), _dt(x), rows, K, _ptr(mu32), _ptr(out))
    return out


def var_scale(x: np.ndarray, v: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """Step 9c: alpha = sqrt(var(x) / var(v * keep)) per token, x the token as
    it came in, v the token the prune ran on (1 if the pruned token has no
    variance)."""
    x = np.ascontiguousarray(x)
    v = np.ascontiguousarray(v, np.uint16)
    keep = np.ascontiguousarray(keep, np.uint8)
    rows, K = v.shape
    out = np.empty(rows, np.float64)
    _load().or_var_scale(_ptr(_as_bits(x)), _dt(x), _ptr(v), _ptr(keep), rows, K, _ptr(out))
    return out


def rowsum_f64(w: np.ndarray) -> np.ndarray:
    """Step 9d: s[o] = sum_k w[o][k] in fp64."""
    w = np.ascontiguousarray(w)
    O, K = w.shape
    out = np.empty(O, np.float64)
    _load().or_rowsum_f64(_ptr(_as_bits(w)), _dt(w), O, K, _ptr(out))
    return out


def act_transform(x: np.ndarray, N: int, M: int, shift: bool, var: bool):
    """The activation operand with the optional corrections of step 9: the
    shift (mu64, mu32; zero without D-PTS), the token the prune runs on
    (xs), its keep mask and compressed form, and the VAR factor (alpha in
    fp64 and rounded to fp32; one without VAR)."""
    rows = x.shape[0]
    if shift:
        mu64, mu32 = row_mean(x)
        xs = shift_bf16(x, mu32)
    else:
        mu64, mu32 = np.zeros(rows, np.float64), np.zeros(rows, np.float32)
        xs = np.ascontiguousarray(x)
    # the compressed form exists for windowable patterns (at most 2n-2 of 2n kept)
    op = sparse_operand(xs, N, M) if N <= (2 if M == 4 else M - 2) else dict(keep=prune(xs, N, M))
    alpha = var_scale(x, xs, op["keep"]) if var else np.ones(rows, np.float64)
    return dict(op, mu64=mu64, mu32=mu32, xs=xs, alpha=alpha, alpha32=alpha.astype(np.float32))


def act_sparse_linear_xf(x: np.ndarray, w: np.ndarray, N: int, M: int, shift: bool, var: bool,
                         rows=None) -> np.ndarray:
    """Y[t][o] = alpha[t] * (prune(xs[t]) . W[o]) + mu32[t] * s[o] in fp64:
    the shifted token pruned and rescaled, the shift added back through the
    weight's row sums."""
    t = act_transform(x, N, M, shift, var)
    y = linear_f64(to_f64(t["xs"], t["keep"]), to_f64(w), rows)
    sel = slice(None) if rows is None else np.asarray(rows)
    a = t["alpha"][sel][:, None]
    mu = t["mu32"].astype(np.float64)[sel][:, None]
    return a * y + mu * rowsum_f64(w)[None, :]
