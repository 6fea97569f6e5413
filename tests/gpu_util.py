"""Helpers shared by the GPU tests: host <-> device transfers of bf16 bit
patterns, and the tolerance check for outputs."""
import numpy as np
import torch

REL_FRO = 1e-2      # relative Frobenius error bound
ROW_MAX = 2e-2      # per-element bound, relative to max |Y_ref| of the row


def dev(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits -> cuda bfloat16; float32 -> cuda float32."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    if a.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()
    raise TypeError(a.dtype)


def host_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16).numpy() if hasattr(torch, "uint16") else t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.numpy()
    if t.dtype in (torch.int32, torch.float32):
        return t.numpy().view(np.uint32)
    raise TypeError(t.dtype)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(y: np.ndarray, y_ref: np.ndarray, what: str = ""):
    """Relative Frobenius <= 1e-2 and |y - y_ref|[i, j] <= 2e-2 * max_j |y_ref[i, j]|."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    fro = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert fro <= REL_FRO, f"{what}: relative Frobenius error {fro:.3e}"
    row_max = np.abs(y_ref).max(axis=1, keepdims=True)
    bad = np.abs(y - y_ref) > ROW_MAX * row_max
    assert not bad.any(), f"{what}: {bad.sum()} entries beyond 2e-2*row max (first at {np.argwhere(bad)[0]})"
    return fro
