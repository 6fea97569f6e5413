"""Seeded synthetic inputs shared by the CUDA path's tests, the benchmark and the oracle tests.

This module holds no arithmetic of the sparsity method (no pruning, no window
assignment, no matmul).  It only draws random numbers and rounds them to the
storage formats the kernels read, so that the oracle and the GPU path see the
very same bytes.

Recipe (all workloads):
  * fp64 draws from numpy's PCG64 generator, then one round-to-nearest-even to
    fp32 and, for bf16 tensors, one more round-to-nearest-even from fp32 to bf16;
  * X uses stream ``seed``, W uses ``seed + 1``, the outlier-channel choice uses
    ``seed + 2`` (seed 0 by default); the GLU-MLP workloads take W_up from
    ``seed + 1``, W_gate from ``seed + 3`` and W_down from ``seed + 4``;
  * N(0, s) means standard deviation s;
  * Student-t(nu=4) is divided by sqrt(2) so that its variance is 1;
  * "0.1% of channels scaled x20" picks round(0.001*K) K-columns by a seeded
    permutation and multiplies them by 20 before rounding.

The workloads mirror LLM linear layers (Llama-8B up_proj / down_proj shapes)
that the pages benchmark on real models; synthetic tensors stand in for the
models' weights and activations.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "bf16_from_f64", "bf16_to_f64", "bf16_to_f32", "f32_bits",
    "normal_bf16", "student_t_bf16", "Workload", "WORKLOADS", "make_workload", "make_mlp_weights",
]


def bf16_from_f64(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE); returns the bf16 bit patterns as uint16."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    out = r.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    return bf16_from_f64(_rng(seed).standard_normal(shape) * std)


def student_t_bf16(shape, nu: float, seed: int) -> np.ndarray:
    # variance of Student-t(nu) is nu / (nu - 2); rescale to unit variance
    scale = 1.0 / math.sqrt(nu / (nu - 2.0))
    return bf16_from_f64(_rng(seed).standard_t(nu, size=shape) * scale)


def normal_with_outlier_channels_bf16(shape, frac: float, factor: float, seed: int) -> np.ndarray:
    rows, K = shape
    x = _rng(seed).standard_normal(shape)
    n_out = int(round(frac * K))
    cols = _rng(seed + 2).permutation(K)[:n_out]
    x[:, cols] *= factor
    return bf16_from_f64(x)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload of the sparse linear layer Y = X . W^T.

    side: "act"    -> X is pruned N:M along K at run time (activation sparsity)
          "weight" -> W is pruned N:M along K offline (weight sparsity)
          "hybrid" -> W keeps a dense share of K columns, the rest is 2:4
          "mlp"    -> a GLU MLP (W_up, W_gate [O x K], W_down [K x O]) whose
                      dense share of intermediate indices stays dense in all
                      three projections, the rest 2:4 (K = model width,
                      O = intermediate width)
    """
    name: str
    side: str
    T: int          # tokens (rows of X)
    K: int          # reduction dim
    O: int          # output features (rows of W)
    N: int
    M: int
    x_dtype: str    # "bf16" | "fp32"
    out_dtype: str  # "bf16" | "fp32"
    x_dist: str     # "normal" | "student_t4" | "normal_outliers"
    w_std: float = 0.02
    dense_frac: float = 0.0
    fp8: bool = False   # 8-bit (E4M3) operands: X quantised per token, W per output row
    xf: int = 0         # per-token corrections of the activation prune: 1 shift (D-PTS), 2 VAR, 3 both

    @property
    def K_lift(self) -> int:
        if self.side in ("hybrid", "mlp"):
            return self.K
        n = self.M // 2
        return self.K * (2 * n - 2) // n


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_2of4_act_fp32", "act", 16, 256, 128, 2, 4, "fp32", "fp32", "normal"),
        Workload("up_proj_8of16_act", "act", 2048, 4096, 14336, 8, 16, "bf16", "bf16", "student_t4"),
        # the same shape pruned 2:4: the 2:4 prefill GEMM measurement
        Workload("up_proj_2of4_act", "act", 2048, 4096, 14336, 2, 4, "bf16", "bf16", "student_t4"),
        # the same 8:16 product with 8-bit operands (X per token, W per output channel)
        Workload("up_proj_8of16_act_fp8", "act", 2048, 4096, 14336, 8, 16, "bf16", "bf16", "student_t4", fp8=True),
        # the same 8:16 product with the D-PTS shift and the VAR rescale around the prune
        Workload("up_proj_8of16_act_xf", "act", 2048, 4096, 14336, 8, 16, "bf16", "bf16", "student_t4", xf=3),
        Workload("slide_6of8_wt_prefill", "weight", 4096, 4096, 4096, 6, 8, "bf16", "bf16", "normal"),
        Workload("slide_6of8_wt_decode", "weight", 16, 4096, 4096, 6, 8, "bf16", "bf16", "normal"),
        Workload("slide_6of8_wt_decode_fp8", "weight", 16, 4096, 4096, 6, 8, "bf16", "bf16", "normal", fp8=True),
        # the same prefill product with 8-bit operands (the pages' B200 precision)
        Workload("slide_6of8_wt_prefill_fp8", "weight", 4096, 4096, 4096, 6, 8, "bf16", "bf16", "normal",
                 fp8=True),
        Workload("down_proj_16of32_act", "act", 4096, 14336, 4096, 16, 32, "bf16", "bf16", "normal_outliers"),
    ] + [
        Workload(f"hybrid_decode_b{b}", "hybrid", b, 4096, 14336, 2, 4, "bf16", "bf16", "normal",
                 dense_frac=0.25) for b in (1, 8, 32, 128)
    ] + [
        Workload(f"spense_mlp_decode_b{b}", "mlp", b, 4096, 14336, 2, 4, "bf16", "bf16", "normal",
                 dense_frac=0.25) for b in (1, 8, 32, 128)
    ]
}


def make_x(w: Workload, seed: int = 0, T: int | None = None) -> np.ndarray:
    """X [T x K]: uint16 bf16 bits, or float32 for the fp32 workload."""
    T = w.T if T is None else T
    if w.x_dtype == "fp32":
        return _rng(seed).standard_normal((T, w.K)).astype(np.float32)
    if w.x_dist == "student_t4":
        return student_t_bf16((T, w.K), 4.0, seed)
    if w.x_dist == "normal_outliers":
        return normal_with_outlier_channels_bf16((T, w.K), 0.001, 20.0, seed)
    return normal_bf16((T, w.K), 1.0, seed)


def make_w(w: Workload, seed: int = 0) -> np.ndarray:
    """W [O x K]: uint16 bf16 bits, or float32 for the fp32 workload."""
    if w.x_dtype == "fp32":
        return (_rng(seed + 1).standard_normal((w.O, w.K)) * w.w_std).astype(np.float32)
    return normal_bf16((w.O, w.K), w.w_std, seed + 1)


def make_mlp_weights(w: Workload, seed: int = 0):
    """(W_up [O x K], W_gate [O x K], W_down [K x O]) of a GLU-MLP workload."""
    return (normal_bf16((w.O, w.K), w.w_std, seed + 1), normal_bf16((w.O, w.K), w.w_std, seed + 3),
            normal_bf16((w.K, w.O), w.w_std, seed + 4))


def make_workload(name: str, seed: int = 0, T: int | None = None):
    w = WORKLOADS[name]
    return w, make_x(w, seed, T), make_w(w, seed)
