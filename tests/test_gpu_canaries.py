"""Guard bands around every output buffer: each kernel writes exactly its
output and nothing before or after it, on ragged shapes where a stray tile
edge would show."""
import numpy as np
import pytest
import torch

from semi_structured_sparse_nm_b200 import _lib as nm
from semi_structured_sparse_nm_b200 import inputs
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps 16-byte alignment)
PATTERN = 0xA5


class Guarded:
    """A device buffer of `nbytes` between two guard bands of PATTERN bytes."""

    def __init__(self, nbytes):
        self.n = nbytes
        self.raw = torch.full((GUARD + max(nbytes, 16) + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        return self.raw[GUARD:GUARD + self.n].view(dtype).view(shape)

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool((r[:GUARD] == PATTERN).all() and (r[GUARD + self.n:] == PATTERN).all())


def _compressed(rows, K, N, M, with_mask=True):
    Kl = nm.lifted_k(K, M)
    g = [Guarded(rows * Kl), Guarded(max(nm.meta_bytes(rows, K, M), 16)), Guarded(rows * ((K + 31) // 32) * 4)]
    c = nm.Compressed(g[0].view(torch.bfloat16, (rows, Kl // 2)), g[1].view(torch.uint8, (-1,)), rows, K, N, M,
                      g[2].view(torch.int32, (rows, (K + 31) // 32)) if with_mask else None)
    return c, g


@pytest.mark.parametrize("rows,K,N,M", [(37, 520, 2, 4), (129, 1088, 8, 16), (5, 448, 16, 32), (200, 96, 6, 8)])
def test_prune_and_lift_stay_inside(rows, K, N, M):
    x = dev(inputs.student_t_bf16((rows, K), 4.0, rows))
    c, g = _compressed(rows, K, N, M)
    nm.prune_compress(x, N, M, out=c)
    gl = Guarded(rows * nm.lifted_k(K, M) * 2)
    nm.lift(x, M, out=gl.view(torch.bfloat16, (rows, nm.lifted_k(K, M))))
    torch.cuda.synchronize()
    assert all(b.intact() for b in g) and gl.intact()


@pytest.mark.parametrize("T,K,O,N,M,side", [(37, 512, 200, 2, 4, "act"), (300, 1024, 520, 8, 16, "act"),
                                            (16, 768, 384, 6, 8, "weight"), (130, 512, 256, 6, 8, "weight"),
                                            (512, 512, 600, 8, 16, "act")])
def test_gemm_stays_inside(T, K, O, N, M, side):
    x = dev(inputs.student_t_bf16((T, K), 4.0, T))
    w = dev(inputs.normal_bf16((O, K), 0.02, O))
    for out_dt, esz in ((torch.bfloat16, 2), (torch.float32, 4)):
        gy = Guarded(T * O * esz)
        if side == "act":
            nm.sparse_gemm(nm.prune_compress(x, N, M), nm.lift(w, M), nm.NM_ACT, out_dt, out=gy.view(out_dt, (T, O)))
        else:
            nm.sparse_gemm(nm.slide_decompose(w, N, M), nm.lift(x, M), nm.NM_WEIGHT, out_dt,
                           out=gy.view(out_dt, (T, O)))
        torch.cuda.synchronize()
        assert gy.intact(), (side, out_dt)


@pytest.mark.parametrize("B", [1, 33, 130])
def test_hybrid_and_mlp_stay_inside(B):
    K, O = 512, 384
    x = dev(inputs.normal_bf16((B, K), 1.0, B))
    h = nm.hybrid_prepare(dev(inputs.normal_bf16((O, K), 0.02, 1)), 0.25)
    gy = Guarded(B * O * 2)
    nm.hybrid_gemm(x, h, torch.bfloat16, out=gy.view(torch.bfloat16, (B, O)))
    I, d = 1024, 256
    W = nm.spense_mlp_prepare(dev(inputs.normal_bf16((I, d), 0.02, 2)), dev(inputs.normal_bf16((I, d), 0.02, 3)),
                              dev(inputs.normal_bf16((d, I), 0.02, 4)), 0.25)
    gm = Guarded(B * d * 2)
    nm.spense_mlp(dev(inputs.normal_bf16((B, d), 1.0, 5)), W, out=gm.view(torch.bfloat16, (B, d)))
    torch.cuda.synchronize()
    assert gy.intact() and gm.intact()


def test_eight_bit_and_corrections_stay_inside():
    T, K, O = 40, 768, 256
    x = dev(inputs.student_t_bf16((T, K), 4.0, 1))
    w = dev(inputs.normal_bf16((O, K), 0.02, 2))
    Kl = nm.lifted_k(K, 8)
    gc, gs = Guarded(T * Kl), Guarded(T * 4)
    q = nm.Fp8Operand(gc.view(torch.uint8, (T, Kl)), gs.view(torch.float32, (T,)), T, K, 0, 8)
    nm.quant_lift_fp8(x, 8, out=q)
    P = nm.slide_decompose_fp8(w, 6, 8)
    gy = Guarded(T * O * 2)
    nm.sparse_gemm_fp8(P, q, nm.NM_WEIGHT, torch.bfloat16, out=gy.view(torch.bfloat16, (T, O)))
    X = nm.prune_compress_xf(x, 8, 16, nm.NM_XF_SHIFT | nm.NM_XF_VAR)
    gx = Guarded(T * O * 4)
    nm.sparse_gemm_xf(X, nm.lift(w, 16), nm.row_sums(w), torch.float32, out=gx.view(torch.float32, (T, O)))
    torch.cuda.synchronize()
    assert gc.intact() and gs.intact() and gy.intact() and gx.intact()
