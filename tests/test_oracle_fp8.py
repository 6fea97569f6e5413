"""The oracle's 8-bit (E4M3) step pinned to what the format and the
mathematics fix: values of codes from the format's definition, nearest-even
rounding at every midpoint, a library conversion routine, quantisation
invariants, and exact products when quantisation is lossless."""
import math

import numpy as np
import pytest
import torch

import oracle
from semi_structured_sparse_nm_b200 import inputs

# Code -> value, from the E4M3 definition: bias 7, 3 mantissa bits, subnormals
# (m/8) 2^-6, S.1111.111 is NaN, largest finite 1.75 * 2^8.
DECODE = [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0),
    (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x77, 240.0), (0x7E, 448.0), (0xB8, -1.0), (0xFE, -448.0),
]
# value -> code, nearest with ties to even, saturating
ENCODE = [
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (448.0, 0x7E), (450.0, 0x7E), (1e9, 0x7E), (math.inf, 0x7E),
    (-1e9, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (5 * 2.0 ** -10, 0x02),
    (1.0625, 0x38), (1.1875, 0x3A), (1.0625 * (1 + 2 ** -20), 0x39), (464.0, 0x7E), (0.3, 0x2A),          # 0.3 = 1.2 * 2^-2: exponent field 5, mantissa 2 (1.25)
]


@pytest.mark.parametrize("code,value", DECODE)
def test_decode_values(code, value):
    assert oracle.e4m3_to_f64([code])[0] == value


def test_nan_codes():
    v = oracle.e4m3_to_f64([0x7F, 0xFF])
    assert np.isnan(v).all()
    assert oracle.e4m3_from_f32([np.nan])[0] == 0x7F


@pytest.mark.parametrize("value,code", ENCODE)
def test_encode_values(value, code):
    assert oracle.e4m3_from_f32([value])[0] == code


def test_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_from_f32(vals), codes)


def test_midpoints_round_to_even():
    codes = np.arange(0, 0x7E, dtype=np.uint8)
    v0 = oracle.e4m3_to_f64(codes)
    v1 = oracle.e4m3_to_f64(codes + 1)
    mid = ((v0 + v1) / 2).astype(np.float32)                 # at most 5 significant bits: exact
    assert np.array_equal(mid.astype(np.float64), (v0 + v1) / 2)
    even = np.where(codes % 2 == 0, codes, codes + 1)
    assert np.array_equal(oracle.e4m3_from_f32(mid), even)
    up = (mid.astype(np.float64) * (1 + 2.0 ** -20)).astype(np.float32)
    down = (mid.astype(np.float64) * (1 - 2.0 ** -20)).astype(np.float32)
    assert np.array_equal(oracle.e4m3_from_f32(up[1:]), (codes + 1)[1:])
    assert np.array_equal(oracle.e4m3_from_f32(down[1:]), codes[1:])


def test_agrees_with_library_conversion_in_range():
    rng = np.random.default_rng(3)
    mag = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 20000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_from_f32(x), ref)


def test_quant_rows_invariants():
    x = inputs.student_t_bf16((40, 512), 4.0, seed=5)
    x[7] = 0                                                   # an all-zero row
    codes, scale = oracle.quant_rows(x)
    xf = inputs.bf16_to_f64(x)
    dec = oracle.e4m3_to_f64(codes)
    assert scale[7] == 1.0 and not codes[7].any()
    nz = np.arange(40) != 7
    # the row maximum maps to the largest code
    assert np.array_equal(np.abs(dec[nz]).max(axis=1), np.full(39, 448.0))
    assert np.array_equal(scale[nz], (np.abs(xf[nz]).max(axis=1) / 448.0).astype(np.float32))
    # within half a step of the value (3 mantissa bits; subnormal step 2^-9)
    err = np.abs(dec * scale[:, None].astype(np.float64) - xf)
    bound = (2.0 ** -4) * np.abs(xf) + 2.0 ** -10 * scale[:, None].astype(np.float64) * (1 + 1e-6)
    assert (err <= bound * (1 + 1e-6)).all()


def test_lift_u8_is_the_lift_map():
    codes = np.random.default_rng(1).integers(0, 256, size=(9, 96), dtype=np.uint8)
    for M in (4, 8, 16, 32):
        ref = oracle.lift(codes.astype(np.uint16), M).astype(np.uint8)
        assert np.array_equal(oracle.lift_u8(codes, M), ref)


def _decode_meta8_tensor_view(meta, rows, Kl):
    """Independent reading of the 8-bit sparse-MMA metadata image, as the
    tensor core sees it (PTX ISA, tcgen05.cp and the sparse metadata of
    tcgen05.mma.sp with kind::f8f6f4).  A copy of shape 128x128b moves one
    2048-byte block into tensor memory as 128 lanes of four 32-bit columns:
    lane m receives the m-th 16 bytes, column c the c-th little-endian word of
    them.  An 8-bit sparse MMA covers 64 lifted K and reads a 64-bit metadata
    word per row from a pair of columns, the lower column holding the low 32
    bits; the 4-bit field i of that word belongs to the i-th group of four K.
    The two MMAs of a 128-K block use column pairs (0, 1) and (2, 3).
    Returns the nibble of every (row, window) over the padded extent."""
    RB, KB = -(-rows // 128), -(-Kl // 128)
    words = np.ascontiguousarray(meta[:RB * KB * 2048]).view("<u4").reshape(RB, KB, 128, 4)
    out = np.zeros((RB * 128, KB * 32), np.uint8)
    for mma in range(2):
        w64 = words[..., 2 * mma].astype(np.uint64) | (words[..., 2 * mma + 1].astype(np.uint64) << np.uint64(32))
        for i in range(16):
            field = ((w64 >> np.uint64(4 * i)) & np.uint64(0xF)).astype(np.uint8)      # [RB, KB, 128]
            for kb in range(KB):
                out[:, kb * 32 + 16 * mma + i] = field[:, kb, :].reshape(RB * 128)
    return out


def test_meta8_decodes_to_nibbles():
    rng = np.random.default_rng(2)
    rows, Kl = 150, 384
    nib = rng.choice(np.array([0x4, 0x8, 0xC, 0x9, 0xD, 0xE], np.uint8), size=(rows, Kl // 4))
    img = oracle.meta8(nib, Kl)
    assert img.size == 2 * 3 * 2048
    dec = _decode_meta8_tensor_view(img, rows, Kl)
    np.testing.assert_array_equal(dec[:rows, :Kl // 4], nib)
    # padding rows and windows carry the valid index pair (0, 1)
    assert (dec[rows:, :] == 0x4).all() and (dec[:, Kl // 4:] == 0x4).all()
    assert (oracle.meta8(np.full((3, 32), 0x4, np.uint8), 128) == 0x44).all()


@pytest.mark.parametrize("rows,K,N,M", [(130, 512, 6, 8), (64, 640, 2, 4), (40, 1024, 14, 16), (9, 2048, 30, 32)])
def test_meta8_tensor_view_reproduces_the_pruned_product(rows, K, N, M):
    """Emulates the 8-bit sparse MMA from the packed weight alone: each
    window's two codes, placed at the lifted positions the tensor-view decode
    of the metadata gives, times integer activations lifted by the lift map,
    summed exactly; this equals the product of the pruned weight's codes with
    the unlifted activations."""
    w = inputs.normal_bf16((rows, K), 0.02, seed=rows + K)
    P = oracle.fp8_weight(w, N, M)
    Kl = P["K_lift"]
    dec = _decode_meta8_tensor_view(P["meta"], rows, Kl)[:rows, :Kl // 4].astype(np.int64)
    codes = oracle.e4m3_to_f64(P["vals"])                        # [rows, Kl / 2] kept values, window order
    dense_lifted = np.zeros((rows, Kl))
    r = np.arange(rows)[:, None]
    j = np.arange(Kl // 4)[None, :]
    np.add.at(dense_lifted, (r, 4 * j + (dec & 3)), codes[:, 0::2])
    np.add.at(dense_lifted, (r, 4 * j + ((dec >> 2) & 3)), codes[:, 1::2])
    xi = np.random.default_rng(5).integers(-3, 4, size=(7, K)).astype(np.float64)
    xl = inputs.bf16_to_f64(oracle.lift(inputs.bf16_from_f64(xi), M))
    got = dense_lifted @ xl.T
    q, _ = oracle.quant_rows(w)
    kept = oracle.e4m3_to_f64(q) * P["keep"]
    np.testing.assert_array_equal(got, kept @ xi.T)


@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (14, 16)])
def test_fp8_product_exact_when_quantisation_is_lossless(N, M):
    """Inputs on the E4M3 grid whose row maxima are 448 (scale 1) or 112
    (scale 1/4, a power of two): the 8-bit product equals the plain one."""
    rng = np.random.default_rng(N + M)
    grid = oracle.e4m3_to_f64(np.arange(0x00, 0x77, dtype=np.uint8))    # 0 .. 240
    for top in (448.0, 112.0):
        def make(rows, K, seed):
            r = np.random.default_rng(seed)
            v = r.choice(grid, size=(rows, K)) * r.choice([-1.0, 1.0], size=(rows, K)) * (top / 448.0)
            v[:, 0] = top
            return inputs.bf16_from_f64(v)
        x = make(12, 64, 1)
        w = make(40, 64, 2)
        y8 = oracle.fp8_weight_sparse_linear(x, w, N, M)
        y = oracle.weight_sparse_linear(x, w, N, M)
        assert np.array_equal(y8, y)


@pytest.mark.parametrize("N,M", [(8, 16), (2, 4), (16, 32)])
def test_fp8_act_product_exact_when_quantisation_is_lossless(N, M):
    """The activation-sparse 8-bit product on lossless inputs equals the plain
    activation-sparse product."""
    grid = oracle.e4m3_to_f64(np.arange(0x00, 0x77, dtype=np.uint8))
    for top in (448.0, 112.0):
        def make(rows, K, seed):
            r = np.random.default_rng(seed)
            v = r.choice(grid, size=(rows, K)) * r.choice([-1.0, 1.0], size=(rows, K)) * (top / 448.0)
            v[:, 0] = top
            return inputs.bf16_from_f64(v)
        x = make(10, 128, 3)
        w = make(24, 128, 4)
        assert np.array_equal(oracle.fp8_act_sparse_linear(x, w, N, M), oracle.act_sparse_linear(x, w, N, M))


def test_fp8_act_operand_codes_are_the_kept_values():
    """Decoded codes times the scale reproduce the kept bf16 values within
    half an E4M3 step, in the window order of the 16-bit operand."""
    x = inputs.student_t_bf16((20, 256), 4.0, seed=8)
    ref16 = oracle.sparse_operand(x, 8, 16)
    ref8 = oracle.fp8_act_operand(x, 8, 16)
    assert np.array_equal(ref8["mask"], ref16["mask"])
    assert np.array_equal(ref8["nib"], ref16["nib"])
    v = inputs.bf16_to_f64(ref16["vals"])
    d = oracle.e4m3_to_f64(ref8["vals"]) * ref8["scale"][:, None].astype(np.float64)
    assert (np.abs(d - v) <= 2.0 ** -4 * np.abs(v) + 2.0 ** -10 * ref8["scale"][:, None] * 1.000001).all()


def test_quant_vals_are_the_row_codes_of_the_kept_entries():
    """The 8-bit weight packing quantises the window-compressed values with
    each row's dense-row scale: scattered back to their positions, those codes
    must be the per-row codes of quant_rows at every kept entry (a wrong row's
    scale or a misplaced window fails)."""
    w = inputs.normal_bf16((40, 256), 0.02, seed=12)
    for N, M in [(6, 8), (2, 4), (14, 16)]:
        keep = oracle.prune(w, N, M)
        vals, nib = oracle.compress(w, keep, M)
        row_codes, scale = oracle.quant_rows(w)
        qv = oracle.quant_vals(vals, scale)
        placed = oracle.decompress(qv.astype(np.uint16), nib, w.shape[1], M)
        assert np.array_equal(placed, np.where(keep, row_codes, 0).astype(np.uint16)), (N, M)
        packed = oracle.fp8_weight(w, N, M)
        assert np.array_equal(packed["vals"], qv) and np.array_equal(packed["scale"], scale)


def test_fp8_activation_lift_is_the_lift_map():
    """The quantise + lift step's byte lift equals the bf16 lift applied to the
    same codes (two independent implementations of the lift map)."""
    x = inputs.student_t_bf16((24, 512), 4.0, seed=13)
    for M in (4, 8, 16, 32):
        a = oracle.fp8_activation(x, M)
        assert np.array_equal(a["lifted"], oracle.lift(a["codes"].astype(np.uint16), M).astype(np.uint8)), M
        codes, scale = oracle.quant_rows(x)
        assert np.array_equal(a["codes"], codes) and np.array_equal(a["scale"], scale)
