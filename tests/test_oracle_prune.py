"""Pins for the oracle's prune step (top-N |value| per aligned group of M, ties
to the lower index), checked against brute force, counting and invariants --
never against the oracle itself."""
import itertools
import math

import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs

NM_CASES = [(1, 4), (2, 4), (4, 8), (6, 8), (3, 8), (8, 16), (14, 16), (16, 32), (30, 32), (4, 6), (8, 10)]


def _keys_bf16(bits):
    return (bits.astype(np.uint32) & 0x7FFF)


def _brute_force_groups(bits_row, N, M):
    """All N-subsets of each group that satisfy: every kept entry beats every
    dropped entry (larger key, or equal key and lower index)."""
    out = []
    for g in range(len(bits_row) // M):
        keys = [int(k) for k in _keys_bf16(bits_row[g * M:(g + 1) * M])]
        good = []
        for S in itertools.combinations(range(M), N):
            s = set(S)
            ok = all(keys[a] > keys[b] or (keys[a] == keys[b] and a < b)
                     for a in s for b in range(M) if b not in s)
            if ok:
                good.append(S)
        out.append(good)
    return out


@pytest.mark.parametrize("N,M", NM_CASES)
def test_exactly_n_kept_per_group(N, M):
    x = inputs.normal_bf16((7, M * 9), 1.0, seed=11 + M)
    keep = oracle.prune(x, N, M)
    per_group = keep.reshape(7, 9, M).sum(axis=2)
    assert (per_group == N).all()


@pytest.mark.parametrize("M", [4, 8, 16, 32])
def test_n_equals_m_keeps_everything(M):
    x = inputs.normal_bf16((3, M * 5), 1.0, seed=5)
    assert oracle.prune(x, M, M).all()


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (4, 8), (6, 8), (3, 8), (2, 6)])
@pytest.mark.parametrize("dist", ["normal", "ties"])
def test_brute_force_unique_subset_small(N, M, dist):
    rng = np.random.default_rng(3)
    if dist == "normal":
        x = inputs.normal_bf16((4, M * 6), 1.0, seed=17)
    else:  # tie torture: values from {-2,-1,-0,0,1,2}
        vals = np.array([-2.0, -1.0, -0.0, 0.0, 1.0, 2.0])
        x = inputs.bf16_from_f64(vals[rng.integers(0, 6, size=(4, M * 6))])
    keep = oracle.prune(x, N, M)
    for r in range(x.shape[0]):
        subsets = _brute_force_groups(x[r], N, M)
        for g, good in enumerate(subsets):
            assert len(good) == 1, "the tie rule must make the kept set unique"
            expect = np.zeros(M, np.uint8)
            expect[list(good[0])] = 1
            np.testing.assert_array_equal(keep[r, g * M:(g + 1) * M], expect)


def test_brute_force_8_of_16_ties():
    vals = np.array([-2.0, -1.0, -0.0, 0.0, 1.0, 2.0])
    rng = np.random.default_rng(99)
    x = inputs.bf16_from_f64(vals[rng.integers(0, 6, size=(1, 32))])
    keep = oracle.prune(x, 8, 16)
    for g, good in enumerate(_brute_force_groups(x[0], 8, 16)):
        assert len(good) == 1
        expect = np.zeros(16, np.uint8)
        expect[list(good[0])] = 1
        np.testing.assert_array_equal(keep[0, g * 16:(g + 1) * 16], expect)


@pytest.mark.parametrize("pattern", ["2:4", "8:16"])
def test_configuration_count_matches_pages(pattern, golden):
    """Every N-subset of a group is reachable, and nothing else is: the number
    of distinct masks equals the count the pages give (6 for 2:4, 12,870 for
    8:16)."""
    N, M = map(int, pattern.split(":"))
    subsets = list(itertools.combinations(range(M), N))
    x = np.full((len(subsets), M), 1.0)
    for i, S in enumerate(subsets):
        x[i, list(S)] = 2.0
    # alternate signs so that the sign never matters
    x *= np.where(np.arange(M) % 3 == 0, -1.0, 1.0)
    keep = oracle.prune(inputs.bf16_from_f64(x), N, M)
    distinct = {tuple(np.flatnonzero(row)) for row in keep}
    assert distinct == set(subsets)
    assert len(distinct) == math.comb(M, N) == golden["configurations_per_block"][pattern]


def test_ties_go_to_lower_index():
    x = inputs.bf16_from_f64(np.array([[1.0, -1.0, 1.0, -1.0, 0.5, -0.5, 0.5, -0.5]]))
    np.testing.assert_array_equal(oracle.prune(x, 2, 4)[0], [1, 1, 0, 0, 1, 1, 0, 0])
    np.testing.assert_array_equal(oracle.prune(x, 3, 8)[0], [1, 1, 1, 0, 0, 0, 0, 0])


def test_signed_zero_share_a_key():
    # bits: +0 = 0x0000, -0 = 0x8000; both have magnitude key 0
    x = np.array([[0x8000, 0x0000, 0x8000, 0x3F80]], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.prune(x, 2, 4)[0], [1, 0, 0, 1])


def test_magnitude_not_signed_value():
    x = inputs.bf16_from_f64(np.array([[-3.0, 2.0, 1.0, -0.5]]))
    np.testing.assert_array_equal(oracle.prune(x, 2, 4)[0], [1, 1, 0, 0])


def test_fp32_keys_see_bits_below_bf16():
    # 1 + 2^-20 and 1 round to the same bf16 but differ in fp32
    x = np.array([[1.0, 1.0 + 2.0 ** -20, -1.0, 0.25]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.prune(x, 1, 4)[0], [0, 1, 0, 0])
    np.testing.assert_array_equal(oracle.prune(x, 2, 4)[0], [1, 1, 0, 0])


def test_mask_pack_layout():
    keep = np.zeros((2, 40), np.uint8)
    keep[0, 0] = keep[0, 31] = keep[0, 33] = keep[1, 5] = 1
    m = oracle.mask_pack(keep)
    assert m.shape == (2, 2)
    assert m[0, 0] == (1 | (1 << 31)) and m[0, 1] == (1 << 1)
    assert m[1, 0] == (1 << 5) and m[1, 1] == 0


def test_rejects_bad_group():
    with pytest.raises(ValueError):
        oracle.prune(inputs.normal_bf16((2, 10), 1.0, 0), 2, 4)
