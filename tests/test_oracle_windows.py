"""Pins for the sliding-window decomposition, the nibble/value encoding and the
lift map: exhaustive enumeration of patterns, capacity arguments, the page's
closed forms and round trips."""
import itertools
import math

import numpy as np
import pytest

import oracle
from semi_structured_sparse_nm_b200 import inputs

VALID_NIBBLES = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}


def _check_assignment(masks, M, win, slot, st):
    n = M // 2
    bits = ((masks[:, None] >> np.arange(M, dtype=np.uint64)) & np.uint64(1)).astype(bool)
    assert (st == 0).all()
    # every kept position has a window, and only kept positions do
    assert ((win >= 0) == bits).all()
    pos = np.arange(M)
    w = win.astype(np.int64)
    # a window w only covers positions 2w .. 2w+3
    inside = (pos[None, :] >= 2 * w) & (pos[None, :] <= 2 * w + 3)
    assert (inside | ~bits).all()
    assert (w < n - 1).all()
    # at most two entries per window, slots 0 and 1 used once each
    for ww in range(n - 1):
        cnt = (win == ww).sum(axis=1)
        assert (cnt <= 2).all()
        s0 = ((win == ww) & (slot == 0)).sum(axis=1)
        s1 = ((win == ww) & (slot == 1)).sum(axis=1)
        assert ((s0 == (cnt >= 1)) & (s1 == (cnt >= 2))).all()
    # order is kept: windows (then slots) never decrease along the positions
    order = np.where(bits, w * 2 + slot, -1)
    for b in range(order.shape[0]):
        o = order[b][bits[b]]
        assert (np.diff(o) > 0).all()


@pytest.mark.parametrize("M", [4, 6, 8, 10, 12, 14, 16])
def test_greedy_fits_every_pattern_exhaustive(M):
    """N-1 windows suffice for every pattern with at most 2n-2 kept entries,
    checked on all 2^M masks for 2n <= 16."""
    masks = np.arange(1 << M, dtype=np.uint64)
    pop = np.array([bin(int(m)).count("1") for m in masks])
    ok = masks[pop <= M - 2]
    win, slot, st = oracle.window_assign_batch(ok, M)
    _check_assignment(ok, M, win, slot, st)
    # one entry more than the windows' capacity never fits
    over = masks[pop == M - 1]
    _, _, st2 = oracle.window_assign_batch(over, M)
    assert (st2 != 0).all()


def test_greedy_fits_random_32():
    rng = np.random.default_rng(7)
    M = 32
    masks = []
    for _ in range(20000):
        k = int(rng.integers(0, 31))
        pos = rng.choice(32, size=k, replace=False)
        masks.append(sum(1 << int(p) for p in pos))
    # adversarial: all kept entries packed at the start / at the end
    masks += [(1 << 30) - 1, ((1 << 30) - 1) << 2, 0xFFFFFFFF & ~0x3, 0xFFFFFFFF & ~(0x3 << 30)]
    masks += [0xFFFFFFFF & ~((1 << a) | (1 << b)) for a, b in itertools.combinations(range(32), 2)]
    masks = np.array(masks, dtype=np.uint64)
    win, slot, st = oracle.window_assign_batch(masks, M)
    _check_assignment(masks, M, win, slot, st)


@pytest.mark.parametrize("n", [2, 3, 4, 8, 16])
def test_fewer_windows_cannot_hold_the_pattern(n):
    """n-2 windows of two entries hold 2n-4 < 2n-2 entries: the page's
    necessity argument is the capacity count."""
    assert 2 * (n - 2) < 2 * n - 2


def test_page_closed_forms(golden):
    g = golden["sliding_window_6_8"]
    M = 8
    n = M // 2
    assert n == g["N_pages"] and n - 1 == g["windows"]
    assert (2 * n - 2) / n == g["gamma"]
    assert oracle.lifted_k(g["K"], M) == g["K_lift"]
    s = golden["theoretical_speedup_6_8"]
    assert math.isclose(n / (n - 1), s["numerator"] / s["denominator"])
    for M in (4, 8, 16, 32):
        n = M // 2
        assert oracle.lifted_k(4096, M) * n == 4096 * (2 * n - 2)


@pytest.mark.parametrize("N,M", [(1, 4), (2, 4), (4, 8), (6, 8), (8, 16), (14, 16), (16, 32), (30, 32), (4, 6)])
def test_round_trip_and_nibbles(N, M):
    x = inputs.student_t_bf16((9, M * 12), 4.0, seed=M + N)
    keep = oracle.prune(x, N, M)
    vals, nib = oracle.compress(x, keep, M)
    assert set(np.unique(nib)) <= VALID_NIBBLES
    back = oracle.decompress(vals, nib, x.shape[1], M)
    np.testing.assert_array_equal(back, np.where(keep == 1, x, np.uint16(0)))
    # every stored value is either a kept value or a +0 pad
    kept_count = keep.sum()
    assert np.count_nonzero(vals) == np.count_nonzero(np.where(keep == 1, x, 0))
    assert vals.size - np.count_nonzero(vals == 0) <= kept_count


def test_window_example_6_of_8():
    # kept {0,2,3,4,6,7}: greedy gives w0 {0,2}, w1 {3,4}, w2 {6,7}
    x = inputs.bf16_from_f64(np.array([[5, 0.1, 5, 5, 5, 0.1, 5, 5]], dtype=np.float64))
    keep = oracle.prune(x, 6, 8)
    np.testing.assert_array_equal(keep[0], [1, 0, 1, 1, 1, 0, 1, 1])
    vals, nib = oracle.compress(x, keep, 8)
    # local indices: w0 (0,2) -> 0x8; w1 covers 2..5, holds 3,4 -> (1,2) -> 0x9;
    # w2 covers 4..7, holds 6,7 -> (2,3) -> 0xE
    np.testing.assert_array_equal(nib[0], [0x8, 0x9, 0xE])


def test_padding_rules():
    # 2:4 with N=1: the single kept entry is paired with the lowest other index
    x = inputs.bf16_from_f64(np.array([[0.1, 0.2, 9.0, 0.3, 7.0, 0.1, 0.2, 0.3]]))
    keep = oracle.prune(x, 1, 4)
    vals, nib = oracle.compress(x, keep, 4)
    np.testing.assert_array_equal(nib[0], [0x8, 0x4])            # (0,2), (0,1)
    np.testing.assert_array_equal(vals[0], [0, x[0, 2], x[0, 4], 0])
    # an empty window of a sparse 6:8 group is (0,1) with zeros
    x = inputs.bf16_from_f64(np.array([[1, 1, 1, 1, 0, 0, 0, 0]], dtype=np.float64))
    keep = oracle.prune(x, 4, 8)
    vals, nib = oracle.compress(x, keep, 8)
    # w0 takes positions 0,1; w1 takes 2,3 (its local 0,1); w2 is empty
    np.testing.assert_array_equal(nib[0], [0x4, 0x4, 0x4])
    np.testing.assert_array_equal(vals[0], [x[0, 0], x[0, 1], x[0, 2], x[0, 3], 0, 0])


@pytest.mark.parametrize("M", [4, 8, 16, 32])
def test_lift_map(M):
    n = M // 2
    K = M * 3
    src = np.arange(1, K + 1, dtype=np.float64)[None, :].repeat(2, axis=0)
    lifted = oracle.lift(inputs.bf16_from_f64(src), M)
    Kl = oracle.lifted_k(K, M)
    assert lifted.shape == (2, Kl)
    got = inputs.bf16_to_f64(lifted[0]).astype(int)
    expect = []
    for g in range(K // M):
        for w in range(n - 1):
            for j in range(4):
                expect.append(g * M + 2 * w + j + 1)
    np.testing.assert_array_equal(got, expect)


@pytest.mark.parametrize("N,M", [(2, 4), (6, 8), (8, 16), (16, 32)])
def test_expand_lifted_sums_back(N, M):
    """Summing the expanded lifted row over the lift map's duplicates gives
    back X (.) mask: every kept value appears exactly once in the windows."""
    x = inputs.normal_bf16((5, M * 7), 1.0, seed=3)
    keep = oracle.prune(x, N, M)
    vals, nib = oracle.compress(x, keep, M)
    ex = oracle.expand_lifted(vals, nib)
    n = M // 2
    K = x.shape[1]
    back = np.zeros((5, K))
    for g in range(K // M):
        for w in range(n - 1):
            for j in range(4):
                back[:, g * M + 2 * w + j] += ex[:, g * 4 * (n - 1) + 4 * w + j]
    np.testing.assert_array_equal(back, oracle.to_f64(x, keep))
