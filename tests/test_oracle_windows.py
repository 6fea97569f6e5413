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


def _check_assignment_fast(masks, M, win, slot, st):
    """The invariants of _check_assignment in whole-array form, for large
    batches of 32-position groups: every kept position is placed once, in a
    window that covers it; along the kept positions the (window, slot) order
    strictly increases, so no window holds more than two entries and no slot
    is used twice; a slot 1 always follows its window's slot 0."""
    assert M == 32
    bits = np.unpackbits(masks.astype("<u4").view(np.uint8).reshape(-1, 4), axis=1, bitorder="little").view(bool)
    assert (st == 0).all()
    assert ((win >= 0) == bits).all()
    half = (np.arange(M) // 2).astype(np.int8)[None, :]
    d = half - win                                  # 0 or 1 for a kept position (window w covers 2w .. 2w+3)
    assert (((d == 0) | (d == 1)) & (win <= M // 2 - 2) | ~bits).all()
    o = np.where(bits, 2 * win + slot, np.int8(-1))
    prev = np.empty_like(o)
    prev[:, 0] = -1
    np.maximum.accumulate(o[:, :-1], axis=1, out=prev[:, 1:])
    assert ((o > prev) | ~bits).all()
    assert ((slot == 0) | (prev == o - 1) | ~bits).all()


def test_greedy_fits_every_pair_count_vector_32():
    """n-1 windows suffice for every pattern of at most 2n-2 kept entries, for
    2n = 32.  The greedy fills window w from pairs w and w+1, so whether a
    pattern fits depends on how many entries of each pair are kept (0, 1 or
    2); all 3^16 such pair-count vectors are enumerated, each as one mask (a
    pair keeping one entry keeps its lower or its upper position, chosen by a
    multiplicative hash), as every pairing of the 3^8 vectors of the lower
    eight pairs with the 3^8 of the upper eight.  The 17 vectors with 31 or
    32 kept entries must fail."""
    M, H = 32, 8                                  # two halves of 8 pairs: 3^8 vectors each
    v = np.arange(3 ** H, dtype=np.int64)
    cnt = (v[:, None] // (3 ** np.arange(H, dtype=np.int64))[None, :]) % 3
    h = (v.astype(np.uint64) * np.uint64(0x9E3779B1)) >> np.uint64(7)
    upper = ((h[:, None] >> np.arange(H, dtype=np.uint64)) & np.uint64(1)).astype(bool)
    lo = (cnt == 2) | ((cnt == 1) & ~upper)
    hi = (cnt == 2) | ((cnt == 1) & upper)
    sh = (2 * np.arange(H)).astype(np.uint64)
    half = ((lo.astype(np.uint64) << sh) | (hi.astype(np.uint64) << (sh + np.uint64(1)))).sum(axis=1, dtype=np.uint64)
    half_pop = cnt.sum(axis=1)
    # the upper half's choice of position is decorrelated from the lower's
    half_hi = np.roll(half, 1234)
    pop_hi = np.roll(half_pop, 1234)
    failing = 0
    step = 256
    for b0 in range(0, v.size, step):
        masks = (half[None, :] | (half_hi[b0:b0 + step, None] << np.uint64(16))).ravel()
        pop = (half_pop[None, :] + pop_hi[b0:b0 + step, None]).ravel()
        win, slot, st = oracle.window_assign_batch(masks, M)
        fits = pop <= M - 2
        if fits.all():
            _check_assignment_fast(masks, M, win, slot, st)
        else:
            _check_assignment_fast(masks[fits], M, win[fits], slot[fits], st[fits])
            assert (st[~fits] != 0).all()
            failing += int((~fits).sum())
    assert failing == 17


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
