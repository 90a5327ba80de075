"""A model of the per-group selection's decisions (topk_kernel.cuh), run on
the CPU against the oracle's select_kv.

The kernel finds the k-th largest score T by a radix select over the 31
magnitude bits in digits of 12, 10 and 9 bits, on a candidate list when it
can.  Its one walk over a row lists the keys whose first digit is at least a
guess (the previous row's threshold digit less one bin); when at least k keys
are listed and the list (6144 entries) did not overflow, it resolves all
three digits on the list alone.  Otherwise it counts the first digit over
the row and lists the keys at or above the threshold's first digit, or, if
those overflow the list too, resolves the digits over the whole row.  The
model keeps exactly those decisions and checks, row after row, that every
path gives the oracle's selection: the exactness argument is that the
listed keys include the k largest and every key equal to the k-th.
"""
import numpy as np
import pytest

from oracle import mcs_oracle as orc

DIGITS = ((19, 12), (9, 10), (0, 9))   # (shift, width) of the three digits
NB1 = 1 << 12
CAP = 6144
MARGIN = 1


def radix_threshold(bits: np.ndarray, k: int):
    """T (the k-th largest of `bits`) and how many keys equal to T are kept,
    digit by digit from the top, each digit's histogram over the keys that
    match the digits found so far."""
    kk, prefix, mask = k, 0, 0
    for shift, width in DIGITS:
        nb = 1 << width
        sel = bits[(bits & mask) == prefix]
        hist = np.bincount((sel >> shift) & (nb - 1), minlength=nb)
        from_top = np.cumsum(hist[::-1])
        i = int(np.searchsorted(from_top, kk))      # first bin from the top reaching kk
        b = nb - 1 - i
        kk -= int(from_top[i] - hist[b])
        prefix |= b << shift
        mask |= (nb - 1) << shift
    return prefix, kk


def select_model(row: np.ndarray, k: int, guess: int):
    """(selected indices ascending, the threshold's first digit, path)."""
    bits = row.view(np.uint32) & np.uint32(0x7FFFFFFF)
    N = bits.size
    if k >= N:
        return np.arange(N), NB1, "all"
    d1 = bits >> 19
    cand, path, miss = None, "walk", ""
    if guess < NB1:
        listed = np.nonzero(d1 >= guess)[0]
        if k <= listed.size <= CAP:
            cand, path = listed, "guess"
        else:
            miss = " (too few listed)" if listed.size < k else " (list overflow)"
    if cand is None:
        hist = np.bincount(d1, minlength=NB1)
        from_top = np.cumsum(hist[::-1])
        b1 = NB1 - 1 - int(np.searchsorted(from_top, k))
        if int(from_top[NB1 - 1 - b1]) <= CAP:      # keys at or above b1's bin
            cand, path = np.nonzero(d1 >= b1)[0], "relist" + miss
    src = bits[cand] if cand is not None else bits
    T, need_eq = radix_threshold(src, k)
    gt = np.nonzero(bits > T)[0]
    eq = np.nonzero(bits == T)[0][:need_eq]
    return np.sort(np.concatenate([gt, eq])), int(T >> 19), path


def run_rows(rows: np.ndarray, k: int):
    guess, paths = NB1, []
    for r in range(rows.shape[0]):
        got, b1, path = select_model(rows[r], k, guess)
        ref = orc.select_kv(rows[r].astype(np.float64), k)
        assert np.array_equal(got, ref), f"row {r} ({path}): {np.setxor1d(got, ref).size} indices differ"
        paths.append(path)
        guess = b1 - MARGIN if b1 > MARGIN else 0
    return paths


def test_alike_rows_take_the_guessed_list():
    rng = np.random.default_rng(1)
    rows = rng.lognormal(-9.0, 0.6, size=(40, 8000)).astype(np.float32)
    paths = run_rows(rows, 400)
    assert paths[0] == "relist" and paths[1:].count("guess") >= 35


def test_scale_jumps_miss_the_guess_both_ways():
    """Runs of alike rows broken by rows scaled by 2^12 either way: a row far
    above its guess lists too few keys, a row far below lists them all and
    overflows the list; both are listed again at their own threshold."""
    rng = np.random.default_rng(2)
    rows = rng.lognormal(-9.0, 0.6, size=(30, 8000)).astype(np.float32)
    rows[2::5] *= np.float32(2.0 ** 12)
    rows[4::5] *= np.float32(2.0 ** -12)
    paths = run_rows(rows, 400)
    assert paths.count("guess") >= 5
    assert "relist (too few listed)" in paths and "relist (list overflow)" in paths


def test_ties_and_constant_rows():
    rng = np.random.default_rng(3)
    few = rng.choice(np.array([0.0, 1e-6, 2.5e-3, 0.125], np.float32), size=(6, 9000), p=[0.4, 0.3, 0.25, 0.05])
    const = np.full((3, 9000), 3.0e-4, np.float32)
    zeros = np.zeros((2, 9000), np.float32)
    rows = np.concatenate([few, const, few[:2], zeros])
    paths = run_rows(rows, 1000)
    assert "walk" in paths                  # a constant row's first bin holds all 9000 keys


@pytest.mark.parametrize("k", [1, 2, CAP - 1, CAP, CAP + 1])
def test_list_capacity_edges(k):
    """n listed == k and n listed == capacity, exactly."""
    rng = np.random.default_rng(k)
    N = 3 * CAP
    rows = np.empty((6, N), np.float32)
    for r in range(6):
        # a block of exactly CAP keys in one high bin above a spread of low keys
        low = rng.uniform(1e-6, 2e-6, size=N - CAP).astype(np.float32)
        high = np.float32(0.5) + rng.integers(0, 1 << 12, size=CAP).astype(np.float32) * np.float32(2.0 ** -24)
        rows[r] = rng.permutation(np.concatenate([low, high]))
    paths = run_rows(rows, min(k, N))
    if k <= CAP:
        assert paths[1:].count("guess") == 5
