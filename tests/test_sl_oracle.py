"""Pins of the Stochastic Length oracle (``oracle/stochastic_length.py``), CPU only.

Each test ties the oracle to something it does not compute itself: the pair of
lengths the HSTU walkthrough prints ("Three more scaling components /
Stochastic Length": alpha = 1.6 maps 4,096 to 776, 64%-84% sparsity), closed
forms at exact powers of two, a brute-force rank definition of the selected
subset, the exact integer threshold of the keep-whole draw, invariants of the
output batch, and sampling statistics (uniform inclusion, keep-whole rate,
expected kept attention cost).  ``test_sl_pins_catch_planted_mistakes`` plants
plausible mistakes in the oracle and checks that a pin fails on each.
"""
import math
import os

import numpy as np
import pytest

from oracle import stochastic_length as SL
from hstu_sequential_transducer_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "stochastic_length.txt")):
        if line.strip() and not line.startswith("#"):
            n, a, L = line.split()
            rows.append((int(n), float(a), int(L)))
    return rows


def check_lengths():
    for n, a, L in golden_rows():
        assert SL.subsequence_length(n, a) == L, (n, a)
    L = SL.subsequence_length(4096, 1.6)
    assert 0.64 <= 1.0 - L / 4096 <= 0.84


def brute_select(keys, L):
    """Position j is selected iff fewer than L pairs (key, position) are
    smaller than (key_j, j)."""
    h = len(keys)
    out = []
    for j in range(h):
        smaller = 0
        for i in range(h):
            if int(keys[i]) < int(keys[j]) or (keys[i] == keys[j] and i < j):
                smaller += 1
        if smaller < L:
            out.append(j)
    return np.array(out, dtype=np.int64)


def check_brute_select():
    rng = np.random.default_rng(7)
    for trial in range(60):
        h = int(rng.integers(1, 40))
        L = int(rng.integers(0, h + 1))
        hi = 4 if trial % 2 else 1 << 32
        keys = rng.integers(0, hi, size=h, dtype=np.uint64).astype(np.uint32)
        np.testing.assert_array_equal(SL.select_history(keys, L), brute_select(keys, L))


def check_keep_threshold():
    # L = 776, h = 4096: L^2/h^2 * 2^32 = 776^2 * 256 = 154,157,056 exactly.
    thr = 776 * 776 * 256
    assert SL.keep_whole(4096, 776, thr - 1)
    assert not SL.keep_whole(4096, 776, thr)
    # h <= L always keeps; the largest draw never keeps a longer history.
    assert SL.keep_whole(776, 776, 0xFFFFFFFF)
    assert not SL.keep_whole(777, 776, 0xFFFFFFFF)


def check_batch_invariants():
    rng = np.random.default_rng(3)
    for trial in range(20):
        B = int(rng.integers(1, 12))
        lengths = rng.integers(0, 300, size=B)
        offs = W.offsets_from_lengths(lengths)
        nt = None
        if trial % 2:
            nt = np.array([int(rng.integers(0, n + 1)) for n in lengths], dtype=np.int32)
        L = int(rng.integers(0, 120))
        keep, keys = W.sl_draws(100 + trial, B, int(offs[-1]), key_range=8 if trial % 3 == 0 else None)
        new_offs, gi = SL.sample(offs, nt, L, keep, keys)
        assert new_offs[0] == 0 and new_offs[-1] == len(gi)
        for b in range(B):
            s, e = int(offs[b]), int(offs[b + 1])
            m = 0 if nt is None else int(nt[b])
            h = e - s - m
            rows = gi[new_offs[b]:new_offs[b + 1]]
            assert np.all(np.diff(rows) > 0)
            assert rows.size == 0 or (rows[0] >= s and rows[-1] < e)
            np.testing.assert_array_equal(rows[rows >= s + h], np.arange(s + h, e))
            whole = h <= L or float(keep[b]) < (L * L) / (h * h) * 2.0 ** 32
            if whole:
                np.testing.assert_array_equal(rows, np.arange(s, e))
            else:
                assert rows.size == L + m
                np.testing.assert_array_equal(rows[:L] - s, brute_select(keys[s:s + h], L)
                                              if h <= 150 else SL.select_history(keys[s:s + h], L))


def check_statistics():
    # One history of h = 4096 at L = 776, many independent draws.
    h, L, trials = 4096, 776, 4000
    p = (L / h) ** 2
    offs = np.array([0, h], dtype=np.int64)
    kept, cost, incl = 0, 0.0, np.zeros(h)
    for t in range(trials):
        keep, keys = W.sl_draws(10_000 + t, 1, h)
        new_offs, gi = SL.sample(offs, None, L, keep, keys)
        n = int(new_offs[-1])
        kept += n == h
        cost += n * n
        if n == L:
            incl[gi] += 1
    sd = math.sqrt(trials * p * (1 - p))
    assert abs(kept - trials * p) < 5 * sd
    # E[h_kept^2] = p h^2 + (1 - p) L^2 = 2 L^2 - L^4 / h^2.
    expect = 2 * L * L - L ** 4 / h ** 2
    var = p * (1 - p) * (h * h - L * L) ** 2
    assert abs(cost / trials - expect) < 5 * math.sqrt(var / trials)
    # Uniform inclusion: each position selected with probability L / h in the
    # sampled draws; compare the early, middle and late thirds.
    sampled = trials - kept
    frac = incl / sampled
    for part in np.array_split(frac, 3):
        assert abs(part.mean() - L / h) < 0.01
    assert abs(frac.mean() - L / h) < 1e-12


def test_sl_lengths_golden():
    check_lengths()


def test_sl_select_brute_force():
    check_brute_select()


def test_sl_keep_threshold_exact():
    check_keep_threshold()


def test_sl_batch_invariants():
    check_batch_invariants()


def test_sl_statistics():
    check_statistics()


def test_sl_gather_rows():
    x = np.arange(30, dtype=np.float64).reshape(10, 3)
    gi = np.array([0, 3, 4, 9], dtype=np.int64)
    np.testing.assert_array_equal(SL.gather(x, gi), x[[0, 3, 4, 9]])


def test_sl_alpha_two_is_identity():
    lengths = [5, 4096, 100, 0, 3000]
    offs = W.offsets_from_lengths(lengths)
    keep, keys = W.sl_draws(1, len(lengths), int(offs[-1]))
    L = SL.subsequence_length(4096, 2.0)
    new_offs, gi = SL.sample(offs, None, L, keep, keys)
    np.testing.assert_array_equal(new_offs, offs)
    np.testing.assert_array_equal(gi, np.arange(offs[-1]))


# ----------------------------------------------------------------------------
# Planted mistakes: each must make a pin above fail.
# ----------------------------------------------------------------------------

def _fails(check):
    try:
        check()
    except AssertionError:
        return True
    return False


def test_sl_pins_catch_planted_mistakes(monkeypatch):
    orig_keep, orig_sel, orig_len = SL.keep_whole, SL.select_history, SL.subsequence_length

    def keep_linear(h, L, draw):  # probability L/h instead of (L/h)^2
        return h <= L or float(draw) < (L / h) * SL.TWO32

    def sel_largest(keys_b, L):  # largest keys instead of smallest
        pos = np.arange(len(keys_b))
        order = np.lexsort((pos, -keys_b.astype(np.int64)))
        return np.sort(order[:L])

    def sel_ties_late(keys_b, L):  # ties broken by the later position
        pos = np.arange(len(keys_b))
        order = np.lexsort((-pos, keys_b.astype(np.int64)))
        return np.sort(order[:L])

    def sel_most_recent(keys_b, L):  # the last L positions, not a random subset
        h = len(keys_b)
        return np.arange(max(0, h - L), h)

    def len_ceil(n, a):
        return int(math.ceil(float(n) ** (a / 2.0)))

    def len_full_exponent(n, a):  # N^alpha instead of N^(alpha/2)
        return int(math.floor(float(n) ** a)) if n > 0 else 0

    cases = [
        ("keep_whole", keep_linear, check_keep_threshold),
        ("select_history", sel_largest, check_brute_select),
        ("select_history", sel_ties_late, check_brute_select),
        ("select_history", sel_most_recent, check_statistics),
        ("subsequence_length", len_ceil, check_lengths),
        ("subsequence_length", len_full_exponent, check_lengths),
    ]
    for name, bad, check in cases:
        monkeypatch.setattr(SL, name, bad)
        assert _fails(check), (name, bad.__name__)
        monkeypatch.setattr(SL, "keep_whole", orig_keep)
        monkeypatch.setattr(SL, "select_history", orig_sel)
        monkeypatch.setattr(SL, "subsequence_length", orig_len)

    def sample_drop_targets(seq_offsets, num_targets, L, keep_draw, keys):
        offs = np.asarray(seq_offsets)
        nt = None if num_targets is None else np.zeros_like(num_targets)
        new_offs, gi = orig_sample(offs, nt, L, keep_draw, keys)
        return new_offs, gi

    orig_sample = SL.sample
    monkeypatch.setattr(SL, "sample", sample_drop_targets)
    assert _fails(check_batch_invariants)
    monkeypatch.setattr(SL, "sample", orig_sample)
