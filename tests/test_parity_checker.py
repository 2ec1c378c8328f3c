"""The near-tie rule the parity tests apply to selections (CPU only).

Where the oracle's fp64 gap at the cut is not decisive (at most 1e-3 relative), several index
sets are correct; valid_near_tie accepts exactly those that differ from the exact top-k only
inside the decisive rule's band.  Each planted wrong choice below must be refused.
"""
from __future__ import annotations

import numpy as np

from oracle import infllm_oracle as O
from tests._parity import valid_near_tie


def test_exact_topk_is_always_valid():
    rng = np.random.default_rng(5)
    for _ in range(200):
        n = int(rng.integers(1, 40))
        s = rng.normal(size=n) * 10.0 ** rng.integers(-3, 4)
        if rng.random() < 0.3:
            s = np.round(s)  # exact ties
        k = int(rng.integers(1, n + 2))
        assert valid_near_tie(s, O.topk_stable(s, min(k, n)), k)


def test_clear_winner_must_be_kept():
    # {A: 10, B: 5, C: 5.0001}, k = 2: A must be chosen; B and C are a near-tie
    s = [10.0, 5.0, 5.0001]
    assert not O.decisive(s, 2)
    assert valid_near_tie(s, [0, 2], 2)
    assert valid_near_tie(s, [0, 1], 2)
    assert not valid_near_tie(s, [1, 2], 2)


def test_clear_loser_must_be_left_out():
    s = [10.0, 5.0, 5.0001, 4.0]
    assert not valid_near_tie(s, [0, 3], 2)
    assert not valid_near_tie(s, [2, 3], 2)


def test_count_distinctness_and_range():
    s = [3.0, 2.0, 2.0, 1.0]
    assert valid_near_tie(s, [0, 2], 2)
    assert not valid_near_tie(s, [0, 0], 2)      # repeated id
    assert not valid_near_tie(s, [0], 2)         # too few
    assert not valid_near_tie(s, [0, 1, 2], 2)   # too many
    assert not valid_near_tie(s, [0, 4], 2)      # out of range
    assert not valid_near_tie(s, [0, -1], 2)
    assert valid_near_tie(s, [3, 1, 2, 0], 9)    # k above n: every id, once


def test_band_is_the_decisive_rule():
    # s_(k) = 100, s_(k+1) = 100 - g: swapping is allowed only while g <= 1e-3 * 100
    for g, ok in ((0.05, True), (0.1, True), (0.2, False), (1.0, False)):
        s = [200.0, 100.0, 100.0 - g, 50.0]
        assert O.decisive(s, 2) == (not ok)
        assert valid_near_tie(s, [0, 2], 2) == ok
