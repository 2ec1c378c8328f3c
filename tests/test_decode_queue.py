"""The one-launch decode step's work queue, modelled on the CPU.

`k_decode_step` (decode_tc.cu) runs a whole decode step in one cooperative launch: every CTA is
resident, and each takes items from a shared counter until none is left.  Some items wait for
others (bounded spins on per-head flags), so the order of the item list is what rules out a
deadlock: every item that waits comes after every item that it (transitively) waits for, and a
CTA only waits while it holds a claimed item, so all earlier items are claimed by CTAs that never
wait on later ones.  This model runs the item list with any number of resident CTAs under random
interleavings and checks:
- every wait ends (no deadlock), for every grid size;
- a unit tile reads its head's selection only after the selection is final;
- a head's final merge reads the merged sinks-and-window slot only after it is written;
- each head's output is written exactly once, after all of its tiles.
Planted mistakes (unit tiles listed before the scoring items; the window flag published before its
merge; the final merge not waiting for the window flag) must each fail a check.
"""
from __future__ import annotations

import random

import pytest


def items(hkv, n_win, n_score, n_unit, plant=None):
    win = [("win", h, i) for h in range(hkv) for i in range(n_win)]
    score = [("score", h, i) for h in range(hkv) for i in range(n_score)]
    unit = [("unit", h, i) for h in range(hkv) for i in range(n_unit)]
    return win + unit + score if plant == "units_first" else win + score + unit


def run(grid, hkv, n_win, n_score, n_unit, seed, plant=None):
    rnd = random.Random(seed)
    todo = items(hkv, n_win, n_score, n_unit, plant)
    nxt = [0]
    cnt = {(k, h): 0 for k in ("win", "score", "unit") for h in range(hkv)}
    sel_flag = [False] * hkv      # selection final
    win_flag = [False] * hkv      # sinks and window merged into their slot
    win_slot = [False] * hkv      # the merged slot's contents are written
    sel_done = [False] * hkv
    out = [0] * hkv
    unit_done = [0] * hkv

    def cta():
        while True:
            i = nxt[0]
            nxt[0] += 1
            yield
            if i >= len(todo):
                return
            kind, h, _ = todo[i]
            if kind == "unit":
                while not sel_flag[h]:  # bounded spin in the kernel; the model counts steps instead
                    yield
                assert sel_done[h], f"unit tile of head {h} read an unfinished selection"
            yield  # the item's work
            if kind == "unit":
                unit_done[h] += 1
            cnt[(kind, h)] += 1
            last = cnt[(kind, h)] == {"win": n_win, "score": n_score, "unit": n_unit}[kind]
            if not last:
                continue
            if kind == "score":
                sel_done[h] = True
                yield
                sel_flag[h] = True
            elif kind == "win":
                if plant == "flag_before_merge":
                    win_flag[h] = True
                    yield
                    win_slot[h] = True
                else:
                    win_slot[h] = True
                    yield
                    win_flag[h] = True
            else:
                if plant != "merge_skips_window_flag":
                    while not win_flag[h]:
                        yield
                assert win_slot[h], f"head {h} merged before its sinks and window were merged"
                assert unit_done[h] == n_unit
                out[h] += 1

    ctas = [cta() for _ in range(grid)]
    alive = list(range(grid))
    # CTAs progress at very different rates (a random speed each), so one can lag far behind
    speed = [rnd.choice((0.002, 0.05, 1.0)) for _ in range(grid)]
    steps = 0
    while alive:
        k = rnd.choices(alive, weights=[speed[a] for a in alive])[0]
        try:
            next(ctas[k])
        except StopIteration:
            alive.remove(k)
        steps += 1
        assert steps < 60000, "deadlock"
    assert out == [1] * hkv


@pytest.mark.parametrize("grid", [1, 2, 3, 7, 40, 500])
def test_every_wait_ends_and_every_handoff_is_ordered(grid):
    for seed in range(60):
        run(grid, hkv=3, n_win=4, n_score=5, n_unit=3, seed=seed)


@pytest.mark.parametrize("plant", ["units_first", "flag_before_merge", "merge_skips_window_flag"])
def test_planted_mistakes_are_caught(plant):
    caught = 0
    for grid in (1, 2, 5):
        for seed in range(60):
            try:
                run(grid, hkv=3, n_win=4, n_score=5, n_unit=3, seed=seed, plant=plant)
            except AssertionError:
                caught += 1
    assert caught > 0, plant
