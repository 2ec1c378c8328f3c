"""The one-launch decode step's schedule, modelled on the CPU.

`k_decode_step` (decode_tc.cu) runs a whole decode step in one cooperative launch: every CTA is
resident.  CTA c of a grid of G, in order:
  1. the window items c, c + G, ... (sink and window tiles); the head's last one merges them, after
     step 2 when the grid covers every window tile;
  2. its static range of the scoring rows, head-major; at the end of each head's part it publishes
     its list; the head's last CTA to publish selects, and publishes each selected slot (with the
     unit id) on the slot's flag;
  3. the deferred window merge, published on the head's window flag;
  4. unit tiles claimed from a counter (the next claim made as an item starts): each waits for its
     slot's flag; the head's last one waits for the window flag and merges into the output.
Steps 1-3 wait for nothing and the unit tiles wait only for steps 1-3, so every wait ends.  This
model runs the schedule with several grid sizes under random interleavings and checks:
- every wait ends (no deadlock);
- a unit tile reads its slot only after the head's selection is final;
- a head's final merge reads the merged sinks-and-window slot only after it is written;
- each head's output is written exactly once, after all of its tiles;
- the claim counter ends at (unit tiles) + G: the host's base for the next step.
Planted mistakes (unit tiles claimed before the CTA's scoring range; a slot flag published before
the selection is final; the window flag published before its merge; the final merge not waiting for
the window flag) must each fail a check.
"""
from __future__ import annotations

import random

import pytest


def run(grid, hkv, n_win, nm, n_unit, seed, plant=None):
    rnd = random.Random(seed)
    n_total = hkv * nm
    # static scoring ranges: [c N / G, (c + 1) N / G) of flat units (plain split)
    f0 = [c * n_total // grid for c in range(grid + 1)]
    parts = [sorted({c for c in range(grid) for f in range(f0[c], f0[c + 1]) if f // nm == h}) for h in range(hkv)]
    nw = hkv * n_win
    n_units = hkv * n_unit
    claim = [0]
    win_cnt = [0] * hkv
    pub_cnt = [0] * hkv
    unit_cnt = [0] * hkv
    slot_flag = [[False] * n_unit for _ in range(hkv)]
    sel_done = [False] * hkv
    win_slot = [False] * hkv
    win_flag = [False] * hkv
    out = [0] * hkv

    def cta(c):
        deferred = []

        def window_merge(h):
            if plant == "flag_before_merge":
                win_flag[h] = True
                yield
                win_slot[h] = True
            else:
                win_slot[h] = True
                yield
                win_flag[h] = True

        def units():
            nxt = claim[0]
            claim[0] += 1
            yield
            while True:
                i = nxt
                if i >= n_units:
                    return
                nxt = claim[0]
                claim[0] += 1
                h, s = divmod(i, n_unit)
                while not slot_flag[h][s]:  # bounded spin in the kernel; the model counts steps
                    yield
                assert sel_done[h], f"unit tile of head {h} read slot {s} of an unfinished selection"
                yield  # the tile
                unit_cnt[h] += 1
                if unit_cnt[h] == n_unit:
                    if plant != "merge_skips_window_flag":
                        while not win_flag[h]:
                            yield
                    assert win_slot[h], f"head {h} merged before its sinks and window were merged"
                    out[h] += 1

        if plant == "units_before_scoring":
            yield from units()
        for w in range(c, nw, grid):  # 1. window tiles
            yield
            h = w // n_win
            win_cnt[h] += 1
            if win_cnt[h] == n_win:
                if grid >= nw:
                    deferred.append(h)
                else:
                    yield from window_merge(h)
        heads = sorted({f // nm for f in range(f0[c], f0[c + 1])})  # 2. scoring range
        for h in heads:
            yield  # this head's part of the range
            pub_cnt[h] += 1
            if pub_cnt[h] == len(parts[h]):  # the head's last list: select, publish slot by slot
                if plant == "slot_before_select":
                    slot_flag[h][0] = True
                    yield
                yield
                sel_done[h] = True
                for s in range(n_unit):
                    yield
                    slot_flag[h][s] = True
        for h in deferred:  # 3. deferred window merges
            yield from window_merge(h)
        if plant != "units_before_scoring":
            yield from units()  # 4. unit tiles

    ctas = [cta(c) for c in range(grid)]
    alive = list(range(grid))
    speed = [rnd.choice((0.002, 0.05, 1.0)) for _ in range(grid)]  # CTAs progress at very different rates
    steps = 0
    while alive:
        k = rnd.choices(alive, weights=[speed[a] for a in alive])[0]
        try:
            next(ctas[k])
        except StopIteration:
            alive.remove(k)
        steps += 1
        assert steps < 80000, "deadlock"
    assert out == [1] * hkv
    assert claim[0] == n_units + grid  # every CTA's last claim overshoots once


@pytest.mark.parametrize("grid", [1, 2, 3, 7, 13, 40])
def test_every_wait_ends_and_every_handoff_is_ordered(grid):
    for seed in range(40):
        run(grid, hkv=3, n_win=4, nm=10, n_unit=3, seed=seed)


@pytest.mark.parametrize("plant", ["units_before_scoring", "slot_before_select", "flag_before_merge",
                                   "merge_skips_window_flag"])
def test_planted_mistakes_are_caught(plant):
    caught = 0
    for grid in (1, 2, 5, 13):
        for seed in range(40):
            try:
                run(grid, hkv=3, n_win=4, nm=10, n_unit=3, seed=seed, plant=plant)
            except AssertionError:
                caught += 1
    assert caught > 0, plant


def _f0(c, gs, n, t, wr, nw_cta, weighted):
    """Start of CTA c's scoring range, as `score_f0` in decode_tc.cu computes it."""
    if c >= gs:
        return n
    if weighted:
        r = c * t // gs - wr * min(c, nw_cta)
        return min(max(r, 0), n)
    return c * n // gs


def _split(grid, hkv, nm, nw, wr, splits_max):
    """The host's choice of split (launch_decode_step): weighted when every CTA's share of rows
    plus window rows exceeds a window tile, else plain with ranges of at least 16 rows; halved
    until every head's parts fit its list slots."""
    n = hkv * nm
    nw_cta = min(nw, grid)
    t = n + nw_cta * wr
    weighted = grid > nw and t // grid >= wr + 1
    gs = grid if weighted else max(1, min(grid, n // 16))

    def owner(f):
        lo, hi = 0, gs - 1
        while lo < hi:
            mid = (lo + hi + 1) // 2
            if _f0(mid, gs, n, t, wr, nw_cta, weighted) <= f:
                lo = mid
            else:
                hi = mid - 1
        return lo

    while True:
        worst = max(owner((h + 1) * nm - 1) - owner(h * nm) + 1 for h in range(hkv))
        if worst <= splits_max:
            break
        weighted = False
        gs = max(1, gs // 2)
    return [_f0(c, gs, n, t, wr, nw_cta, weighted) for c in range(grid + 1)], owner, worst


@pytest.mark.parametrize("grid,hkv,nm,nw,wr,units_max", [
    (444, 8, 8192, 272, 64, 8300),     # 1M-token memory, REPS rows (1 KB): weighted
    (444, 8, 8192, 272, 256, 8300),    # MEANKEY rows (256 B): weighted, barely
    (444, 8, 8192, 272, 128, 8300),    # REPSUM rows (512 B)
    (444, 2, 20, 10, 64, 40),          # a small memory: plain, ranges of >= 16 rows
    (444, 2, 3, 10, 64, 4),            # three units per head, four list slots
    (296, 8, 1000, 300, 64, 1100),     # more window tiles than CTAs: plain
    (148, 1, 1, 5, 64, 2),             # one unit
])
def test_scoring_split_covers_every_unit_once(grid, hkv, nm, nw, wr, units_max):
    f, owner, worst = _split(grid, hkv, nm, nw, wr, units_max // 4 + 1)
    n = hkv * nm
    assert f[0] == 0 and f[-1] == n
    assert all(a <= b for a, b in zip(f, f[1:]))  # non-decreasing: every unit in exactly one range
    nonempty = [c for c in range(grid) if f[c] < f[c + 1]]
    assert nonempty == list(range(len(nonempty)))  # the non-empty ranges are the first ones, contiguous
    for h in range(hkv):  # the head's parts are CTAs owner(h nm) .. owner((h + 1) nm - 1), all non-empty
        first, last = owner(h * nm), owner((h + 1) * nm - 1)
        assert all(f[c] < f[c + 1] for c in range(first, last + 1))
        assert f[first] <= h * nm < f[first + 1] and f[last] <= (h + 1) * nm - 1 < f[last + 1]
    assert worst <= units_max // 4 + 1
