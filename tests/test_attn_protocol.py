"""The tcgen05 prefill attention kernel's barrier protocol, modelled and explored on the CPU.

No compute-sanitizer run of this kernel exists, so its synchronisation is checked on a model
instead: the roles of `k_attn_tc` (attend_tc.cu) as coroutines that a seeded scheduler
interleaves at random, with exact mbarrier parity semantics.
- TMA producer: two query tiles, then K and V tiles through 2-stage rings. Slot s is refilled
  with tile i once QK(i - 2) / PV(i - 2) is complete, seen on the S / PV barriers of parity s
  (there are no separate slot-release barriers).
- MMA issuer: QK(i) into S buffer i & 1, then PV(i - 1) into O_{(i - 1) & 1} after P(i - 1) is
  released.
- Tensor pipe: executes one thread's MMAs in issue order; each commit arrives when every
  earlier MMA is done.
- TMA engine: lands copies in any order.
- Two softmax groups: group g takes the tiles i with i & 1 == g, reads all of S(i), writes P(i)
  over it and keeps its own online softmax and accumulator O_g. Before it waits for S(i) it
  consumes its previous PV, so it rescales O_g and releases P(i) only after that PV is complete
  (and the PV barrier of its parity is never two phases ahead of it).

Every data hand-off is asserted where it happens:
- a ring slot is refilled only after the MMA that read it has executed;
- S(i) is read only once QK(i) has written it, and is not overwritten before its group read it;
- PV(j) reads P(j), and never a stale one;
- O_g is read or rescaled only when no PV that writes it is pending;
- a parity wait never runs two or more phases behind its barrier, where parity aliases, nor
  starts before the previous phase completed, where it would pass early;
- no interleaving deadlocks (bounded step count).
A planted protocol mistake must fail the same checks (last test).
"""
from __future__ import annotations

import os
import random
import re

import pytest

NSTAGE = 2
KERNEL = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "block_memory_sparse_b200", "csrc",
                      "attend_tc.cu")


class Bar:
    """mbarrier: `count` arrivals complete a phase; a parity wait for phase j is true once phase j
    has completed. It aliases if two or more phases completed past it (it would wait for a third),
    and it passes early if phase j - 1 has not completed yet (phase j - 2 has j's parity)."""

    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1

    def done(self, j):
        assert self.phase < j + 2, f"{self.name}: parity wait for phase {j} after {self.phase} completed phases"
        assert self.phase >= j, f"{self.name}: parity wait for phase {j} with only {self.phase} completed (passes early)"
        return self.phase > j


def run(NT, seed, plant=None):
    rnd = random.Random(seed)
    bars = {"q": Bar("q", 1)}
    for g in (0, 1):
        for x in ("sfull", "pfull", "pvdone"):
            bars[f"{x}{g}"] = Bar(f"{x}{g}", 1)  # pfull: one arrival stands for the group's threads
    for s in range(NSTAGE):
        for x in ("kfull", "vfull"):
            bars[f"{x}{s}"] = Bar(f"{x}{s}", 1)
    kslot = [None] * NSTAGE   # tile whose K occupies the slot
    vslot = [None] * NSTAGE
    kread = [-1] * NSTAGE     # last tile whose QK has executed on that slot
    vread = [-1] * NSTAGE
    S = [None, None]          # per buffer: [tile, read by its group?]
    P = [None, None]          # per buffer: tile of the P stored there, or ("used", tile)
    pv_done = []              # PV tiles executed, in order
    pipe = []                 # issued, not yet executed tensor-pipe ops
    tma = []                  # copies in flight
    q_landed = [False]

    def wait(name, j):
        while not bars[name].done(j):
            yield

    def producer():
        tma.append(("q", None, None))
        for i in range(NT):
            s, use = i % NSTAGE, i // NSTAGE
            if i >= NSTAGE and plant != "k_slot_not_released":
                yield from wait(f"sfull{s}", use - 1)
            tma.append(("k", s, i))
            yield
            if i >= NSTAGE:
                yield from wait(f"pvdone{s}", use - 1)
            tma.append(("v", s, i))
            yield

    def tma_engine():
        while True:
            if tma:
                op, s, i = tma.pop(rnd.randrange(len(tma)))
                if op == "q":
                    q_landed[0] = True
                    bars["q"].arrive()
                elif op == "k":
                    assert i < NSTAGE or kread[s] == i - NSTAGE, \
                        f"K slot {s} refilled with tile {i} before QK({i - NSTAGE}) ran"
                    kslot[s] = i
                    bars[f"kfull{s}"].arrive()
                else:
                    assert i < NSTAGE or vread[s] == i - NSTAGE, \
                        f"V slot {s} refilled with tile {i} before PV({i - NSTAGE}) ran"
                    vslot[s] = i
                    bars[f"vfull{s}"].arrive()
            yield

    def mma():
        yield from wait("q", 0)
        for i in range(NT + 1):
            if i < NT:
                s, use = i % NSTAGE, i // NSTAGE
                yield from wait(f"kfull{s}", use)
                pipe.extend([("qk", i), ("commit", f"sfull{i & 1}")])
                yield
            if i >= 1:
                j = i - 1
                yield from wait(f"pfull{j & 1}", j >> 1)
                if plant != "pv_skips_v_wait":
                    yield from wait(f"vfull{j % NSTAGE}", j // NSTAGE)
                pipe.extend([("pv", j), ("commit", f"pvdone{j & 1}")])
                yield

    def tensor_pipe():
        while True:
            if pipe:
                op, x = pipe.pop(0)
                if op == "qk":
                    b, s = x & 1, x % NSTAGE
                    assert q_landed[0]
                    assert kslot[s] == x, f"QK({x}) read K slot {s} holding {kslot[s]}"
                    if S[b] is not None:
                        assert S[b][1], f"QK({x}) overwrote S({S[b][0]}) before its group read it"
                        assert P[b] == ("used", x - 2), f"QK({x}) overwrote P: {P[b]}"
                    S[b] = [x, False]
                    P[b] = None
                    kread[s] = x
                elif op == "pv":
                    b, s = x & 1, x % NSTAGE
                    assert vslot[s] == x, f"PV({x}) read V slot {s} holding {vslot[s]}"
                    assert P[b] == x, f"PV({x}) read P {P[b]}"
                    P[b] = ("used", x)
                    vread[s] = x
                    pv_done.append(x)
                else:
                    bars[x].arrive()
            yield

    def softmax(g):
        seen = [0]  # this group's PV products known complete

        def upto(x):  # the x-th PV of group g (tile g + 2x) completes phase x of pvdone[g]
            while seen[0] <= x:
                yield from wait(f"pvdone{g}", seen[0])
                seen[0] += 1

        for i in range(g, NT, 2):
            x = i >> 1
            # the group's previous PV is consumed before the wait for S(i) (it completes first anyway:
            # PV(i - 2) was issued before QK(i)); rescaling O_g and releasing P(i) both follow it
            if x >= 1 and plant not in ("rescale_without_pv_wait", "release_without_pv_wait"):
                yield from upto(x - 1)
            yield from wait(f"sfull{g}", x)
            assert S[g] is not None and S[g][0] == i, f"group {g} read S buffer {g} = {S[g]} for tile {i}"
            S[g][1] = True
            yield
            P[g] = i  # over S(i), which this group has read
            yield
            if x >= 1:
                if rnd.random() < 0.3 or plant == "rescale_without_pv_wait":  # the group's max grew
                    mine = [j for j in pv_done if j % 2 == g]
                    assert mine == list(range(g, i, 2)), f"group {g} rescaled O at tile {i} with PVs done {pv_done}"
            bars[f"pfull{g}"].arrive()
            yield
        mine = len(range(g, NT, 2))
        if mine:
            yield from upto(mine - 1)
        assert [j for j in pv_done if j % 2 == g] == list(range(g, NT, 2)), f"group {g} read O with PVs done {pv_done}"

    actors = [producer(), mma(), softmax(0), softmax(1)]
    engines = [tma_engine(), tensor_pipe()]
    done = [False] * len(actors)
    steps = 0
    while not all(done):
        k = rnd.randrange(len(actors) + len(engines))
        if k >= len(actors):
            next(engines[k - len(actors)])
        elif not done[k]:
            try:
                next(actors[k])
            except StopIteration:
                done[k] = True
        steps += 1
        assert steps < 200000, "deadlock"
    assert pv_done == list(range(NT))


@pytest.mark.parametrize("NT", [1, 2, 3, 4, 5, 8, 17])
def test_protocol_random_interleavings(NT):
    for seed in range(300):
        run(NT, seed)


@pytest.mark.parametrize("plant", ["pv_skips_v_wait", "rescale_without_pv_wait", "release_without_pv_wait",
                                   "k_slot_not_released"])
def test_planted_protocol_mistakes_are_caught(plant):
    """Each planted mistake drops one wait of the protocol; some interleaving must trip a check."""
    caught = 0
    for seed in range(300):
        try:
            run(6, seed, plant=plant)
        except AssertionError:
            caught += 1
    assert caught > 0, plant


def test_model_matches_kernel_source():
    """The model's ring depth and barrier arrival counts are the kernel's: two K/V stages released
    through the S and PV barriers, one arrival (the TMA transaction) for the query tiles, the
    threads of one softmax group for P, one commit for each of the tensor-pipe barriers."""
    src = open(KERNEL).read()
    assert int(re.search(r"constexpr int NSTAGE = (\d+);", src).group(1)) == NSTAGE
    for init in ("mbar_init(&bars->q, 1)", "mbar_init(&bars->pfull[b], NSOFT / 2)", "mbar_init(&bars->pvdone[b], 1)",
                 "mbar_init(&bars->sfull[b], 1)", "mbar_init(&bars->kfull[s], 1)", "mbar_init(&bars->vfull[s], 1)",
                 "wait_bar(&bars->sfull[s], (use - 1) & 1", "wait_bar(&bars->pvdone[s], (use - 1) & 1"):
        assert init in src, init
    # no separate slot-release barriers, and the two groups never exchange inside the tile loop
    for gone in ("kempty", "vempty", "bars->mx"):
        assert gone not in src, gone
