"""The tcgen05 prefill attention kernel's barrier protocol, modelled and explored on the CPU.

No compute-sanitizer run of this kernel exists, so its synchronisation is checked on a model
instead: the roles of `k_attn_tc` (attend_tc.cu) as coroutines that a seeded scheduler
interleaves at random, with exact mbarrier parity semantics.
- TMA producer: two query tiles, then K and V tiles through 2-stage rings.
- MMA issuer: QK(i) into S buffer i & 1, then PV(i - 1) after P(i - 1) is released.
- Tensor pipe: executes one thread's MMAs in issue order; each commit arrives when every
  earlier MMA is done.
- TMA engine: lands copies in any order.
- Two softmax threads: the two column halves of a row, each with its own online softmax. A
  half may rescale its accumulator O_h (only after PV(i - 1) is complete) and writes its half
  of P(i) over its half of S(i); it releases P(i) once PV(i - 2) is complete, so PV(i - 1) can
  run while it works on the next tile.  P releases and PV completions alternate between two
  barriers each (by tile parity), which keeps every consumer within one phase of its barrier.

Every data hand-off is asserted where it happens:
- a ring slot is refilled only after the MMA that read it has executed;
- S(i) is read only once QK(i) has written it, and is not overwritten before both halves are
  done;
- PV(j) reads both halves of P(j), and never a stale one;
- O_h is read or rescaled only when no PV that writes it is pending;
- a parity wait never runs two or more phases behind its barrier, where parity aliases;
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
    has completed, and is ambiguous (aliases) if two or more phases completed past it."""

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
        return self.phase > j


def run(NT, seed, plant=None):
    rnd = random.Random(seed)
    bars = {"q": Bar("q", 1), "pfull0": Bar("pfull0", 2), "pfull1": Bar("pfull1", 2), "pvdone0": Bar("pvdone0", 1), "pvdone1": Bar("pvdone1", 1),
            "sfull0": Bar("sfull0", 1), "sfull1": Bar("sfull1", 1)}
    for s in range(NSTAGE):
        for x in ("kfull", "kempty", "vfull", "vempty"):
            bars[f"{x}{s}"] = Bar(f"{x}{s}", 1)
    kslot = [None] * NSTAGE   # tile whose K occupies the slot (None: empty)
    vslot = [None] * NSTAGE
    kread = [-1] * NSTAGE     # last tile whose QK has executed on that slot
    vread = [-1] * NSTAGE
    S = [None, None]          # per buffer: (tile, set of halves that have read it)
    P = [dict(), dict()]      # per buffer: half -> tile of the P half stored there
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
            if i >= NSTAGE:
                yield from wait(f"kempty{s}", use - 1)
            tma.append(("k", s, i))
            yield
            if i >= NSTAGE:
                yield from wait(f"vempty{s}", use - 1)
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
                pipe.extend([("qk", i), ("commit", f"sfull{i & 1}"), ("commit", f"kempty{s}")])
                yield
            if i >= 1:
                j = i - 1
                yield from wait(f"pfull{j & 1}", j >> 1)
                if plant != "pv_skips_v_wait":
                    yield from wait(f"vfull{j % NSTAGE}", j // NSTAGE)
                pipe.extend([("pv", j), ("commit", f"pvdone{j & 1}"), ("commit", f"vempty{j % NSTAGE}")])
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
                        assert S[b][1] == {0, 1}, f"QK({x}) overwrote S({S[b][0]}) before both halves read it"
                        assert all(v == ("used", x - 2) for v in P[b].values()), f"QK({x}) overwrote P: {P[b]}"
                    S[b] = (x, set())
                    P[b] = {}
                    kread[s] = x
                elif op == "pv":
                    b, s = x & 1, x % NSTAGE
                    assert vslot[s] == x, f"PV({x}) read V slot {s} holding {vslot[s]}"
                    assert P[b] == {0: x, 1: x}, f"PV({x}) read P {P[b]}"
                    P[b] = {h: ("used", x) for h in (0, 1)}
                    vread[s] = x
                    pv_done.append(x)
                else:
                    bars[x].arrive()
            yield

    def softmax(h):
        seen = [0]  # PV completions consumed: tiles [0, seen)

        def upto(j):  # PV(x) completes phase x >> 1 of pvdone[x & 1]
            while seen[0] <= j:
                yield from wait(f"pvdone{seen[0] & 1}", seen[0] >> 1)
                seen[0] += 1

        for i in range(NT):
            b = i & 1
            yield from wait(f"sfull{b}", i >> 1)
            assert S[b] is not None and S[b][0] == i, f"half {h} read S buffer {b} = {S[b]} for tile {i}"
            yield
            if i >= 1 and rnd.random() < 0.3:  # the half's running max grew: rescale O_h
                if plant != "rescale_without_pv_wait":
                    yield from upto(i - 1)
                assert pv_done == list(range(i)), f"half {h} rescaled O at tile {i} with PVs done {pv_done}"
            S[b][1].add(h)
            P[b][h] = i  # over this half's own S columns (it has read them; the partner never does)
            yield
            # PV(i - 2) is consumed before P(i) is released: PV(i) is issued only after the release, so
            # the barrier is then at most one phase ahead of this consumer (no parity aliasing), and
            # PV(i - 1) may still run while this half works on tile i + 1
            if i >= 2 and plant != "release_without_pv_wait":
                yield from upto(i - 2)
            bars[f"pfull{i & 1}"].arrive()
            yield
        yield from upto(NT - 1)
        assert pv_done == list(range(NT)), f"half {h} read O with PVs done {pv_done}"

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


@pytest.mark.parametrize("plant", ["pv_skips_v_wait", "rescale_without_pv_wait", "release_without_pv_wait"])
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
    """The model's ring depth and barrier arrival counts are the kernel's: two K/V stages, one
    arrival (the TMA transaction) for the query tiles, every softmax thread for P, one commit
    for each of the tensor-pipe barriers."""
    src = open(KERNEL).read()
    assert int(re.search(r"constexpr int NSTAGE = (\d+);", src).group(1)) == NSTAGE
    for init in ("mbar_init(&bars->q, 1)", "mbar_init(&bars->pfull[b], NSOFT)", "mbar_init(&bars->pvdone[b], 1)",
                 "mbar_init(&bars->sfull[b], 1)", "mbar_init(&bars->kfull[s], 1)", "mbar_init(&bars->vempty[s], 1)"):
        assert init in src, init
    # the two halves of a row never wait for each other inside the tile loop (no exchange barrier)
    assert "bars->mx" not in src
