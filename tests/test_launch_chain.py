"""Launch chaining (programmatic dependent launch) of the library's kernel sequences, on a model.

Within one C-ABI call, every launch after the first may start before its predecessor has
finished. Each kernel has one of three codes (the griddepcontrol instructions it executes):
- early: trigger at entry, and one thread waits at exit. Its body may run beside the kernels
  before it; it completes only after its predecessor has.
- late: wait at entry, then trigger. Past the wait, every earlier kernel is complete.
Plainly launched kernels (the first of each call, every launch with chaining off, and the
kernels launched without the attribute) start only once their predecessor is complete.

Completion is transitive along the chain, so kernel b's body can overlap kernel a (a < b) only
if b is an early kernel launched with the attribute, and no kernel between them triggers only
after its predecessor completed (a late or plain one).

This file transcribes the launch sequences of the C ABI (`api.cu`): per-chunk append / attend
calls, the whole-prompt prefill with its one-chunk lookahead, and decode steps. Each kernel
carries the buffers it reads and writes: store positions, query block sums, units'
representatives, query slots, selection and query-sum buffers, the scoring scratch, and the
decode partials. The check: no two kernels that may overlap touch the same buffer where one
of them writes it. Planted schedule mistakes must be caught by the same check.
"""
from __future__ import annotations

import math

import pytest

EARLY, LATE, NOPDL = "early", "late", "no_pdl"
PLAIN = "plain"


class Schedule:
    def __init__(self, S, U, W, topk, chaining=True, prefill_lookup=True, tc_decode=True, G=4, plant=None):
        self.S, self.U, self.W, self.topk = S, U, W, topk
        self.gblk = math.gcd(U, W)
        self.chaining, self.prefill_lookup, self.tc_decode, self.G = chaining, prefill_lookup, tc_decode, G
        self.plant = plant
        self.tokens = 0
        self.units_done = 0
        self.nlook = 0
        self.chain = False
        self.launches = []  # (name, mode, reads, writes)

    # ---- helpers -------------------------------------------------------------------------------
    def n_mem(self, c0):
        x = c0 - self.W - self.S
        return x // self.U if x > 0 else 0

    def keys(self, lo, hi):
        return {("K", t) for t in range(max(lo, 0), hi)}

    def yblocks(self, lo, hi):
        lo = max(lo, self.S)
        return {("Y", (t - self.S) // self.gblk) for t in range(lo, hi)}

    def launch(self, name, code, reads, writes, attr=True):
        mode = code if (attr and code != NOPDL and self.chaining and self.chain) else PLAIN
        self.launches.append((name, mode, frozenset(reads), frozenset(writes)))

    def qslot(self, L):
        return ("Q", L % (2 if self.plant == "two_query_slots" else 3))

    def selbuf(self, L):
        return ("sel", 0 if self.plant == "one_selection_buffer" else L % 2)

    def qbar(self, L):
        return ("qbar", L % 2)

    # ---- stages (api.cu) ------------------------------------------------------------------------
    def reps_to(self, target):
        if target <= self.units_done:
            return False
        reads, writes = set(), set()
        for j in range(self.units_done, target):
            e = self.S + (j + 1) * self.U
            reads |= self.keys(e - self.U, e) | self.yblocks(e, e + self.W)
            writes.add(("rep", j))
        self.launch("reps", EARLY, reads, writes)
        self.chain = True
        self.units_done = target
        return True

    def stage_store(self, n, tag):
        c0 = self.tokens
        self.reps_to(self.n_mem(c0))
        self.launch("append", EARLY, {("in", tag)}, self.keys(c0, c0 + n) | {("cs_chunk",)})
        self.chain = True
        if c0 + n > self.S:
            yb = self.yblocks(c0, c0 + n)
            self.launch("ysum", EARLY, {("in", tag)} | yb, yb)
        self.tokens = c0 + n

    def stage_prep(self, L, tag):
        self.launch("prep", EARLY, {("in", tag)}, {self.qslot(L), self.qbar(L)})
        self.chain = True

    def stage_select(self, L, nm, qraw_tag, wait_first):
        if nm <= 0 or self.topk <= 0:
            return
        fast = self.topk <= 32
        reads = {("rep", j) for j in range(nm)} | ({("in", qraw_tag)} if qraw_tag is not None else {self.qbar(L)})
        writes = {("uscore",), ("cand",), ("counters",)} | ({self.selbuf(L)} if fast else set())
        self.launch("score", LATE if wait_first else EARLY, reads, writes)
        self.chain = True
        if not fast:  # launched without the attribute
            self.launch("topk_sort", NOPDL, {("uscore",)}, {self.selbuf(L)}, attr=False)

    def stage_attend(self, L, c0, n, lookup, tag):
        nm = self.n_mem(c0)
        kk = min(self.topk, nm) if lookup else 0
        B = self.S + self.U * nm
        reads = {self.qslot(L)} | self.keys(0, min(self.S, c0 + n)) | self.keys(B, c0 + n)
        if kk > 0:
            reads |= {self.selbuf(L)} | self.keys(self.S, self.S + nm * self.U)
        code = EARLY if self.plant == "attention_early" else LATE
        self.launch("attend", code, reads, {("out", tag)})
        self.chain = True

    # ---- entry points ---------------------------------------------------------------------------
    def append_chunk(self, n, tag):
        self.chain = False
        self.pending_c0 = self.tokens
        self.stage_store(n, tag)

    def attend_chunk(self, n, tag, decoding=False):
        if not decoding:
            self.chain = False
        c0 = self.pending_c0
        L = self.nlook
        self.nlook += 1
        nm = self.n_mem(c0)
        lookup = decoding or self.prefill_lookup
        self.stage_prep(L, tag)
        if lookup and min(self.topk, nm) > 0:
            self.stage_select(L, nm, None, True)
        self.stage_attend(L, c0, n, lookup, tag)

    def prefill(self, n, chunk, tag):
        self.chain = False
        N = (n + chunk - 1) // chunk
        L0, t0 = self.nlook, self.tokens
        ln = [min(chunk, n - i * chunk) for i in range(N)]

        def store_pack(i):
            self.stage_store(ln[i], (tag, i))
            self.stage_prep(L0 + i, (tag, i))

        def lookup(i, wait_first):
            nm = self.n_mem(t0 + i * chunk)
            if self.prefill_lookup and min(self.topk, nm) > 0:
                self.stage_select(L0 + i, nm, None, wait_first)

        store_pack(0)
        before = len(self.launches)
        lookup(0, True)
        if len(self.launches) == before and self.plant != "chunk1_chained_without_lookup":
            self.chain = False
        for i in range(N):
            if i + 1 < N:
                store_pack(i + 1)
            if i > 0:
                lookup(i, False)
            self.stage_attend(L0 + i, t0 + i * chunk, ln[i], self.prefill_lookup, (tag, i))
        self.nlook = L0 + N

    def decode_step(self, tag):
        self.chain = False
        t = self.tokens
        if self.tc_decode and self.G <= 8:
            # representatives of a newly evicted unit; part 0: the token's store, the sink and window
            # tiles and their merge (early); the lookup alongside it (late after new representatives);
            # part 1: the selected units' tiles and the final merge (late)
            new_reps = self.reps_to(self.n_mem(t))
            L = self.nlook
            self.nlook += 1
            nm = self.n_mem(t)
            kk = min(self.topk, nm)
            B = self.S + self.U * nm
            w0 = self.keys(t, t + 1) | self.yblocks(t, t + 1) | {("dpart", 0)} | ({("out", tag)} if kk == 0 else set())
            self.launch("decode_part0", EARLY, {("in", tag)} | self.keys(0, min(self.S, t + 1)) | self.keys(B, t + 1), w0)
            self.chain = True
            self.tokens = t + 1
            if kk > 0:
                wait_first = new_reps and self.plant != "decode_score_never_waits"
                self.stage_select(L, nm, tag, wait_first)
                self.launch("decode_part1", LATE, {("in", tag), self.selbuf(L), ("dpart", 0)} |
                            self.keys(self.S, self.S + nm * self.U), {("dpart", 1), ("out", tag)})
            return
        self.pending_c0 = t
        self.stage_store(1, tag)
        if self.G > 8:
            self.attend_chunk(1, tag, decoding=True)
            return
        L = self.nlook
        self.nlook += 1
        nm = self.n_mem(t)
        kk = min(self.topk, nm)
        if kk > 0:
            self.stage_select(L, nm, tag, True)
        self.launch("decode", NOPDL, {("in", tag), ("cs_chunk",), self.selbuf(L)} | self.keys(0, t + 1),
                    {("out", tag)}, attr=False)


def overlapping_conflicts(launches):
    """Pairs (a, b), a < b, that launch chaining may run at the same time and that touch one
    buffer with at least one write."""
    body_waits = {PLAIN, LATE}           # the body starts only after the predecessor completed
    trigger_waits = {PLAIN, LATE}        # the trigger comes only after the predecessor completed
    found = []
    for b, (nb, mb, rb, wb) in enumerate(launches):
        if mb in body_waits:
            continue
        for a in range(b - 1, -1, -1):
            na, ma, ra, wa = launches[a]
            clash = (wa & (rb | wb)) | (ra & wb)
            if clash:
                found.append((a, na, b, nb, sorted(clash)[:3]))
            if ma in trigger_waits:
                break  # a kernel that triggers only after its predecessor completed separates the rest
    return found


# ---- scenarios -----------------------------------------------------------------------------------
SHAPES = [
    dict(S=4, U=8, W=16, topk=2),     # fused top-k in the scoring kernel
    dict(S=0, U=8, W=24, topk=40),    # k > 32: separate sort kernel
    dict(S=6, U=12, W=8, topk=3),     # gcd(U, W) = 4: windows in several query-sum blocks
    dict(S=4, U=8, W=16, topk=0),     # no lookup at all
]


def scenarios(sched_kwargs):
    """(label, callable building a schedule)"""
    out = []

    def prefill_whole(chunk):
        def f():
            s = Schedule(**sched_kwargs)
            s.prefill(230, chunk, "p")
            for i in range(12):
                s.decode_step(("d", i))
            return s
        return f

    def prefill_pieces(cut, chunk):
        def f():
            s = Schedule(**sched_kwargs)
            s.prefill(cut, chunk, "p1")
            s.prefill(200 - cut, chunk, "p2")
            s.prefill(7, chunk, "p3")
            for i in range(6):
                s.decode_step(("d", i))
            s.prefill(40, chunk, "p4")  # prompt continued after decoding
            return s
        return f

    def per_chunk(chunk):
        def f():
            s = Schedule(**sched_kwargs)
            t = 0
            while t < 170:
                n = min(chunk, 170 - t)
                s.append_chunk(n, ("c", t))
                s.attend_chunk(n, ("c", t))
                t += n
            for i in range(5):
                s.decode_step(("d", i))
            return s
        return f

    for chunk in (5, 8, 13, 32):
        out.append((f"prefill chunk {chunk}", prefill_whole(chunk)))
        out.append((f"per-chunk calls {chunk}", per_chunk(chunk)))
    for cut, chunk in ((40, 8), (64, 16), (33, 11), (96, 32)):
        out.append((f"prefill in pieces {cut}/{chunk}", prefill_pieces(cut, chunk)))
    return out


VARIANTS = [
    dict(),
    dict(prefill_lookup=False),
    dict(tc_decode=False),
    dict(G=16),
    dict(chaining=False),
]


@pytest.mark.parametrize("shape", range(len(SHAPES)))
@pytest.mark.parametrize("variant", range(len(VARIANTS)))
def test_no_overlapping_kernels_share_a_written_buffer(shape, variant):
    kw = {**SHAPES[shape], **VARIANTS[variant]}
    for label, build in scenarios(kw):
        s = build()
        assert s.launches, label
        bad = overlapping_conflicts(s.launches)
        assert not bad, (label, bad[:3])


def test_chaining_actually_overlaps_kernels():
    """The model is not vacuous: with chaining on, attention runs beside the next chunk's store
    side and lookup; with chaining off, nothing overlaps."""
    s = Schedule(**SHAPES[0])
    s.prefill(230, 8, "p")
    names = [n for n, *_ in s.launches]
    modes = [m for _, m, *_ in s.launches]
    i = names.index("attend")
    assert modes[i + 1] == EARLY  # the next chunk's store side starts beside the attention
    assert EARLY in modes and LATE in modes
    off = Schedule(**SHAPES[0], chaining=False)
    off.prefill(230, 8, "p")
    assert {m for _, m, *_ in off.launches} == {PLAIN}


# planted mistake -> the clash it must produce: (earlier kernel, later kernel, buffer kind)
PLANTS = {
    "two_query_slots": ("attend", "prep", "Q"),                  # chunk c+1 packed over chunk c-1's queries
    "one_selection_buffer": ("attend", "score", "sel"),          # lookup c over the selection attend c-1 reads
    "attention_early": ("score", "attend", "sel"),               # attention before its selection is final
    "chunk1_chained_without_lookup": ("ysum", "reps", "Y"),      # chunk 1's representatives beside chunk 0's sums
    "decode_score_never_waits": ("reps", "score", "rep"),        # a decode lookup beside its new representatives
}


@pytest.mark.parametrize("plant", list(PLANTS))
def test_planted_schedule_mistakes_are_caught(plant):
    want = PLANTS[plant]
    seen = set()
    for shape in SHAPES:
        for label, build in scenarios({**shape, "plant": plant}):
            for a, na, b, nb, clash in overlapping_conflicts(build().launches):
                seen |= {(na, nb, c[0]) for c in clash}
    assert want in seen, (plant, sorted(seen))
