"""A CPU model of the decode attention kernel's synchronisation.

decode_attn_kernel (csrc/decode.cu) has one producer warp (attn_producer)
streaming K and V of each span into a three-stage ring, and four consumer
warps (attn_consumer) that each take their share of every span on their
own and merge at the end of every run of spans through shared memory and a
named barrier over the 128 consumer threads.  Every mbarrier wait is bounded
and, when it gives up, raises the CTA's abort flag, after which every other
bounded wait returns at once; a consumer warp whose wait gave up turns
"dead": it walks the rest of the schedule without waiting or computing, but
still reaches every named barrier, because a named barrier has no time
limit.  List-1 spans (the selected blocks) are read only after the
selection grid has finished (griddepcontrol.wait in both roles).

This file restates both roles as Python generators and runs them under
random interleavings, on CTA schedules of runs drawn at random (runs
without spans included), and checks:
  * without faults: no wait ever gives up, every consumer warp reads K, V
    and the key count of exactly the span it expects, no stage is reloaded
    while a warp still has to read it, and each merge reads every warp's
    values of this run and head tile, none overwritten early;
  * with random give-ups (any bounded wait may run out): every role still
    ends (no warp is left at a named barrier) and the producer leaves no
    copy in flight.
Planted mistakes must each be caught.
"""

from __future__ import annotations

import random
from dataclasses import dataclass, field

import pytest

RING = 3  # kRingStages
WARPS = 4  # kConsumerWarps


class ProtocolError(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise ProtocolError(msg)


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.done = name, count, count, 0, 0

    def arrive(self):
        check(self.pending >= 1, f"{self.name}: more arrivals than its phase expects")
        self.pending -= 1
        self._complete()

    def expect_tx(self, units):
        self.tx += units

    def complete_tx(self, units):
        self.tx -= units
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.done & 1) != parity


@dataclass
class Stage:
    span: object = None
    owed: set = field(default_factory=set)  # consumer warps that still read this content


class Model:
    def __init__(self, runs, nt, faults, rng, mistake=None):
        self.runs, self.nt, self.faults, self.rng, self.mistake = runs, nt, faults, rng, mistake
        empty_count = WARPS - 1 if mistake == "empty_count_short" else WARPS
        self.k_full = [Bar(f"k_full[{i}]", 1) for i in range(RING)]
        self.v_full = [Bar(f"v_full[{i}]", 1) for i in range(RING)]
        self.empty = [Bar(f"empty[{i}]", empty_count) for i in range(RING)]
        self.k = [Stage() for _ in range(RING)]
        self.v = [Stage() for _ in range(RING)]
        self.nk = [None] * RING
        self.named_arrived, self.named_generation = 0, 0
        self.merge = [None] * WARPS  # each warp's wm / wl / wo slot
        self.merge_owed = [set() for _ in range(WARPS)]  # warps still to read a slot
        self.abort = False
        self.gave_up = 0
        self.selection_done = False
        self.tma = []

    def schedule(self, li):
        return [(run_id, n) for run_id, (l, n) in enumerate(self.runs) if l == li]

    def bounded_wait(self, bar, parity, phase, abort_aware=True):
        """Generator returning True when the phase completes, False when the
        wait gives up (its time limit, or the abort flag of another wait)."""
        check(parity == (phase & 1), f"{bar.name}: parity {parity} does not name phase {phase}")
        while True:
            if abort_aware and self.abort:
                return False
            if bar.passes(parity):
                check(bar.done == phase + 1, f"{bar.name}: wait for phase {phase} passed at {bar.done}")
                return True
            if self.faults and abort_aware and self.rng.random() < 0.03:
                timed_out = True
            else:
                timed_out = yield ("wait", bar, parity, abort_aware)
            if timed_out:
                self.abort = self.abort or abort_aware
                self.gave_up += 1
                return False

    def griddep_wait(self):
        while not self.selection_done:
            yield ("griddep",)

    def named_sync(self):
        gen = self.named_generation
        self.named_arrived += 1
        if self.named_arrived == WARPS:
            self.named_arrived = 0
            self.named_generation += 1
            return
        while self.named_generation == gen:
            yield ("named", gen)

    # ------------------------------------------------------------ roles
    def producer(self):
        issued = 0
        ok = True
        for li in (0, 1):
            runs = self.schedule(li)
            if not ok or not runs:
                continue
            if li == 1:
                yield from self.griddep_wait()
            for run_id, n_spans in runs:
                for s in range(n_spans):
                    if not ok:
                        break
                    st, u = issued % RING, issued // RING
                    if self.mistake == "producer_parity":
                        got = yield from self.bounded_wait(self.empty[st], u & 1, u)
                    else:
                        got = yield from self.bounded_wait(self.empty[st], (u & 1) ^ 1, u - 1)
                    if not got:
                        ok = False
                        break
                    for stage in (self.k[st], self.v[st]):
                        check(not stage.owed, f"stage {st} reloaded while warps {sorted(stage.owed)} still read it")
                    self.nk[st] = (run_id, s)
                    for bar, stage in ((self.k_full[st], self.k[st]), (self.v_full[st], self.v[st])):
                        bar.expect_tx(1)
                        bar.arrive()
                        self.tma.append((bar, stage, (run_id, s)))
                    issued += 1
                    yield
        # wait for the copies that may still be in flight before the CTA exits
        for d in range(min(RING, issued)):
            e = issued - 1 - d
            yield from self.bounded_wait(self.k_full[e % RING], (e // RING) & 1, e // RING, abort_aware=False)
            yield from self.bounded_wait(self.v_full[e % RING], (e // RING) & 1, e // RING, abort_aware=False)
        check(not self.tma, "the producer ended with copies in flight")

    def consumer(self, w):
        used = 0
        dead = False
        for li in (0, 1):
            runs = self.schedule(li)
            if not runs:
                continue
            if li == 1:
                yield from self.griddep_wait()
            for run_id, n_spans in runs:
                for s in range(n_spans):
                    u = used
                    used += 1
                    if dead:
                        continue
                    st, ph = u % RING, (u // RING) & 1
                    if not (yield from self.bounded_wait(self.k_full[st], ph, u // RING)):
                        dead = True
                        if self.mistake == "dead_warp_leaves":
                            return
                        continue
                    check(self.nk[st] == (run_id, s), f"warp {w}: key count of {self.nk[st]}, wants {(run_id, s)}")
                    check(self.k[st].span == (run_id, s), f"warp {w}: K holds {self.k[st].span}, wants {(run_id, s)}")
                    yield
                    if not (yield from self.bounded_wait(self.v_full[st], ph, u // RING)):
                        dead = True
                        if self.mistake == "dead_warp_leaves":
                            return
                        continue
                    check(self.v[st].span == (run_id, s), f"warp {w}: V holds {self.v[st].span}, wants {(run_id, s)}")
                    self.k[st].owed.discard(w)
                    self.v[st].owed.discard(w)
                    yield
                    self.empty[st].arrive()
                    yield
                # end of the run: merge the four warps, one tile of 8 heads at a time
                for t in range(self.nt):
                    check(not self.merge_owed[w],
                          f"warp {w}: merge slot rewritten before warps {sorted(self.merge_owed[w])} read it")
                    self.merge[w] = (run_id, t)
                    self.merge_owed[w] = set(range(WARPS))
                    yield
                    yield from self.named_sync()  # every warp's m, l and O^T are posted
                    for v in range(WARPS):
                        check(self.merge[v] == (run_id, t),
                              f"warp {w}: merge slot {v} holds {self.merge[v]}, wants {(run_id, t)}")
                        self.merge_owed[v].discard(w)
                        yield
                    if self.mistake != "single_merge_sync":
                        yield from self.named_sync()  # the slots are free again


def run(runs, nt, seed, faults=False, mistake=None, max_steps=500_000):
    rng = random.Random(seed)
    m = Model(runs, nt, faults, rng, mistake)
    roles = [m.producer()] + [m.consumer(w) for w in range(WARPS)]
    state = [None] * len(roles)
    live = set(range(len(roles)))

    def enabled(i):
        s = state[i]
        if s is None:
            return True
        if s[0] == "wait":
            return s[1].passes(s[2]) or (s[3] and m.abort)
        if s[0] == "griddep":
            return m.selection_done
        return m.named_generation != s[1]  # named barrier released

    def resume(i, value=None):
        try:
            state[i] = roles[i].send(value) if value is not None else next(roles[i])
        except StopIteration:
            live.discard(i)
            state[i] = None

    for _ in range(max_steps):
        choices = [i for i in live if enabled(i)]
        if m.tma:
            choices.append("tma")
        if not m.selection_done:
            choices.append("selection")
        if not choices:
            if not live:
                check(faults or m.gave_up == 0, "a wait gave up in a run without faults")
                return m
            waiting = [i for i in live if state[i][0] == "wait"]
            check(waiting, "hang: " + ", ".join(state[i][0] for i in live))
            # nothing else can move: a bounded wait reaches its time limit
            check(faults, "a bounded wait had to time out in a run without faults: "
                  + ", ".join(state[i][1].name for i in waiting))
            resume(rng.choice(waiting), True)
            continue
        c = rng.choice(choices)
        if c == "tma":
            bar, stage, span = m.tma.pop(rng.randrange(len(m.tma)))
            stage.span, stage.owed = span, set(range(WARPS))
            bar.complete_tx(1)
        elif c == "selection":
            m.selection_done = True
        else:
            resume(c)
    raise ProtocolError("step limit")


def random_runs(rng, max_runs=4, max_spans=6):
    runs = [(li, rng.randint(0, max_spans)) for li in (0, 1) for _ in range(rng.randint(0, max_runs))]
    return runs or [(0, 1)]


@pytest.mark.parametrize("nt", [1, 2])
def test_protocol_holds_under_random_interleavings(nt):
    for seed in range(200):
        rng = random.Random(700 + seed)
        run(random_runs(rng), nt, seed)


def test_every_role_ends_when_waits_give_up():
    gave_up = 0
    for seed in range(300):
        rng = random.Random(900 + seed)
        m = run(random_runs(rng), rng.choice((1, 2)), seed, faults=True)
        gave_up += m.gave_up > 0
    assert gave_up > 50  # the fault path really ran


MISTAKES = [
    ("empty_count_short", False),   # a stage released after three of the four warps
    ("producer_parity", False),     # the producer waits for the wrong phase of a free stage
    ("single_merge_sync", False),   # merge slots reused without the second named barrier
    ("dead_warp_leaves", True),     # a warp whose wait gave up skips the remaining merges
]


@pytest.mark.parametrize("mistake,faults", MISTAKES, ids=[m[0] for m in MISTAKES])
def test_planted_mistakes_are_caught(mistake, faults):
    for seed in range(300):
        rng = random.Random(3000 + seed)
        try:
            run(random_runs(rng), rng.choice((1, 2)), seed, faults=faults, mistake=mistake)
        except ProtocolError:
            return
    pytest.fail(f"planted mistake {mistake} was not caught in 300 interleavings")
