"""A CPU model of the prefill kernel's barrier protocol.

hybrid_prefill_kernel (csrc/prefill.cu) runs its roles in one CTA and hands
data between them only through mbarriers: the producer warp loads Q, K and
V by TMA (run_producer), one thread issues the tensor-core MMAs
(run_mma), and four softmax warps per query head turn S into P and write
the output (run_softmax).  S and P share tensor-memory columns, O lives in
tensor memory, and the K/V tiles sit in two-stage rings.

This file restates each role's sequence of waits, arrivals, copies and MMA
issues as a Python generator, mirroring the kernel line for line, and runs
the roles under many random interleavings.  The tensor pipe executes the
MMAs one at a time in issue order, a commit arrives on its barrier only
once every MMA issued before it has executed, and TMA copies complete in
any order.  It checks that:
  * no interleaving deadlocks;
  * every parity wait sees the phase it means: when it passes, the barrier
    has completed exactly that phase (a parity test cannot tell phase k
    from k + 2, so a signaller two phases ahead is an error);
  * every read sees the data its role expects: Q of this item, K/V of this
    tile, S of this tile, every warp's P of this tile, and O accumulated
    over exactly this item's tiles so far (at the lazy rescale and at the
    epilogue);
  * no buffer is overwritten while a reader of its previous content is
    still to come.
Both instantiations are modelled: shared selections (every tile belongs to
both heads of the pair) and per-head selections (a tile may belong to one
head only; the other head's S, P V and P handshake are skipped as the
kernel skips them).  Planted protocol mistakes must each be caught.
The bounded-wait give-up paths are not modelled; they only run after a
time-out.
"""

from __future__ import annotations

import random
from dataclasses import dataclass, field

import pytest

K_STAGES = 2  # kKStages
V_STAGES = 2  # kVStages
P_CHUNKS = 2  # kPChunks (RTP_P_CHUNKS)
WARPS = 4  # softmax warps per head (32 rows each)
TILE = 1  # tx units of one TMA tile


class ProtocolError(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise ProtocolError(msg)


class Bar:
    """An mbarrier: `count` arrivals plus all expected tx complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.done = name, count, count, 0, 0

    def arrive(self, n=1):
        check(self.pending >= n, f"{self.name}: more arrivals than its phase expects")
        self.pending -= n
        self._complete()

    def expect_tx(self, units):
        self.tx += units

    def complete_tx(self, units):
        self.tx -= units
        check(self.tx >= 0, f"{self.name}: tx underflow")
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity):
        # try_wait.parity: true once the phase of that parity has completed,
        # i.e. when the phase in progress has the other parity
        return (self.done & 1) != parity


@dataclass
class Item:
    mem: list  # per tile: bit 0 = head 0 attends to it, bit 1 = head 1

    @property
    def n(self):
        return len(self.mem)


@dataclass
class Buf:
    content: object = None
    readers: set = field(default_factory=set)  # reads still owed to the current content


class Model:
    def __init__(self, items, per_head, mistake=None):
        self.items, self.per_head, self.mistake = items, per_head, mistake
        B = Bar
        self.q_full = [B(f"q_full[{h}]", 1) for h in range(2)]
        self.q_empty = [B(f"q_empty[{h}]", 1) for h in range(2)]
        self.k_full = [B(f"k_full[{s}]", 1) for s in range(K_STAGES)]
        self.k_empty = [B(f"k_empty[{s}]", 1) for s in range(K_STAGES)]
        self.v_full = [B(f"v_full[{s}]", 1) for s in range(V_STAGES)]
        self.v_empty = [B(f"v_empty[{s}]", 1) for s in range(V_STAGES)]
        self.s_full = [B(f"s_full[{h}]", 1) for h in range(2)]
        self.o_full = [B(f"o_full[{h}]", 1) for h in range(2)]
        self.p_full = [[B(f"p_full[{h}][{q}]", 32 * WARPS) for q in range(P_CHUNKS)] for h in range(2)]
        self.q = [Buf() for _ in range(2)]
        self.k = [Buf() for _ in range(K_STAGES)]
        self.v = [Buf() for _ in range(V_STAGES)]
        self.tile_mem = [None] * K_STAGES
        # tensor memory, per head and softmax warp (32 rows each)
        self.s = [[Buf() for _ in range(WARPS)] for _ in range(2)]  # S columns (holds S, then P over it)
        self.p = [[[Buf() for _ in range(P_CHUNKS)] for _ in range(WARPS)] for _ in range(2)]
        self.o = [[{"item": None, "parts": set(), "read": True} for _ in range(WARPS)] for _ in range(2)]
        self.pipe = []  # tensor-core operations in issue order
        self.tma = []  # copies in flight

    # ------------------------------------------------------------ helpers
    def wait(self, bar, parity, phase):
        """Generator: a parity wait meant for `phase` (-1: the phase before the first)."""
        check(parity == (phase & 1), f"{bar.name}: parity {parity} does not name phase {phase}")
        while not bar.passes(parity):
            check(bar.done <= phase + 1, f"{bar.name}: signaller ran two phases past a waiter (phase {phase})")
            yield ("blocked", bar, parity, phase)
        check(bar.done == phase + 1, f"{bar.name}: wait for phase {phase} passed at {bar.done} completed phases")

    def read_tile_mem(self, st, it, j):
        tm = self.tile_mem[st]
        check(tm is not None and tm[:2] == (it, j), f"tile_mem[{st}] holds {tm}, wants tile {(it, j)}")
        return tm[2]

    def member(self, it, j, h):
        return bool((self.items[it].mem[j] >> h) & 1)

    # ------------------------------------------------------------ tensor pipe
    def run_op(self, op):
        kind = op[0]
        if kind == "commit":
            op[1].arrive()
        elif kind == "qk":
            _, h, st, it, j = op
            check(self.q[h].content == it, f"QK{h}: Q holds {self.q[h].content}, wants item {it}")
            check(self.k[st].content == (it, j), f"QK{h}: K[{st}] holds {self.k[st].content}, wants {(it, j)}")
            self.q[h].readers.discard(("qk", it, j))
            self.k[st].readers.discard(h)
            for w in range(WARPS):
                check(not self.s[h][w].readers, f"QK{h} overwrites S[{h}] before the softmax read it")
                for q in range(P_CHUNKS):
                    check(not self.p[h][w][q].readers, f"QK{h} overwrites P[{h}] before P V read it")
                self.s[h][w] = Buf((it, j), {"softmax"})
                for q in range(P_CHUNKS):
                    self.p[h][w][q] = Buf()
        elif kind == "pv":
            _, h, q, st, it, j, accumulate = op
            check(self.v[st].content == (it, j), f"PV{h}: V[{st}] holds {self.v[st].content}, wants {(it, j)}")
            self.v[st].readers.discard((h, q))
            for w in range(WARPS):
                pb = self.p[h][w][q]
                check(pb.content == (it, j), f"PV{h}: P chunk {q} of warp {w} holds {pb.content}, wants {(it, j)}")
                pb.readers.clear()
                o = self.o[h][w]
                if not accumulate and q == 0:
                    check(o["read"], f"PV{h} overwrites O[{h}] before the epilogue read it")
                    o.update(item=it, parts=set(), read=False)
                check(o["item"] == it, f"PV{h}: O holds item {o['item']}, accumulating item {it}")
                o["parts"].add((j, q))

    # ------------------------------------------------------------ roles
    def producer(self):
        gt = 0
        for it, item in enumerate(self.items):
            for h in range(2):
                yield from self.wait(self.q_empty[h], (it & 1) ^ 1, it - 1)
                check(not self.q[h].readers, f"Q[{h}] reloaded while S MMAs still need it")
                self.q_full[h].expect_tx(TILE)
                self.q_full[h].arrive()
                reads = {("qk", it, j) for j in range(item.n) if self.member(it, j, h)}
                self.tma.append((self.q_full[h], self.q[h], it, reads))
                yield
            for j in range(item.n):
                sk, sv = gt % K_STAGES, gt % V_STAGES
                uk, uv = gt // K_STAGES, gt // V_STAGES
                par = (uk & 1) if self.mistake == "producer_empty_parity" else (uk & 1) ^ 1
                if self.mistake == "producer_empty_parity":
                    yield from self.wait(self.k_empty[sk], par, uk)
                else:
                    yield from self.wait(self.k_empty[sk], par, uk - 1)
                self.tile_mem[sk] = (it, j, item.mem[j])  # published by the arrive below
                self.k_full[sk].expect_tx(TILE)
                self.k_full[sk].arrive()
                self.tma.append((self.k_full[sk], self.k[sk], (it, j),
                                 {h for h in range(2) if self.member(it, j, h)}))
                yield
                yield from self.wait(self.v_empty[sv], (uv & 1) ^ 1, uv - 1)
                self.v_full[sv].expect_tx(TILE)
                self.v_full[sv].arrive()
                self.tma.append((self.v_full[sv], self.v[sv], (it, j),
                                 {(h, q) for h in range(2) if self.member(it, j, h) for q in range(P_CHUNKS)}))
                yield
                gt += 1

    def mma(self):
        gt = pc = 0
        M = self.mistake
        for it, item in enumerate(self.items):
            n = item.n
            yield from self.wait(self.q_full[0], it & 1, it)
            yield from self.wait(self.q_full[1], it & 1, it)
            started = [False, False]
            st0 = gt % K_STAGES
            yield from self.wait(self.k_full[st0], (gt // K_STAGES) & 1, gt // K_STAGES)
            mem_cur = self.read_tile_mem(st0, it, 0) if self.per_head else 3
            if mem_cur & 1:
                self.pipe.append(("qk", 0, st0, it, 0))
            self.pipe.append(("commit", self.s_full[0]))
            if M == "s_full_twice":
                self.pipe.append(("commit", self.s_full[0]))
            if M == "k_empty_early":
                self.pipe.append(("commit", self.k_empty[st0]))
            if mem_cur & 2:
                self.pipe.append(("qk", 1, st0, it, 0))
            self.pipe.append(("commit", self.s_full[1]))
            if M != "k_empty_early":
                self.pipe.append(("commit", self.k_empty[st0]))
            if n == 1:
                self.pipe.append(("commit", self.q_empty[0]))
                self.pipe.append(("commit", self.q_empty[1]))
            elif n == 2 and M == "q_empty_one_early":
                self.pipe.append(("commit", self.q_empty[0]))
            yield
            for j in range(n):
                g = gt + j
                st, st2 = g % V_STAGES, (g + 1) % K_STAGES
                has_next = j + 1 < n
                yield from self.wait(self.v_full[st], (g // V_STAGES) & 1, g // V_STAGES)
                mem_next = 3
                if M == "o_full_early" and not has_next:
                    self.pipe.append(("commit", self.o_full[0]))
                # head 0: O0 += P0 V, then S0 of the next tile
                yield from self.pv_or_skip(0, bool(mem_cur & 1), pc, st, it, j, started[0] if self.per_head else j > 0)
                if mem_cur & 1:
                    started[0] = True
                if M == "v_empty_after_head0":
                    self.pipe.append(("commit", self.v_empty[st]))
                if not has_next:
                    if M != "o_full_early":
                        self.pipe.append(("commit", self.o_full[0]))
                else:
                    yield from self.wait(self.k_full[st2], ((g + 1) // K_STAGES) & 1, (g + 1) // K_STAGES)
                    mem_next = self.read_tile_mem(st2, it, j + 1) if self.per_head else 3
                    if mem_next & 1:
                        self.pipe.append(("qk", 0, st2, it, j + 1))
                    self.pipe.append(("commit", self.s_full[0]))
                    if j + (3 if M == "q_empty_one_early" else 2) == n:
                        self.pipe.append(("commit", self.q_empty[0]))
                if M == "s1_before_pv1" and has_next:
                    if mem_next & 2:
                        self.pipe.append(("qk", 1, st2, it, j + 1))
                    self.pipe.append(("commit", self.s_full[1]))
                # head 1
                yield from self.pv_or_skip(1, bool(mem_cur & 2), pc, st, it, j, started[1] if self.per_head else j > 0)
                if mem_cur & 2:
                    started[1] = True
                if M != "v_empty_after_head0":
                    self.pipe.append(("commit", self.v_empty[st]))
                if not has_next:
                    self.pipe.append(("commit", self.o_full[1]))
                else:
                    if M != "s1_before_pv1":
                        if mem_next & 2:
                            self.pipe.append(("qk", 1, st2, it, j + 1))
                        self.pipe.append(("commit", self.s_full[1]))
                    self.pipe.append(("commit", self.k_empty[st2]))
                    if j + 2 == n:
                        self.pipe.append(("commit", self.q_empty[1]))
                mem_cur = mem_next
                pc += 1
                yield
            gt += n

    def pv_or_skip(self, h, member, pc, st, it, j, accumulate):
        for q in range(P_CHUNKS):
            yield from self.wait(self.p_full[h][q], pc & 1, pc)
            if member:
                self.pipe.append(("pv", h, q, st, it, j, accumulate))
            yield

    def softmax(self, h, w):
        sc = 0
        for it, item in enumerate(self.items):
            started = False
            for j in range(item.n):
                yield from self.wait(self.s_full[h], sc & 1, sc)
                sc += 1
                if not self.member(it, j, h):
                    if self.mistake != "skip_without_handshake":
                        for q in range(P_CHUNKS):
                            self.p_full[h][q].arrive(32)
                    yield
                    continue
                sb = self.s[h][w]
                check(sb.content == (it, j), f"softmax {h}.{w}: S holds {sb.content}, wants {(it, j)}")
                sb.readers.clear()
                yield
                if started:  # the lazy rescale reads and writes O
                    o = self.o[h][w]
                    want = {(jj, q) for jj in range(j) if self.member(it, jj, h) for q in range(P_CHUNKS)}
                    check(o["item"] == it and o["parts"] == want,
                          f"softmax {h}.{w}: rescale sees O of item {o['item']} with {sorted(o['parts'])}")
                    yield
                started = True
                for q in range(P_CHUNKS):
                    pb = self.p[h][w][q]
                    check(not pb.readers, f"softmax {h}.{w}: P chunk {q} rewritten before P V read it")
                    self.p[h][w][q] = Buf((it, j), {"pv"})
                    self.p_full[h][q].arrive(32)
                    yield
            yield from self.wait(self.o_full[h], it & 1, it)
            o = self.o[h][w]
            want = {(jj, q) for jj in range(item.n) if self.member(it, jj, h) for q in range(P_CHUNKS)}
            check(o["item"] == it and o["parts"] == want,
                  f"epilogue {h}.{w}: O of item {o['item']} holds {sorted(o['parts'])}, wants {sorted(want)}")
            o["read"] = True
            yield


def run(items, per_head, seed, mistake=None, max_steps=2_000_000):
    """One random interleaving of all roles; raises ProtocolError on a violation."""
    m = Model(items, per_head, mistake)
    rng = random.Random(seed)
    roles = [m.producer(), m.mma()] + [m.softmax(h, w) for h in range(2) for w in range(WARPS)]
    state = [None] * len(roles)  # None: runnable; ("blocked", bar, parity, phase): waiting
    live = set(range(len(roles)))
    for _ in range(max_steps):
        for i in live:  # a blocked waiter whose barrier ran two phases on would never see its phase
            if state[i] is not None:
                _, bar, _, phase = state[i]
                check(bar.done <= phase + 1, f"{bar.name}: signaller ran two phases past a waiter (phase {phase})")
        choices = [i for i in live if state[i] is None or state[i][1].passes(state[i][2])]
        if m.pipe:
            choices.append("pipe")
        if m.tma:
            choices.append("tma")
        if not choices:
            if not live:
                return m
            blocked = ", ".join(f"{state[i][1].name}" for i in live)
            raise ProtocolError(f"deadlock: waiting on {blocked}")
        c = rng.choice(choices)
        if c == "pipe":
            m.run_op(m.pipe.pop(0))
        elif c == "tma":
            bar, buf, content, readers = m.tma.pop(rng.randrange(len(m.tma)))
            check(not buf.readers, f"TMA into a buffer with reads still owed ({sorted(map(str, buf.readers))})")
            buf.content, buf.readers = content, set(readers)
            bar.complete_tx(TILE)
        else:
            try:
                state[c] = next(roles[c])
            except StopIteration:
                live.discard(c)
                state[c] = None
    raise ProtocolError("step limit")


def random_items(rng, per_head, n_items=4, max_tiles=5):
    items = []
    for _ in range(n_items):
        n = rng.randint(1, max_tiles)
        if per_head:  # the diagonal tile (last) is in both heads' lists
            mem = [rng.choice((1, 2, 3)) for _ in range(n - 1)] + [3]
        else:
            mem = [3] * n
        items.append(Item(mem))
    return items


@pytest.mark.parametrize("per_head", [False, True], ids=["shared", "per_head"])
def test_protocol_holds_under_random_interleavings(per_head):
    for seed in range(150):
        rng = random.Random(1000 + seed)
        run(random_items(rng, per_head), per_head, seed)


def test_protocol_single_tile_items_and_long_items():
    for seed in range(40):
        run([Item([3]) for _ in range(5)], False, seed)
        run([Item([3] * 9), Item([3]), Item([3] * 2)], False, seed)
        run([Item([1, 2, 1, 3]), Item([2, 2, 2, 3]), Item([3])], True, seed)


MISTAKES = [
    ("producer_empty_parity", False),   # producer waits for the wrong phase of k_empty
    ("k_empty_early", False),           # K stage released before head 1's S MMA read it
    ("v_empty_after_head0", False),     # V stage released before head 1's P V read it
    ("o_full_early", False),            # O declared final before the last P V of head 0
    ("s1_before_pv1", False),           # head 1's next S issued before its P V read P
    ("q_empty_one_early", False),       # Q released one tile before its last S MMA
    ("skip_without_handshake", True),   # a skipped tile's P handshake left out
    ("s_full_twice", False),            # S announced twice: the softmax's parity wait aliases
]


@pytest.mark.parametrize("mistake,per_head", MISTAKES, ids=[m[0] for m in MISTAKES])
def test_planted_protocol_mistakes_are_caught(mistake, per_head):
    for seed in range(300):
        rng = random.Random(5000 + seed)
        items = random_items(rng, per_head, n_items=3, max_tiles=5)
        if per_head:
            items.append(Item([1, 3]))  # at least one tile that head 1 skips
        try:
            run(items, per_head, seed, mistake)
        except ProtocolError:
            return
    pytest.fail(f"planted mistake {mistake} was not caught in 300 interleavings")
