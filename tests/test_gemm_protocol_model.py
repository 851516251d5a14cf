"""A host model of the tensor-core GEMM's pipeline protocol (gemm.cu), run
under random interleavings: the TMA producer, the four weight-unpack warps,
the MMA warp and the epilogue as separate agents, with copies and MMA
completions as asynchronous events.

What it checks, for the 4-bit weights (unpacked into tensor-memory A slots)
and the int8 weights (the MMA's shared-memory operand), with units issued
one or two at a time:
  * every mbarrier wait is resolved on the phase it means: the barrier's
    completed-phase count is the awaited phase or one more when a
    parity test is made, never one behind or two ahead (the hardware
    compares parities only);
  * no copy is issued into a stage region, and no unpack writes an A slot,
    while an earlier unit may still read it; every read sees its own unit;
  * every run finishes (no deadlock).
The ring sizes follow the kernel's limits: stages <= 16, A slots <= 8, a
ring of 32 completion barriers.  The producer sends a stage's next weight
copy when the stage's `ready` phase of the previous unit completes (its
weights are in tensor memory), and the activation copy after that unit's
MMA completion.  A variant that sends the weight copy one stage too early
must be caught.
"""
import random

import pytest

DONE_RING = 32


class Protocol(Exception):
    pass


class Barrier:
    """An mbarrier: arrivals and transaction bytes; a phase completes when
    both reach zero, then the counts reset."""

    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        if self.pending < 0:
            raise Protocol(f"{self.name}: more arrivals than expected in phase {self.completed}")
        self._maybe_complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def test(self, phase):
        """try_wait.parity for `phase`: the hardware's answer, checked against
        the phase actually meant."""
        c = self.completed
        if c < phase or c > phase + 1:
            raise Protocol(f"{self.name}: wait for phase {phase} while {c} phases completed (parity aliasing)")
        return (c & 1) != (phase & 1)


class Model:
    def __init__(self, ns, nas, total, kbn, w8, pair, early_w=True, bad_w=False, seed=0):
        self.rng = random.Random(seed)
        self.ns, self.nas, self.total, self.kbn = ns, nas, total, kbn
        self.w8, self.pair, self.early_w, self.bad_w = w8, pair, early_w, bad_w
        self.wfull = [Barrier(f"wfull[{s}]", 1) for s in range(ns)]
        self.ready = [Barrier(f"ready[{s}]", 2 if w8 else 5) for s in range(ns)]
        self.done = [Barrier(f"done[{j}]", 1) for j in range(DONE_RING)]
        self.acc_full = [Barrier(f"acc_full[{b}]", 1) for b in range(2)]
        self.acc_empty = [Barrier(f"acc_empty[{b}]", 8) for b in range(2)]
        # region contents: (unit, landed) per stage's weight and activation region, unit per A slot
        self.w_region = [None] * ns
        self.x_region = [None] * ns
        self.a_slot = [None] * nas
        self.unpacked = {}            # unit -> unpack warps done
        self.mma_done = set()         # units whose MMA completed
        self.epi_done = set()         # segments the epilogue has drained
        self.copies = []              # in-flight copies: (barrier, nbytes, region, stage, unit)
        self.mma_queue = []           # in-order tensor-core work: ("mma", unit, seg) / ("commit", barrier)
        self.segments = self._segments()

    def _segments(self):
        seg_of, i, kb, seg = {}, 0, 0, 0
        while i < self.total:
            n = min(self.total - i, self.kbn - kb)
            for u in range(i, i + n):
                seg_of[u] = seg
            i, kb, seg = i + n, 0, seg + 1
        self.nseg = seg
        return seg_of

    # --- asynchronous engines
    def _issue_copy(self, kind, s, u):
        region = self.w_region if kind == "w" else self.x_region
        if kind == "w" and not self.w8:
            prev = u - self.ns
            if prev >= 0 and self.unpacked.get(prev, 0) < 4:
                raise Protocol(f"weight copy of unit {u} into stage {s} before unit {prev} was unpacked")
        if kind == "x" or self.w8:
            prev = u - self.ns
            if prev >= 0 and prev not in self.mma_done:
                raise Protocol(f"{kind} copy of unit {u} into stage {s} before unit {prev}'s MMA completed")
        region[s] = (u, False)
        bar = self.wfull[s] if (kind == "w" and not self.w8) else self.ready[s]
        self.copies.append((bar, 1, region, s, u))

    def _land_copy(self, k):
        bar, nbytes, region, s, u = self.copies.pop(k)
        region[s] = (u, True)
        bar.complete_tx(nbytes)

    def _run_tensor(self):
        op = self.mma_queue.pop(0)
        if op[0] == "mma":
            _, u, seg = op
            s = u % self.ns
            if self.x_region[s] != (u, True):
                raise Protocol(f"MMA of unit {u} reads stage {s} holding {self.x_region[s]}")
            if self.w8:
                if self.w_region[s] != (u, True):
                    raise Protocol(f"MMA of unit {u} reads weights of stage {s} holding {self.w_region[s]}")
            elif self.a_slot[u % self.nas] != u or self.unpacked.get(u, 0) < 4:
                raise Protocol(f"MMA of unit {u} reads A slot {u % self.nas} holding {self.a_slot[u % self.nas]}")
            if seg >= 2 and (seg - 2) not in self.epi_done:
                raise Protocol(f"MMA of segment {seg} writes an accumulator the epilogue still reads")
            self.mma_done.add(u)
        else:
            op[1].arrive()

    # --- agents (generators yielding a barrier test to block on)
    def wait(self, bar, phase):
        while not bar.test(phase):
            yield

    def load_w(self, s, u):
        # 4-bit weights complete on wfull[s]; int8 weights on ready[s] (their own arrival)
        (self.ready[s] if self.w8 else self.wfull[s]).arrive(1)
        self._issue_copy("w", s, u)

    def load_x(self, s, u):
        self.ready[s].arrive(1)
        self._issue_copy("x", s, u)

    def producer(self):
        ns, total = self.ns, self.total
        prime = min(total, ns)
        for i in range(prime):
            self.load_w(i, i)
        for i in range(prime):  # after the wait for the preceding kernel
            self.load_x(i, i)
        for it in range(prime, total):
            s, w = it % ns, it - ns
            if not self.w8 and self.early_w:
                # the stage's weight region: free once unit w's ready phase completed
                ph = (w // ns) - (1 if self.bad_w else 0)
                if ph >= 0:
                    yield from self.wait(self.ready[s], ph)
                self.load_w(s, it)
            yield from self.wait(self.done[w % DONE_RING], w // DONE_RING)
            if self.w8 or not self.early_w:
                self.load_w(s, it)
            self.load_x(s, it)
        for i in range(max(total - ns, 0), total):
            if not self.w8:
                yield from self.wait(self.wfull[i % ns], i // ns)
            yield from self.wait(self.ready[i % ns], i // ns)

    def unpack(self, warp):
        for it in range(self.total):
            s, a = it % self.ns, it % self.nas
            yield from self.wait(self.wfull[s], it // self.ns)
            if it >= self.nas:
                u = it - self.nas
                yield from self.wait(self.done[u % DONE_RING], u // DONE_RING)
            if self.w_region[s] != (it, True):
                raise Protocol(f"unpack of unit {it} reads stage {s} holding {self.w_region[s]}")
            prev = self.a_slot[a]
            if prev is not None and prev != it and prev not in self.mma_done:
                raise Protocol(f"unpack of unit {it} overwrites A slot {a} before unit {prev}'s MMA")
            self.a_slot[a] = it
            yield  # the tensor-memory stores take time
            self.unpacked[it] = self.unpacked.get(it, 0) + 1
            self.ready[s].arrive()

    def mma(self):
        i, seg = 0, 0
        while i < self.total:
            n = sum(1 for u in range(i, self.total) if self.segments[u] == seg)
            b = seg & 1
            if seg >= 2:
                yield from self.wait(self.acc_empty[b], seg // 2 - 1)
            j = 0
            if self.pair:
                while j + 1 < n:
                    yield from self.wait(self.ready[i % self.ns], i // self.ns)
                    yield from self.wait(self.ready[(i + 1) % self.ns], (i + 1) // self.ns)
                    self.mma_queue += [("mma", i, seg), ("mma", i + 1, seg),
                                       ("commit", self.done[i % DONE_RING]),
                                       ("commit", self.done[(i + 1) % DONE_RING])]
                    i, j = i + 2, j + 2
            while j < n:
                yield from self.wait(self.ready[i % self.ns], i // self.ns)
                self.mma_queue += [("mma", i, seg), ("commit", self.done[i % DONE_RING])]
                i, j = i + 1, j + 1
            self.mma_queue.append(("commit", self.acc_full[b]))
            seg += 1

    def epilogue(self):
        for seg in range(self.nseg):
            b = seg & 1
            yield from self.wait(self.acc_full[b], seg // 2)
            yield  # reading the accumulator
            self.epi_done.add(seg)
            for _ in range(8):
                self.acc_empty[b].arrive()

    def run(self, max_steps=200000):
        agents = [self.producer(), self.mma(), self.epilogue()]
        if not self.w8:
            agents += [self.unpack(w) for w in range(4)]
        live = list(agents)
        for _ in range(max_steps):
            choices = [("agent", a) for a in live]
            choices += [("copy", k) for k in range(len(self.copies))]
            if self.mma_queue:
                choices.append(("tensor", None))
            if not choices:
                raise Protocol("nothing can run")
            kind, x = self.rng.choice(choices)
            if kind == "agent":
                try:
                    next(x)
                except StopIteration:
                    live.remove(x)
            elif kind == "copy":
                self._land_copy(x)
            else:
                self._run_tensor()
            if not live and not self.copies and not self.mma_queue:
                if len(self.mma_done) != self.total or len(self.epi_done) != self.nseg:
                    raise Protocol("finished without every unit's MMA and every segment's epilogue")
                return
        raise Protocol("no progress: deadlock or livelock")


CASES = [
    # (stages, A slots, units, units per tile, int8 weights, pair issue)
    (3, 2, 40, 10, False, False),   # BT = 192: 3 stages, 2 A slots
    (3, 2, 37, 12, False, False),
    (4, 4, 50, 10, False, True),    # BT <= 128: pair issue
    (10, 7, 90, 16, False, True),   # BT = 16..64: many stages
    (16, 7, 120, 48, False, False),
    (16, 8, 70, 5, False, True),
    (3, 2, 40, 10, True, False),    # int8 weights
    (6, 4, 33, 11, True, True),
]


@pytest.mark.parametrize("ns,nas,total,kbn,w8,pair", CASES)
def test_pipeline_protocol_random_interleavings(ns, nas, total, kbn, w8, pair):
    for seed in range(100):
        Model(ns, nas, total, kbn, w8, pair, seed=seed).run()


@pytest.mark.parametrize("ns,nas,total,kbn", [(3, 2, 40, 10), (10, 7, 90, 16)])
def test_the_previous_order_passes_too(ns, nas, total, kbn):
    # weight copy after the MMA's completion, as before
    for seed in range(20):
        Model(ns, nas, total, kbn, False, False, early_w=False, seed=seed).run()


def test_a_weight_copy_one_stage_early_is_caught():
    caught = 0
    for seed in range(40):
        try:
            Model(3, 2, 40, 10, False, False, bad_w=True, seed=seed).run()
        except Protocol:
            caught += 1
    assert caught > 0
