"""The streaming lookup-table kernel's sign-word ring, run as a model on the CPU.

lut_gemv_stream_kernel streams a CTA's TS = nchunks x nt stages (the quads of one row tile
for one chunk of units) through a ring of NS shared-memory slots. Every stage k has its own
pair of mbarriers: full[k] (the bulk copies' bytes, one arrival by the issuing lane) and
empty[k] (one arrival per unit-group warp that read it). The 12 warps form gt tile groups x
gu unit groups; at kernel start warp w issues stages w, w + 12, ... below NS; per chunk the
CTA synchronises twice (tables are rebuilt) and each warp walks its tile group's stages of
the chunk in the interleaved order of stage_in_chunk, waits full[k], reads slot k % NS and,
if stage k + NS exists, arrives on empty[k]; the group's first warp then waits empty[k]
and issues stage k + NS into the same slot. This test replays those programs against the
mbarrier phase rules (the same model as the tensor-core protocol test) with random
interleavings and copy latencies, and checks that every run finishes, every warp reads the
stage it expects, and no slot is refilled before every reader of its stage has read it.
"""

import random

import pytest

from test_tc_pipeline_model import MBar

KSW = 12  # warps of the streaming kernel


def stage_in_chunk(g, s, nt, gt):
    # position of (tile group g, step s) among a chunk's stages, tile groups interleaved
    q = nt // gt
    return s * gt + g if s < q else q * gt + (g * nt // gt - g * q)


def stage_tile(j, nt, gt):
    q = nt // gt
    if j < q * gt:
        s, g = j // gt, j % gt
        return g * nt // gt + s
    r, g = j - q * gt, 0
    while g < gt - 1:
        if (g + 1) * nt // gt - g * nt // gt > q:
            if r == 0:
                break
            r -= 1
        g += 1
    return g * nt // gt + q


class CtaBarrier:
    def __init__(self, n):
        self.n, self.arrived, self.gen = n, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.n:
            self.arrived, self.gen = 0, self.gen + 1


class Sim:
    def __init__(self, nt, nchunks, gu, NS, seed):
        self.nt, self.nchunks, self.gu, self.gt, self.NS = nt, nchunks, gu, KSW // gu, NS
        self.TS = nchunks * nt
        self.rng = random.Random(seed)
        self.full = [MBar(1) for _ in range(self.TS)]
        self.empty = [MBar(gu) for _ in range(self.TS)]
        self.slot = [None] * NS
        self.readers = [set() for _ in range(NS)]
        self.bar = CtaBarrier(KSW)
        self.events, self.now = [], 0

    def issue(self, k):
        s = k % self.NS
        assert not self.readers[s], f"slot {s} refilled before every reader of its stage read it"
        self.slot[s] = None
        self.full[k].expect_tx(512)
        g = self._group_of(k)

        def land():
            self.slot[s] = k
            self.readers[s] = {(g, b) for b in range(self.gu)}
            self.full[k].complete_tx(512)
        self.events.append((self.now + self.rng.randint(1, 15), land))

    def _group_of(self, k):
        t = stage_tile(k % self.nt, self.nt, self.gt)
        return next(g for g in range(self.gt) if g * self.nt // self.gt <= t < (g + 1) * self.nt // self.gt)

    def warp(self, w):
        ga, gb = w // self.gu, w % self.gu
        for k in range(w, min(self.NS, self.TS), KSW):
            self.issue(k)
        sz = (ga + 1) * self.nt // self.gt - ga * self.nt // self.gt
        for c in range(self.nchunks):
            for _ in range(2):  # __syncthreads before and after the chunk's tables
                gen = self.bar.gen
                self.bar.arrive()
                yield ("cta", gen)
            for st in range(sz):
                k = c * self.nt + stage_in_chunk(ga, st, self.nt, self.gt)
                assert stage_tile(k % self.nt, self.nt, self.gt) == ga * self.nt // self.gt + st
                yield ("mbar", self.full[k], 0)
                s = k % self.NS
                assert self.slot[s] == k, f"warp {w} read slot {s} holding stage {self.slot[s]}, expected {k}"
                self.readers[s].discard((ga, gb))
                if k + self.NS < self.TS:
                    self.empty[k].arrive()
                    if gb == 0:
                        yield ("mbar", self.empty[k], 0)
                        self.issue(k + self.NS)

    def _ready(self, wait):
        if wait is None:
            return True
        if wait[0] == "cta":
            return self.bar.gen != wait[1]
        return wait[1].done(wait[2])

    def run(self):
        progs = [self.warp(w) for w in range(KSW)]
        waiting = [None] * KSW
        live = list(range(KSW))
        for _ in range(500000):
            runnable = [w for w in live if self._ready(waiting[w])]
            if not runnable and not self.events:
                raise AssertionError(f"deadlock: warps {live} wait forever")
            if runnable and (not self.events or self.rng.random() < 0.6):
                w = self.rng.choice(runnable)
                try:
                    waiting[w] = next(progs[w])
                except StopIteration:
                    live.remove(w)
            else:
                self.events.sort(key=lambda e: e[0])
                t, fn = self.events.pop(0)
                self.now = max(self.now, t)
                fn()
            if not live and not self.events:
                return
        raise AssertionError("did not finish")


def test_stage_order_is_a_permutation_of_the_tiles():
    for nt in range(1, 40):
        for gt in (1, 2, 3, 4, 6, 12):
            pos = sorted(stage_in_chunk(g, s, nt, gt) for g in range(gt)
                         for s in range((g + 1) * nt // gt - g * nt // gt))
            assert pos == list(range(nt))
            for j in range(nt):  # stage_tile inverts stage_in_chunk
                t = stage_tile(j, nt, gt)
                g = next(g for g in range(gt) if g * nt // gt <= t < (g + 1) * nt // gt)
                assert stage_in_chunk(g, t - g * nt // gt, nt, gt) == j


@pytest.mark.parametrize("nt,nchunks,gu,NS", [(16, 1, 1, 4), (20, 2, 2, 6), (29, 3, 3, 5), (12, 4, 4, 12),
                                               (45, 2, 6, 8), (17, 3, 12, 3), (8, 2, 2, 16), (30, 1, 3, 30)])
def test_ring_finishes_and_every_warp_reads_its_stage(nt, nchunks, gu, NS):
    for seed in range(25):
        sim = Sim(nt, nchunks, gu, NS, seed)
        sim.run()
        for b in sim.full + sim.empty:
            assert b.tx == 0


def test_per_slot_barriers_would_alias_phases():
    # The form the kernel replaced: one (full, empty) pair per ring slot, waited on with the
    # stage's round parity. A warp of a later stage of the same slot can then pass the full
    # wait on the earlier stage's completed phase and read the wrong data (or a refill can
    # happen early): the model must find such a run.
    class SlotSim(Sim):
        def __init__(self, *a):
            super().__init__(*a)
            self.full = [MBar(1) for _ in range(self.NS)]
            self.empty = [MBar(self.gu) for _ in range(self.NS)]

        def issue(self, k):
            s = k % self.NS
            self.slot[s] = None
            self.full[s].expect_tx(512)
            g = self._group_of(k)

            def land():
                self.slot[s] = k
                self.readers[s] = {(g, b) for b in range(self.gu)}
                self.full[s].complete_tx(512)
            self.events.append((self.now + self.rng.randint(1, 15), land))

        def warp(self, w):
            ga, gb = w // self.gu, w % self.gu
            for k in range(w, min(self.NS, self.TS), KSW):
                self.issue(k)
            sz = (ga + 1) * self.nt // self.gt - ga * self.nt // self.gt
            for c in range(self.nchunks):
                for _ in range(2):
                    gen = self.bar.gen
                    self.bar.arrive()
                    yield ("cta", gen)
                for st in range(sz):
                    k = c * self.nt + stage_in_chunk(ga, st, self.nt, self.gt)
                    s = k % self.NS
                    yield ("mbar", self.full[s], (k // self.NS) & 1)
                    assert self.slot[s] == k, "read another stage's data"
                    if k + self.NS < self.TS:
                        self.empty[s].arrive()
                        if gb == 0:
                            yield ("mbar", self.empty[s], (k // self.NS) & 1)
                            self.issue(k + self.NS)

    found = False
    for seed in range(200):
        try:
            SlotSim(20, 2, 2, 3, seed).run()
        except AssertionError:
            found = True
            break
    assert found
