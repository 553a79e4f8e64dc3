"""The tensor-core kernel's hand-over protocol, run as a model on the CPU.

tc_gemm_kernel passes each (segment, K tile, part) step between four warp roles through
mbarriers in shared memory: the sign loader fills raw slot i % R (raw_full / raw_free), the
activation loader fills B stage i % nB (b_full / b_free), the producers expand step i into
A stage i % nA in tensor memory (a_full / a_free) and the MMA thread consumes A and B stages
and commits to a_free / b_free when its MMAs complete. This test replays those programs
(the order of waits, arrivals, expected bytes and commits as the kernel issues them) against
a model of the mbarrier rules, under random interleavings and random completion delays of
the asynchronous copies and MMAs, for ring sizes around the ones the planner picks. It
checks that every run finishes (no role waits forever), that a consumer only sees the data
of its own step, and that no stage or slot is overwritten while an earlier reader may
still use it.
"""

import random

import pytest


class MBar:
    """mbarrier phase rules: a phase completes when its expected arrivals have all arrived
    and its transaction count is back to zero; waiting on parity p succeeds once the phase
    with parity p has completed (the current phase's parity is then 1 - p)."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, n=1):
        assert self.pending >= n, "more arrivals than expected in one phase"
        self.pending -= n
        self._maybe_complete()

    def expect_tx(self, nbytes):  # arrive.expect_tx: one arrival plus expected bytes
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def done(self, parity):
        return (self.phase & 1) != parity


class Sim:
    def __init__(self, n, nA, nB, R, tma_steps, producers, seed):
        self.n, self.nA, self.nB, self.R = n, nA, nB, R
        self.tma = tma_steps  # steps whose B tile comes through a tensor copy
        self.rng = random.Random(seed)
        self.raw_full = [MBar(33) for _ in range(R)]
        self.raw_free = [MBar(producers) for _ in range(R)]
        self.a_full = [MBar(producers) for _ in range(nA)]
        self.a_free = [MBar(1) for _ in range(nA)]
        self.b_full = [MBar(1) for _ in range(nB)]
        self.b_free = [MBar(1) for _ in range(nB)]
        self.raw = [None] * R          # step whose sign words are in the slot (None: in flight)
        self.A = [None] * nA           # step expanded into the stage
        self.B = [None] * nB
        self.producers = producers
        self.raw_readers = [set() for _ in range(R)]   # producers yet to read the landed slot
        self.mma_live = {}             # step -> (A stage, B stage) of MMAs not complete yet
        self.events = []               # (time, callback)
        self.now = 0

    def later(self, fn):
        self.events.append((self.now + self.rng.randint(1, 12), fn))

    # -- role programs (generators yielding a (barrier, parity) to wait on) ----------
    def sign_loader(self):
        for i in range(self.n):
            rs = i % self.R
            if i >= self.R:
                yield self.raw_free[rs], (i // self.R - 1) & 1
            assert not self.raw_readers[rs], "raw slot refilled before every producer read it"
            self.raw[rs] = None
            self.raw_full[rs].expect_tx(2048 + 256)          # lane 0: bytes of both tensor copies

            def land(rs=rs, i=i):
                self.raw[rs] = i
                self.raw_readers[rs] = set(range(self.producers))
                self.raw_full[rs].complete_tx(2048 + 256)
            self.later(land)
            self.raw_full[rs].arrive(32)                     # every lane after its plain stores

    def act_loader(self):
        for j in range(self.n):
            sb = j % self.nB
            if j >= self.nB:
                yield self.b_free[sb], (j // self.nB - 1) & 1
            assert all(s[1] != sb for s in self.mma_live.values()), "B stage reloaded under a live MMA"
            if j in self.tma:
                self.B[sb] = None
                self.b_full[sb].expect_tx(4096)

                def land(sb=sb, j=j):
                    self.B[sb] = j
                    self.b_full[sb].complete_tx(4096)
                self.later(land)
            else:
                self.b_full[sb].arrive()

    def producer(self, p):
        for i in range(self.n):
            sa, sb, rs = i % self.nA, i % self.nB, i % self.R
            if i >= self.nA:
                yield self.a_free[sa], (i // self.nA - 1) & 1
            yield self.raw_full[rs], (i // self.R) & 1
            assert self.raw[rs] == i, "producer read sign words of another step"
            assert all(s[0] != sa for s in self.mma_live.values()), "A stage rewritten under a live MMA"
            self.A[sa] = i
            if i not in self.tma:  # producers write the B tile themselves
                if i >= self.nB:
                    yield self.b_free[sb], (i // self.nB - 1) & 1
                assert all(s[1] != sb for s in self.mma_live.values()), "B stage rewritten under a live MMA"
                self.B[sb] = i
            self.raw_readers[rs].discard(p)
            self.a_full[sa].arrive()
            self.raw_free[rs].arrive()

    def mma(self):
        for i in range(self.n):
            sa, sb = i % self.nA, i % self.nB
            yield self.a_full[sa], (i // self.nA) & 1
            yield self.b_full[sb], (i // self.nB) & 1
            assert self.A[sa] == i and self.B[sb] == i, "MMA read a stage of another step"
            self.mma_live[i] = (sa, sb)

            def complete(i=i, sa=sa, sb=sb):  # commit: arrivals once the MMAs are done
                del self.mma_live[i]
                self.a_free[sa].arrive()
                self.b_free[sb].arrive()
            self.later(complete)

    def run(self):
        roles = [self.sign_loader(), self.act_loader(), self.mma()] + [self.producer(p) for p in range(self.producers)]
        waiting = [None] * len(roles)
        live = list(range(len(roles)))
        for _ in range(200000):
            runnable = [k for k in live if waiting[k] is None or waiting[k][0].done(waiting[k][1])]
            if not runnable and not self.events:
                raise AssertionError(f"deadlock: roles {live} wait forever")
            if runnable and (not self.events or self.rng.random() < 0.7):
                k = self.rng.choice(runnable)
                try:
                    waiting[k] = next(roles[k])
                except StopIteration:
                    live.remove(k)
                    waiting[k] = None
            else:
                self.events.sort(key=lambda e: e[0])
                t, fn = self.events.pop(0)
                self.now = max(self.now, t)
                fn()
            if not live and not self.events:
                return
        raise AssertionError("did not finish")


@pytest.mark.parametrize("n,nA,nB,R", [(1, 2, 3, 4), (5, 2, 3, 4), (16, 4, 6, 4), (16, 4, 3, 56), (17, 3, 5, 8),
                                       (64, 4, 6, 64), (40, 2, 2, 3), (9, 4, 6, 2)])
def test_protocol_finishes_and_hands_over_the_right_data(n, nA, nB, R):
    for seed in range(40):
        tma = {i for i in range(n) if (i * 7 + seed) % 5 != 0}   # some steps with producer-written B tiles
        sim = Sim(n, nA, nB, R, tma, producers=3, seed=seed)
        sim.run()
        assert not sim.mma_live
        for b in sim.a_full + sim.a_free + sim.b_full + sim.b_free + sim.raw_full + sim.raw_free:
            assert b.pending == b.count and b.tx == 0


PLANTED = {
    # each replaces one line of the role programs above with a protocol mistake
    "producers skip the A-stage free wait": (
        "                yield self.a_free[sa], (i // self.nA - 1) & 1\n", "                pass\n"),
    "sign loader waits on the wrong parity": (
        "                yield self.raw_free[rs], (i // self.R - 1) & 1\n",
        "                yield self.raw_free[rs], (i // self.R) & 1\n"),
    "activation loader skips the B-stage free wait": (
        "                yield self.b_free[sb], (j // self.nB - 1) & 1\n            assert all",
        "                pass\n            if False:\n                yield None\n            assert all"),
    "MMA skips the B-stage full wait": ("            yield self.b_full[sb], (i // self.nB) & 1\n", ""),
    "producers skip the raw-slot full wait": ("            yield self.raw_full[rs], (i // self.R) & 1\n", ""),
    "MMA frees the A stage at issue": (
        "                self.a_free[sa].arrive()\n                self.b_free[sb].arrive()\n            self.later(complete)",
        "                self.b_free[sb].arrive()\n            self.a_free[sa].arrive()\n            self.later(complete)"),
}


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_model_catches_planted_protocol_mistakes(name):
    import os
    import types
    with open(os.path.abspath(__file__)) as f:
        src = f.read()
    old, new = PLANTED[name]
    assert src.count(old) >= 1
    mod = types.ModuleType("planted")
    exec(compile(src.replace(old, new, 1), "planted", "exec"), mod.__dict__)
    for args in [(1, 2, 3, 4), (5, 2, 3, 4), (16, 4, 6, 4), (16, 4, 3, 56), (17, 3, 5, 8), (40, 2, 2, 3), (9, 4, 6, 2)]:
        try:
            mod.test_protocol_finishes_and_hands_over_the_right_data(*args)
        except (AssertionError, KeyError):
            return
    raise AssertionError(f"planted mistake not caught: {name}")
