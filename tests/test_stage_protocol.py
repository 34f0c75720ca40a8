"""Randomised-schedule model of the replay kernel's stage protocol (CPU, no GPU).

The kernel (csrc/replay_kernel.cuh) streams a CTA's units through NS shared-memory stages:
a producer warp fills unit i into stage i mod NS, two units per batch, after waiting for the
release of each stage's previous use on its "empty" mbarrier; consumer group g (of two)
takes units g, g + 2, ..., waiting first for the release of the stage's previous use (phase
k-1 of "empty") and then for its own fill (phase k of "full"), and releases the stage when
done. mbarrier waits test a phase by its parity only, so a wait is exact only while the
barrier is at most one phase away. This model runs the producer, both groups and the copy
engine as coroutines under random schedules, with the parity semantics of the hardware,
and checks that every consumer reads its own unit's data for as long as it holds the stage
and that no schedule deadlocks. It also checks that the protocol needs the consumers' wait
on "empty": without it some schedule reads a stale stage.
"""
import random

import pytest


class MBarrier:
    """Arrival count + transaction bytes; a phase completes when both reach zero."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0  # phases completed so far

    def arrive(self):
        self.pending -= 1
        self._check()

    def arrive_expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def try_wait(self, parity):
        # true once the phase with this parity has completed: the current (incomplete)
        # phase has parity `completed & 1`, so a wait on the other parity passes at once
        return (self.completed & 1) != parity


def run(total, NS, seed, U=2, NG=2, consumer_empty_wait=True, max_steps=400_000):
    rnd = random.Random(seed)
    full = [MBarrier(1) for _ in range(NS)]
    empty = [MBarrier(1) for _ in range(NS)]  # one arrival per group release (after its barrier)
    data = [None] * NS  # the unit whose tile a stage holds
    meta = [None] * NS  # the unit descriptor the producer wrote
    inflight = []

    def producer():
        for i0 in range(0, total, U):
            for jj in range(U):  # wait for the releases of the batch's stages' previous uses
                i = i0 + jj
                if i < total and i >= NS:
                    while not empty[i % NS].try_wait(((i // NS) - 1) & 1):
                        yield
            for jj in range(U):
                i = i0 + jj
                if i < total:
                    s = i % NS
                    meta[s] = i
                    full[s].arrive_expect_tx(1)
                    inflight.append((s, i))
            yield

    def group(g):
        for i in range(g, total, NG):
            s, k = i % NS, i // NS
            if consumer_empty_wait and k > 0:
                while not empty[s].try_wait((k - 1) & 1):
                    yield
            while not full[s].try_wait(k & 1):
                yield
            if data[s] != i or meta[s] != i:
                raise AssertionError(("stale stage", i, data[s], meta[s]))
            for _ in range(rnd.randrange(3)):  # work on the unit
                yield
                if data[s] != i or meta[s] != i:
                    raise AssertionError(("stage overwritten while in use", i, data[s], meta[s]))
            empty[s].arrive()
            yield

    def copies():  # bulk copies land in any order
        while True:
            if inflight and rnd.random() < 0.5:
                s, i = inflight.pop(rnd.randrange(len(inflight)))
                data[s] = i
                full[s].complete_tx(1)
            yield

    roles = [producer()] + [group(g) for g in range(NG)]
    land = copies()
    steps = 0
    while roles:
        steps += 1
        if steps > max_steps:
            raise RuntimeError(("deadlock", total, NS, seed))
        next(land)
        r = rnd.choice(roles)
        try:
            next(r)
        except StopIteration:
            roles.remove(r)
    while inflight:  # the producer's final drain
        next(land)
    return True


@pytest.mark.parametrize("NS", [2, 3, 4, 5, 6, 7, 8])
def test_every_read_sees_its_own_unit(NS):
    for seed in range(60):
        total = 1 + (seed * 7) % 45
        assert run(total, NS, seed)


def test_the_consumer_wait_on_empty_is_needed():
    # With an odd number of stages a stage's consecutive uses alternate between the groups,
    # so a group that runs ahead can test "full" while the stage is a whole phase behind.
    failures = 0
    for seed in range(300):
        try:
            run(40, 5, seed, consumer_empty_wait=False)
        except AssertionError:
            failures += 1
    assert failures > 0
