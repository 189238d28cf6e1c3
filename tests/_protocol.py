"""Shared pieces of the barrier-protocol models: an mbarrier with parity waits, and a random
scheduler over cooperative actors (generators that yield wait predicates) plus background
engines (the tensor pipe, the copy engine) that the scheduler steps at random."""
import random


class Bar:
    """An mbarrier: `count` arrivals complete a phase; `done` = completed phases."""

    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.done = name, count, 0, 0

    def arrive(self, n=1):
        self.arrived += n
        assert self.arrived <= self.count, f"{self.name}: too many arrivals in one phase"
        if self.arrived == self.count:
            self.arrived = 0
            self.done += 1

    def passes(self, parity):
        # try_wait.parity passes once the phase of that parity has completed: the current
        # (incomplete) phase has the other parity
        return (self.done & 1) != parity



def wait_for(bar, n):
    """Wait for completion n (0-based) of `bar` with parity n & 1, as the kernels do; assert on
    passing that exactly completions 0..n have happened (a parity wait cannot tell n-1 or n+1
    from n)."""
    yield lambda: bar.passes(n & 1)
    assert bar.done == n + 1, f"{bar.name}: wait for completion {n} passed with {bar.done} completions"


def wait_released(bar, n):
    """A producer's wait before use n of a stage: completion n-1 of its 'empty' barrier (use 0
    passes at once on the fresh barrier's previous-phase parity)."""
    yield lambda: bar.passes((n & 1) ^ 1)
    assert bar.done == n, f"{bar.name}: use {n} started after {bar.done} releases"


def run_actors(actors, engines, rng: random.Random, before_step=None, max_events=2_000_000):
    """Interleave `actors` (generators yielding predicates to wait on) and `engines` (callables
    returning False when idle) at random until every actor has finished; assert on deadlock."""
    waiting = [None] * len(actors)
    live = set(range(len(actors)))
    for _ in range(max_events):
        if before_step is not None:
            before_step()
        ready = [k for k in live if waiting[k] is None or waiting[k]()]
        busy = [e for e in engines if e(probe=True)]
        choices = [("a", k) for k in ready] + [("e", e) for e in busy]
        if not choices:
            assert not live, f"deadlock: {len(live)} actors blocked"
            return
        kind, c = rng.choice(choices)
        if kind == "e":
            c()
        else:
            try:
                waiting[c] = next(actors[c])
            except StopIteration:
                live.discard(c)
                waiting[c] = None
    raise AssertionError("no progress bound reached")
