"""The barrier protocol of the bf16 attention kernel (attend_tc.cu), checked by randomized
interleavings on the CPU.

The kernel's correctness rests on ordering arguments: every mbarrier parity wait must pass on
exactly the phase it means (a wait for completion n passes wrongly if completion n-1 is still
pending, since the parities agree, or if completion n+1 already happened), TMEM buffers must
hold what each reader expects, the PV products must accumulate into O in step order, and O may
only be rescaled between PV(i-1) and PV(i).  This module restates the kernel's roles as
cooperative actors (K and V producers, the two MMA issuers, the in-order tensor pipe with its
commits, and the two softmax warpgroups as four independently scheduled warps each), runs them
under many random schedules and list lengths, and asserts those properties at every step.

It models the protocol, not the arithmetic; the GPU parity tests cover the arithmetic.
"""
import random

import pytest

from tests._protocol import Bar, run_actors, wait_for, wait_released

KSTAGES, VSTAGES, NSBUF = 3, 2, 3


class Sim:
    def __init__(self, nsteps, rng, rescale_prob, mistake=None):
        self.n, self.rng, self.rescale_prob, self.mistake = nsteps, rng, rescale_prob, mistake
        B = {}
        for s in range(KSTAGES):
            B[f"kfull{s}"], B[f"kempty{s}"] = Bar(f"kfull{s}", 1), Bar(f"kempty{s}", 1)
        for s in range(VSTAGES):
            B[f"vfull{s}"], B[f"vempty{s}"] = Bar(f"vfull{s}", 1), Bar(f"vempty{s}", 1)
        for b in range(NSBUF):
            B[f"sfull{b}"], B[f"pfull{b}"] = Bar(f"sfull{b}", 1), Bar(f"pfull{b}", 128)
        for w in range(2):   # P-ready per warpgroup (used only by a planted mistake)
            B[f"pfullwg{w}"] = Bar(f"pfullwg{w}", 128)
        for p in range(2):
            B[f"pvdone{p}"] = Bar(f"pvdone{p}", 1)
            B[f"xdone{p}"] = Bar(f"xdone{p}", 128)
        B["mmadone"] = Bar("mmadone", 2)
        self.B = B
        # what each TMEM S/P buffer holds, per lane quadrant (a warp stores only its 32 rows)
        self.buf = [[None] * 4 for _ in range(NSBUF)]
        self.kst = [None] * KSTAGES        # which step's K a stage holds
        self.vst = [None] * VSTAGES
        self.pv_done = -1                  # last PV executed (O accumulates in order)
        self.mref = {}                     # row reference max: version = last step that set it
        self.pipe = {0: [], 1: []}         # per issuing thread, in order: (kind, step)
        self.pending_commits = []          # (issuer, seq of its last batch, barrier)
        self.issued = {0: 0, 1: 0}         # batches issued per issuer
        self.completed = {0: 0, 1: 0}      # batches completed per issuer
        self.loads = []                    # in-flight TMA loads: (barrier, kind, stage, step)

    def wait(self, bar, n):
        yield from wait_for(self.B[bar], n)

    def wait_free(self, bar, n):
        yield from wait_released(self.B[bar], n)

    def issue(self, who, kind, step):
        self.pipe[who].append((kind, step))
        self.issued[who] += 1

    def commit(self, who, bar):
        self.pending_commits.append((who, self.issued[who], bar))

    # -- actors
    def k_producer(self):
        for i in range(self.n):
            s = i % KSTAGES
            yield from self.wait_free(f"kempty{s}", max(0, i // KSTAGES - (self.mistake == "k_stage_reused_early")))
            self.loads.append((f"kfull{s}", "k", s, i))

    def v_producer(self):
        for j in range(self.n):
            s = j % VSTAGES
            yield from self.wait_free(f"vempty{s}", j // VSTAGES)
            self.loads.append((f"vfull{s}", "v", s, j))

    def issuer(self, w):
        def qk(i):
            yield from self.wait(f"kfull{i % KSTAGES}", i // KSTAGES)
            self.issue(w, "qk", i)
            self.commit(w, f"sfull{i % NSBUF}")
            self.commit(w, f"kempty{i % KSTAGES}")

        if self.n == 0:
            return   # the kernel's issuers do nothing without steps
        for j in range(w, min(NSBUF, self.n), 2):
            yield from qk(j)
        for i in range(w, self.n, 2):
            if i >= 1 and self.mistake != "pv_not_ordered":
                yield from self.wait(f"pvdone{(i - 1) & 1}", (i - 1) >> 1)
            yield from self.wait(f"vfull{i % VSTAGES}", i // VSTAGES)
            if self.mistake == "p_ready_per_warpgroup":
                yield from self.wait(f"pfullwg{i & 1}", i >> 1)
            else:
                yield from self.wait(f"pfull{i % NSBUF}", i // NSBUF)
            if self.mistake == "qk_before_pv" and i + NSBUF < self.n:
                yield from qk(i + NSBUF)
            self.issue(w, "pv", i)
            self.commit(w, f"vempty{i % VSTAGES}")
            self.commit(w, f"pvdone{i & 1}")
            if i + NSBUF < self.n and self.mistake != "qk_before_pv":
                yield from qk(i + NSBUF)
        self.commit(w, "mmadone")

    def warp(self, wg, wq):
        for i in range(wg, self.n, 2):
            b = i % NSBUF
            yield from self.wait(f"sfull{b}", i // NSBUF)
            assert self.buf[b][wq] == ("S", i), f"step {i}: buffer {b} rows {wq} hold {self.buf[b][wq]}"
            if i >= 1:
                yield from self.wait(f"xdone{wg ^ 1}", (i - 1) >> 1)
            # the row's reference maximum: step i reads what step i-1 published
            got = self.mref.get(wq, -1)
            assert got == i - 1, f"step {i} warp {wg}.{wq}: reference from step {got}"
            if self.mistake == "reference_after_handoff":
                if i + 1 < self.n:
                    self.B[f"xdone{wg}"].arrive(32)
                yield lambda: True
            self.mref[wq] = i
            rescale = i >= 1 and self.rng.random() < self.rescale_prob
            # exponentials, then P over the consumed S columns
            yield lambda: True
            if i + 1 < self.n and self.mistake != "reference_after_handoff":
                self.B[f"xdone{wg}"].arrive(32)
            if rescale and self.mistake != "rescale_without_wait":
                yield from self.wait(f"pvdone{(i - 1) & 1}", (i - 1) >> 1)
            if rescale:
                assert self.pv_done == i - 1, f"O rescaled at step {i} after PV({self.pv_done})"
            assert self.buf[b][wq] == ("S", i), f"P({i}) stored over {self.buf[b][wq]}"
            self.buf[b][wq] = ("P", i)
            self.B[f"pfullwg{wg}" if self.mistake == "p_ready_per_warpgroup" else f"pfull{b}"].arrive(32)
        if self.n > 0:
            yield from self.wait("mmadone", 0)

    # -- the tensor pipe (each issuing thread's MMAs in its issue order; no order between the
    # two threads) and the copy engine, stepped by the scheduler
    def pipe_step(self, probe=False):
        busy = [w for w in (0, 1) if self.pipe[w]]
        if probe or not busy:
            return bool(busy)
        who = self.rng.choice(busy)
        kind, i = self.pipe[who].pop(0)
        b = i % NSBUF
        if kind == "qk":
            assert self.kst[i % KSTAGES] == i, f"QK({i}) read K stage holding {self.kst[i % KSTAGES]}"
            for q in range(4):
                assert self.buf[b][q] is None or self.buf[b][q] == ("P", i - NSBUF) and self.pv_done >= i - NSBUF, \
                    f"QK({i}) overwrote {self.buf[b][q]} before its PV"
            self.buf[b] = [("S", i)] * 4
        else:
            assert self.buf[b] == [("P", i)] * 4, f"PV({i}) read {self.buf[b]}"
            assert self.vst[i % VSTAGES] == i, f"PV({i}) read V stage holding {self.vst[i % VSTAGES]}"
            assert self.pv_done == i - 1, f"PV({i}) after PV({self.pv_done})"
            self.pv_done = i
        self.completed[who] += 1
        keep = []
        for c in self.pending_commits:
            if c[0] == who and c[1] <= self.completed[who]:
                self.B[c[2]].arrive()
            else:
                keep.append(c)
        self.pending_commits = keep
        return True

    def load_step(self, probe=False):
        if probe or not self.loads:
            return bool(self.loads)
        bar, kind, s, i = self.loads.pop(self.rng.randrange(len(self.loads)))
        (self.kst if kind == "k" else self.vst)[s] = i
        self.B[bar].arrive()
        return True

    def commits_without_mmas(self):
        # a commit with nothing outstanding on its thread arrives at once
        keep = []
        for c in self.pending_commits:
            if c[1] <= self.completed[c[0]]:
                self.B[c[2]].arrive()
            else:
                keep.append(c)
        self.pending_commits = keep

    def run(self):
        actors = [self.k_producer(), self.v_producer(), self.issuer(0), self.issuer(1)]
        actors += [self.warp(wg, wq) for wg in (0, 1) for wq in range(4)]
        run_actors(actors, [self.pipe_step, self.load_step], self.rng, before_step=self.commits_without_mmas)


@pytest.mark.parametrize("nsteps", [0, 1, 2, 3, 4, 5, 7, 12, 40])
def test_attend_barrier_protocol_random_schedules(nsteps):
    for seed in range(40):
        rng = random.Random(seed * 1000 + nsteps)
        sim = Sim(nsteps, rng, rescale_prob=0.3)
        sim.run()
        assert sim.pv_done == nsteps - 1
        assert sim.B["mmadone"].done == (1 if nsteps > 0 else 0)


MISTAKES = ["pv_not_ordered", "qk_before_pv", "reference_after_handoff", "rescale_without_wait",
            "p_ready_per_warpgroup", "k_stage_reused_early"]


@pytest.mark.parametrize("mistake", MISTAKES)
def test_attend_protocol_checks_catch_planted_mistakes(mistake):
    """Each planted mistake (PV not ordered by the previous PV's completion, the next QK issued
    before PV, the reference maximum published after the hand-off, O rescaled without waiting for
    PV(i-1), one P-ready barrier per warpgroup instead of per buffer, a K stage reloaded one use
    early) must trip an assertion or deadlock under some schedule."""
    caught = 0
    for nsteps in (4, 7, 12, 40):
        for seed in range(60):
            rng = random.Random(seed * 7919 + nsteps)
            try:
                Sim(nsteps, rng, rescale_prob=0.5, mistake=mistake).run()
            except AssertionError:
                caught += 1
    assert caught > 0, mistake
