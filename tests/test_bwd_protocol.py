"""The barrier protocol of the backward's dK/dV pass (attend_bwd.cu, bwd_dkdv_kernel), checked by
randomized interleavings on the CPU.

Roles, as in the kernel: one producer thread loads the CTA's K, V pair once and then Q, dO and
the query block's log-sum-exp and D rows of each step into a ring of three stages; one issuing
thread puts S^T = K Q^T and dP^T = V dO^T of step j into TMEM buffer j mod 2 once the dV/dK
products of step j-2 have freed it; a second issuing thread accumulates dV += P^T dO and
dK += dS^T Q of every step in order, then releases the step's stage and buffer; the two
warpgroups (four independently scheduled warps each) take alternate steps, read the stage's
log-sum-exp and D rows and S^T, dP^T, and store P^T, dS^T over them.  The model asserts that
every parity wait lands on its intended phase, that every read finds the expected step in the
stage or buffer it reads, that dV and dK accumulate in step order, and that nothing deadlocks;
three planted protocol mistakes must each be caught.  It models the protocol, not the
arithmetic; the GPU parity tests cover the arithmetic.
"""
import random

import pytest

from tests._protocol import Bar, run_actors, wait_for, wait_released

QST = 3   # query-block stages (Q, dO, log-sum-exp and D rows)


class DkdvSim:
    def __init__(self, nsteps, rng, mistake=None):
        self.n, self.rng, self.mistake = nsteps, rng, mistake
        self.B = {"kvfull": Bar("kvfull", 1), "mmadone": Bar("mmadone", 2)}
        for s in range(QST):
            self.B[f"qfull{s}"], self.B[f"qempty{s}"] = Bar(f"qfull{s}", 1), Bar(f"qempty{s}", 1)
        for b in range(2):
            self.B[f"sfull{b}"], self.B[f"bfree{b}"] = Bar(f"sfull{b}", 1), Bar(f"bfree{b}", 1)
            self.B[f"pfull{b}"] = Bar(f"pfull{b}", 128)
        self.stage = [None] * QST                    # which step's Q, dO and rows a stage holds
        self.buf = [[None] * 4 for _ in range(2)]    # per buffer and lane quadrant: ("S"|"P", j)
        self.kv_loaded = False
        self.dkdv_done = -1                          # last step whose dV/dK products ran
        self.pipe = {"s": [], "d": []}               # each issuing thread's MMAs, in order
        self.issued = {"s": 0, "d": 0}
        self.completed = {"s": 0, "d": 0}
        self.commits = []                            # (thread, batches before the commit, barrier)
        self.loads = []                              # in flight: (barrier, what, stage, step)

    def commit(self, who, bar):
        self.commits.append((who, self.issued[who], bar))

    def flush_commits(self):
        keep = []
        for c in self.commits:
            if c[1] <= self.completed[c[0]]:
                self.B[c[2]].arrive()
            else:
                keep.append(c)
        self.commits = keep

    # -- actors
    def producer(self):
        if self.n == 0:
            return
        self.loads.append(("kvfull", "kv", None, None))
        for j in range(self.n):
            s = j % QST
            yield from wait_released(self.B[f"qempty{s}"], j // QST)
            self.loads.append((f"qfull{s}", "q", s, j))

    def issuer_s(self):
        if self.n == 0:
            return
        yield from wait_for(self.B["kvfull"], 0)
        for j in range(self.n):
            b = j & 1
            if j >= 2 and self.mistake != "s_before_buffer_free":
                yield from wait_for(self.B[f"bfree{b}"], (j - 2) >> 1)
            yield from wait_for(self.B[f"qfull{j % QST}"], j // QST)
            self.pipe["s"].append(("st", j))
            self.issued["s"] += 1
            self.commit("s", f"sfull{b}")
        self.commit("s", "mmadone")

    def issuer_d(self):
        if self.n == 0:
            return
        for j in range(self.n):
            b, s = j & 1, j % QST
            yield from wait_for(self.B[f"pfull{b}"], j >> 1)
            if self.mistake == "stage_released_before_dkdv":
                self.B[f"qempty{s}"].arrive()
            self.pipe["d"].append(("dkdv", j))
            self.issued["d"] += 1
            if self.mistake != "stage_released_before_dkdv":
                self.commit("d", f"qempty{s}")
            self.commit("d", f"bfree{b}")
        self.commit("d", "mmadone")

    def warp(self, wg, wq):
        for j in range(wg, self.n, 2):
            s, b = j % QST, j & 1
            # (For ordering alone this wait is implied by the S-full wait below; the kernel keeps
            # it because it is what makes the stage's TMA-written rows visible to these threads.)
            yield from wait_for(self.B[f"qfull{s}"], j // QST)
            yield from wait_for(self.B[f"sfull{b}"], j >> 1)
            assert self.buf[b][wq] == ("S", j), f"step {j}: buffer {b} rows {wq} hold {self.buf[b][wq]}"
            assert self.stage[s] == j, f"step {j}: log-sum-exp and D rows from stage holding {self.stage[s]}"
            yield lambda: True                       # P^T and dS^T formed
            assert self.stage[s] == j, f"step {j}: stage {s} reloaded during the formation"
            self.buf[b][wq] = ("P", j)
            if self.mistake == "p_ready_from_one_warp":
                if wq == 0:
                    self.B[f"pfull{b}"].arrive(128)
            else:
                self.B[f"pfull{b}"].arrive(32)
        if self.n > 0:
            yield from wait_for(self.B["mmadone"], 0)

    # -- engines
    def pipe_step(self, probe=False):
        busy = [w for w in ("s", "d") if self.pipe[w]]
        if probe or not busy:
            return bool(busy)
        who = self.rng.choice(busy)
        kind, j = self.pipe[who].pop(0)
        b, s = j & 1, j % QST
        assert self.stage[s] == j, f"{kind}({j}) read stage {s} holding {self.stage[s]}"
        if kind == "st":
            assert self.kv_loaded
            for q in range(4):
                prev = self.buf[b][q]
                assert prev is None or (prev == ("P", j - 2) and self.dkdv_done >= j - 2), \
                    f"S^T({j}) overwrote {prev} before its dV/dK"
            self.buf[b] = [("S", j)] * 4
        else:
            assert self.buf[b] == [("P", j)] * 4, f"dV/dK({j}) read {self.buf[b]}"
            assert self.dkdv_done == j - 1, f"dV/dK({j}) after dV/dK({self.dkdv_done})"
            self.dkdv_done = j
        self.completed[who] += 1
        return True

    def load_step(self, probe=False):
        if probe or not self.loads:
            return bool(self.loads)
        bar, what, s, j = self.loads.pop(self.rng.randrange(len(self.loads)))
        if what == "kv":
            self.kv_loaded = True
        else:
            self.stage[s] = j
        self.B[bar].arrive()
        return True

    def run(self):
        actors = [self.producer(), self.issuer_s(), self.issuer_d()]
        actors += [self.warp(wg, wq) for wg in (0, 1) for wq in range(4)]
        run_actors(actors, [self.pipe_step, self.load_step], self.rng, before_step=self.flush_commits)


@pytest.mark.parametrize("nsteps", [0, 1, 2, 3, 4, 5, 8, 13, 40])
def test_dkdv_barrier_protocol_random_schedules(nsteps):
    for seed in range(40):
        sim = DkdvSim(nsteps, random.Random(seed * 1000 + nsteps))
        sim.run()
        assert sim.dkdv_done == nsteps - 1
        assert sim.B["mmadone"].done == (1 if nsteps > 0 else 0)


MISTAKES = ["s_before_buffer_free", "stage_released_before_dkdv", "p_ready_from_one_warp"]


@pytest.mark.parametrize("mistake", MISTAKES)
def test_dkdv_protocol_checks_catch_planted_mistakes(mistake):
    """S^T/dP^T issued without waiting for the buffer's dV/dK, a stage released before the dV/dK
    products that read it have run, and a P-ready barrier completed by one warp's arrivals
    instead of all four warps': each must trip an assertion or deadlock under some schedule."""
    caught = 0
    for nsteps in (4, 8, 13, 40):
        for seed in range(60):
            try:
                DkdvSim(nsteps, random.Random(seed * 7919 + nsteps), mistake=mistake).run()
            except AssertionError:
                caught += 1
    assert caught > 0, mistake
