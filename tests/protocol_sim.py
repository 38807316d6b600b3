"""Discrete-event engine for the barrier-protocol models of the CUDA kernels (CPU only).

Roles are Python generators that yield commands: ("wait", barrier, phase) waits for an
explicit phase of an mbarrier to complete, ("delay", cycles) models work, and
("turn", value) waits for a shared turn counter.  The engine checks the parity rule
every kernel wait relies on: a waiter may target the barrier's current phase or the
one just completed, never a phase that has already come round again (a parity wait
two phases behind would wait forever or pass early).  The tensor pipe executes MMA
groups in issue order; a commit completes once every group issued before it is done.
"""

import heapq
import random


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, sim, name, count):
        self.sim, self.name, self.count = sim, name, count
        self.pending = count
        self.completions = 0
        self.waiters = []  # (agent, phase)

    def arrive(self, n=1):
        self.pending -= n
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: more arrivals than the count in one phase")
        if self.pending == 0:
            self.completions += 1
            self.pending = self.count
            woken, self.waiters = self.waiters, []
            for agent, phase in woken:
                self.sim.wait_on(agent, self, phase)


class Engine:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.t = 0
        self.q = []
        self.seq = 0
        self.turn = 0
        self.turn_waiters = []
        self.pipe_free_at = 0
        self.readers = {}  # buffer -> completion time of the last MMA reading it
        self.waiting = {}  # agent -> (barrier, phase) of its last wait
        self.done = set()
        self.agents = {}

    def barrier(self, name, count):
        return Barrier(self, name, count)

    # -- scheduling -------------------------------------------------------------------
    def at(self, t, agent, value=None):
        self.seq += 1
        heapq.heappush(self.q, (t, self.seq, agent, value))

    def wait_on(self, agent, bar, phase):
        self.waiting[agent] = (bar, phase)
        if bar.completions >= phase + 2:
            raise ProtocolError(f"{bar.name}: waiter {agent} targets phase {phase}, "
                                f"but {bar.completions} phases have completed")
        if bar.completions >= phase + 1:
            self.at(self.t + self.rng.randint(1, 20), agent)
        else:
            bar.waiters.append((agent, phase))

    def later(self, dt, fn):
        self.seq += 1
        heapq.heappush(self.q, (self.t + dt, self.seq, None, fn))

    # -- tensor pipe and copies -------------------------------------------------------
    def mma(self, duration, reads=()):
        start = max(self.t, self.pipe_free_at)
        self.pipe_free_at = start + duration
        for buf in reads:
            self.readers[buf] = max(self.readers.get(buf, 0), self.pipe_free_at)
        return self.pipe_free_at

    def commit(self, bar):
        done = max(self.t, self.pipe_free_at)
        self.later(done - self.t + 1, lambda: bar.arrive())

    def tma(self, bar, buf, lo=200, hi=3000):
        if self.readers.get(buf, 0) > self.t:
            raise ProtocolError(f"{buf} refilled at {self.t} while an MMA reads it until {self.readers[buf]}")
        self.later(self.rng.randint(lo, hi), lambda: bar.arrive())

    def pass_turn(self, value):
        self.turn = value
        keep = []
        for agent, want in self.turn_waiters:
            if want == value:
                self.at(self.t + 1, agent)
            else:
                keep.append((agent, want))
        self.turn_waiters = keep

    def run(self, agents, limit=10 ** 9):
        self.agents = agents
        for name in self.agents:
            self.at(0, name)
        while self.q:
            t, _, agent, value = heapq.heappop(self.q)
            self.t = t
            if t > limit:
                break
            if agent is None:
                value()
                continue
            gen = self.agents[agent]
            if agent in self.waiting:
                bar, phase = self.waiting.pop(agent)
                if bar.completions != phase + 1:  # a poll here would see the wrong parity
                    raise ProtocolError(f"{bar.name}: {agent} resumes for phase {phase} after "
                                        f"{bar.completions} completions")
            try:
                cmd = next(gen)
            except StopIteration:
                self.done.add(agent)
                continue
            kind = cmd[0]
            if kind == "wait":
                self.wait_on(agent, cmd[1], cmd[2])
            elif kind == "delay":
                self.at(self.t + cmd[1], agent)
            elif kind == "turn":
                if self.turn == cmd[1]:
                    self.at(self.t + 1, agent)
                else:
                    self.turn_waiters.append((agent, cmd[1]))
        if len(self.done) != len(self.agents):
            stuck = sorted(set(self.agents) - self.done)
            raise ProtocolError(f"deadlock: {stuck} never finished")
