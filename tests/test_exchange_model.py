"""A model check of the cross-rank exchange protocol of the branch-sharded
up-projection, on the CPU.

The protocol (as the kernel runs it): each rank owns a region with a call
counter per tile and two buffers of 64-bit words [2][world][tiles].  For a
call, each tile of each rank reads its counter c (and advances it), stores
its value tagged c + 1 into slot `rank` of buffer c & 1 of EVERY rank's
region (one single-copy-atomic word per store), then reads slot src of
buffer c & 1 of its OWN region for every src, waiting while the tag is not
c + 1, and adds the values in rank order.  On one rank, a call's tiles run in
any interleaving, and the next call starts only when all of them are done
(kernels on one stream); ranks run independently.

The model runs every step (one store, one poll) as an atomic action and
picks the next action at random among the runnable ones.  Checked over many
schedules: every rank's result of every call is the sum of all ranks' values
of that call, and the protocol never deadlocks.  A planted mistake -- one
buffer instead of two -- must be caught (a fast rank's next-call word
overwrites a word a slow rank has not read yet, so the slow rank waits for a
tag that never comes).
"""
import random

import pytest


class Model:
    def __init__(self, world, tiles, calls, buffers, seed):
        self.world, self.tiles, self.calls, self.buffers = world, tiles, calls, buffers
        self.rng = random.Random(seed)
        # region of rank p: epoch[t], data[buffer][src][t] = (value, tag)
        self.epoch = [[0] * tiles for _ in range(world)]
        self.data = [[[[(0, 0)] * tiles for _ in range(world)] for _ in range(buffers)] for _ in range(world)]
        self.value = {(r, e, t): self.rng.randint(-1000, 1000)
                      for r in range(world) for e in range(calls) for t in range(tiles)}
        self.result = {}
        self.launch = [0] * world  # call each rank's current launch runs
        # per (rank, tile): program counter within the current launch
        self.pc = [[None] * tiles for _ in range(world)]
        for r in range(world):
            self._start_launch(r)

    def _start_launch(self, r):
        if self.launch[r] < self.calls:
            for t in range(self.tiles):
                self.pc[r][t] = {"phase": "read", "call": None, "push": 0, "src": 0, "acc": 0}

    def _buf(self, call):
        return call % self.buffers

    def runnable(self):
        out = []
        for r in range(self.world):
            for t in range(self.tiles):
                st = self.pc[r][t]
                if st is None or st["phase"] == "done":
                    continue
                if st["phase"] == "wait":
                    v, tag = self.data[r][self._buf(st["call"])][st["src"]][t]
                    if tag != st["call"] + 1:
                        continue  # the poll would fail: not a step that makes progress
                out.append((r, t))
        return out

    def step(self, r, t):
        st = self.pc[r][t]
        if st["phase"] == "read":
            st["call"] = self.epoch[r][t]
            self.epoch[r][t] = st["call"] + 1
            st["phase"] = "push"
        elif st["phase"] == "push":
            p = st["push"]
            e = st["call"]
            self.data[p][self._buf(e)][r][t] = (self.value[(r, e, t)], e + 1)
            st["push"] += 1
            if st["push"] == self.world:
                st["phase"] = "wait"
        elif st["phase"] == "wait":
            v, tag = self.data[r][self._buf(st["call"])][st["src"]][t]
            assert tag == st["call"] + 1
            st["acc"] += v
            st["src"] += 1
            if st["src"] == self.world:
                self.result[(r, st["call"], t)] = st["acc"]
                st["phase"] = "done"
        # a launch ends when all its tiles are done; the next one may start
        if all(s is not None and s["phase"] == "done" for s in self.pc[r]):
            self.launch[r] += 1
            self.pc[r] = [None] * self.tiles
            self._start_launch(r)

    def run(self, max_steps=100000):
        for _ in range(max_steps):
            live = self.runnable()
            if not live:
                finished = all(self.launch[r] == self.calls for r in range(self.world))
                return "done" if finished else "deadlock"
            self.step(*self.rng.choice(live))
        return "too long"


@pytest.mark.parametrize("world,tiles", [(2, 1), (2, 3), (4, 2), (8, 1)])
def test_double_buffered_exchange_is_exact_and_never_deadlocks(world, tiles):
    for seed in range(150):
        m = Model(world, tiles, calls=5, buffers=2, seed=seed)
        assert m.run() == "done", seed
        for e in range(5):
            for t in range(tiles):
                want = sum(m.value[(r, e, t)] for r in range(world))
                for r in range(world):
                    assert m.result[(r, e, t)] == want, (seed, r, e, t)


def test_a_single_buffer_is_caught():
    outcomes = set()
    for seed in range(300):
        m = Model(2, 2, calls=5, buffers=1, seed=seed)
        status = m.run()
        if status == "done":
            for (r, e, t), got in m.result.items():
                if got != sum(m.value[(s, e, t)] for s in range(2)):
                    status = "wrong"
        outcomes.add(status)
    assert outcomes & {"deadlock", "wrong"}, outcomes
