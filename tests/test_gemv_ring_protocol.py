"""Randomized model check of the decode GEMV's copy-ring protocol (CPU).

One warp of ``w4a8_gemv_kernel`` (csrc/qoq_gemv.cu) streams its k-tiles
through a ring of S shared-memory slots.  Per k-tile every lane copies its own
row's code chunks into the slot, and lanes 0 .. 3 gpt - 1 copy the group
scales and zero points that every lane reads.  Each lane commits one
``cp.async`` group per k-tile index (empty past the warp's last k-tile), and
before reading k-tile i it waits until at most S - 1 of its groups are pending,
then meets the other lanes at a warp barrier; after reading it meets them
again before it refills the slot with k-tile i + S.

Here every lane is a generator that performs those steps in program order,
each copy is a separate event that lands at a random later time, and a seeded
random scheduler interleaves it all.  What is checked on every run:

* every read of a slot sees the k-tile it expects: its own code chunk and all
  of the shared scale parts (neither a stale k-tile nor a refill);
* visibility: a lane reads another lane's copy only if that lane had waited
  for the copy's group before a warp barrier the reader has since passed
  (``cp.async.wait_group`` makes a copy visible to the issuing thread;
  ``__syncwarp`` orders it for the others);
* completion: after the final ``wait_group 0`` no copy is still in flight.

Mutant protocols (the wait allowing S pending groups, either warp barrier
left out) must each fail on some seed.
"""
import random

import pytest


def lane_program(lane, S, n, gpt, variant):
    """The kernel's per-lane sequence of copy-ring operations."""
    for i in range(S):
        yield ("issue", i)
    for i in range(n):
        yield ("wait", S if variant == "wait_S" else S - 1)
        if variant != "no_sync1":
            yield ("sync",)
        yield ("read", i)
        if variant != "no_sync2":
            yield ("sync",)
        yield ("issue", i + S)
    yield ("wait", 0)


class RingModel:
    def __init__(self, S, n, gpt, lanes, rng, variant="ok"):
        assert lanes >= 3 * gpt
        self.S, self.n, self.gpt, self.lanes, self.rng = S, n, gpt, lanes, rng
        self.codes = [[None] * lanes for _ in range(S)]        # slot -> lane -> k-tile
        self.scales = [[None] * (3 * gpt) for _ in range(S)]   # slot -> part -> k-tile
        self.inflight = []                 # (lane, group, kind, index, slot, k-tile)
        self.committed = [0] * lanes
        self.pending = [dict() for _ in range(lanes)]          # group -> copies in flight
        self.acquired = {}                 # (lane, group) -> warp barriers passed at the wait
        self.synced = [0] * lanes          # warp barriers passed
        self.at_sync = set()
        self.progs = [lane_program(l, S, n, gpt, variant) for l in range(lanes)]
        self.op = [next(p) for p in self.progs]
        self.done = [False] * lanes

    # ---- lane operations -------------------------------------------------
    def issue(self, lane, j):
        g = self.committed[lane]
        assert g == j, "one commit group per k-tile index"
        if j < self.n:
            slot = j % self.S
            copies = [("code", lane)]
            if lane < 3 * self.gpt:
                copies.append(("scale", lane))
            for kind, idx in copies:
                self.inflight.append((lane, g, kind, idx, slot, j))
            self.pending[lane][g] = len(copies)
        self.committed[lane] += 1

    def wait_ready(self, lane, N):
        older = self.committed[lane] - N
        return all(self.pending[lane].get(g, 0) == 0 for g in range(older))

    def wait(self, lane, N):
        for g in range(self.committed[lane] - N):
            self.acquired.setdefault((lane, g), self.synced[lane])

    def read(self, lane, i):
        slot = i % self.S
        assert self.codes[slot][lane] == i, (
            f"lane {lane} read code k-tile {self.codes[slot][lane]} for {i}")
        assert (lane, i) in self.acquired, "own copy read before its wait"
        for part in range(3 * self.gpt):
            got = self.scales[slot][part]
            assert got == i, f"lane {lane} read scale part {part} of k-tile {got} for {i}"
            writer = part
            acq = self.acquired.get((writer, i))
            assert acq is not None and self.synced[lane] > acq, (
                f"lane {lane} read lane {writer}'s copy of k-tile {i} without ordering")

    # ---- scheduler -------------------------------------------------------
    def land(self, k):
        lane, g, kind, idx, slot, j = self.inflight.pop(k)
        if kind == "code":
            self.codes[slot][idx] = j
        else:
            self.scales[slot][idx] = j
        self.pending[lane][g] -= 1

    def runnable(self, lane):
        if self.done[lane]:
            return False
        op = self.op[lane]
        if op[0] == "wait":
            return self.wait_ready(lane, op[1])
        if op[0] == "sync":
            return lane not in self.at_sync
        return True

    def step_lane(self, lane):
        op = self.op[lane]
        if op[0] == "issue":
            self.issue(lane, op[1])
        elif op[0] == "wait":
            self.wait(lane, op[1])
        elif op[0] == "read":
            self.read(lane, op[1])
        elif op[0] == "sync":
            self.at_sync.add(lane)
            live = {l for l in range(self.lanes) if not self.done[l]}
            if self.at_sync >= live:
                for l in self.at_sync:
                    self.synced[l] += 1
                    self.advance(l)
                self.at_sync = set()
            return
        self.advance(lane)

    def advance(self, lane):
        try:
            self.op[lane] = next(self.progs[lane])
        except StopIteration:
            self.done[lane] = True

    def run(self, max_steps=200000):
        for _ in range(max_steps):
            if all(self.done):
                assert not self.inflight, "copies still in flight at the end"
                return
            lanes = [l for l in range(self.lanes) if self.runnable(l)]
            # land copies lazily so that early reads and late refills are tried
            if self.inflight and (not lanes or self.rng.random() < 0.3):
                self.land(self.rng.randrange(len(self.inflight)))
                continue
            assert lanes, "deadlock: no lane can run and no copy is in flight"
            self.step_lane(self.rng.choice(lanes))
        raise AssertionError("model did not finish")


CASES = [(S, n, gpt) for S in (2, 4) for n in (0, 1, 2, 3, 5, 9) for gpt in (1, 2)]


@pytest.mark.parametrize("S,n,gpt", CASES, ids=[f"S{s}_n{n}_gpt{g}" for s, n, g in CASES])
def test_ring_protocol_holds(S, n, gpt):
    for seed in range(40):
        RingModel(S, n, gpt, lanes=8, rng=random.Random(seed * 1000 + S * 10 + n)).run()


@pytest.mark.parametrize("variant", ["wait_S", "no_sync1", "no_sync2"])
def test_mutant_protocols_fail(variant):
    failures = 0
    for seed in range(200):
        try:
            RingModel(2, 6, 2, lanes=8, rng=random.Random(seed), variant=variant).run()
        except AssertionError:
            failures += 1
    assert failures > 0, f"the {variant} protocol was never caught"
