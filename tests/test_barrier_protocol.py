"""Randomized model check of the GEMM kernel's mbarrier protocol (CPU).

Every warp role of ``w4a8_gemm_kernel`` (csrc/qoq_gemm.cu) is written here as
a generator that performs the kernel's waits and arrivals in program order:
the X producer, the weight producer, the MMA warp, each warp of each
dequantizing warpgroup, and the four epilogue warps.  The asynchronous parts
are separate events: TMA copies land in any order, and tcgen05 MMA groups
complete in issue order.  A seeded random scheduler interleaves all of it.

What is checked on every run:

* every parity wait for phase k is evaluated only while its barrier has
  completed k or k + 1 phases.  With k - 1 completed the wait would pass
  early; with k + 2 completed it would miss its phase.  (An mbarrier's parity
  test cannot tell these cases apart, which is why the kernel orders its waits
  so that they cannot arise);
* slot ownership: no copy overwrites a slot whose previous stage is still in
  use; every consumer reads the stage it expects; the MMA overwrites an
  accumulator only after the epilogue released it;
* completion: every role finishes, and no copy is still in flight when they
  have all finished.

The ring sizes, warpgroup counts and accumulator counts are those of the
kernel's token tiles.  The model also replays an older dequantizer wait
order (the weight slot tested before the A slot).  That order failed its
bounded waits on the GPU, and the model must catch it.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase."""

    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending = count
        self.completed = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def try_wait(self, k):
        """mbarrier.try_wait.parity for phase k, with the exactness check."""
        c = self.completed
        assert k <= c <= k + 1, f"{self.name}: wait for phase {k} at {c} completed phases"
        return (c & 1) != (k & 1)


class KernelModel:
    def __init__(self, S, G, kAcc, unit_stages, seed, weights_first=False):
        self.S, self.G, self.kAcc = S, G, kAcc
        self.units = unit_stages
        self.rng = random.Random(seed)
        self.weights_first = weights_first
        self.xfull = [Bar(f"xfull{i}", 1) for i in range(S)]
        self.empty = [Bar(f"empty{i}", 1) for i in range(S)]
        self.wfull = [Bar(f"wfull{i}", 1) for i in range(S)]
        self.wempty = [Bar(f"wempty{i}", 4) for i in range(S)]
        self.dqfull = [Bar(f"dqfull{i}", 4) for i in range(S)]
        self.accfull = [Bar(f"accfull{i}", 1) for i in range(kAcc)]
        self.accempty = [Bar(f"accempty{i}", 4) for i in range(kAcc)]
        self.drain = Bar("drain", 1)
        self.xslot = [None] * S
        self.wslot = [None] * S
        self.aslot = [None] * S
        self.acc_unit = [None] * kAcc
        self.w_reads = {}
        self.mma_done = -1
        self.epi_done = {}
        self.tma = []
        self.mma_q = []

    # ------------------------------------------------------------------ roles
    def x_producer(self):
        S, g = self.S, 0
        for n in self.units:
            for _ in range(n):
                s = g % S
                if g >= S:
                    yield ("wait", self.empty[s], g // S - 1)
                    assert self.mma_done >= g - S, "X slot refilled before its MMAs completed"
                self.xslot[s] = ("inflight", g)
                self.tma.append(("x", g))
                g += 1

    def w_producer(self):
        S, g = self.S, 0
        for n in self.units:
            for _ in range(n):
                s = g % S
                if g >= S:
                    yield ("wait", self.wempty[s], g // S - 1)
                    assert self.w_reads.get(g - S, 0) == 4, "weight slot refilled before read"
                self.wslot[s] = ("inflight", g)
                self.tma.append(("w", g))
                g += 1

    def mma(self):
        S, kAcc, g = self.S, self.kAcc, 0
        for lt, n in enumerate(self.units):
            b = lt % kAcc
            if lt >= kAcc:
                yield ("wait", self.accempty[b], lt // kAcc - 1)
                assert self.epi_done.get(lt - kAcc) == 4, "accumulator reused early"
            for _ in range(n):
                s = g % S
                yield ("wait", self.dqfull[s], g // S)
                assert self.xslot[s] == ("landed", g), (g, self.xslot[s])
                assert self.aslot[s] == ("written", g), (g, self.aslot[s])
                self.mma_q.append(("stage", g))
                g += 1
            self.mma_q.append(("acc", lt))
        self.mma_q.append(("drain", None))
        yield ("wait", self.drain, 0)

    def dequant_warp(self, wg, q4):
        S, G, g0 = self.S, self.G, 0
        for n in self.units:
            i = (wg + G - g0 % G) % G          # this warpgroup's first stage of the unit
            while i < n:
                g = g0 + i
                s = g % S
                if self.weights_first:
                    yield ("wait", self.wfull[s], g // S)
                    self.w_reads[g] = self.w_reads.get(g, 0) + 1
                    yield ("arrive", self.wempty[s])
                    if g >= S:
                        yield ("wait", self.empty[s], g // S - 1)
                else:
                    if g >= S:
                        yield ("wait", self.empty[s], g // S - 1)
                    yield ("wait", self.wfull[s], g // S)
                    assert self.wslot[s] == ("landed", g), (g, self.wslot[s])
                    self.w_reads[g] = self.w_reads.get(g, 0) + 1
                    yield ("arrive", self.wempty[s])
                assert g < S or self.mma_done >= g - S, "A slot written before its MMAs completed"
                if q4 == 0:
                    self.aslot[s] = ("writing", g)
                yield ("yield",)
                yield ("wait", self.xfull[s], g // S)
                if q4 == 0:
                    self.aslot[s] = ("written", g)
                yield ("arrive", self.dqfull[s])
                i += G
            g0 += n

    def epilogue_warp(self):
        for lt in range(len(self.units)):
            b = lt % self.kAcc
            yield ("wait", self.accfull[b], lt // self.kAcc)
            assert self.acc_unit[b] == lt, (lt, self.acc_unit[b])
            yield ("yield",)
            self.epi_done[lt] = self.epi_done.get(lt, 0) + 1
            yield ("arrive", self.accempty[b])

    # -------------------------------------------------------------- scheduler
    def complete_one(self):
        kinds = (["tma"] if self.tma else []) + (["mma"] if self.mma_q else [])
        if not kinds:
            return False
        if self.rng.choice(kinds) == "tma":
            kind, g = self.tma.pop(self.rng.randrange(len(self.tma)))
            slots, bars = (self.xslot, self.xfull) if kind == "x" else (self.wslot, self.wfull)
            s = g % self.S
            assert slots[s] == ("inflight", g)
            slots[s] = ("landed", g)
            bars[s].arrive()
        else:
            kind, v = self.mma_q.pop(0)
            if kind == "stage":
                self.mma_done = v
                self.empty[v % self.S].arrive()
            elif kind == "acc":
                self.acc_unit[v % self.kAcc] = v
                self.accfull[v % self.kAcc].arrive()
            else:
                self.drain.arrive()
        return True

    def run(self):
        gens = {"xp": self.x_producer(), "wp": self.w_producer(), "mma": self.mma()}
        for wg in range(self.G):
            for q4 in range(4):
                gens[f"dq{wg}.{q4}"] = self.dequant_warp(wg, q4)
        for ew in range(4):
            gens[f"epi{ew}"] = self.epilogue_warp()
        waiting = {name: None for name in gens}
        live = set(gens)
        for _ in range(2_000_000):
            if not live:
                break
            runnable = [n for n in sorted(live)
                        if waiting[n] is None or waiting[n][1].try_wait(waiting[n][2])]
            if not runnable or (self.rng.random() < 0.3 and (self.tma or self.mma_q)):
                if not self.complete_one():
                    assert runnable, f"deadlock: {[(n, waiting[n][1].name) for n in live]}"
                continue
            name = self.rng.choice(runnable)
            waiting[name] = None
            try:
                op = next(gens[name])
            except StopIteration:
                live.discard(name)
                continue
            if op[0] == "wait":
                waiting[name] = op
            elif op[0] == "arrive":
                op[1].arrive()
        assert not live, "no progress"
        # every copy was consumed: nothing is in flight once all roles finished
        assert not self.tma and not self.mma_q


# (X/weight ring stages S, dequantizing warpgroups G, accumulators) per token tile
KERNEL_CONFIGS = {16: (7, 4, 2), 32: (7, 4, 2), 64: (6, 4, 2), 128: (4, 3, 2),
                  176: (5, 3, 2), 192: (4, 3, 2), 256: (4, 3, 1)}


@pytest.mark.parametrize("tok", sorted(KERNEL_CONFIGS))
def test_protocol_is_exact_for_every_token_tile(tok):
    S, G, kAcc = KERNEL_CONFIGS[tok]
    assert S >= G       # the condition under which the A-slot wait is exact
    for seed in range(60):
        rng = random.Random(tok * 1000 + seed)
        units = [rng.randint(1, 3 * S) for _ in range(rng.randint(1, 5))]
        KernelModel(S, G, kAcc, units, seed).run()


def test_model_catches_the_older_wait_order():
    caught = 0
    for seed in range(200):
        rng = random.Random(seed)
        units = [rng.randint(1, 9) for _ in range(rng.randint(1, 6))]
        try:
            KernelModel(4, 3, 2, units, seed, weights_first=True).run()
        except AssertionError:
            caught += 1
    assert caught > 0


def test_model_catches_fewer_stages_than_warpgroups():
    caught = 0
    for seed in range(200):
        rng = random.Random(seed)
        units = [rng.randint(4, 12) for _ in range(rng.randint(1, 4))]
        try:
            KernelModel(2, 3, 2, units, seed).run()
        except AssertionError:
            caught += 1
    assert caught > 0
