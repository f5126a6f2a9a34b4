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
    """One CTA of the kernel.  ``abort_prob`` > 0 lets a blocked wait give up
    at random (the kernel's bounded wait running out): the role raises the
    CTA's abort flag, and from then on every wait that is not already
    satisfied gives up too, as the kernel's waits do when they see the flag.
    The producers' final drains wait regardless of the flag."""

    def __init__(self, S, G, kAcc, unit_stages, seed, weights_first=False, SW=None,
                 abort_prob=0.0):
        SW = S if SW is None else SW
        self.S, self.SW, self.G, self.kAcc = S, SW, G, kAcc
        self.units = unit_stages
        self.rng = random.Random(seed)
        self.weights_first = weights_first
        self.abort_prob = abort_prob
        self.aborted = False
        self.xfull = [Bar(f"xfull{i}", 1) for i in range(S)]
        self.empty = [Bar(f"empty{i}", 1) for i in range(S)]
        self.wfull = [Bar(f"wfull{i}", 1) for i in range(SW)]
        self.wempty = [Bar(f"wempty{i}", 4) for i in range(SW)]
        self.dqfull = [Bar(f"dqfull{i}", 4) for i in range(S)]
        self.accfull = [Bar(f"accfull{i}", 1) for i in range(kAcc)]
        self.accempty = [Bar(f"accempty{i}", 4) for i in range(kAcc)]
        self.drain = Bar("drain", 1)
        self.xslot = [None] * S
        self.wslot = [None] * SW
        self.aslot = [None] * S
        self.acc_unit = [None] * kAcc
        self.w_reads = {}
        self.mma_done = -1
        self.epi_done = {}
        self.tma = []
        self.mma_q = []

    # ------------------------------------------------------------------ roles
    # A role yields ("wait", bar, phase) and receives True (the phase
    # completed) or False (the wait gave up); ("drain", bar, phase) always
    # returns once the phase completed.
    def x_producer(self):
        S, g = self.S, 0
        ok = True
        for n in self.units:
            for _ in range(n):
                s = g % S
                if g >= S:
                    ok = yield ("wait", self.empty[s], g // S - 1)
                    if not ok:
                        break
                    assert self.mma_done >= g - S, "X slot refilled before its MMAs completed"
                self.xslot[s] = ("inflight", g)
                self.tma.append(("x", g))
                g += 1
            if not ok:
                break
        # every copy issued lands before the CTA exits
        for j in range(max(0, g - S), g):
            yield ("drain", self.xfull[j % S], j // S)

    def w_producer(self):
        SW, g = self.SW, 0
        ok = True
        for n in self.units:
            for _ in range(n):
                s = g % SW
                if g >= SW:
                    ok = yield ("wait", self.wempty[s], g // SW - 1)
                    if not ok:
                        break
                    assert self.w_reads.get(g - SW, 0) == 4, "weight slot refilled before read"
                self.wslot[s] = ("inflight", g)
                self.tma.append(("w", g))
                g += 1
            if not ok:
                break
        for j in range(max(0, g - SW), g):
            yield ("drain", self.wfull[j % SW], j // SW)

    def mma(self):
        S, kAcc, g = self.S, self.kAcc, 0
        for lt, n in enumerate(self.units):
            b = lt % kAcc
            if lt >= kAcc:
                if not (yield ("wait", self.accempty[b], lt // kAcc - 1)):
                    break
                assert self.epi_done.get(lt - kAcc) == 4, "accumulator reused early"
            ok = True
            for _ in range(n):
                s = g % S
                ok = yield ("wait", self.dqfull[s], g // S)
                if not ok:
                    break
                assert self.xslot[s] == ("landed", g), (g, self.xslot[s])
                assert self.aslot[s] == ("written", g), (g, self.aslot[s])
                self.mma_q.append(("stage", g))
                g += 1
            if not ok:
                break
            self.mma_q.append(("acc", lt))
        self.mma_q.append(("drain", None))
        yield ("drain", self.drain, 0)

    def dequant_warp(self, wg, q4):
        S, SW, G, g0 = self.S, self.SW, self.G, 0
        for n in self.units:
            i = (wg + G - g0 % G) % G          # this warpgroup's first stage of the unit
            while i < n:
                g = g0 + i
                s, sw = g % S, g % SW
                if self.weights_first:
                    if not (yield ("wait", self.wfull[sw], g // SW)):
                        return
                    self.w_reads[g] = self.w_reads.get(g, 0) + 1
                    yield ("arrive", self.wempty[sw])
                    if g >= S and not (yield ("wait", self.empty[s], g // S - 1)):
                        return
                else:
                    if g >= S and not (yield ("wait", self.empty[s], g // S - 1)):
                        return
                    if not (yield ("wait", self.wfull[sw], g // SW)):
                        return
                    assert self.wslot[sw] == ("landed", g), (g, self.wslot[sw])
                    self.w_reads[g] = self.w_reads.get(g, 0) + 1
                    yield ("arrive", self.wempty[sw])
                assert g < S or self.mma_done >= g - S, "A slot written before its MMAs completed"
                if q4 == 0:
                    self.aslot[s] = ("writing", g)
                yield ("yield",)
                if not (yield ("wait", self.xfull[s], g // S)):
                    return
                if q4 == 0:
                    self.aslot[s] = ("written", g)
                yield ("arrive", self.dqfull[s])
                i += G
            g0 += n

    def epilogue_warp(self):
        for lt in range(len(self.units)):
            b = lt % self.kAcc
            if not (yield ("wait", self.accfull[b], lt // self.kAcc)):
                return
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
            if kind == "x":
                slots, bars, s = self.xslot, self.xfull, g % self.S
            else:
                slots, bars, s = self.wslot, self.wfull, g % self.SW
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
        reply = {name: None for name in gens}
        live = set(gens)
        for _ in range(2_000_000):
            if not live:
                break
            runnable = []
            for n in sorted(live):
                w = waiting[n]
                if w is None:
                    runnable.append(n)
                elif w[1].try_wait(w[2]):
                    reply[n] = True
                    runnable.append(n)
                elif w[0] == "wait" and (self.aborted or self.rng.random() < self.abort_prob):
                    # the bounded wait gives up: the CTA's abort flag is raised
                    self.aborted = True
                    reply[n] = False
                    runnable.append(n)
            if not runnable or (self.rng.random() < 0.3 and (self.tma or self.mma_q)):
                if not self.complete_one():
                    assert runnable, f"deadlock: {[(n, waiting[n][1].name) for n in live]}"
                continue
            name = self.rng.choice(runnable)
            waiting[name] = None
            try:
                op = gens[name].send(reply[name])
            except StopIteration:
                live.discard(name)
                continue
            reply[name] = None
            if op[0] in ("wait", "drain"):
                waiting[name] = op
            elif op[0] == "arrive":
                op[1].arrive()
        assert not live, "no progress"
        # every copy and every MMA group has completed once all roles finished
        # (the CTA's teardown): nothing lands in shared or tensor memory later
        assert not self.tma and not self.mma_q, (self.tma, self.mma_q)


# (X ring stages S, weight ring stages SW, dequantizing warpgroups G,
# accumulators) per token tile
KERNEL_CONFIGS = {16: (7, 7, 4, 2), 32: (7, 7, 4, 2), 64: (6, 6, 4, 2), 128: (4, 5, 3, 2),
                  176: (5, 10, 3, 2), 192: (4, 10, 3, 2), 256: (4, 8, 3, 1)}


@pytest.mark.parametrize("tok", sorted(KERNEL_CONFIGS))
def test_protocol_is_exact_for_every_token_tile(tok):
    S, SW, G, kAcc = KERNEL_CONFIGS[tok]
    assert S >= G       # the condition under which the A-slot wait is exact
    assert SW >= S      # the weight slot's older phase belongs to a stage <= g - S
    for seed in range(60):
        rng = random.Random(tok * 1000 + seed)
        units = [rng.randint(1, 3 * SW) for _ in range(rng.randint(1, 5))]
        KernelModel(S, G, kAcc, units, seed, SW=SW).run()


@pytest.mark.parametrize("tok", sorted(KERNEL_CONFIGS))
def test_abort_at_any_wait_leaves_nothing_in_flight(tok):
    """Any role's wait may give up at any point; every role then leaves its
    loop, the producers drain the copies they issued, the MMA warp drains its
    MMAs, and at teardown no copy or MMA is still in flight.  Every parity
    wait stays exact on the way."""
    S, SW, G, kAcc = KERNEL_CONFIGS[tok]
    aborted = 0
    for seed in range(80):
        rng = random.Random(tok * 7919 + seed)
        units = [rng.randint(1, 3 * SW) for _ in range(rng.randint(1, 5))]
        m = KernelModel(S, G, kAcc, units, seed, SW=SW, abort_prob=0.02)
        m.run()
        aborted += m.aborted
    assert aborted > 10     # the aborts were exercised


def test_model_catches_a_producer_that_does_not_drain():
    """Without the producers' final drain (the older kernel drained only when
    the producer itself gave up), an abort elsewhere can end the CTA with
    copies still landing."""
    class NoDrain(KernelModel):
        def x_producer(self):
            S, g = self.S, 0
            for n in self.units:
                for _ in range(n):
                    s = g % S
                    if g >= S:
                        if not (yield ("wait", self.empty[s], g // S - 1)):
                            for j in range(max(0, g - S), g):
                                yield ("drain", self.xfull[j % S], j // S)
                            return
                    self.xslot[s] = ("inflight", g)
                    self.tma.append(("x", g))
                    g += 1
    caught = 0
    for seed in range(300):
        rng = random.Random(seed)
        units = [rng.randint(1, 6) for _ in range(rng.randint(1, 3))]
        try:
            NoDrain(4, 3, 2, units, seed, abort_prob=0.05).run()
        except AssertionError:
            caught += 1
    assert caught > 0


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


class ClusterReductionModel:
    """The K split across a cluster: per unit, every non-leader CTA's
    epilogue warp q waits for red_free[q] (its own barrier, phase lt - 1),
    writes its INT32 slice into the leader's buffer slot and arrives on the
    leader's red_full[q] (count cs - 1); the leader's warp q waits for
    red_full[q] (phase lt), adds the slots up and, if a unit follows, arrives
    on every non-leader's red_free[q].  Checks parity exactness, that no slot
    is overwritten before the leader consumed it, that the leader reads every
    slot of the right unit, and that nothing is left pending at the end."""

    def __init__(self, cs, units, seed):
        self.cs, self.units = cs, units
        self.rng = random.Random(seed)
        self.red_full = [Bar(f"red_full{q}", cs - 1) for q in range(4)]
        self.red_free = {(r, q): Bar(f"red_free{r}.{q}", 1) for r in range(1, cs) for q in range(4)}
        self.slot = {}          # (r, q) -> unit whose slice the slot holds
        self.consumed = {}      # (r, q) -> last unit the leader added up

    def non_leader(self, r, q):
        for lt in range(self.units):
            if lt > 0:
                yield ("wait", self.red_free[(r, q)], lt - 1)
                assert self.consumed.get((r, q)) == lt - 1, "slot overwritten before it was read"
            self.slot[(r, q)] = lt
            yield ("yield",)
            yield ("arrive", self.red_full[q])

    def leader(self, q):
        for lt in range(self.units):
            yield ("wait", self.red_full[q], lt)
            for r in range(1, self.cs):
                assert self.slot.get((r, q)) == lt, (r, q, lt, self.slot.get((r, q)))
                self.consumed[(r, q)] = lt
            yield ("yield",)
            if lt + 1 < self.units:
                for r in range(1, self.cs):
                    yield ("arrive", self.red_free[(r, q)])

    def run(self):
        gens = {f"L{q}": self.leader(q) for q in range(4)}
        for r in range(1, self.cs):
            for q in range(4):
                gens[f"N{r}.{q}"] = self.non_leader(r, q)
        waiting = {n: None for n in gens}
        live = set(gens)
        for _ in range(1_000_000):
            if not live:
                break
            runnable = [n for n in sorted(live)
                        if waiting[n] is None or waiting[n][1].try_wait(waiting[n][2])]
            assert runnable, f"deadlock: {[(n, waiting[n][1].name) for n in live]}"
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
        assert not live
        # every phase a waiter expects completed, none is left half-arrived
        for q in range(4):
            assert self.red_full[q].completed == self.units
            assert self.red_full[q].pending == self.cs - 1
        for b in self.red_free.values():
            assert b.completed == self.units - 1 and b.pending == 1


@pytest.mark.parametrize("cs", [2, 3, 4, 8])
def test_cluster_reduction_protocol(cs):
    for seed in range(60):
        units = random.Random(seed).randint(1, 7)
        ClusterReductionModel(cs, units, seed).run()


def test_model_catches_a_leader_that_frees_before_reading():
    class Early(ClusterReductionModel):
        def leader(self, q):
            for lt in range(self.units):
                yield ("wait", self.red_full[q], lt)
                if lt + 1 < self.units:
                    for r in range(1, self.cs):
                        yield ("arrive", self.red_free[(r, q)])
                yield ("yield",)
                for r in range(1, self.cs):
                    assert self.slot.get((r, q)) == lt, "slot overwritten before it was read"
                    self.consumed[(r, q)] = lt
    caught = 0
    for seed in range(200):
        try:
            Early(3, 5, seed).run()
        except AssertionError:
            caught += 1
    assert caught > 0
