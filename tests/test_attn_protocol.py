"""Model check of the sparse attention kernel's barrier protocol (host only, no GPU).

The attention kernel (svg2_attn.cu) hands its work from agent to agent through mbarriers that are
waited on by phase parity:

* the producer warps (three, each writing its own rows of a tile) gather K(j) and V(j) into
  shared-memory stage j % 2 with cp.async. Each warp's copies land asynchronously and arrive on
  k_full / v_full, which complete once every warp has arrived. Each warp waits on k_empty / v_empty
  before it reuses a stage.
* the MMA thread issues S = Q K^T into a tensor-memory slot, and PV in two 64-key halves. Its
  commits arrive on s_full, k_empty, v_empty, pv_done and o_full once every earlier product has
  completed. The tensor core runs the products in issue order.
* four softmax warps per Q tile read S, rescale O when their running maximum grows, write P over S
  in two halves and arrive on p_full, and at the end wait on o_full.

This module restates that protocol as Python generators: which barrier each agent waits on, with
which parity, and in which order. It runs the agents under many seeded random interleavings. A
parity wait is satisfied only while the awaited phase is complete and not yet overtaken, so a
barrier that runs two phases ahead of its waiter shows up here, as it does on the device, as a wait
that never ends. The data checks compare each tile's operands at the moment a product runs
against what the schedule intends, which catches a stage or slot overwritten too early.

The model restates the protocol, not the code. A change to the kernel's barrier scheme must be
made here too. ``test_shared_p_barriers_in_ring_mode_deadlock`` plants the single P barrier pair
that ring mode once shared between consecutive tiles. It checks that the model finds the resulting
hang, which the device reported as a bounded-wait timeout in the MMA thread, and the early reads
the same sharing allows.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase; wait(parity) passes once the phase of that
    parity has completed and the barrier is not yet back in a phase of the same parity."""

    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


class ProtocolError(AssertionError):
    pass


def check(cond, what):
    if not cond:
        raise ProtocolError(what)


class Kernel:
    """One CTA of the attention kernel: one unit of one or two Q tiles over T key tiles."""

    def __init__(self, T, has_b, rng, shared_p=False, producers=3):
        self.T, self.has_b, self.rng, self.shared_p, self.producers = T, has_b, rng, shared_p, producers
        self.k_full = [Bar(producers), Bar(producers)]
        self.v_full = [Bar(producers), Bar(producers)]
        self.k_empty = [Bar(1), Bar(1)]
        self.v_empty = [Bar(1), Bar(1)]
        self.s_full = [Bar(1), Bar(1)]
        self.p_full = [[Bar(4), Bar(4)], [Bar(4), Bar(4)]]
        self.pv_done, self.o_full = Bar(1), Bar(1)
        # shared memory: per stage, the tile each producer's rows hold
        self.k_smem = [[None] * producers for _ in range(2)]
        self.v_smem = [[None] * producers for _ in range(2)]
        # tensor memory: per slot and warp quarter, the S tile held and the P halves written over it
        self.s_tm = [[None] * 4 for _ in range(2)]
        self.p_tm = [[[None, None] for _ in range(4)] for _ in range(2)]
        self.o_halves = [[0] * 4 for _ in range(2)]  # PV halves applied to O_x, per warp quarter
        self.in_rescale = [[False] * 4 for _ in range(2)]
        self.tc_queue, self.copies = [], []

    # ---- tensor core: runs queued products and commits in issue order ----
    def run_tc_op(self):
        op = self.tc_queue.pop(0)
        kind = op[0]
        if kind == "S":
            _, x, j, stage, slot = op
            check(all(r == ("K", j) for r in self.k_smem[stage]), f"S_{x}({j}) read stage {stage} holding {self.k_smem[stage]}")
            for q in range(4):
                self.s_tm[slot][q] = (x, j)
                self.p_tm[slot][q] = [None, None]
        elif kind == "PV":
            _, x, j, slot, stage, h = op
            check(all(r == ("V", j) for r in self.v_smem[stage]), f"PV_{x}({j}) read stage {stage} holding {self.v_smem[stage]}")
            for q in range(4):
                check(self.p_tm[slot][q][h] == (x, j), f"PV_{x}({j}) half {h} read {self.p_tm[slot][q][h]}")
                check(not self.in_rescale[x][q], f"PV_{x}({j}) ran during a rescale of O_{x}")
                check(self.o_halves[x][q] == 2 * j + h, f"PV_{x}({j}) half {h} out of order")
                self.o_halves[x][q] += 1
        else:
            op[1].arrive()

    def run_copy(self):
        i = self.rng.randrange(len(self.copies))
        rows, w, val, bar = self.copies.pop(i)
        rows[w] = val
        bar.arrive()

    # ---- agents: each yields a wait condition (or None for a plain step) ----
    def wait(self, bar, parity):
        return lambda: bar.done(parity)

    def producer(self, w):
        for j in range(self.T):
            st = j & 1
            if j >= 2:
                yield self.wait(self.k_empty[st], ((j >> 1) - 1) & 1)
            self.k_smem[st][w] = ("landing", j)
            self.copies.append((self.k_smem[st], w, ("K", j), self.k_full[st]))
            yield None
            if j >= 2:
                yield self.wait(self.v_empty[st], ((j >> 1) - 1) & 1)
            self.v_smem[st][w] = ("landing", j)
            self.copies.append((self.v_smem[st], w, ("V", j), self.v_full[st]))
            yield None

    def mma(self):
        T, q = self.T, self.tc_queue
        if T > 0:
            yield self.wait(self.k_full[0], 0)
            q.append(("S", 0, 0, 0, 0))
            q.append(("commit", self.s_full[0]))
            if self.has_b:
                q.append(("S", 1, 0, 0, 1))
                q.append(("commit", self.s_full[1]))
            q.append(("commit", self.k_empty[0]))
            yield None
        if not self.has_b:
            if T > 1:
                yield self.wait(self.k_full[1], 0)
                q.append(("S", 0, 1, 1, 1))
                q.append(("commit", self.s_full[1]))
                q.append(("commit", self.k_empty[1]))
                yield None
            for j in range(T):
                st = j & 1
                pb, pp = (self.p_full[0], j & 1) if self.shared_p else (self.p_full[st], (j >> 1) & 1)
                yield self.wait(pb[0], pp)
                yield self.wait(self.v_full[st], (j >> 1) & 1)
                q.append(("PV", 0, j, st, st, 0))
                yield self.wait(pb[1], pp)
                q.append(("PV", 0, j, st, st, 1))
                q.append(("commit", self.pv_done))
                q.append(("commit", self.v_empty[st]))
                yield None
                if j + 2 < T:
                    yield self.wait(self.k_full[st], ((j + 2) >> 1) & 1)
                    q.append(("S", 0, j + 2, st, st))
                    q.append(("commit", self.s_full[st]))
                    q.append(("commit", self.k_empty[st]))
                    yield None
        else:
            for j in range(T):
                st, nst, more = j & 1, (j + 1) & 1, j + 1 < T
                yield self.wait(self.p_full[0][0], j & 1)
                yield self.wait(self.v_full[st], (j >> 1) & 1)
                q.append(("PV", 0, j, 0, st, 0))
                yield self.wait(self.p_full[0][1], j & 1)
                q.append(("PV", 0, j, 0, st, 1))
                if more:
                    yield self.wait(self.k_full[nst], ((j + 1) >> 1) & 1)
                    q.append(("S", 0, j + 1, nst, 0))
                    q.append(("commit", self.s_full[0]))
                yield self.wait(self.p_full[1][0], j & 1)
                q.append(("PV", 1, j, 1, st, 0))
                yield self.wait(self.p_full[1][1], j & 1)
                q.append(("PV", 1, j, 1, st, 1))
                q.append(("commit", self.v_empty[st]))
                if more:
                    q.append(("S", 1, j + 1, nst, 1))
                    q.append(("commit", self.s_full[1]))
                    q.append(("commit", self.k_empty[nst]))
                yield None
        q.append(("commit", self.o_full))

    def softmax(self, x, w):
        ring = not self.has_b
        for j in range(self.T):
            slot = (j & 1) if ring else x
            par = ((j >> 1) & 1) if ring else (j & 1)
            yield self.wait(self.s_full[slot], par)
            check(self.s_tm[slot][w] == (x, j), f"softmax {x}.{w} tile {j} read S {self.s_tm[slot][w]}")
            if j > 0 and self.rng.random() < 0.5:  # the running maximum grew: rescale O_x
                if ring:
                    yield self.wait(self.pv_done, (j - 1) & 1)
                check(self.o_halves[x][w] == 2 * j, f"rescale of O_{x} at tile {j} saw {self.o_halves[x][w]} halves")
                self.in_rescale[x][w] = True
                yield None
                self.in_rescale[x][w] = False
            for hh in range(2):
                check(self.s_tm[slot][w] == (x, j), f"P_{x}({j}) written over S {self.s_tm[slot][w]}")
                self.p_tm[slot][w][hh] = (x, j)
                yield None
                (self.p_full[x] if self.shared_p else self.p_full[slot])[hh].arrive()
                yield None
        if self.T > 0:
            yield self.wait(self.o_full, 0)
            check(self.o_halves[x][w] == 2 * self.T, f"epilogue of O_{x} saw {self.o_halves[x][w]} halves")


def run_schedule(T, has_b, seed, shared_p=False, max_steps=100000):
    """Run one random interleaving; raise ProtocolError on a hazard or a deadlock."""
    rng = random.Random(seed)
    k = Kernel(T, has_b, rng, shared_p)
    agents = {f"producer{w}": k.producer(w) for w in range(k.producers)}
    agents["mma"] = k.mma()
    for x in range(2 if has_b else 1):
        for w in range(4):
            agents[f"softmax{x}.{w}"] = k.softmax(x, w)
    waiting = {name: None for name in agents}
    for _ in range(max_steps):
        runnable = [n for n in agents if waiting[n] is None or waiting[n]()]
        if k.tc_queue:
            runnable.append("tc")
        if k.copies:
            runnable.append("copy")
        if not runnable:
            if agents:
                raise ProtocolError(f"deadlock: {sorted(agents)} wait forever")
            return
        name = rng.choice(runnable)
        if name == "tc":
            k.run_tc_op()
        elif name == "copy":
            k.run_copy()
        else:
            try:
                waiting[name] = next(agents[name])
            except StopIteration:
                del agents[name]
                del waiting[name]
    raise ProtocolError("schedule did not finish")


@pytest.mark.parametrize("has_b", [False, True], ids=["one-q-tile-ring", "two-q-tiles"])
@pytest.mark.parametrize("T", [0, 1, 2, 3, 4, 7])
def test_protocol_has_no_deadlock_or_hazard(T, has_b):
    for seed in range(400):
        run_schedule(T, has_b, seed)


@pytest.mark.parametrize("T", [2, 3, 5])
def test_shared_p_barriers_in_ring_mode_deadlock(T):
    """One P barrier pair shared by consecutive ring-mode tiles lets the softmax complete two
    phases before the MMA thread waits for the first, so some interleavings hang. Others let a
    phase complete on arrivals meant for two different tiles (one softmax warp a tile ahead of
    another), or let a wait pass on the wrong phase, so a PV product reads P before it is written.
    Every tile count shows the fault; from three tiles on, 400 schedules show both forms."""
    deadlocks = hazards = 0
    for seed in range(400):
        try:
            run_schedule(T, False, seed, shared_p=True)
        except ProtocolError as e:
            if "deadlock" in str(e):
                deadlocks += 1
            else:
                hazards += 1
    assert deadlocks + hazards > 0
    if T >= 3:
        assert deadlocks > 0 and hazards > 0
