"""CPU model check of the prefill kernel's synchronisation protocol.

csrc/prefill_sm100.cu runs four roles that meet only on mbarriers: a TMA
producer, a single-thread tcgen05 MMA issuer and two softmax warpgroups.  This
model replays each role's sequence of waits, arrivals, MMA issues and commits
(as written in the kernel) against a model of the hardware:

* an mbarrier completes a phase when its arrival count is reached;
  ``try_wait.parity(P)`` succeeds iff the barrier's current phase parity is
  not P -- the model also knows which phase each waiter means and reports a
  wait that would succeed early or block on a later phase (parity aliasing);
* tcgen05 MMAs from one thread execute in issue order, and a commit arrives
  once every earlier MMA has executed;
* TMA loads land at arbitrary later times.

Random interleavings are explored for several tile counts.  Besides deadlock
and aliasing, every tensor-memory buffer and ring slot carries the tag of what
was last written to it, so a role reading stale or overwritten data (an S
buffer reused too early, a key tile released before its MMA ran, an output
rescaled before its last PV executed) fails the check.

The role scripts mirror the kernel; a change to the kernel's protocol must be
made here too.
"""
import random

import pytest

BN = 64  # keys per tile


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class ProtocolError(AssertionError):
    pass


class Model:
    def __init__(self, n_sub, ns, rng):
        self.rng = rng
        self.n_sub = list(n_sub)
        self.n_kv = max(n_sub)
        self.ns = ns
        B = Bar
        self.q = B("q", 1)
        self.full = [B(f"full{i}", 1) for i in range(ns)]
        self.empty = [B(f"empty{i}", 1) for i in range(ns)]
        self.s = [[B(f"s{a}{b}", 1) for b in range(2)] for a in range(2)]
        self.p = [[B(f"p{a}{b}", 1) for b in range(2)] for a in range(2)]  # one arrival per warpgroup in the model
        self.o = [B(f"o{a}", 1) for a in range(2)]
        self.done_bar = B("done", 1)
        self.slot = [None] * ns           # tag of the tile in each ring slot
        self.sbuf = [[None, None], [None, None]]  # tag in each S/P tensor-memory buffer
        self.o_applied = [0, 0]           # PVs executed into O[sub]
        self.pipe = []                    # in-order tensor pipe
        self.tma = []                     # (slot, tag) loads in flight

    # -- hardware -------------------------------------------------------
    def check_wait(self, bar, parity, phase):
        hw = (bar.done & 1) != parity
        truth = bar.done > phase
        if hw and not truth:
            raise ProtocolError(f"{bar.name}: parity wait for phase {phase} passes early (done={bar.done})")
        if not hw and truth:
            raise ProtocolError(f"{bar.name}: parity wait for phase {phase} aliased to a later phase (done={bar.done})")
        return hw

    def exec_pipe(self):
        op = self.pipe.pop(0)
        kind = op[0]
        if kind == "commit":
            op[1].arrive()
        elif kind == "qk":
            _, sub, buf, slot, j = op
            if self.slot[slot] != ("K", j):
                raise ProtocolError(f"S{sub}({j}) reads slot {slot} holding {self.slot[slot]}")
            if self.sbuf[sub][buf] is not None and self.sbuf[sub][buf][0] == "P":
                pj = self.sbuf[sub][buf][1]
                if self.o_applied[sub] <= pj:
                    raise ProtocolError(f"S{sub}({j}) overwrites P({pj}) before its PV ran")
            self.sbuf[sub][buf] = ("S", j)
            self._s_exec[sub] = max(self._s_exec[sub], j + 1)
        elif kind == "pv":
            _, sub, buf, slot, j = op
            if self.slot[slot] != ("V", j):
                raise ProtocolError(f"PV{sub}({j}) reads slot {slot} holding {self.slot[slot]}")
            if self.sbuf[sub][buf] != ("P", j):
                raise ProtocolError(f"PV{sub}({j}) reads buffer holding {self.sbuf[sub][buf]}")
            if self.o_applied[sub] != j:
                raise ProtocolError(f"PV{sub}({j}) out of order")
            self.o_applied[sub] = j + 1

    def land_tma(self, k):
        slot, tag = self.tma.pop(k)
        self.slot[slot] = tag
        self.full[slot].arrive()

    # -- roles (generators yielding callables that return True when they could act)
    def producer(self):
        self.q.arrive()  # Q lands (modelled as immediate)
        t = 0
        for j in range(self.n_kv):
            for which in "KV":
                slot = t % self.ns
                yield ("wait", self.empty[slot], ((t // self.ns) & 1) ^ 1, t // self.ns - 1)
                # the slot is free: nothing may still need its old tile
                old = self.slot[slot]
                if old is not None:
                    self.assert_released(old)
                self.slot[slot] = ("loading",)
                self.tma.append((slot, (which, j)))
                t += 1

    def assert_released(self, tag):
        kind, j = tag
        for sub in range(2):
            if j < self.n_sub[sub]:
                if kind == "V" and self.o_applied[sub] <= j:
                    raise ProtocolError(f"V{j} slot refilled before PV{sub}({j}) ran")
                if kind == "K" and self._s_exec[sub] <= j:
                    raise ProtocolError(f"K{j} slot refilled before S{sub}({j}) ran")

    def mma(self):
        yield ("wait", self.q, 0, 0)
        ns = self.ns

        def qk(sub, buf, slot, j):
            self.pipe.append(("qk", sub, buf, slot, j))

        for j in range(min(2, self.n_kv)):
            kt = 2 * j
            kslot = kt % ns
            yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
            for sub in range(2):
                if j < self.n_sub[sub]:
                    qk(sub, j & 1, kslot, j)
                    self.pipe.append(("commit", self.s[sub][j & 1]))
            self.pipe.append(("commit", self.empty[kslot]))
        for j in range(self.n_kv):
            vt = 2 * j + 1
            vslot = vt % ns
            kt = 2 * (j + 2)
            kslot = kt % ns
            k_ready = False
            yield ("wait", self.full[vslot], (vt // ns) & 1, vt // ns)
            for sub in range(2):
                if j >= self.n_sub[sub]:
                    continue
                yield ("wait", self.p[sub][j & 1], (j >> 1) & 1, j >> 1)
                self.pipe.append(("pv", sub, j & 1, vslot, j))
                if j + 2 >= self.n_sub[sub]:
                    self.pipe.append(("commit", self.o[sub]))
                if j + 2 < self.n_sub[sub]:
                    if not k_ready:
                        yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
                        k_ready = True
                    qk(sub, j & 1, kslot, j + 2)
                    self.pipe.append(("commit", self.s[sub][j & 1]))
            self.pipe.append(("commit", self.empty[vslot]))
            if j + 2 < self.n_kv:
                if not k_ready:
                    yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
                self.pipe.append(("commit", self.empty[kslot]))
        self.pipe.append(("commit", self.done_bar))
        yield ("wait", self.done_bar, 0, 0)

    def softmax(self, sub):
        n = self.n_sub[sub]
        for j in range(n):
            buf = j & 1
            yield ("wait", self.s[sub][buf], (j >> 1) & 1, j >> 1)
            if self.sbuf[sub][buf] != ("S", j):
                raise ProtocolError(f"softmax{sub}({j}) reads {self.sbuf[sub][buf]}")
            self.sbuf[sub][buf] = ("P", j)
            rescale = j > 0 and self.rng.random() < 0.3
            if j > 0 and j + 1 == n:
                yield ("wait", self.o[sub], 0, 0)
            elif j > 0 and rescale:
                yield ("wait", self.s[sub][(j + 1) & 1], ((j + 1) >> 1) & 1, (j + 1) >> 1)
            if rescale and self.o_applied[sub] != j:
                raise ProtocolError(f"softmax{sub}({j}) rescales O with {self.o_applied[sub]} PVs applied")
            self.p[sub][buf].arrive()
        if n > 0:
            yield ("wait", self.o[sub], 1 if n >= 2 else 0, 1 if n >= 2 else 0)
            if self.o_applied[sub] != n:
                raise ProtocolError(f"epilogue{sub} reads O with {self.o_applied[sub]} of {n} PVs")

    def run(self):
        self._s_exec = [0, 0]
        roles = [self.producer(), self.mma(), self.softmax(0), self.softmax(1)]
        pending = [None] * len(roles)
        alive = [True] * len(roles)
        for steps in range(200000):
            choices = []
            # Advance every role to its next wait first (advancing may arrive
            # on barriers), then see which waits can pass.
            for i, g in enumerate(roles):
                if alive[i] and pending[i] is None:
                    try:
                        pending[i] = next(g)
                    except StopIteration:
                        alive[i] = False
            for i in range(len(roles)):
                if alive[i]:
                    _, bar, parity, phase = pending[i]
                    if self.check_wait(bar, parity, phase):
                        choices.append(("role", i))
            if self.pipe:
                choices.append(("pipe", None))
            for k in range(len(self.tma)):
                choices.append(("tma", k))
            if not choices:
                if any(alive):
                    stuck = [pending[i][1].name for i in range(len(roles)) if alive[i]]
                    raise ProtocolError(f"deadlock: roles wait on {stuck}")
                return
            kind, arg = self.rng.choice(choices)
            if kind == "role":
                pending[arg] = None
            elif kind == "pipe":
                self.exec_pipe()
            else:
                self.land_tma(arg)
        raise ProtocolError("did not finish")


CASES = [
    (1, 0), (2, 0), (1, 1), (2, 2), (3, 3), (4, 4), (9, 9), (2, 4), (6, 8), (30, 32), (5, 0), (17, 17),
]


@pytest.mark.parametrize("n_sub", CASES)
@pytest.mark.parametrize("ns", [8, 16])
def test_protocol_random_interleavings(n_sub, ns):
    for seed in range(25):
        Model(n_sub, ns, random.Random(seed * 1000 + n_sub[0] * 37 + n_sub[1])).run()


def test_model_catches_single_p_barrier_aliasing():
    """The protocol with ONE P-ready barrier per sub-tile (instead of one per S
    buffer) lets the softmax finish two tiles before the MMA issuer waits,
    aliasing the barrier's parity; the model must flag it."""

    class OneP(Model):
        def __init__(self, *a):
            super().__init__(*a)
            shared = [Bar("p0", 1), Bar("p1", 1)]
            self.p = [[shared[0], shared[0]], [shared[1], shared[1]]]

        def mma(self):
            seen = {"p0": 0, "p1": 0}
            for item in Model.mma(self):
                if item[0] == "wait" and item[1].name in seen:
                    j = seen[item[1].name]
                    seen[item[1].name] += 1
                    item = ("wait", item[1], j & 1, j)
                yield item

    caught = False
    for seed in range(200):
        try:
            OneP((6, 6), 8, random.Random(seed)).run()
        except ProtocolError:
            caught = True
            break
    assert caught
