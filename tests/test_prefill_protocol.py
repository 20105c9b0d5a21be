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
was last written to it, so a role reading stale or overwritten data (scores
issued over a P that its PV has not read, a key tile released before its MMA
ran, an output rescaled before the previous PV executed) fails the check.

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
    """The kernel's protocol: per sub-tile one score buffer S (P is written
    over it), one output accumulator O; barriers q, full/empty[ns] (ring),
    s[sub] (S computed), p[sub] (P written, O rescaled), o[sub] (O final)."""

    def __init__(self, n_kv, ns, rng):
        self.rng = rng
        self.n_kv = n_kv
        self.ns = ns
        B = Bar
        self.q = B("q", 1)
        self.full = [B(f"full{i}", 1) for i in range(ns)]
        self.empty = [B(f"empty{i}", 1) for i in range(ns)]
        self.s = [B(f"s{a}", 1) for a in range(2)]
        self.p = [B(f"p{a}", 1) for a in range(2)]  # one arrival per warpgroup in the model
        self.o = [B(f"o{a}", 1) for a in range(2)]
        self.slot = [None] * ns           # tag of the tile in each ring slot
        self.sbuf = [None, None]          # tag in each S/P tensor-memory buffer
        self.o_applied = [0, 0]           # PVs executed into O[sub]
        self.s_exec = [0, 0]              # S MMAs executed per sub-tile
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
            _, sub, slot, j = op
            if self.slot[slot] != ("K", j):
                raise ProtocolError(f"S{sub}({j}) reads slot {slot} holding {self.slot[slot]}")
            if self.sbuf[sub] is not None and self.sbuf[sub][0] == "P" and self.o_applied[sub] <= self.sbuf[sub][1]:
                raise ProtocolError(f"S{sub}({j}) overwrites P({self.sbuf[sub][1]}) before its PV ran")
            self.sbuf[sub] = ("S", j)
            self.s_exec[sub] = j + 1
        elif kind == "pv":
            _, sub, slot, j = op
            if self.slot[slot] != ("V", j):
                raise ProtocolError(f"PV{sub}({j}) reads slot {slot} holding {self.slot[slot]}")
            if self.sbuf[sub] != ("P", j):
                raise ProtocolError(f"PV{sub}({j}) reads buffer holding {self.sbuf[sub]}")
            if self.o_applied[sub] != j:
                raise ProtocolError(f"PV{sub}({j}) out of order")
            self.o_applied[sub] = j + 1

    def land_tma(self, k):
        slot, tag = self.tma.pop(k)
        self.slot[slot] = tag
        self.full[slot].arrive()

    # -- roles: generators yielding ("wait", barrier, parity, phase) ----------
    def producer(self):
        self.q.arrive()  # Q lands (modelled as immediate)
        t = 0
        for j in range(self.n_kv):
            for which in "KV":
                slot = t % self.ns
                yield ("wait", self.empty[slot], ((t // self.ns) & 1) ^ 1, t // self.ns - 1)
                old = self.slot[slot]
                if old is not None:  # nothing may still need the old tile
                    kind, oj = old
                    for sub in range(2):
                        if kind == "V" and self.o_applied[sub] <= oj:
                            raise ProtocolError(f"V{oj} slot refilled before PV{sub}({oj}) ran")
                        if kind == "K" and self.s_exec[sub] <= oj:
                            raise ProtocolError(f"K{oj} slot refilled before S{sub}({oj}) ran")
                self.slot[slot] = ("loading",)
                self.tma.append((slot, (which, j)))
                t += 1

    def mma(self):
        ns = self.ns
        yield ("wait", self.q, 0, 0)
        yield ("wait", self.full[0], 0, 0)
        for sub in range(2):
            self.pipe.append(("qk", sub, 0, 0))
            self.pipe.append(("commit", self.s[sub]))
        self.pipe.append(("commit", self.empty[0]))
        for j in range(self.n_kv):
            vt = 2 * j + 1
            vslot = vt % ns
            yield ("wait", self.full[vslot], (vt // ns) & 1, vt // ns)
            kslot = None
            for sub in range(2):
                yield ("wait", self.p[sub], j & 1, j)
                self.pipe.append(("pv", sub, vslot, j))
                if j + 1 == self.n_kv:
                    self.pipe.append(("commit", self.o[sub]))
                if j + 1 < self.n_kv:
                    if sub == 0:
                        kt = 2 * (j + 1)
                        kslot = kt % ns
                        yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
                    self.pipe.append(("qk", sub, kslot, j + 1))
                    self.pipe.append(("commit", self.s[sub]))
            self.pipe.append(("commit", self.empty[vslot]))
            if kslot is not None:
                self.pipe.append(("commit", self.empty[kslot]))
        yield ("wait", self.o[0], 0, 0)

    def softmax(self, sub):
        for j in range(self.n_kv):
            yield ("wait", self.s[sub], j & 1, j)
            if self.sbuf[sub] != ("S", j):
                raise ProtocolError(f"softmax{sub}({j}) reads {self.sbuf[sub]}")
            self.sbuf[sub] = ("P", j)
            if j > 0 and self.rng.random() < 0.3 and self.o_applied[sub] != j:  # rescale O
                raise ProtocolError(f"softmax{sub}({j}) rescales O with {self.o_applied[sub]} PVs applied")
            self.p[sub].arrive()
        yield ("wait", self.o[sub], 0, 0)
        if self.o_applied[sub] != self.n_kv:
            raise ProtocolError(f"epilogue{sub} reads O with {self.o_applied[sub]} of {self.n_kv} PVs")

    def run(self):
        roles = [self.producer(), self.mma(), self.softmax(0), self.softmax(1)]
        pending = [None] * len(roles)
        alive = [True] * len(roles)
        for _ in range(200000):
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


CASES = [1, 2, 3, 4, 5, 9, 16, 33]


@pytest.mark.parametrize("n_kv", CASES)
@pytest.mark.parametrize("ns", [4, 8])
def test_protocol_random_interleavings(n_kv, ns):
    for seed in range(40):
        Model(n_kv, ns, random.Random(seed * 1000 + n_kv * 37 + ns)).run()


def _caught(cls, n_kv=6, ns=4):
    for seed in range(300):
        try:
            cls(n_kv, ns, random.Random(seed)).run()
        except ProtocolError:
            return True
    return False


def test_model_catches_scores_issued_before_the_pv():
    """Issuing S(j+1) before PV(j) overwrites P(j) (which lives in S's
    tensor-memory columns) before the PV reads it."""

    class Early(Model):
        def mma(self):
            for item in Model.mma(self):
                # after each PV is queued, move a following S of the same
                # sub-tile in front of it
                for k in range(len(self.pipe) - 1):
                    a, b = self.pipe[k], self.pipe[k + 1]
                    if a[0] == "pv" and b[0] == "qk" and a[1] == b[1]:
                        self.pipe[k], self.pipe[k + 1] = b, a
                yield item

    assert _caught(Early)


def test_model_catches_parity_off_by_one():
    """A softmax that waits for S with the wrong parity passes early."""

    class OffByOne(Model):
        def softmax(self, sub):
            for item in Model.softmax(self, sub):
                if item[1] is self.s[sub]:
                    item = ("wait", item[1], (item[3] + 1) & 1, item[3])
                yield item

    assert _caught(OffByOne)
