"""CPU model check of the prefill kernel's synchronisation protocol.

csrc/prefill_sm100.cu is a persistent kernel whose four roles meet only on
mbarriers: a TMA producer, a single-thread tcgen05 MMA issuer and two softmax
warpgroups (one per 128-row sub-tile, each also writing its sub-tile's output
at the end of a unit).  A CTA works
through a list of units (256 query rows each) with a per-unit number of key
tiles; the producer takes the units and publishes them to the other roles
through a four-entry ring in shared memory.  This model replays each role's
sequence of waits, arrivals, MMA issues and commits (as written in the kernel)
against a model of the hardware:

* an mbarrier completes a phase when its arrival count is reached;
  ``try_wait.parity(P)`` succeeds iff the barrier's current phase parity is
  not P -- the model also knows which phase each waiter means and reports a
  wait that would succeed early or block on a later phase (parity aliasing);
* tcgen05 MMAs from one thread execute in issue order, and a commit arrives
  once every earlier MMA has executed;
* TMA loads land at arbitrary later times.

A unit is given as its number of key tiles n, or as (n0, n1), the tiles each
sub-tile takes: n0 = n - 1 when under a causal mask the last key tile of a
256-row block lies wholly above sub-tile 0's rows, n1 = 0 when a short
segment leaves sub-tile 1 without rows; the kernel skips those tiles' scores,
softmax and PV (a sub-tile without tiles still takes its Q load and its
output barrier, so every barrier keeps one phase per unit).

Random interleavings are explored for several unit lists.  Besides deadlock and
aliasing, every buffer (Q_i, the key/value ring slots, S/P and O in tensor
memory) carries the tag of what
was last written to it, so a role reading stale or overwritten data fails the
check: scores issued over a P that its PV has not read, a ring slot or the Q
buffer refilled before the MMAs reading it ran, an output rescaled before the
previous PV executed, the next unit's first PV overwriting an output that has
not been read out.

The role scripts mirror the kernel; a change to the kernel's protocol must be
made here too.
"""
import random

import pytest


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
    """Barriers: q[sub] (Q_sub landed), q_free[sub] (last score MMAs of a
    unit for Q_sub ran), full/empty[ns] (ring), s[sub] (S computed), p[sub]
    (P written, O rescaled), o[sub] (O final), unit_full/unit_empty[4]
    (unit ring).  The next unit's first PV needs that unit's first P, which
    the softmax warpgroup writes only after reading O out, so O needs no
    release barrier.  Warpgroup arrivals (count 128 in
    the kernel) and the per-warp unit-ring releases are one arrival per role
    here."""

    RING = 4
    READERS = 3  # MMA, softmax 0, softmax 1

    def __init__(self, units, ns, rng):
        self.ntiles = [u if isinstance(u, tuple) else (u, u) for u in units]
        self.units = [max(u) for u in self.ntiles]
        self.ns, self.rng = ns, rng
        B = Bar
        self.q = [B(f"q{a}", 1) for a in range(2)]
        self.q_free = [B(f"q_free{a}", 1) for a in range(2)]
        self.full = [B(f"full{i}", 1) for i in range(ns)]
        self.empty = [B(f"empty{i}", 1) for i in range(ns)]
        self.s = [B(f"s{a}", 1) for a in range(2)]
        self.p = [B(f"p{a}", 1) for a in range(2)]
        self.o = [B(f"o{a}", 1) for a in range(2)]
        self.unit_full = [B(f"unit_full{e}", 1) for e in range(self.RING)]
        self.unit_empty = [B(f"unit_empty{e}", self.READERS) for e in range(self.RING)]
        self.unit = [None] * self.RING   # published unit numbers (-1: no more)
        self.slot = [None] * ns          # tag of the tile in each ring slot
        self.qbuf = [None, None]         # tag of each Q_sub buffer
        self.sbuf = [None, None]         # tag in each S/P tensor-memory buffer
        self.obuf = [None, None]         # (unit, PVs applied) in each O buffer
        self.o_read = [None, None]       # last unit whose output step ran
        self.o_consumed = [None, None]   # unit of the O buffer contents last read out
        self.s_exec = [(-1, 0), (-1, 0)]  # last (unit, tile) S MMA executed per sub-tile
        self.pipe = []                   # in-order tensor pipe
        self.tma = []                    # (slot, tag) loads in flight

    def nsub(self, k, sub):
        """Key tiles sub-tile `sub` of unit k takes."""
        return self.ntiles[k][0] if sub == 0 else self.ntiles[k][1]

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
        if op[0] == "commit":
            op[1].arrive()
            return
        _, sub, slot, k, j = op
        if op[0] == "qk":
            if self.qbuf[sub] != ("Q", k):
                raise ProtocolError(f"S{sub}({k},{j}) reads the Q{sub} buffer holding {self.qbuf[sub]}")
            if self.slot[slot] != ("K", k, j):
                raise ProtocolError(f"S{sub}({k},{j}) reads slot {slot} holding {self.slot[slot]}")
            sb = self.sbuf[sub]
            if sb is not None and sb[0] == "P":
                read = self.obuf[sub] is not None and self.obuf[sub][0] == sb[1] and self.obuf[sub][1] > sb[2]
                if not read:
                    raise ProtocolError(f"S{sub}({k},{j}) overwrites P{sb[1:]} before its PV ran")
            if sb is not None and sb[0] == "S":
                raise ProtocolError(f"S{sub}({k},{j}) overwrites S{sb[1:]} before the softmax read it")
            self.sbuf[sub] = ("S", k, j)
            self.s_exec[sub] = (k, j)
        else:  # pv
            if self.slot[slot] != ("V", k, j):
                raise ProtocolError(f"PV{sub}({k},{j}) reads slot {slot} holding {self.slot[slot]}")
            if self.sbuf[sub] != ("P", k, j):
                raise ProtocolError(f"PV{sub}({k},{j}) reads a buffer holding {self.sbuf[sub]}")
            if j == 0:
                if self.obuf[sub] is not None and self.o_consumed[sub] != self.obuf[sub][0]:
                    raise ProtocolError(f"PV{sub}({k},0) overwrites O of unit {self.obuf[sub][0]} before it was read out")
                self.obuf[sub] = (k, 1)
            else:
                if self.obuf[sub] != (k, j):
                    raise ProtocolError(f"PV{sub}({k},{j}) out of order: O holds {self.obuf[sub]}")
                self.obuf[sub] = (k, j + 1)

    def land_tma(self, i):
        slot, tag = self.tma.pop(i)
        if slot in ("q0", "q1"):
            sub = int(slot[1])
            self.qbuf[sub] = tag
            self.q[sub].arrive()
        else:
            self.slot[slot] = tag
            self.full[slot].arrive()

    # -- unit ring --------------------------------------------------------
    def read_unit(self, k):
        e = k % self.RING
        yield ("wait", self.unit_full[e], (k // self.RING) & 1, k // self.RING)
        got = self.unit[e]
        self.unit_empty[e].arrive()
        return got

    # -- roles: generators yielding ("wait", barrier, parity, phase) ----------
    def producer(self):
        t = 0
        nq = [0, 0]
        units = list(range(len(self.units))) + [-1]
        for ku, k in enumerate(units):
            e = ku % self.RING
            yield ("wait", self.unit_empty[e], ((ku // self.RING) & 1) ^ 1, ku // self.RING - 1)
            self.unit[e] = k
            self.unit_full[e].arrive()
            if k < 0:
                return
            n = self.units[k]
            for j in range(n):
                for which in "KV":
                    if j == 0 and which == "V":
                        for sub in range(2):
                            if nq[sub] > 0:
                                yield ("wait", self.q_free[sub], (nq[sub] - 1) & 1, nq[sub] - 1)
                                if self.nsub(k - 1, sub) > 0 and self.s_exec[sub] < (k - 1, self.nsub(k - 1, sub) - 1):
                                    raise ProtocolError(f"Q{sub} of unit {k} loaded under pending score MMAs of unit {k - 1}")
                            self.qbuf[sub] = ("loading",)
                            self.tma.append((f"q{sub}", ("Q", k)))
                            nq[sub] += 1
                    slot = t % self.ns
                    yield ("wait", self.empty[slot], ((t // self.ns) & 1) ^ 1, t // self.ns - 1)
                    old = self.slot[slot]
                    if old is not None:  # nothing may still need the old tile
                        kind, ok, oj = old
                        for sub in range(2):
                            if oj >= self.nsub(ok, sub):
                                continue  # a tile this sub-tile skips
                            if kind == "K" and self.s_exec[sub] < (ok, oj):
                                raise ProtocolError(f"K({ok},{oj}) slot refilled before S{sub} read it")
                            if kind == "V" and (self.obuf[sub] is None or self.obuf[sub] < (ok, oj + 1)):
                                raise ProtocolError(f"V({ok},{oj}) slot refilled before PV{sub} read it")
                    self.slot[slot] = ("loading", -1, -1)
                    self.tma.append((slot, (which, k, j)))
                    t += 1

    def mma(self):
        ns = self.ns
        t, k, tile = 0, 0, [0, 0]
        cur = yield from self.read_unit(0)
        if cur < 0:
            return
        yield ("wait", self.full[0], 0, 0)
        for sub in range(2):
            yield ("wait", self.q[sub], 0, 0)
            if self.nsub(cur, sub) > 0:
                self.pipe.append(("qk", sub, 0, cur, 0))
                self.pipe.append(("commit", self.s[sub]))
            if self.nsub(cur, sub) <= 1:
                self.pipe.append(("commit", self.q_free[sub]))
        self.pipe.append(("commit", self.empty[0]))
        while True:
            n = self.units[cur]
            # steady key tiles: PV_i(j) then S_i(j+1)
            for j in range(n - 1):
                vt, kt = t + 2 * j + 1, t + 2 * (j + 1)
                vslot, kslot = vt % ns, kt % ns
                yield ("wait", self.full[vslot], (vt // ns) & 1, vt // ns)
                for sub in range(2):
                    nsub = self.nsub(cur, sub)
                    if nsub == 0:
                        continue
                    yield ("wait", self.p[sub], tile[sub] & 1, tile[sub])
                    tile[sub] += 1
                    self.pipe.append(("pv", sub, vslot, cur, j))
                    if sub == 0:
                        yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
                    if j + 1 < nsub:
                        self.pipe.append(("qk", sub, kslot, cur, j + 1))
                        self.pipe.append(("commit", self.s[sub]))
                        if j + 2 == nsub:
                            self.pipe.append(("commit", self.q_free[sub]))
                self.pipe.append(("commit", self.empty[vslot]))
                self.pipe.append(("commit", self.empty[kslot]))
            # last key tile, then the next unit's first scores
            vt, kt = t + 2 * n - 1, t + 2 * n
            vslot, kslot = vt % ns, kt % ns
            yield ("wait", self.full[vslot], (vt // ns) & 1, vt // ns)
            nxt = yield from self.read_unit(k + 1)
            for sub in range(2):
                if self.nsub(cur, sub) == n:  # else its last PV ran in the steady loop
                    yield ("wait", self.p[sub], tile[sub] & 1, tile[sub])
                    tile[sub] += 1
                    self.pipe.append(("pv", sub, vslot, cur, n - 1))
                self.pipe.append(("commit", self.o[sub]))
                if nxt < 0:
                    continue
                if sub == 0:
                    yield ("wait", self.full[kslot], (kt // ns) & 1, kt // ns)
                yield ("wait", self.q[sub], (k + 1) & 1, k + 1)
                if self.nsub(nxt, sub) > 0:
                    self.pipe.append(("qk", sub, kslot, nxt, 0))
                    self.pipe.append(("commit", self.s[sub]))
                if self.nsub(nxt, sub) <= 1:
                    self.pipe.append(("commit", self.q_free[sub]))
            self.pipe.append(("commit", self.empty[vslot]))
            if nxt < 0:
                return
            self.pipe.append(("commit", self.empty[kslot]))
            t += 2 * n
            k += 1
            cur = nxt

    def softmax(self, sub):
        tile, k = 0, 0
        while True:
            cur = yield from self.read_unit(k)
            if cur < 0:
                return
            n = self.nsub(cur, sub)
            for j in range(n):
                yield ("wait", self.s[sub], tile & 1, tile)
                if self.sbuf[sub] != ("S", cur, j):
                    raise ProtocolError(f"softmax{sub}({cur},{j}) reads {self.sbuf[sub]}")
                self.sbuf[sub] = ("P", cur, j)
                if j > 0 and self.rng.random() < 0.3 and self.obuf[sub] != (cur, j):  # rescale O
                    raise ProtocolError(f"softmax{sub}({cur},{j}) rescales O holding {self.obuf[sub]}")
                self.p[sub].arrive()
                tile += 1
            # the unit's output of this sub-tile
            yield ("wait", self.o[sub], k & 1, k)
            if n > 0 and self.obuf[sub] != (cur, n):
                raise ProtocolError(f"output({cur},{sub}) reads O holding {self.obuf[sub]}")
            self.o_read[sub] = cur
            if self.obuf[sub] is not None:
                self.o_consumed[sub] = self.obuf[sub][0]
            k += 1

    def run(self):
        roles = [self.producer(), self.mma(), self.softmax(0), self.softmax(1)]
        pending = [None] * len(roles)
        alive = [True] * len(roles)
        for _ in range(400000):
            # Advance every role to its next wait first (advancing may arrive
            # on barriers), then see which waits can pass.
            for i, g in enumerate(roles):
                if alive[i] and pending[i] is None:
                    try:
                        pending[i] = next(g)
                    except StopIteration:
                        alive[i] = False
            choices = [("role", i) for i in range(len(roles)) if alive[i] and self.check_wait(*pending[i][1:])]
            if self.pipe:
                choices.append(("pipe", None))
            choices += [("tma", i) for i in range(len(self.tma))]
            if not choices:
                if any(alive):
                    stuck = [pending[i][1].name for i in range(len(roles)) if alive[i]]
                    raise ProtocolError(f"deadlock: roles wait on {stuck}")
                if self.o_read != [len(self.units) - 1] * 2 and self.units:
                    raise ProtocolError(f"finished with outputs read up to {self.o_read}")
                return
            kind, arg = self.rng.choice(choices)
            if kind == "role":
                pending[arg] = None
            elif kind == "pipe":
                self.exec_pipe()
            else:
                self.land_tma(arg)
        raise ProtocolError("did not finish")


UNIT_LISTS = [[1], [2], [3], [5], [16], [33], [1, 1, 1], [3, 1, 2], [5, 5], [1, 4, 2, 6, 1], [16, 8, 2], [2, 2, 2, 2, 2],
              # sub-tile 0 skipping the last key tile (causal row blocks)
              [(1, 2)], [(15, 16), (7, 8), (1, 2)], [(1, 2), (1, 2), (1, 2)], [(3, 4), 2, (1, 2), 1, (5, 6)],
              [1, (1, 2), (2, 3), 3],
              # sub-tile 1 without rows (short last row block of a segment)
              [(1, 0)], [(3, 0), 2, (2, 0), (1, 2), (4, 0)], [(5, 0), (5, 0)], [(1, 0), (1, 0), (1, 2), (2, 0)]]


@pytest.mark.parametrize("units", UNIT_LISTS, ids=lambda u: "-".join(map(str, u)).replace(" ", ""))
@pytest.mark.parametrize("ns", [4, 8])
def test_protocol_random_interleavings(units, ns):
    for seed in range(30):
        Model(units, ns, random.Random(seed * 1000 + sum(u if isinstance(u, int) else u[1] for u in units) * 37 + ns)).run()


def _caught(cls, units=(3, 1, 4, 2), ns=4):
    for seed in range(300):
        try:
            cls(list(units), ns, random.Random(seed)).run()
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


def test_model_catches_output_read_before_the_last_pv():
    """Reading O out without waiting for the unit's last PV reads a partial
    sum."""

    class NoWait(Model):
        def softmax(self, sub):
            for item in Model.softmax(self, sub):
                if item[1] is self.o[sub]:
                    continue
                yield item

    assert _caught(NoWait)


def test_model_catches_q_released_too_early():
    """Releasing Q_i right after a unit's first scores (instead of its last)
    lets the producer load the next unit's Q under pending score MMAs."""

    class EarlyQ(Model):
        def mma(self):
            gen = Model.mma(self)
            item = next(gen)
            while True:
                # drop the kernel's q_free commits; release right after each
                # sub-tile's first scores of a unit instead
                for sub in range(2):
                    qf = ("commit", self.q_free[sub])
                    while qf in self.pipe:
                        self.pipe.remove(qf)
                for i, op in enumerate(list(self.pipe)):
                    if op[0] == "qk" and op[4] == 0 and ("released", op[1], op[3]) not in self.__dict__.setdefault("rel", set()):
                        self.rel.add(("released", op[1], op[3]))
                        self.pipe.insert(self.pipe.index(op) + 1, ("commit", self.q_free[op[1]]))
                try:
                    item = gen.send((yield item))
                except StopIteration:
                    return

    assert _caught(EarlyQ)



def test_model_catches_a_skipped_tile_still_waited_for():
    """Sub-tile 0's softmax taking all n tiles of a unit whose last tile the
    MMA issuer skips for it waits on scores that never come."""

    class Mismatch(Model):
        def nsub(self, k, sub):
            n0 = Model.nsub(self, k, sub)
            import inspect
            caller = inspect.stack()[1].function
            return self.ntiles[k][1] if caller == "softmax" else n0

    assert _caught(Mismatch, units=((1, 2), (3, 4)))


def test_model_catches_a_skipped_q_wait_for_an_empty_sub_tile():
    """Not waiting for Q_1 of a unit whose sub-tile 1 has no rows lets the
    next unit's wait on the same barrier pass on the wrong phase."""

    class SkipWait(Model):
        def mma(self):
            for item in Model.mma(self):
                if item[1] is self.q[1] and self.nsub(item[3], 1) == 0:
                    continue
                yield item

    assert _caught(SkipWait, units=((2, 0), (1, 2), (3, 0), (2, 3)))
