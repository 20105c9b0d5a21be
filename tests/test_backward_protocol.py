"""CPU model check of the synchronisation protocols of the two tensor-core
backward kernels in csrc/backward_sm100.cu (the same hardware model as
tests/test_prefill_protocol.py: mbarrier phases with parity waits checked for
aliasing, an in-order tensor pipe whose commits arrive after every earlier
MMA, TMA loads landing at arbitrary later times).  Every buffer carries the
tag of what was last written to it, so reading stale data or overwriting data
before its reader ran fails the check.  The role scripts mirror the kernels.
"""
import random

import pytest

from test_prefill_protocol import Bar, ProtocolError


class _Hw:
    def __init__(self, rng):
        self.rng, self.pipe, self.tma = rng, [], []

    @staticmethod
    def check_wait(bar, parity, phase):
        hw = (bar.done & 1) != parity
        truth = bar.done > phase
        if hw and not truth:
            raise ProtocolError(f"{bar.name}: wait for phase {phase} passes early (done={bar.done})")
        if not hw and truth:
            raise ProtocolError(f"{bar.name}: wait for phase {phase} aliased (done={bar.done})")
        return hw

    def run(self, roles):
        pending = [None] * len(roles)
        alive = [True] * len(roles)
        for _ in range(400000):
            for i, g in enumerate(roles):
                if alive[i] and pending[i] is None:
                    try:
                        pending[i] = next(g)
                    except StopIteration:
                        alive[i] = False
            ch = [("role", i) for i in range(len(roles)) if alive[i] and self.check_wait(*pending[i][1:])]
            if self.pipe:
                ch.append(("pipe", None))
            ch += [("tma", i) for i in range(len(self.tma))]
            if not ch:
                if any(alive):
                    raise ProtocolError(f"deadlock: {[pending[i][1].name for i in range(len(roles)) if alive[i]]}")
                return
            kind, a = self.rng.choice(ch)
            if kind == "role":
                pending[a] = None
            elif kind == "pipe":
                op = self.pipe.pop(0)
                if op[0] == "commit":
                    op[1].arrive()
                else:
                    op[1]()
            else:
                fn = self.tma.pop(a)
                fn()
        raise ProtocolError("did not finish")


class DqModel(_Hw):
    """dQ kernel: rings K (3 slots) and V (2 slots); S, dP and dS buffers."""

    def __init__(self, n, rng):
        super().__init__(rng)
        B = Bar
        self.n = n
        self.qg = B("qg", 1)
        self.kfull = [B(f"kfull{i}", 1) for i in range(3)]
        self.kempty = [B(f"kempty{i}", 1) for i in range(3)]
        self.vfull = [B(f"vfull{i}", 1) for i in range(2)]
        self.vempty = [B(f"vempty{i}", 1) for i in range(2)]
        self.sdp_ready, self.sdp_free = B("sdp_ready", 1), B("sdp_free", 1)
        self.ds_ready, self.ds_free, self.done = B("ds_ready", 1), B("ds_free", 1), B("done", 1)
        self.kslot, self.vslot = [None] * 3, [None] * 2
        self.sbuf = None      # tile whose S/dP are in tensor memory
        self.sread = set()    # tiles whose S/dP the elementwise role has read
        self.dsbuf = None
        self.dq_done = []     # dQ products executed, in order

    def _land(self, ring, slot, tag, full):
        def f():
            ring[slot] = tag
            full.arrive()
        return f

    def producer(self):
        self.tma.append(lambda: self.qg.arrive())
        for j in range(self.n):
            ks, vs = j % 3, j % 2
            yield ("wait", self.kempty[ks], ((j // 3) & 1) ^ 1, j // 3 - 1)
            if self.kslot[ks] is not None and self.kslot[ks] not in self.dq_done:
                raise ProtocolError(f"K slot {ks} refilled before dQ({self.kslot[ks]}) read it")
            self.kslot[ks] = None
            self.tma.append(self._land(self.kslot, ks, j, self.kfull[ks]))
            yield ("wait", self.vempty[vs], ((j // 2) & 1) ^ 1, j // 2 - 1)
            self.vslot[vs] = None
            self.tma.append(self._land(self.vslot, vs, j, self.vfull[vs]))

    def _sdp(self, j):
        def f():
            if self.kslot[j % 3] != j or self.vslot[j % 2] != j:
                raise ProtocolError(f"S/dP({j}) read rings holding K {self.kslot[j % 3]} V {self.vslot[j % 2]}")
            if self.sbuf is not None and self.sbuf not in self.sread:
                raise ProtocolError(f"S/dP({j}) overwrite tile {self.sbuf} before it was read")
            self.sbuf = j
        return f

    def _dq(self, j):
        def f():
            if self.dsbuf != j or self.kslot[j % 3] != j:
                raise ProtocolError(f"dQ({j}) reads dS {self.dsbuf} and K {self.kslot[j % 3]}")
            self.dq_done.append(j)
        return f

    def mma(self):
        n = self.n
        yield ("wait", self.qg, 0, 0)
        yield ("wait", self.kfull[0], 0, 0)
        yield ("wait", self.vfull[0], 0, 0)
        self.pipe += [("op", self._sdp(0)), ("commit", self.sdp_ready), ("commit", self.vempty[0])]
        for j in range(n):
            if j + 1 < n:
                ks, vs = (j + 1) % 3, (j + 1) % 2
                yield ("wait", self.sdp_free, j & 1, j)
                yield ("wait", self.kfull[ks], ((j + 1) // 3) & 1, (j + 1) // 3)
                yield ("wait", self.vfull[vs], ((j + 1) // 2) & 1, (j + 1) // 2)
                self.pipe += [("op", self._sdp(j + 1)), ("commit", self.sdp_ready), ("commit", self.vempty[vs])]
            yield ("wait", self.ds_ready, j & 1, j)
            self.pipe += [("op", self._dq(j)), ("commit", self.ds_free), ("commit", self.kempty[j % 3])]
        self.pipe.append(("commit", self.done))

    def elementwise(self):
        for j in range(self.n):
            yield ("wait", self.sdp_ready, j & 1, j)
            if self.sbuf != j:
                raise ProtocolError(f"elementwise({j}) reads S/dP of tile {self.sbuf}")
            self.sread.add(j)
            self.sdp_free.arrive()
            if j > 0:
                yield ("wait", self.ds_free, (j - 1) & 1, j - 1)
            if self.dsbuf is not None and self.dsbuf not in self.dq_done:
                raise ProtocolError(f"dS({j}) overwrites dS({self.dsbuf}) before its dQ ran")
            self.dsbuf = j
            self.ds_ready.arrive()
        yield ("wait", self.done, 0, 0)
        if self.dq_done != list(range(self.n)):
            raise ProtocolError(f"dQ written after {self.dq_done}")

    def go(self):
        self.run([self.producer(), self.mma(), self.elementwise()])


class DkdvModel(_Hw):
    """dK/dV kernel: K and V once, a 2-slot ring of (Q_i, grad_i) tiles; the
    query columns in two halves, one per elementwise warpgroup, each with its
    own S^T / dP^T columns (half h: 64h..64h+63) and barriers."""

    def __init__(self, iters, rng):
        super().__init__(rng)
        B = Bar
        self.iters = iters
        self.kv = B("kv", 1)
        self.qfull = [B(f"qfull{i}", 1) for i in range(2)]
        self.qempty = [B(f"qempty{i}", 1) for i in range(2)]
        self.sdp_ready = [B(f"sdp_ready{h}", 1) for h in range(2)]
        self.pds_ready = [B(f"pds_ready{h}", 1) for h in range(2)]
        self.done = B("done", 1)
        self.slot = [None, None]
        self.slot_uses = {}   # tile -> products that read its slot
        self.buf = [None, None]  # per half: ("S", it) or ("P", it) or ("used", it)
        self.acc = [[], []]

    def producer(self):
        self.tma.append(lambda: self.kv.arrive())
        for it in range(self.iters):
            s = it & 1
            yield ("wait", self.qempty[s], ((it >> 1) & 1) ^ 1, (it >> 1) - 1)
            old = self.slot[s]
            if old is not None and self.slot_uses.get(old, 0) < 4:
                raise ProtocolError(f"slot {s} refilled before tile {old} was fully read")
            self.slot[s] = None

            def land(s=s, it=it):
                self.slot[s] = it
                self.qfull[s].arrive()
            self.tma.append(land)

    def _sdp(self, it, h):
        def f():
            if self.slot[it & 1] != it:
                raise ProtocolError(f"S^T({it},{h}) reads slot holding {self.slot[it & 1]}")
            if self.buf[h] is not None and self.buf[h][0] != "used":
                raise ProtocolError(f"S^T({it},{h}) overwrites {self.buf[h]}")
            self.slot_uses[it] = self.slot_uses.get(it, 0) + 1
            self.buf[h] = ("S", it)
        return f

    def _acc(self, it, h):
        def f():
            if self.buf[h] != ("P", it) or self.slot[it & 1] != it:
                raise ProtocolError(f"dV/dK({it},{h}) read {self.buf[h]} and slot {self.slot[it & 1]}")
            self.slot_uses[it] = self.slot_uses.get(it, 0) + 1
            self.buf[h] = ("used", it)
            self.acc[h].append(it)
        return f

    def mma(self):
        if self.iters == 0:
            self.pipe.append(("commit", self.done))
            return
        yield ("wait", self.kv, 0, 0)
        yield ("wait", self.qfull[0], 0, 0)
        for h in range(2):
            self.pipe += [("op", self._sdp(0, h)), ("commit", self.sdp_ready[h])]
        for it in range(self.iters):
            nxt = it + 1 < self.iters
            ns = (it + 1) & 1
            yield ("wait", self.pds_ready[0], it & 1, it)
            self.pipe.append(("op", self._acc(it, 0)))
            if nxt:
                yield ("wait", self.qfull[ns], ((it + 1) >> 1) & 1, (it + 1) >> 1)
                self.pipe += [("op", self._sdp(it + 1, 0)), ("commit", self.sdp_ready[0])]
            yield ("wait", self.pds_ready[1], it & 1, it)
            self.pipe += [("op", self._acc(it, 1)), ("commit", self.qempty[it & 1])]
            if nxt:
                self.pipe += [("op", self._sdp(it + 1, 1)), ("commit", self.sdp_ready[1])]
        self.pipe.append(("commit", self.done))

    def elementwise(self, h):
        for it in range(self.iters):
            yield ("wait", self.sdp_ready[h], it & 1, it)
            if self.buf[h] != ("S", it):
                raise ProtocolError(f"elementwise({it},{h}) reads {self.buf[h]}")
            self.buf[h] = ("P", it)
            self.pds_ready[h].arrive()
        yield ("wait", self.done, 0, 0)
        if self.acc[h] != list(range(self.iters)):
            raise ProtocolError(f"accumulated {self.acc[h]}")

    def go(self):
        self.run([self.producer(), self.mma(), self.elementwise(0), self.elementwise(1)])


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 7, 16])
def test_dq_protocol(n):
    for seed in range(60):
        DqModel(n, random.Random(seed * 31 + n)).go()


@pytest.mark.parametrize("iters", [0, 1, 2, 3, 6, 17])
def test_dkdv_protocol(iters):
    for seed in range(60):
        DkdvModel(iters, random.Random(seed * 17 + iters)).go()


def test_models_catch_mistakes():
    class NoDsFree(DqModel):
        def elementwise(self):
            for item in DqModel.elementwise(self):
                if item[1] is self.ds_free:
                    continue
                yield item

    class EarlyQempty(DkdvModel):
        def mma(self):
            for item in DkdvModel.mma(self):
                # release the slot after the first half's products only
                if item[1] is self.pds_ready[1]:
                    self.pipe.append(("commit", self.qempty[item[3] & 1]))
                    self.pipe[:] = [op for op in self.pipe[:-1] if not (op[0] == "commit" and op[1] in self.qempty)] + self.pipe[-1:]
                yield item

    def caught(cls, arg):
        for seed in range(300):
            try:
                cls(arg, random.Random(seed)).go()
            except ProtocolError:
                return True
        return False

    assert caught(NoDsFree, 5)
    assert caught(EarlyQempty, 6)
