"""Pins of the backward's per-element error budget (oracle/budget.py,
``backward_budget``).

Two sides, as for the forward:

* an independent low-precision emulation of the FlashAttention-style
  backward the kernels run (the forward emulated first, its output rounded
  to the input dtype and its fp32 logsumexp kept; then per key tile P
  recomputed in fp32 from the logsumexp, dP = grad V^T in fp32,
  D = rowsum(grad * out), dS = P (dP - D), P and dS rounded to the input
  dtype before the products, fp32 accumulators, one final rounding) stays
  inside the budget on random inputs, causal masks, GQA and every dtype;
* plausible mistakes leave it: the scale left out of dK, D taken from the
  unrounded P V of another row, dS without the subtraction of D, one key's
  contribution to dV dropped.
"""
import numpy as np
import pytest
import torch

from oracle import sdpa_backward
from oracle.budget import backward_budget
from tests.test_budget_pins import _round, emulate

L2E = np.float32(1.4426950408889634)


def emulate_backward(q, k, v, g, dtype_name, *, is_causal=False, scale=None, tile=128, mistake=None):
    q, k, v, g = (np.asarray(t, dtype=np.float32) for t in (q, k, v, g))
    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    grp = Hq // Hkv
    out, lse = emulate(q, k, v, dtype_name, is_causal=is_causal, scale=scale)
    s = np.float32(1.0 / np.sqrt(E) if scale is None else scale)
    rnd = (lambda x: _round(x, dtype_name)) if dtype_name != "float32" else (lambda x: x)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kv = h // grp
            qa, ka, va, ga = q[b, h], k[b, kv], v[b, kv], g[b, h]
            D = (ga * out[b, h]).sum(axis=1, keepdims=True, dtype=np.float32)
            if mistake == "D_row":
                D = np.roll(D, 1, axis=0)
            l2 = (lse[b, h] * L2E).astype(np.float32)[:, None]
            acc_q = np.zeros((L, E), dtype=np.float32)
            for j0 in range(0, S, tile):
                kt, vt = ka[j0:j0 + tile], va[j0:j0 + tile]
                sc = (qa @ kt.T).astype(np.float32) * np.float32(s * L2E)
                keys = np.arange(j0, min(S, j0 + tile))
                if is_causal:
                    sc = np.where(keys[None, :] <= np.arange(L)[:, None], sc, -np.inf).astype(np.float32)
                with np.errstate(invalid="ignore"):
                    p = np.where(np.isfinite(l2), np.exp2(sc - l2), 0).astype(np.float32)
                dp = (ga @ vt.T).astype(np.float32)
                ds = p * (dp if mistake == "no_D" else dp - D)
                pr, dsr = rnd(p), rnd(ds)
                contrib_v = (pr.T @ ga).astype(np.float32)
                if mistake == "drop_dv_key" and j0 == 0:
                    contrib_v[0] = 0
                dv[b, kv, j0:j0 + tile] += contrib_v
                sk = np.float32(1.0) if mistake == "dk_scale" else s
                dk[b, kv, j0:j0 + tile] += (dsr.T @ qa).astype(np.float32) * sk
                acc_q += (dsr @ kt).astype(np.float32)
            dq[b, h] = acc_q * s
    return rnd(dq), rnd(dk), rnd(dv)


def _inputs(shapes, dtype_name, seed):
    rng = np.random.default_rng(seed)
    return tuple(_round(rng.standard_normal(sh), dtype_name).astype(np.float64) for sh in shapes)


CASES = [
    ("bfloat16", (1, 2, 200, 64), (1, 2, 300, 64), (1, 2, 300, 64), dict()),
    ("bfloat16", (1, 2, 257, 128), (1, 2, 257, 128), (1, 2, 257, 128), dict(is_causal=True)),
    ("float16", (1, 4, 130, 96), (1, 2, 260, 96), (1, 2, 260, 96), dict(enable_gqa=True)),
    ("float16", (1, 1, 150, 64), (1, 1, 200, 64), (1, 1, 200, 32), dict(scale=2.0 / 64)),
    ("float32", (1, 2, 100, 40), (1, 2, 170, 40), (1, 2, 170, 24), dict(is_causal=True)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1][2]}x{c[2][2]}x{c[1][3]}-{list(c[4])}")
def test_backward_emulation_stays_inside_the_budget(case):
    dt, sq, sk, sv, kw = case
    q, k, v, g = _inputs((sq, sk, sv, sq[:3] + sv[3:]), dt, 5)
    rq, rk, rv = sdpa_backward(q, k, v, g, **kw)
    tq, tk, tv = backward_budget(q, k, v, g, dtype_name=dt, **kw)
    eq, ek, ev = emulate_backward(q, k, v, g, dt, **{a: b for a, b in kw.items() if a != "enable_gqa"})
    for name, e, r, t in (("dq", eq, rq, tq), ("dk", ek, rk, tk), ("dv", ev, rv, tv)):
        assert (np.abs(e - r) <= t).all(), (name, float((np.abs(e - r) / t).max()))


@pytest.mark.parametrize("mistake", ["dk_scale", "D_row", "no_D", "drop_dv_key"])
def test_plausible_backward_mistakes_leave_the_budget(mistake):
    dt = "float16"
    q, k, v, g = _inputs(((1, 2, 128, 64), (1, 2, 192, 64), (1, 2, 192, 64), (1, 2, 128, 64)), dt, 13)
    rq, rk, rv = sdpa_backward(q, k, v, g)
    tq, tk, tv = backward_budget(q, k, v, g, dtype_name=dt)
    eq, ek, ev = emulate_backward(q, k, v, g, dt, mistake=mistake)
    assert ((np.abs(eq - rq) > tq).any() or (np.abs(ek - rk) > tk).any() or (np.abs(ev - rv) > tv).any())
