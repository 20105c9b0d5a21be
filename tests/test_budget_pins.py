"""Pins of the per-element error budget (oracle/budget.py).

The budget is an upper bound on how far an implementation of the named
algorithm the kernels use (fp32 scores, online softmax with a lagging
maximum, P rounded to the input dtype, fp32 accumulation, one final
rounding) can be from the exact result.  Two sides are pinned:

* an independent low-precision emulation of that algorithm (numpy float32
  arithmetic, torch for the 16-bit roundings, 128-key tiles with the 2^8
  rescale threshold) stays inside the budget on random inputs, masks, GQA and
  every dtype;
* the budget is tight enough that plausible mistakes leave it: a scale off
  by 0.5 %, one kept key dropped, an lse off by 1e-3.  (A worst-case bound
  does not catch errors that only change the size of random roundings, such
  as P rounded to bf16 instead of fp16: those stay a parity-test matter.)
"""
import numpy as np
import pytest
import torch

from oracle import sdpa
from oracle.budget import forward_budget, unit_roundoff

_TD = {"bfloat16": torch.bfloat16, "float16": torch.float16, "float32": torch.float32}


def _round(x, dtype_name):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(_TD[dtype_name]).to(torch.float32).numpy()


def emulate(q, k, v, dtype_name, *, is_causal=False, scale=None, bias=None, enable_gqa=False, tile=128,
            p_dtype=None, scale_err=1.0, drop_last_key=False):
    """FlashAttention-style forward in float32 with 16-bit roundings."""
    q, k, v = (np.asarray(t, dtype=np.float32) for t in (q, k, v))
    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    g = Hq // Hkv
    s = np.float32((1.0 / np.sqrt(E) if scale is None else scale) * scale_err)
    sl = np.float32(s * np.float32(1.4426950408889634))
    out = np.zeros((B, Hq, L, v.shape[-1]), dtype=np.float32)
    lse = np.zeros((B, Hq, L), dtype=np.float32)
    pd = p_dtype or dtype_name
    for b in range(B):
        for h in range(Hq):
            qa, ka, va = q[b, h], k[b, h // g], v[b, h // g]
            m = np.full((L, 1), -np.inf, dtype=np.float32)
            lsum = np.zeros((L, 1), dtype=np.float32)
            acc = np.zeros((L, va.shape[1]), dtype=np.float32)
            for j0 in range(0, S, tile):
                sc = (qa @ ka[j0:j0 + tile].T).astype(np.float32) * sl  # log2 units
                if bias is not None:
                    sc = sc + np.float32(1.4426950408889634) * bias[b, h, :, j0:j0 + tile].astype(np.float32)
                keys = np.arange(j0, min(S, j0 + tile))
                keep = np.ones((L, len(keys)), dtype=bool)
                if is_causal:
                    keep &= keys[None, :] <= np.arange(L)[:, None]
                if drop_last_key:
                    keep &= keys[None, :] != S - 1
                sc = np.where(keep, sc, -np.inf).astype(np.float32)
                mt = sc.max(axis=1, keepdims=True)
                mn = np.maximum(m, mt)
                need = mn > m + 8
                fac = np.where(need, np.exp2(np.where(need, m - mn, 0)).astype(np.float32), 1).astype(np.float32)
                lsum *= fac
                acc *= fac
                m = np.where(need, mn, m)
                neg = np.where(np.isfinite(m), -m, 0).astype(np.float32)
                with np.errstate(invalid="ignore"):
                    p = np.exp2(sc + neg).astype(np.float32)
                lsum += p.sum(axis=1, keepdims=True, dtype=np.float32)
                pr = _round(p, pd) if pd != "float32" else p
                acc += (pr @ va[j0:j0 + tile]).astype(np.float32)
            with np.errstate(invalid="ignore", divide="ignore"):
                o = np.where(lsum > 0, acc / lsum, 0)
                ls = np.where(lsum > 0, (m + np.log2(lsum)) * np.float32(0.6931471805599453), -np.inf)
            out[b, h] = _round(o, dtype_name) if dtype_name != "float32" else o
            lse[b, h] = ls[:, 0]
    return out, lse


def _inputs(shape_q, shape_k, shape_v, dtype_name, seed):
    rng = np.random.default_rng(seed)
    return tuple(_round(rng.standard_normal(sh), dtype_name).astype(np.float64) for sh in (shape_q, shape_k, shape_v))


CASES = [
    ("bfloat16", (1, 2, 200, 64), (1, 2, 300, 64), (1, 2, 300, 64), dict()),
    ("bfloat16", (1, 2, 257, 128), (1, 2, 257, 128), (1, 2, 257, 128), dict(is_causal=True)),
    ("float16", (2, 4, 130, 96), (2, 2, 260, 96), (2, 2, 260, 96), dict(enable_gqa=True)),
    ("float16", (1, 1, 150, 64), (1, 1, 400, 64), (1, 1, 400, 32), dict(scale=1.0 / 64)),
    ("float32", (1, 2, 100, 40), (1, 2, 170, 40), (1, 2, 170, 24), dict(is_causal=True)),
    ("bfloat16", (1, 1, 64, 32), (1, 1, 300, 32), (1, 1, 300, 32), dict(scale=2.0)),  # peaky weights
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1][2]}x{c[2][2]}x{c[1][3]}-{list(c[4])}")
def test_emulation_stays_inside_the_budget(case):
    dt, sq, sk, sv, kw = case
    q, k, v = _inputs(sq, sk, sv, dt, 7)
    ro, rl = sdpa(q, k, v, **kw)
    tol_o, tol_l = forward_budget(q, k, v, dtype_name=dt, **kw)
    eo, el = emulate(q, k, v, dt, **{a: b for a, b in kw.items() if a != "enable_gqa"})
    assert (np.abs(eo - ro) <= tol_o).all(), float((np.abs(eo - ro) / tol_o).max())
    assert (np.abs(el - rl) <= tol_l).all(), float((np.abs(el - rl) / tol_l).max())
    # and, for 16-bit inputs, the budget is a few unit roundoffs of the output
    # scale: far sharper than the flat 2e-2 (for float32 the worst-case
    # gamma_n terms dominate and the flat 1e-5 bar stays the sharper one)
    scale_o = np.abs(ro).mean() + np.abs(v).mean()
    if dt != "float32":
        assert np.median(tol_o) < 8 * unit_roundoff(dt) * scale_o
    else:
        assert np.median(tol_o) < 1e-3 * scale_o


def test_bias_mask_inside_the_budget():
    dt = "bfloat16"
    q, k, v = _inputs((1, 2, 90, 64), (1, 2, 140, 64), (1, 2, 140, 64), dt, 9)
    bias = np.where(np.random.default_rng(3).random((1, 2, 90, 140)) < 0.2, -np.inf,
                    np.random.default_rng(4).standard_normal((1, 2, 90, 140)))
    ro, rl = sdpa(q, k, v, attn_mask=bias)
    tol_o, tol_l = forward_budget(q, k, v, dtype_name=dt, attn_mask=bias)
    eo, el = emulate(q, k, v, dt, bias=bias)
    assert (np.abs(eo - ro) <= tol_o).all() and (np.abs(el - rl) <= tol_l).all()


@pytest.mark.parametrize("mistake", ["scale", "drop_key", "lse"])
def test_plausible_mistakes_leave_the_budget(mistake):
    dt = "float16"
    q, k, v = _inputs((1, 2, 128, 64), (1, 2, 256, 64), (1, 2, 256, 64), dt, 11)
    ro, rl = sdpa(q, k, v)
    tol_o, tol_l = forward_budget(q, k, v, dtype_name=dt)
    kw = {"scale": dict(scale_err=1.005), "drop_key": dict(drop_last_key=True), "lse": dict()}[mistake]
    eo, el = emulate(q, k, v, dt, **kw)
    if mistake == "lse":
        el = el + 1e-3
    assert (np.abs(eo - ro) > tol_o).any() or (np.abs(el - rl) > tol_l).any()
