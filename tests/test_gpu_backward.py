"""Parity of the CUDA backward (sdpa_bwd through the C ABI) with the float64
backward oracle on the same seeded inputs.

Tolerances, from the arithmetic: the kernels compute in fp32 from the inputs
as given, recompute P from the forward's fp32 logsumexp and take
D_i = grad_i . out_i from the forward's output; every gradient element is one
fp32 sum over a row's or a key's partners, then one rounding to the dtype.
float32: max |diff| <= 1e-4 * max(1, max |ref|) (sums of up to a few thousand
terms in fp32 plus the cancellation in dP - D); bf16/fp16: max |diff| <=
2e-2 * max(1, max |ref|) (the output rounding, 2^-9 relative for bf16, plus
D taken from the 16-bit forward output).  NaN positions must agree.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import sdpa_backward as ref_bwd
from oracle import sdpa_backward_packed as ref_bwd_packed

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import os

    from scaled_dot_product_15_b200 import api, build

    if not os.path.exists(api.LIB_PATH):
        build.build()
    api.load_library()
    assert torch.cuda.is_available(), "these tests need a GPU"


def _tol(dtype):
    return 1e-4 if dtype == torch.float32 else 2e-2


def _check(got, ref, dtype, what):
    for g, r, name in zip(got, ref, ("dq", "dk", "dv")):
        g = g.detach().double().cpu().numpy()
        r = np.asarray(r, dtype=np.float64)
        assert g.shape == r.shape, (what, name, g.shape, r.shape)
        assert np.array_equal(np.isnan(g), np.isnan(r)), f"{what} {name}: NaN positions differ"
        fin = np.isfinite(r)
        tol = _tol(dtype) * max(1.0, np.abs(r[fin]).max(initial=0.0))
        err = np.abs(g[fin] - r[fin]).max(initial=0.0)
        assert err <= tol, f"{what} {name}: max |diff| = {err:.3e} > {tol:.2e}"


def _run(q, k, v, g, **kw):
    from scaled_dot_product_15_b200 import api, sdpa, sdpa_backward

    qd, kd, vd, gd = (t.to(DEV) for t in (q, k, v, g))
    out, lse = sdpa(qd, kd, vd, **kw)
    grads = sdpa_backward(qd, kd, vd, out, lse, gd, **kw)
    torch.cuda.synchronize()
    assert api.take_device_error() == 0
    assert api.last_launch_count() in (1, 2, 3)
    return grads


CASES = [
    # dtype, B, Hq, Hkv, L, S, E, Ev, causal
    (torch.float32, 1, 2, 2, 37, 37, 16, 16, False),
    (torch.float32, 2, 4, 2, 50, 70, 40, 24, True),
    (torch.bfloat16, 1, 2, 2, 300, 300, 128, 128, True),
    (torch.bfloat16, 2, 8, 2, 129, 129, 64, 64, False),
    (torch.float16, 1, 3, 3, 257, 257, 96, 96, True),
    (torch.float16, 1, 2, 2, 40, 200, 64, 32, False),
    (torch.bfloat16, 1, 2, 1, 300, 100, 128, 128, True),   # L > S: rows past S keep every key
    (torch.float16, 1, 1, 1, 1, 64, 256, 256, False),      # one query row, widest head
    (torch.float16, 1, 2, 2, 17, 400, 96, 96, False),      # few rows, several key tiles, ragged
    (torch.bfloat16, 2, 4, 2, 700, 700, 128, 128, True),   # several tiles both ways, GQA
    (torch.bfloat16, 1, 2, 2, 129, 640, 64, 64, True),     # causal with S > L
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_backward_small(case):
    dt, B, Hq, Hkv, L, S, E, Ev, causal = case
    q, k, v = W.randn((B, Hq, L, E), 401, dt), W.randn((B, Hkv, S, E), 402, dt), W.randn((B, Hkv, S, Ev), 403, dt)
    g = W.randn((B, Hq, L, Ev), 404, dt)
    from scaled_dot_product_15_b200.api import backward_plan

    want = "backward_tcgen05" if (dt != torch.float32 and E == Ev and E in (64, 96, 128)) else "backward_simt"
    qd = q.to(DEV)
    assert backward_plan(qd, k.to(DEV), v.to(DEV), g.to(DEV), mask_kind=1 if causal else 0) == want
    got = _run(q, k, v, g, is_causal=causal, enable_gqa=Hq != Hkv)
    ref = ref_bwd(q, k, v, g, is_causal=causal, enable_gqa=Hq != Hkv)
    _check(got, ref, dt, str(case))


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_backward_masks_and_scale(dt):
    B, H, L, S, E = 1, 2, 48, 64, 32
    q, k, v = W.randn((B, H, L, E), 411, dt), W.randn((B, H, S, E), 412, dt), W.randn((B, H, S, E), 413, dt)
    g = W.randn((B, H, L, E), 414, dt)
    mask = torch.rand((B, H, L, S), generator=torch.Generator().manual_seed(5)) > 0.3
    mask[0, 1, 7] = False  # a row with no kept key: contributes 0
    got = _run(q, k, v, g, attn_mask=mask, scale=0.37)
    ref = ref_bwd(q, k, v, g, attn_mask=mask, scale=0.37)
    _check(got, ref, dt, "bool mask")
    assert (got[0][0, 1, 7] == 0).all()
    bias = W.randn((1, 1, L, S), 415, torch.float32)
    got = _run(q, k, v, g, attn_mask=bias)
    ref = ref_bwd(q, k, v, g, attn_mask=bias)
    _check(got, ref, dt, "float bias")


def test_backward_nan_row():
    dt = torch.float32
    q, k, v = W.randn((1, 1, 20, 16), 421, dt), W.randn((1, 1, 30, 16), 422, dt), W.randn((1, 1, 30, 16), 423, dt)
    g = W.randn((1, 1, 20, 16), 424, dt)
    q[0, 0, 5, 3] = float("nan")
    got = _run(q, k, v, g)
    ref = ref_bwd(q, k, v, g)
    _check(got, ref, dt, "NaN row")
    assert torch.isnan(got[1]).all() and torch.isnan(got[2]).all()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_packed_varlen(causal):
    dt = torch.float16
    seqlens = [100, 3, 260, 1, 77]
    T, H, E = sum(seqlens), 4, 64
    q, k, v, g = (W.randn((1, T, H, E), 430 + i, dt) for i in range(4))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(seqlens)]), dtype=torch.int32, device=DEV)
    got = _run(q, k, v, g, is_causal=causal, layout="bmhk", cu_seqlens=cu, max_seqlen=max(seqlens))
    ref = ref_bwd_packed(q, k, v, g, seqlens, causal=causal)
    _check(got, ref, dt, f"varlen causal={causal}")


def test_autograd_op_matches_backward():
    from scaled_dot_product_15_b200 import attention

    dt = torch.bfloat16
    q, k, v = (W.randn((1, 4, 200, 64), 440 + i, dt).to(DEV).requires_grad_() for i in range(3))
    g = W.randn((1, 4, 200, 64), 443, dt).to(DEV)
    out = attention(q, k, v, is_causal=True)
    out.backward(g)
    ref = ref_bwd(q.detach().cpu(), k.detach().cpu(), v.detach().cpu(), g.cpu(), is_causal=True)
    _check((q.grad, k.grad, v.grad), ref, dt, "autograd")


def test_backward_full_headline_sampled_heads():
    """The headline shape (bf16 causal 4 x 16 x 2048 x 128) in one call; two
    (batch, head) pairs are checked completely against the oracle."""
    w = W.WORKLOADS["bf16_causal_b4_h16_l2048_e128"]
    q, k, v = W.make_inputs(w)
    g = W.randn(tuple(q.shape), 450, q.dtype)
    dq, dk, dv = _run(q, k, v, g, is_causal=True)
    for b, h in ((0, 0), (3, 11)):
        ref = ref_bwd(q[b : b + 1, h : h + 1], k[b : b + 1, h : h + 1], v[b : b + 1, h : h + 1],
                      g[b : b + 1, h : h + 1], is_causal=True)
        got = (dq[b : b + 1, h : h + 1], dk[b : b + 1, h : h + 1], dv[b : b + 1, h : h + 1])
        _check(got, ref, q.dtype, f"headline b={b} h={h}")


BUDGET_CASES = [
    # dtype, B, Hq, Hkv, L, S, E, causal   (16-bit E in {64, 96, 128}: tcgen05 kernels)
    (torch.bfloat16, 1, 2, 2, 300, 300, 128, True),
    (torch.float16, 1, 4, 2, 257, 130, 96, False),
    (torch.bfloat16, 1, 2, 1, 129, 640, 64, True),
    (torch.float16, 1, 2, 2, 90, 70, 32, False),      # general kernels
    (torch.float32, 1, 2, 2, 80, 120, 40, True),
]


@pytest.mark.parametrize("case", BUDGET_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_backward_within_the_error_budget(case):
    """Every gradient element inside the per-element budget of the
    FlashAttention backward (oracle/budget.py, backward_budget), which takes
    the forward's own budget into the recomputed weights and D."""
    from oracle.budget import backward_budget

    dt, B, Hq, Hkv, L, S, E, causal = case
    q, k, v = W.randn((B, Hq, L, E), 541, dt), W.randn((B, Hkv, S, E), 542, dt), W.randn((B, Hkv, S, E), 543, dt)
    g = W.randn((B, Hq, L, E), 544, dt)
    got = _run(q, k, v, g, is_causal=causal, enable_gqa=Hq != Hkv)
    ref = ref_bwd(q, k, v, g, is_causal=causal, enable_gqa=Hq != Hkv)
    name = {torch.float32: "float32", torch.float16: "float16", torch.bfloat16: "bfloat16"}[dt]
    tols = backward_budget(q, k, v, g, dtype_name=name, is_causal=causal, enable_gqa=Hq != Hkv)
    for gr, r, t, what in zip(got, ref, tols, ("dq", "dk", "dv")):
        e = np.abs(gr.detach().double().cpu().numpy() - np.asarray(r))
        assert (e <= t).all(), f"{what} outside the budget: max ratio {float((e / t).max()):.2f}"
