"""Parity of the CUDA library with the float64 oracle on the same seeded inputs.

Tolerances (stated for the method): float32 max |diff| <= 1e-5 * max(1, max|ref|)
on O and on lse; bf16/fp16 max |diff| <= 2e-2 on O and <= 1e-2 on lse.  NaN
and infinity positions must agree exactly.

Small cases are compared element by element; the full-size workloads, in the
launch configuration the benchmark times, on sampled rows that the oracle
computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import sdpa as ref_sdpa
from oracle import sdpa_packed as ref_packed

pytestmark = pytest.mark.gpu

DEV = "cuda"
O_TOL = {torch.float16: 2e-2, torch.bfloat16: 2e-2}
L_TOL = {torch.float16: 1e-2, torch.bfloat16: 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from scaled_dot_product_15_b200 import api, build

    import os

    if not os.path.exists(api.LIB_PATH):
        build.build()
    api.load_library()
    assert torch.cuda.is_available(), "these tests need a GPU"


def _sdpa(*a, **k):
    from scaled_dot_product_15_b200 import api, sdpa

    out, lse = sdpa(*a, **k)
    torch.cuda.synchronize()
    assert api.take_device_error() == 0, "a kernel gave up on a bounded wait"
    return out, lse


def _plan(*a, **k):
    from scaled_dot_product_15_b200 import plan

    return plan(*a, **k)


def assert_close(out, lse, ref_o, ref_l, dtype, what=""):
    got_o = out.detach().double().cpu().numpy() if torch.is_tensor(out) else np.asarray(out)
    got_l = lse.detach().double().cpu().numpy() if torch.is_tensor(lse) else np.asarray(lse)
    ref_o = np.asarray(ref_o, dtype=np.float64)
    ref_l = np.asarray(ref_l, dtype=np.float64)
    assert got_o.shape == ref_o.shape, (got_o.shape, ref_o.shape)
    assert got_l.shape == ref_l.shape, (got_l.shape, ref_l.shape)
    for g, r, name in ((got_o, ref_o, "O"), (got_l, ref_l, "lse")):
        assert np.array_equal(np.isnan(g), np.isnan(r)), f"{what} {name}: NaN positions differ"
        fin = np.isfinite(r)
        assert np.array_equal(g[~fin & ~np.isnan(r)], r[~fin & ~np.isnan(r)]), f"{what} {name}: inf differ"
    fo, fl = np.isfinite(ref_o), np.isfinite(ref_l)
    if dtype == torch.float32:
        to = 1e-5 * max(1.0, np.abs(ref_o[fo]).max(initial=0.0))
        tl = 1e-5 * max(1.0, np.abs(ref_l[fl]).max(initial=0.0))
    else:
        to, tl = O_TOL[dtype], L_TOL[dtype]
    eo = np.abs(got_o[fo] - ref_o[fo]).max(initial=0.0)
    el = np.abs(got_l[fl] - ref_l[fl]).max(initial=0.0)
    assert eo <= to, f"{what}: max |dO| = {eo:.3e} > {to:.1e}"
    assert el <= tl, f"{what}: max |dlse| = {el:.3e} > {tl:.1e}"
    return eo, el


def _rand(shape, seed, dtype):
    return W.randn(shape, seed, dtype)


# ---------------------------------------------------------------- small, full compare


@pytest.mark.parametrize("name", ["fp32_b1_h2_l64_e16", "fp32_b1_h2_l64_e16_causal"])
def test_fp32_small_workload(name):
    w = W.WORKLOADS[name]
    q, k, v = W.make_inputs(w)
    for _ in range(2):  # run twice: same result
        out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=w.mask == "causal")
        ro, rl = ref_sdpa(q, k, v, is_causal=w.mask == "causal")
        assert_close(out, lse, ro, rl, torch.float32, name)


PREFILL_CASES = [
    # dtype, B, Hq, Hkv, L, S, E, Ev, causal
    (torch.bfloat16, 1, 2, 2, 300, 300, 128, 128, True),
    (torch.bfloat16, 2, 2, 2, 256, 256, 128, 128, False),
    (torch.float16, 1, 2, 2, 200, 333, 64, 64, False),
    (torch.float16, 1, 2, 2, 257, 257, 96, 96, True),
    (torch.float16, 1, 3, 3, 129, 129, 64, 64, True),
    (torch.bfloat16, 1, 8, 2, 200, 200, 128, 128, True),   # GQA prefill
    (torch.bfloat16, 1, 2, 2, 300, 100, 128, 128, True),   # L > S: rows past S keep all keys
    (torch.float16, 1, 2, 2, 17, 400, 96, 96, False),
    (torch.bfloat16, 1, 2, 2, 70, 70, 32, 48, False),     # odd head sizes: general kernel
    (torch.float32, 1, 2, 2, 100, 77, 40, 24, True),
    (torch.bfloat16, 1, 2, 2, 1, 300, 128, 128, True),    # one query row: key 0 only
    (torch.float16, 2, 4, 4, 700, 700, 128, 128, True),   # several 256-row blocks, ragged tail
    (torch.bfloat16, 1, 2, 2, 513, 1500, 64, 64, False),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_prefill_small(case):
    dt, B, Hq, Hkv, L, S, E, Ev, causal = case
    q = _rand((B, Hq, L, E), 101, dt)
    k = _rand((B, Hkv, S, E), 102, dt)
    v = _rand((B, Hkv, S, Ev), 103, dt)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    want = "prefill_tcgen05" if (dt != torch.float32 and E == Ev and E in (64, 96, 128)) else "simt"
    assert _plan(qd, kd, vd, mask_kind=1 if causal else 0) == want
    out, lse = _sdpa(qd, kd, vd, is_causal=causal, enable_gqa=Hq != Hkv)
    ro, rl = ref_sdpa(q, k, v, is_causal=causal, enable_gqa=Hq != Hkv)
    assert_close(out, lse, ro, rl, dt, str(case))


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("order", ["growing", "shrinking"])
def test_prefill_row_maximum_moves_across_tiles(dt, causal, order):
    """Key norms that grow (or shrink) from tile to tile make every row's
    maximum jump by far more than the 2^8 the kernel lets its running maximum
    lag: the rescale of O and the recomputation of a tile's weights must both
    be exact."""
    B, H, L, S, E = 1, 2, 300, 1024, 64
    q = _rand((B, H, L, E), 301, torch.float32)
    k = _rand((B, H, S, E), 302, torch.float32)
    v = _rand((B, H, S, E), 303, torch.float32)
    t = torch.arange(S, dtype=torch.float32) // 128
    gain = 1.0 + 3.2 * (t if order == "growing" else (t.max() - t))
    k = k * gain[None, None, :, None]
    q, k, v = q.to(dt), k.to(dt), v.to(dt)
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=causal)
    ro, rl = ref_sdpa(q, k, v, is_causal=causal)
    assert_close(out, lse, ro, rl, dt, f"{order} causal={causal}")


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_zero_head_size_logits_are_the_mask(dt):
    """E = 0: every dot product is 0, so only the mask shapes the logits
    (exactref "Full specification"); without a mask the weights are uniform."""
    B, H, L, S, Ev = 1, 2, 40, 70, 32
    q = torch.empty((B, H, L, 0), dtype=dt)
    k = torch.empty((B, H, S, 0), dtype=dt)
    v = _rand((B, H, S, Ev), 501, dt)
    bias = W.randn((1, H, L, S), 502, torch.float32)
    for kw in (dict(), dict(is_causal=True), dict(attn_mask=bias)):
        out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), **kw)
        ro, rl = ref_sdpa(q, k, v, **kw)
        assert_close(out, lse, ro, rl, dt, f"E=0 {list(kw)}")
    from oracle import sdpa_backward as ref_bwd
    from scaled_dot_product_15_b200 import sdpa, sdpa_backward

    g = _rand((B, H, L, Ev), 503, dt)
    out, lse = sdpa(q.to(DEV), k.to(DEV), v.to(DEV), attn_mask=bias)
    dq, dk, dv = sdpa_backward(q.to(DEV), k.to(DEV), v.to(DEV), out, lse, g.to(DEV), attn_mask=bias)
    rq, rk, rv = ref_bwd(q, k, v, g, attn_mask=bias)
    assert dq.shape == q.shape and dk.shape == k.shape
    tol = (1e-4 if dt == torch.float32 else 2e-2) * max(1.0, float(np.abs(rv).max()))
    assert float(np.abs(dv.double().cpu().numpy() - rv).max()) <= tol


def test_bmghk_layout_is_grouped_query_attention():
    """xFormers BMGHK (G key/value groups, H query heads per group, the key's
    H axis broadcast) equals GQA with contiguous grouping, on the oracle."""
    from scaled_dot_product_15_b200 import sdpa

    dt = torch.bfloat16
    B, M, G, H, K = 2, 300, 2, 4, 128
    q = _rand((B, M, G, H, K), 511, dt)
    kk = _rand((B, M, G, 1, K), 512, dt).expand(B, M, G, H, K)
    vv = _rand((B, M, G, 1, K), 513, dt).expand(B, M, G, H, K)
    out, lse = sdpa(q.to(DEV), kk.to(DEV), vv.to(DEV), is_causal=True, layout="bmghk")
    torch.cuda.synchronize()
    assert out.shape == (B, M, G, H, K) and lse.shape == (B, G, H, M)
    # the oracle on (B, G*H, M, K) with key/value heads = G
    qo = q.reshape(B, M, G * H, K).permute(0, 2, 1, 3)
    ko = kk[:, :, :, 0].permute(0, 2, 1, 3)
    vo = vv[:, :, :, 0].permute(0, 2, 1, 3)
    ro, rl = ref_sdpa(qo, ko, vo, is_causal=True, enable_gqa=True)
    assert_close(out.reshape(B, M, G * H, K).permute(0, 2, 1, 3), lse.reshape(B, G * H, M), ro, rl, dt, "bmghk")


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_empty_dimensions(dt):
    """No keys: every row has no kept key (out 0, lse -inf); no query rows or
    no batch: nothing is written and nothing fails; the gradients of a
    problem without keys are zero for the queries."""
    from scaled_dot_product_15_b200 import sdpa, sdpa_backward

    q = _rand((2, 3, 17, 64), 521, dt).to(DEV)
    k0 = torch.empty((2, 3, 0, 64), dtype=dt, device=DEV)
    v0 = torch.empty((2, 3, 0, 64), dtype=dt, device=DEV)
    out, lse = _sdpa(q, k0, v0)
    assert (out == 0).all() and torch.isneginf(lse).all()
    g = _rand((2, 3, 17, 64), 522, dt).to(DEV)
    dq, dk, dv = sdpa_backward(q, k0, v0, out, lse, g)
    torch.cuda.synchronize()
    assert (dq == 0).all() and dk.numel() == 0 and dv.numel() == 0
    k = _rand((2, 3, 9, 64), 523, dt).to(DEV)
    v = _rand((2, 3, 9, 64), 524, dt).to(DEV)
    out, lse = _sdpa(q[:, :, :0], k, v)
    assert out.shape == (2, 3, 0, 64) and lse.shape == (2, 3, 0)
    dq, dk, dv = sdpa_backward(q[:, :, :0], k, v, out, lse, out)
    torch.cuda.synchronize()
    assert (dk == 0).all() and (dv == 0).all()
    out, lse = _sdpa(q[:0], k[:0], v[:0])
    assert out.numel() == 0


BUDGET_CASES = [
    # dtype, B, Hq, Hkv, L, S, E, causal
    (torch.bfloat16, 1, 2, 2, 300, 300, 128, True),
    (torch.float16, 1, 2, 2, 257, 257, 96, True),
    (torch.bfloat16, 1, 8, 2, 200, 200, 128, False),
    (torch.float16, 1, 2, 2, 200, 333, 64, False),
    (torch.bfloat16, 2, 8, 2, 1, 3000, 128, False),   # decode kernel
    (torch.float32, 1, 2, 2, 100, 77, 40, True),      # general kernel
]


@pytest.mark.parametrize("case", BUDGET_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_within_the_error_budget(case):
    """Element by element inside the per-element error budget of the
    exactref tolerance model for the algorithm the kernels implement
    (oracle/budget.py), which for 16-bit inputs is far sharper than the flat
    2e-2."""
    from oracle.budget import forward_budget

    dt, B, Hq, Hkv, L, S, E, causal = case
    q, k, v = _rand((B, Hq, L, E), 531, dt), _rand((B, Hkv, S, E), 532, dt), _rand((B, Hkv, S, E), 533, dt)
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=causal, enable_gqa=Hq != Hkv)
    ro, rl = ref_sdpa(q, k, v, is_causal=causal, enable_gqa=Hq != Hkv)
    name = {torch.float32: "float32", torch.float16: "float16", torch.bfloat16: "bfloat16"}[dt]
    to, tl = forward_budget(q, k, v, dtype_name=name, is_causal=causal, enable_gqa=Hq != Hkv)
    eo = np.abs(out.double().cpu().numpy() - ro)
    el = np.abs(lse.double().cpu().numpy() - rl)
    assert (eo <= to).all(), f"out outside the budget: max ratio {float((eo / to).max()):.2f}"
    assert (el <= tl).all(), f"lse outside the budget: max ratio {float((el / tl).max()):.2f}"


DECODE_CASES = [
    # dtype, B, Hq, Hkv, L, S, E
    (torch.bfloat16, 2, 8, 2, 1, 3000, 128),
    (torch.float16, 3, 4, 4, 1, 100, 64),
    (torch.bfloat16, 1, 8, 1, 1, 5000, 256),
    (torch.float16, 2, 8, 2, 2, 1025, 128),     # 8 rows per key head
    (torch.bfloat16, 1, 2, 1, 1, 1, 128),       # one cached key
    (torch.bfloat16, 1, 1, 1, 3, 20000, 64),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_decode_small(case):
    dt, B, Hq, Hkv, L, S, E = case
    q = _rand((B, Hq, L, E), 201, dt)
    k = _rand((B, Hkv, S, E), 202, dt)
    v = _rand((B, Hkv, S, E), 203, dt)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    assert _plan(qd, kd, vd) == "decode_split"
    out, lse = _sdpa(qd, kd, vd, enable_gqa=Hq != Hkv)
    ro, rl = ref_sdpa(q, k, v, enable_gqa=Hq != Hkv)
    assert_close(out, lse, ro, rl, dt, str(case))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dt,E", [(torch.float16, 64), (torch.bfloat16, 128), (torch.float16, 96)])
def test_varlen_small(causal, dt, E):
    seqlens = [5, 130, 1, 257, 64, 300, 128]
    T, H = sum(seqlens), 2
    q = _rand((1, T, H, E), 301, dt)
    k = _rand((1, T, H, E), 302, dt)
    v = _rand((1, T, H, E), 303, dt)
    cu = torch.tensor(W.cu_seqlens_of(seqlens), dtype=torch.int32, device=DEV)
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=causal, cu_seqlens=cu, max_seqlen=max(seqlens))
    ro, rl = ref_packed(q, k, v, seqlens, causal=causal)
    assert_close(out, lse[0], ro, rl, dt, f"varlen causal={causal}")


def test_bmhk_layout_and_strided_views():
    dt = torch.bfloat16
    q = _rand((2, 150, 4, 128), 401, dt)
    k = _rand((2, 150, 4, 128), 402, dt)
    v = _rand((2, 150, 4, 128), 403, dt)
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True, layout="bmhk")
    ro, rl = ref_sdpa(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=True)
    assert_close(out.transpose(1, 2), lse, ro, rl, dt, "bmhk")
    # BHLE views of the same memory (non-contiguous strides)
    out2, lse2 = _sdpa(q.to(DEV).transpose(1, 2), k.to(DEV).transpose(1, 2), v.to(DEV).transpose(1, 2),
                       is_causal=True)
    assert_close(out2, lse2, ro, rl, dt, "bhle view")


def test_masks_and_special_values():
    dt = torch.float16
    B, H, L, S, E = 1, 2, 40, 50, 64
    q = _rand((B, H, L, E), 501, dt)
    k = _rand((B, H, S, E), 502, dt)
    v = _rand((B, H, S, E), 503, dt)
    g = torch.Generator().manual_seed(504)
    bias = torch.randn(B, 1, L, S, generator=g)
    bias[..., 7] = float("-inf")
    bias[0, 0, 3, :] = float("-inf")       # a row with no kept key
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), attn_mask=bias.to(DEV))
    ro, rl = ref_sdpa(q, k, v, attn_mask=bias)
    assert_close(out, lse, ro, rl, dt, "float bias")
    assert (out[0, :, 3] == 0).all() and torch.isneginf(lse[0, :, 3]).all()
    boolm = torch.rand(L, S, generator=g) > 0.5
    boolm[5] = False
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), attn_mask=boolm.to(DEV))
    ro, rl = ref_sdpa(q, k, v, attn_mask=boolm)
    assert_close(out, lse, ro, rl, dt, "bool mask")
    qn = q.clone()
    qn[0, 1, 9, 0] = float("nan")
    out, lse = _sdpa(qn.to(DEV), k.to(DEV), v.to(DEV))
    ro, rl = ref_sdpa(qn, k, v)
    assert_close(out, lse, ro, rl, dt, "NaN row")
    assert torch.isnan(out[0, 1, 9]).all()


@pytest.mark.parametrize("scale", [1.0, 1.0 / 96, 0.0])
def test_explicit_scales(scale):
    dt = torch.float16
    q = _rand((1, 2, 130, 96), 601, dt)
    k = _rand((1, 2, 130, 96), 602, dt)
    v = _rand((1, 2, 130, 96), 603, dt)
    out, lse = _sdpa(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True, scale=scale)
    ro, rl = ref_sdpa(q, k, v, is_causal=True, scale=scale)
    assert_close(out, lse, ro, rl, dt, f"scale={scale}")


def test_dropout_and_dtype_errors():
    q = torch.zeros(1, 1, 4, 64, dtype=torch.float16, device=DEV)
    with pytest.raises(ValueError, match="dropout_p must be 0"):
        _sdpa(q, q, q, dropout_p=0.1)
    with pytest.raises(ValueError):
        _sdpa(q, q.to(torch.bfloat16), q)


# ---------------------------------------------------------------- full sizes, sampled


def _causal_rows_bias(rows, S):
    j = np.arange(S)[None, :]
    return np.where(j <= np.asarray(rows)[:, None], 0.0, -np.inf)


def _sampled_prefill_check(w, samples, rows):
    q, k, v = W.make_inputs(w, DEV)
    causal = w.mask == "causal"
    assert _plan(q, k, v, mask_kind=1 if causal else 0) == "prefill_tcgen05"
    out, lse = _sdpa(q, k, v, is_causal=causal, scale=w.scale)
    worst = (0.0, 0.0)
    for b, h in samples:
        qs = W.make_slice(w, "q", b)[h][rows][None, None]
        ks = W.make_slice(w, "k", b)[h // (w.Hq // w.Hkv)][None, None]
        vs = W.make_slice(w, "v", b)[h // (w.Hq // w.Hkv)][None, None]
        bias = _causal_rows_bias(rows, w.S) if causal else None
        ro, rl = ref_sdpa(qs, ks, vs, attn_mask=bias, scale=w.scale)
        e = assert_close(out[b, h, rows][None, None], lse[b, h, rows][None, None], ro, rl, w.torch_dtype,
                         f"{w.name} b={b} h={h}")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return out, lse, worst


ROWS_2048 = [0, 1, 2, 63, 127, 128, 129, 255, 511, 1000, 1023, 1024, 1500, 2046, 2047]


def test_full_bf16_causal_prefill_sampled():
    w = W.WORKLOADS["bf16_causal_b4_h16_l2048_e128"]
    _sampled_prefill_check(w, [(0, 0), (1, 7), (3, 15)], ROWS_2048)


@pytest.mark.parametrize("name", ["fp16_causal_b1_h64_l2048_e96", "fp16_causal_b1_h64_l2048_e96_scale1_96"])
def test_full_fp16_hd96_sampled(name):
    w = W.WORKLOADS[name]
    out, lse, _ = _sampled_prefill_check(w, [(0, 0), (0, 31), (0, 63)], ROWS_2048)
    if w.scale is not None:
        # double-scaled: logits ~ N(0, 1/96), so over n >= 256 kept keys the
        # weights are near-uniform and lse ~ log(n) + (a few thousandths)
        i = torch.arange(2048, device=DEV, dtype=torch.float32)
        gap = lse[0] - torch.log(i + 1)
        assert gap[:, 255:].abs().max().item() < 0.05
        assert 0.0 < gap[:, 255:].mean().item() < 0.02


def test_full_fp16_varlen_sampled():
    w = W.WORKLOADS["fp16_varlen_t32768_h8_e64"]
    seqlens = W.workload_seqlens(w)
    q, k, v = W.make_inputs(w, DEV)
    cu = torch.tensor(W.cu_seqlens_of(seqlens), dtype=torch.int32, device=DEV)
    out, lse = _sdpa(q, k, v, is_causal=True, cu_seqlens=cu, max_seqlen=max(seqlens))
    qc, kc, vc = W.make_inputs(w, "cpu")
    heads = [0, 5]
    ro, rl = ref_packed(qc, kc, vc, seqlens, causal=True, heads=heads)
    assert_close(out[:, :, heads], lse[0][heads], ro[:, :, heads], rl[heads], w.torch_dtype, w.name)


def test_full_bf16_gqa_decode_sampled():
    w = W.WORKLOADS["bf16_gqa_decode_b64_hq32_hkv8_s16384_e128"]
    q, k, v = W.make_inputs(w, DEV)
    assert _plan(q, k, v) == "decode_split"
    out, lse = _sdpa(q, k, v, enable_gqa=True)
    g = w.Hq // w.Hkv
    for b, kvh in [(0, 0), (17, 3), (63, 7)]:
        qs = W.make_slice(w, "q", b)[kvh * g:(kvh + 1) * g][None]
        ks = W.make_slice(w, "k", b)[kvh][None, None]
        vs = W.make_slice(w, "v", b)[kvh][None, None]
        ro, rl = ref_sdpa(qs, ks, vs, enable_gqa=True)
        assert_close(out[b, kvh * g:(kvh + 1) * g][None], lse[b, kvh * g:(kvh + 1) * g][None], ro, rl,
                     w.torch_dtype, f"decode b={b} kvh={kvh}")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_native_bool_mask_matches_its_bias_form(dt):
    """A bool mask passed natively (one byte per element, broadcast over
    heads) gives the same result as the same mask written as a 0 / -inf
    float bias, and both match the oracle; a NaN score under a removed key
    still makes its row NaN, as a bias would."""
    from scaled_dot_product_15_b200 import plan

    B, Hq, Hkv, L, S, E = 2, 4, 2, 70, 90, 64
    q, k, v = _rand((B, Hq, L, E), 521, dt), _rand((B, Hkv, S, E), 522, dt), _rand((B, Hkv, S, E), 523, dt)
    m = torch.rand((B, 1, L, S), generator=torch.Generator().manual_seed(524)) > 0.4
    m[1, 0, 11] = False                     # a row with no visible key
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    assert plan(qd, kd, vd, mask_kind=5) == "simt"
    out, lse = _sdpa(qd, kd, vd, attn_mask=m.to(DEV), enable_gqa=True)
    bias = torch.where(m, 0.0, float("-inf"))
    ob, lb = _sdpa(qd, kd, vd, attn_mask=bias.to(DEV), enable_gqa=True)
    assert torch.equal(out, ob) and torch.equal(lse, lb)
    ro, rl = ref_sdpa(q, k, v, attn_mask=m, enable_gqa=True)
    assert_close(out, lse, ro, rl, dt, "native bool mask")
    assert (out[1, :, 11] == 0).all() and torch.isneginf(lse[1, :, 11]).all()
    qn = q.clone()
    qn[0, 0, 3, 0] = float("nan")           # NaN in every score of row 3 of head 0
    m2 = m.clone()
    m2[0, 0, 3, :5] = False
    out, lse = _sdpa(qn.to(DEV), kd, vd, attn_mask=m2.to(DEV), enable_gqa=True)
    ro, rl = ref_sdpa(qn, k, v, attn_mask=m2, enable_gqa=True)
    assert_close(out, lse, ro, rl, dt, "NaN under removed keys")
    assert torch.isnan(out[0, 0, 3]).all()
