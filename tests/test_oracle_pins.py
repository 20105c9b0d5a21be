"""Pins for the float64 oracle: checks against what the pages and mathematics
fix, never against the oracle's own formula retyped.

Sources:
- exactref.ai "scaled_dot_product_attention": the worked example and its
  causal / masked / scale-1 variants ("Examples", "Masks, causality and
  scale"), the GQA example, "Special values and dropout", "Padding masks",
  "Full specification".
- hourtab.com xFormers post ("Why double scaling makes attention uniform"):
  scale 1/E makes the weights near-uniform.
- lynx-cortex "Break 00" and khchao.com NN-lab ("Variance stabilization"):
  Var(q.k) = d_k for iid zero-mean unit-variance q, k.
- insureai360 xFormers tutorial, section 4: packed block-diagonal attention
  equals per-segment attention.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

from oracle import default_scale, sdpa, sdpa_packed

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f32(x):
    return np.asarray(x, dtype=np.float32)


# ---------------------------------------------------------------- worked example


@pytest.fixture(scope="module")
def ex():
    return _golden("worked_example.json")


def _qkv(ex):
    return (np.array(ex["q"], dtype=np.float32), np.array(ex["k"], dtype=np.float32),
            np.array(ex["v"], dtype=np.float32))


def _assert_rounds_to(out64, printed):
    """The page prints float32 results of the exact values; the oracle's
    float64 value, rounded to float32, must reproduce each one (one float32
    ulp allowed for the double rounding float64 -> float32)."""
    got = _f32(out64)
    want = _f32(printed)
    ulp = np.spacing(np.abs(want))
    assert np.all(np.abs(got.astype(np.float64) - want.astype(np.float64)) <= ulp), (got, want)


def test_worked_example_plain(ex):
    q, k, v = _qkv(ex)
    out, lse = sdpa(q, k, v)
    assert list(out.shape) == ex["output_shape"]
    assert list(lse.shape) == ex["logsumexp_shape"]
    _assert_rounds_to(out[0], ex["plain"])


def test_worked_example_causal(ex):
    q, k, v = _qkv(ex)
    out, _ = sdpa(q, k, v, is_causal=True)
    _assert_rounds_to(out[0], ex["causal"])


def test_worked_example_masked(ex):
    q, k, v = _qkv(ex)
    mask = np.array([[0.0, -np.inf, 0.0]] * 3, dtype=np.float32)
    out, _ = sdpa(q[:, None], k[:, None], v[:, None], attn_mask=mask)
    _assert_rounds_to(out[0, 0], ex["masked_key1"])


def test_worked_example_scale_one(ex):
    q, k, v = _qkv(ex)
    out, _ = sdpa(q, k, v, scale=1.0)
    _assert_rounds_to(out[0], ex["scale_1"])


def test_worked_example_lse_closed_forms(ex):
    """lse is never printed; on this example three rows have closed forms.
    Query [1,1] scores 1 against every key, so its logits are all s and
    lse = ln 3 + s; causal row 0 sees one key with logit s = 1/sqrt(2)."""
    q, k, v = _qkv(ex)
    s = 1.0 / math.sqrt(2.0)
    _, lse = sdpa(q, k, v)
    assert abs(lse[0, 2] - (math.log(3.0) + s)) < 1e-14
    _, lse_c = sdpa(q, k, v, is_causal=True)
    assert abs(lse_c[0, 0] - s) < 1e-14
    _, lse_1 = sdpa(q, k, v, scale=1.0)
    assert abs(lse_1[0, 2] - (math.log(3.0) + 1.0)) < 1e-14
    # query [1,0] scores (1, 0, 1/2): lse = log(e^s + 1 + e^(s/2))
    assert abs(lse[0, 0] - math.log(math.exp(s) + 1.0 + math.exp(s / 2))) < 1e-14


def test_gqa_example(ex):
    """Two query heads share one key/value head.  Query head 1 = [0,1] against
    keys [1,0],[0,1] is causal row 1 of the worked example (printed); head 0 =
    [1,0] has logits (s, 0): weights (w, 1-w), w = e^s / (e^s + 1)."""
    gq = np.array(ex["gqa_query"], dtype=np.float32)
    gk = np.array(ex["gqa_key"], dtype=np.float32)
    gv = np.array(ex["gqa_value"], dtype=np.float32)
    out, lse = sdpa(gq, gk, gv, enable_gqa=True)
    assert list(out.shape) == ex["gqa_output_shape"]
    _assert_rounds_to(out[0, 1], [ex["causal"][1]])
    s = 1.0 / math.sqrt(2.0)
    w = math.exp(s) / (math.exp(s) + 1.0)
    np.testing.assert_allclose(out[0, 0, 0], [3.0 - 2.0 * w, 4.0 - 2.0 * w], rtol=0, atol=1e-15)
    with pytest.raises(ValueError):
        sdpa(gq, gk, gv)  # fewer key heads without enable_gqa


def test_gqa_grouping_is_contiguous():
    """Query head h reads key head h // (Hq/Hkv) (BMGHK: query head (g, j) uses
    key head g).  A strided h % Hkv mapping gives a different answer here."""
    g = torch.Generator().manual_seed(11)
    q = torch.randn(2, 6, 5, 8, generator=g, dtype=torch.float64)
    k = torch.randn(2, 2, 7, 8, generator=g, dtype=torch.float64)
    v = torch.randn(2, 2, 7, 3, generator=g, dtype=torch.float64)
    out, lse = sdpa(q, k, v, enable_gqa=True)
    out_c, lse_c = sdpa(q, k.repeat_interleave(3, dim=1), v.repeat_interleave(3, dim=1))
    np.testing.assert_array_equal(out, out_c)
    np.testing.assert_array_equal(lse, lse_c)
    out_s, _ = sdpa(q, k.repeat(1, 3, 1, 1), v.repeat(1, 3, 1, 1))
    assert np.abs(out - out_s).max() > 1e-3


# --------------------------------------------------- library routine: torch math


@pytest.mark.parametrize(
    "B,Hq,Hkv,L,S,E,Ev,causal,mask",
    [
        (1, 2, 2, 8, 8, 16, 16, False, None),
        (2, 3, 3, 7, 11, 5, 9, True, None),   # L < S, E != Ev
        (1, 2, 2, 13, 6, 4, 4, True, None),   # L > S: rows past S keep all keys
        (2, 4, 2, 9, 9, 8, 8, True, None),    # GQA
        (1, 2, 2, 6, 10, 4, 7, False, "bool"),
        (2, 1, 1, 5, 12, 3, 3, False, "float"),
    ],
)
def test_against_torch_math_path(B, Hq, Hkv, L, S, E, Ev, causal, mask):
    """torch.nn.functional.scaled_dot_product_attention on float64 CPU inputs
    is an independent implementation of the same definition (the exactref page
    checks PyTorch against its reference, "Checking PyTorch")."""
    g = torch.Generator().manual_seed(B * 1000 + L * 10 + S)
    q = torch.randn(B, Hq, L, E, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, S, E, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, S, Ev, generator=g, dtype=torch.float64)
    m = None
    if mask == "bool":
        m = torch.rand(L, S, generator=g) > 0.3
        m[:, 0] = True
    elif mask == "float":
        m = torch.randn(B, 1, L, S, generator=g, dtype=torch.float64)
        m[..., 3] = float("-inf")
    kk, vv = k, v
    if Hkv != Hq:
        kk = k.repeat_interleave(Hq // Hkv, 1)
        vv = v.repeat_interleave(Hq // Hkv, 1)
    want = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, attn_mask=m, is_causal=causal)
    got, lse = sdpa(q, k, v, attn_mask=m, is_causal=causal, enable_gqa=Hkv != Hq)
    np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-12)
    if E == Ev and mask is None:
        _, lse_t = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(q, kk, vv, 0.0, causal)[:2]
        np.testing.assert_allclose(lse, lse_t.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------ brute force, tiny


def _brute(q, k, v, bias):
    """Every logit, exponential and sum in 50-digit arithmetic."""
    mpmath.mp.dps = 50
    L, E = q.shape
    S = k.shape[0]
    Ev = v.shape[1]
    out = np.zeros((L, Ev))
    lse = np.zeros(L)
    for i in range(L):
        logits = []
        for j in range(S):
            dot = mpmath.fsum(mpmath.mpf(float(q[i, e])) * mpmath.mpf(float(k[j, e])) for e in range(E))
            logits.append(dot / mpmath.sqrt(E) + mpmath.mpf(float(bias[i, j])))
        ws = [mpmath.e ** l_ if l_ != mpmath.ninf else mpmath.mpf(0) for l_ in logits]
        z = mpmath.fsum(ws)
        lse[i] = float(mpmath.log(z))
        for c in range(Ev):
            out[i, c] = float(mpmath.fsum(w * mpmath.mpf(float(v[j, c])) for j, w in enumerate(ws)) / z)
    return out, lse


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    L, S, E, Ev = 4, 5, 3, 2
    q = rng.standard_normal((L, E))
    k = rng.standard_normal((S, E))
    v = rng.standard_normal((S, Ev))
    bias = rng.standard_normal((L, S))
    bias[1, 2] = -np.inf
    want, wlse = _brute(q, k, v, bias)
    got, glse = sdpa(q[None, None], k[None, None], v[None, None], attn_mask=bias)
    np.testing.assert_allclose(got[0, 0], want, rtol=0, atol=1e-13)
    np.testing.assert_allclose(glse[0, 0], wlse, rtol=0, atol=1e-13)


# ------------------------------------------------------------ invariants


def test_rows_sum_to_one():
    """Weights are exponentials normalised to sum to 1 (exactref intro): V of
    ones gives an output of ones; V = identity gives the weight matrix, whose
    rows sum to 1 and are non-negative."""
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 2, 9, 6, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, 9, 6, generator=g, dtype=torch.float64)
    ones = torch.ones(1, 2, 9, 4, dtype=torch.float64)
    out, _ = sdpa(q, k, ones, is_causal=True)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-15)
    eye = torch.eye(9, dtype=torch.float64).expand(1, 2, 9, 9)
    w, _ = sdpa(q, k, eye, is_causal=True)
    assert (w >= 0).all()
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.triu(w[0, 0], 1) == 0)  # causal: nothing above the diagonal


def test_weight_ratios_are_exponentials_of_logit_gaps():
    """w_ij / w_ik = exp(s (q_i.k_j - q_i.k_k)): the softmax definition, read
    off the weights obtained with V = identity."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 3, 4))
    k = rng.standard_normal((1, 1, 6, 4))
    w, _ = sdpa(q, k, np.eye(6)[None, None])
    s = 0.5
    for i in range(3):
        for j in range(6):
            r = w[0, 0, i, j] / w[0, 0, i, 0]
            want = math.exp(s * (float(q[0, 0, i] @ k[0, 0, j]) - float(q[0, 0, i] @ k[0, 0, 0])))
            assert abs(r / want - 1.0) < 1e-13


@pytest.mark.parametrize("L", [1, 5, 64, 300])
def test_causal_row_zero_is_v0(L):
    g = torch.Generator().manual_seed(L)
    q = torch.randn(1, 1, L, 8, generator=g).to(torch.float64)
    k = torch.randn(1, 1, L, 8, generator=g).to(torch.float64)
    v = torch.randn(1, 1, L, 5, generator=g).to(torch.float64)
    out, lse = sdpa(q, k, v, is_causal=True)
    np.testing.assert_array_equal(out[0, 0, 0], v[0, 0, 0].numpy())
    assert abs(lse[0, 0, 0] - float(q[0, 0, 0] @ k[0, 0, 0]) / math.sqrt(8)) < 1e-13


def test_scale_zero_gives_mean_of_kept_values():
    """With scale 0 every kept key has logit 0: equal weights, so the output is
    the mean of the kept values and lse = log(number kept)."""
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 1, 7, 4, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, 7, 4, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, 7, 3, generator=g, dtype=torch.float64)
    out, lse = sdpa(q, k, v, scale=0.0, is_causal=True)
    for i in range(7):
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, : i + 1].mean(0).numpy(), rtol=0, atol=1e-15)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-15


def test_default_scale_is_applied_once():
    """scale=None means 1/sqrt(E) (exactref "Arguments"); passing Q pre-scaled
    by 1/sqrt(E) with scale=1 gives the same result (exactref "Full
    specification": a consumer that pre-scales passes scale=1), while
    pre-scaling AND the default gives the double-scaled 1/E result (hourtab)."""
    g = torch.Generator().manual_seed(9)
    E = 96
    q = torch.randn(1, 2, 16, E, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, 16, E, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, 16, E, generator=g, dtype=torch.float64)
    a, la = sdpa(q, k, v)
    b, lb = sdpa(q / math.sqrt(E), k, v, scale=1.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-13)
    c, _ = sdpa(q / math.sqrt(E), k, v)
    d, _ = sdpa(q, k, v, scale=1.0 / E)
    np.testing.assert_allclose(c, d, rtol=0, atol=1e-13)
    assert np.abs(a - c).max() > 1e-2
    assert default_scale(E) == 1.0 / math.sqrt(E)


@pytest.mark.parametrize("E", [16, 96, 128])
def test_logit_variance_is_E(E):
    """Var(q.k) = d_k for iid N(0,1) q, k (lynx-cortex "Predice"; khchao
    "Variance of the Total Sum").  With one key and scale 1 the lse of a row is
    its logit q.k exactly, so the oracle's lse over many independent rows has
    variance E; at the default scale the variance is 1."""
    g = torch.Generator().manual_seed(E)
    H, L = 512, 8
    q = torch.randn(1, H, L, E, generator=g, dtype=torch.float64)
    k = torch.randn(1, H, 1, E, generator=g, dtype=torch.float64)
    v = torch.ones(1, H, 1, 1, dtype=torch.float64)
    _, lse1 = sdpa(q, k, v, scale=1.0)
    var = lse1.var()
    assert abs(var / E - 1.0) < 0.12, var
    _, lse_d = sdpa(q, k, v)
    assert abs(lse_d.var() - 1.0) < 0.12


def test_lse_minus_log_s_at_default_scale():
    """Logits with unit variance over S keys: lse - log S ~ log E[e^l] = 1/2."""
    g = torch.Generator().manual_seed(21)
    q = torch.randn(1, 4, 64, 128, generator=g, dtype=torch.float64)
    k = torch.randn(1, 4, 2048, 128, generator=g, dtype=torch.float64)
    v = torch.zeros(1, 4, 2048, 1, dtype=torch.float64)
    _, lse = sdpa(q, k, v)
    d = (lse - math.log(2048)).mean()
    assert 0.4 < d < 0.6, d


def test_double_scaling_is_near_uniform():
    """At scale 1/E (the double-scaled case) the logits have variance
    |q|^2/E^2 ~ 1/E, so the weights are near-uniform: row entropy ~ log n minus
    about 1/(2E), the largest weight only a little above 1/n."""
    g = torch.Generator().manual_seed(96)
    E, S = 96, 2048
    q = torch.randn(1, 1, 8, E, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, S, E, generator=g, dtype=torch.float64)
    w, _ = sdpa(q, k, torch.eye(S, dtype=torch.float64)[None, None], scale=1.0 / E)
    ent = -(w * np.log(w)).sum(-1)
    deficit = math.log(S) - ent.mean()
    assert 0.002 < deficit < 0.01, deficit
    assert (w.max(-1) * S).max() < 2.0
    w2, _ = sdpa(q, k, torch.eye(S, dtype=torch.float64)[None, None])
    assert math.log(S) - (-(w2 * np.log(w2)).sum(-1)).mean() > 0.3


def test_no_overflow_with_large_logits():
    """Logits near 1000 overflow exp() without the shift by the row maximum;
    the definition's value is the same as for logits shifted down by 1000."""
    q = np.array([[[[30.0, 30.0]]]])
    k = np.array([[[[30.0, 30.0], [29.0, 30.0], [0.0, 0.0]]]])
    v = np.array([[[[1.0], [2.0], [3.0]]]])
    out, lse = sdpa(q, k, v, scale=1.0)
    # logits 1800, 1770, 0: weights ~ (1, e^-30, e^-1800)
    w1 = math.exp(-30.0)
    assert abs(out[0, 0, 0, 0] - (1.0 + 2.0 * w1) / (1.0 + w1)) < 1e-14
    assert abs(lse[0, 0, 0] - (1800.0 + math.log1p(w1))) < 1e-10


def test_joint_key_value_permutation_invariance():
    g = torch.Generator().manual_seed(8)
    q = torch.randn(1, 2, 5, 4, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, 9, 4, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, 9, 3, generator=g, dtype=torch.float64)
    p = torch.randperm(9, generator=g)
    a, la = sdpa(q, k, v)
    b, lb = sdpa(q, k[:, :, p], v[:, :, p])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-14)


def test_row_bias_shift_and_value_linearity():
    """A bias constant along a row cancels in the softmax and adds to lse; the
    output is linear in V."""
    g = torch.Generator().manual_seed(10)
    q = torch.randn(1, 1, 6, 4, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, 8, 4, generator=g, dtype=torch.float64)
    v1 = torch.randn(1, 1, 8, 3, generator=g, dtype=torch.float64)
    v2 = torch.randn(1, 1, 8, 3, generator=g, dtype=torch.float64)
    c = torch.arange(6, dtype=torch.float64)[:, None] * 0.75 - 2.0
    a, la = sdpa(q, k, v1)
    b, lb = sdpa(q, k, v1, attn_mask=c.expand(6, 8))
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lb - la, c[:, 0].numpy()[None, None], rtol=0, atol=1e-13)
    s, _ = sdpa(q, k, 2.0 * v1 - 3.0 * v2)
    a2, _ = sdpa(q, k, v2)
    np.testing.assert_allclose(s, 2.0 * a - 3.0 * a2, rtol=0, atol=1e-13)


# ------------------------------------------------------------ special values


def test_nan_row(ex):
    """exactref "Special values and dropout": a query containing a NaN makes
    its own output row NaN ([[nan, nan]]) and leaves the other rows alone."""
    _, k, v = _qkv(ex)
    out, lse = sdpa(np.array([[[np.nan, 0.0]]], dtype=np.float32), k, v)
    assert np.isnan(out).all() and out.shape == (1, 1, 2)
    assert np.isnan(lse).all()
    q, _, _ = _qkv(ex)
    q = q.copy()
    q[0, 1, 0] = np.nan
    out, _ = sdpa(q, k, v)
    assert np.isnan(out[0, 1]).all() and not np.isnan(out[0, [0, 2]]).any()


def test_dropout_raises(ex):
    q, k, v = _qkv(ex)
    with pytest.raises(ValueError, match="dropout_p must be 0"):
        sdpa(q, k, v, dropout_p=0.1)


def test_fully_masked_row_and_inf_logits():
    """A row with no kept key: weight 0 everywhere, output 0, lse -inf.  A +inf
    logit makes the row NaN with lse +inf; a NaN logit gives lse NaN.  A masked
    key whose value is infinite contributes 0 * inf = NaN."""
    q = np.ones((1, 1, 4, 2))
    k = np.ones((1, 1, 3, 2))
    v = np.arange(6, dtype=np.float64).reshape(1, 1, 3, 2)
    bias = np.zeros((4, 3))
    bias[0, :] = -np.inf
    bias[1, 1] = np.inf
    bias[2, 2] = np.nan
    out, lse = sdpa(q, k, v, attn_mask=bias)
    assert np.all(out[0, 0, 0] == 0.0) and lse[0, 0, 0] == -np.inf
    assert np.isnan(out[0, 0, 1]).all() and lse[0, 0, 1] == np.inf
    assert np.isnan(out[0, 0, 2]).all() and np.isnan(lse[0, 0, 2])
    assert np.isfinite(out[0, 0, 3]).all()
    boolmask = np.array([[False, False, False], [True, True, False], [True] * 3, [True] * 3])
    out_b, lse_b = sdpa(q, k, v, attn_mask=boolmask)
    assert np.all(out_b[0, 0, 0] == 0.0) and lse_b[0, 0, 0] == -np.inf
    np.testing.assert_allclose(out_b[0, 0, 1], v[0, 0, :2].mean(0), rtol=0, atol=1e-15)
    vinf = v.copy()
    vinf[0, 0, 2, 0] = np.inf
    out_i, _ = sdpa(q, k, vinf, attn_mask=boolmask)
    assert np.isnan(out_i[0, 0, 1, 0]) and np.isfinite(out_i[0, 0, 1, 1])
    assert np.isinf(out_i[0, 0, 3, 0])


def test_padding_mask_example():
    """exactref "Padding masks": hiding keys with float32's lowest finite value
    erases the scores of a fully padded row when score and mask are rounded
    once, so its weights come out equal: PyTorch prints [1.5], [1.0], inside
    the page's finite range for correct outputs."""
    gp = _golden("padding_mask.json")
    low = float(np.finfo(np.float32).min)
    mask = np.array([[[low if m == "low" else m for m in row] for row in gp["mask_pattern"][0]]])
    out, _ = sdpa(np.array(gp["query"]), np.array(gp["key"]), np.array(gp["value"]), attn_mask=mask)
    np.testing.assert_allclose(out[0], gp["torch_output"], rtol=0, atol=1e-12)
    lo, hi = gp["finite_range_row0"]
    assert lo <= out[0, 0, 0] <= hi
    assert abs(out[0, 1, 0] - gp["exact_rounded"][1][0]) < 1e-12


def test_head_dim_zero_logits_are_the_mask():
    """exactref "Full specification": with E = 0 every dot product is 0, so
    only the mask shapes the logits."""
    q = np.zeros((1, 1, 2, 0))
    k = np.zeros((1, 1, 3, 0))
    v = np.array([[[[1.0], [2.0], [4.0]]]])
    bias = np.log(np.array([[1.0, 1.0, 2.0], [1.0, 0.0, 1.0]]))
    out, lse = sdpa(q, k, v, attn_mask=bias)
    assert abs(out[0, 0, 0, 0] - (1 + 2 + 8) / 4.0) < 1e-15
    assert abs(out[0, 0, 1, 0] - 2.5) < 1e-15
    assert abs(lse[0, 0, 0] - math.log(4.0)) < 1e-15
    out2, _ = sdpa(q, k, v)
    np.testing.assert_allclose(out2[0, 0, :, 0], 7.0 / 3.0, rtol=0, atol=1e-15)


# ------------------------------------------------------------ packed varlen


def _block_mask(seqlens, causal):
    T = sum(seqlens)
    seg = np.repeat(np.arange(len(seqlens)), seqlens)
    m = seg[:, None] == seg[None, :]
    if causal:
        m &= np.arange(T)[None, :] <= np.arange(T)[:, None]
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_packed_equals_block_diagonal_mask(causal):
    """Packed attention equals full attention over the concatenation with the
    block-diagonal mask written out element by element (segment of i equals
    segment of j, and j <= i when causal)."""
    seqlens = [5, 1, 9, 3]
    T = sum(seqlens)
    g = torch.Generator().manual_seed(17)
    q = torch.randn(1, T, 3, 4, generator=g, dtype=torch.float64)
    k = torch.randn(1, T, 3, 4, generator=g, dtype=torch.float64)
    v = torch.randn(1, T, 3, 6, generator=g, dtype=torch.float64)
    out, lse = sdpa_packed(q, k, v, seqlens, causal=causal)
    full, flse = sdpa(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), attn_mask=_block_mask(seqlens, causal))
    np.testing.assert_allclose(out[0], full[0].transpose(1, 0, 2), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, flse[0], rtol=0, atol=1e-14)
    # segment 0 on its own (the tutorial's check of the packed result)
    o0, _ = sdpa(q[:, :5].transpose(1, 2), k[:, :5].transpose(1, 2), v[:, :5].transpose(1, 2), is_causal=causal)
    np.testing.assert_allclose(out[0, :5], o0[0].transpose(1, 0, 2), rtol=0, atol=1e-14)
