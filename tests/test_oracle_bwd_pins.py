"""Pins of the float64 backward oracle (oracle/sdpa_bwd_ref.py) to what the
mathematics and the pages fix, independently of the oracle's own formulas.

* central finite differences of the forward oracle's loss sum(grad * O): the
  gradient is the derivative of the forward, whatever formula computes it;
* torch's float64 autograd of its math path, which is what the exactref
  page's backward section compares its gradients with;
* invariants: adding one vector to every key of a row's kept set shifts that
  row's logits by a constant, so the key gradients of a head sum to zero;
  the rows of dS sum to zero; grad_value with an all-ones grad is the column
  sums of P;
* closed forms: equal value rows make dP constant along each row, so dS,
  grad_query and grad_key vanish; scale 0 makes grad_query and grad_key 0 and
  grad_value the mean-weight sums;
* special values from the page's backward section: a masked key with an
  infinite value makes D (hence the row's dS) NaN; a NaN forward row makes the
  gradients it touches NaN; a row with no kept key contributes 0.
"""
import numpy as np
import pytest
import torch

from oracle import attention_weights, sdpa, sdpa_backward, sdpa_backward_packed


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _fd_grads(q, k, v, g, h=1e-6, **kw):
    """Central differences of sum(g * O) with respect to every input entry."""
    out = []
    for idx in range(3):
        x = [q, k, v]
        d = np.zeros_like(x[idx])
        it = np.nditer(x[idx], flags=["multi_index"])
        for _ in it:
            m = it.multi_index
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[idx][m] += h
            xm[idx][m] -= h
            fp = (sdpa(*xp, **kw)[0] * g).sum()
            fm = (sdpa(*xm, **kw)[0] * g).sum()
            d[m] = (fp - fm) / (2 * h)
        out.append(d)
    return out


@pytest.mark.parametrize(
    "kw",
    [
        dict(),
        dict(is_causal=True),
        dict(scale=0.7),
        dict(enable_gqa=True),
        dict(attn_mask="bias"),
        dict(is_causal=True, enable_gqa=True, scale=1.3),
    ],
    ids=["plain", "causal", "scale", "gqa", "bias", "causal-gqa-scale"],
)
def test_finite_differences(kw):
    kw = dict(kw)
    Hq, Hkv = (4, 2) if kw.get("enable_gqa") else (2, 2)
    q = _rand((1, Hq, 5, 3), 1)
    k = _rand((1, Hkv, 6, 3), 2)
    v = _rand((1, Hkv, 6, 4), 3)
    g = _rand((1, Hq, 5, 4), 4)
    if kw.get("attn_mask") == "bias":
        kw["attn_mask"] = _rand((1, Hq, 5, 6), 5)
    dq, dk, dv = sdpa_backward(q, k, v, g, **kw)
    fq, fk, fv = _fd_grads(q, k, v, g, **kw)
    for a, b_ in ((dq, fq), (dk, fk), (dv, fv)):
        assert np.abs(a - b_).max() <= 1e-7 * max(1.0, np.abs(b_).max())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("gqa", [False, True])
def test_torch_float64_autograd(causal, gqa):
    Hq, Hkv = (6, 2) if gqa else (3, 3)
    q = torch.tensor(_rand((2, Hq, 9, 8), 11), requires_grad=True)
    k = torch.tensor(_rand((2, Hkv, 13, 8), 12), requires_grad=True)
    v = torch.tensor(_rand((2, Hkv, 13, 5), 13), requires_grad=True)
    g = torch.tensor(_rand((2, Hq, 9, 5), 14))
    kr = k.repeat_interleave(Hq // Hkv, dim=1)
    vr = v.repeat_interleave(Hq // Hkv, dim=1)
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        out = torch.nn.functional.scaled_dot_product_attention(q, kr, vr, is_causal=causal)
    out.backward(g)
    dq, dk, dv = sdpa_backward(q.detach(), k.detach(), v.detach(), g, is_causal=causal, enable_gqa=gqa)
    for a, t in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert np.abs(a - t.numpy()).max() <= 1e-12 * max(1.0, np.abs(a).max())


def test_key_gradients_sum_to_zero_and_ds_rows_sum_to_zero():
    q, k, v, g = _rand((1, 2, 40, 16), 21), _rand((1, 2, 50, 16), 22), _rand((1, 2, 50, 8), 23), _rand((1, 2, 40, 8), 24)
    for causal in (False, True):
        dq, dk, dv = sdpa_backward(q, k, v, g, is_causal=causal)
        assert np.abs(dk.sum(axis=2)).max() < 1e-12
    # dS rows: rebuild P and dS for one head and check row sums directly
    logits = q[0, 0] @ k[0, 0].T / 4.0
    P = attention_weights(logits)
    dP = g[0, 0] @ v[0, 0].T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    assert np.abs(dS.sum(axis=1)).max() < 1e-12


def test_ones_grad_gives_column_sums_of_weights():
    q, k, v = _rand((1, 1, 30, 8), 31), _rand((1, 1, 20, 8), 32), _rand((1, 1, 20, 6), 33)
    g = np.ones((1, 1, 30, 6))
    _, _, dv = sdpa_backward(q, k, v, g)
    P = attention_weights(q[0, 0] @ k[0, 0].T / np.sqrt(8))
    assert np.allclose(dv[0, 0], np.repeat(P.sum(axis=0)[:, None], 6, axis=1), atol=1e-13)
    assert abs(dv[0, 0, :, 0].sum() - 30.0) < 1e-11  # every row's weights sum to 1


def test_equal_value_rows_and_zero_scale():
    q, k, g = _rand((1, 2, 12, 8), 41), _rand((1, 2, 15, 8), 42), _rand((1, 2, 12, 5), 43)
    v = np.broadcast_to(_rand((1, 2, 1, 5), 44), (1, 2, 15, 5)).copy()
    dq, dk, dv = sdpa_backward(q, k, v, g, is_causal=True)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    v = _rand((1, 2, 15, 5), 45)
    dq, dk, dv = sdpa_backward(q, k, v, g, scale=0.0)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    # uniform weights 1/15: grad_value is the column mean of grad, for every key
    assert np.allclose(dv, np.broadcast_to(g.sum(axis=2, keepdims=True) / 15.0, dv.shape), atol=1e-13)


def test_special_values():
    q, k, v, g = _rand((1, 1, 4, 3), 51), _rand((1, 1, 5, 3), 52), _rand((1, 1, 5, 2), 53), _rand((1, 1, 4, 2), 54)
    # key 4 removed from every row: with a finite value it contributes
    # nothing (the gradients equal those without the key, and its own are 0)
    mask = np.ones((4, 5), dtype=bool)
    mask[:, 4] = False
    dq, dk, dv = sdpa_backward(q, k, v, g, attn_mask=mask)
    rq, rk, rv = sdpa_backward(q, k[:, :, :4], v[:, :, :4], g)
    assert np.allclose(dq, rq, atol=1e-14) and np.allclose(dk[:, :, :4], rk, atol=1e-14)
    assert (dk[0, 0, 4] == 0).all() and (dv[0, 0, 4] == 0).all()
    # ... but an infinite value there gives dP = inf where P = 0, so D and
    # every dS entry of each row are NaN (0 * inf)
    v2 = v.copy()
    v2[0, 0, 4, 0] = np.inf
    dq, dk, dv = sdpa_backward(q, k, v2, g, attn_mask=mask)
    assert np.isnan(dq).all() and np.isnan(dk).all()
    # a NaN query row: its forward row is NaN, so every gradient it touches is NaN
    q2 = q.copy()
    q2[0, 0, 2, 1] = np.nan
    dq, dk, dv = sdpa_backward(q2, k, v, g)
    assert np.isnan(dq[0, 0, 2]).all() and np.isnan(dk).all() and np.isnan(dv).all()
    assert np.isfinite(dq[0, 0, [0, 1, 3]]).all()
    # a row with no kept key contributes 0
    mask = np.ones((4, 5), dtype=bool)
    mask[3] = False
    dq, dk, dv = sdpa_backward(q, k, v, g, attn_mask=mask)
    dq0, dk0, dv0 = sdpa_backward(q[:, :, :3], k, v, g[:, :, :3], attn_mask=mask[:3])
    assert (dq[0, 0, 3] == 0).all()
    assert np.allclose(dk, dk0, atol=1e-14) and np.allclose(dv, dv0, atol=1e-14)
    with pytest.raises(ValueError):
        sdpa_backward(q, k, v, g, dropout_p=0.1)


def test_packed_equals_per_segment_and_block_mask():
    seqlens = [5, 1, 9, 4]
    T, H, E = sum(seqlens), 2, 8
    q, k, v, g = (_rand((1, T, H, E), 60 + i) for i in range(4))
    dq, dk, dv = sdpa_backward_packed(q, k, v, g, seqlens, causal=True)
    # the same through an explicit block-diagonal causal bool mask on (1, H, T, E)
    seg = np.repeat(np.arange(len(seqlens)), seqlens)
    pos = np.arange(T)
    mask = (seg[:, None] == seg[None, :]) & (pos[None, :] <= pos[:, None])
    t = lambda x: x[0].transpose(1, 0, 2)[None]
    rq, rk, rv = sdpa_backward(t(q), t(k), t(v), t(g), attn_mask=mask)
    for a, b_ in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a[0].transpose(1, 0, 2) - b_[0]).max() < 1e-12
