"""Pins of the paged-cache decode oracle (oracle/paged_ref.py).

The gather of a row's tokens from its pages is what the oracle adds to plain
attention; each pin checks it against something other than itself:

* a contiguous cache cut into pages laid out in order (identity table) gives
  the result of plain attention on the contiguous cache (torch's float64
  math path, an independent library routine);
* shuffling the pool's pages together with the table changes nothing, and a
  table pointing at the wrong page does change the result;
* tokens past seq_lens in a row's last page, and pages past it in the table,
  are never read (NaN there leaves the result finite);
* seq_lens = 0 gives output 0 and lse -inf (exactref "Full specification":
  a row with no key);
* equal keys give equal weights: the output is the mean of the row's values
  and lse = q.k * scale + log n, in closed form.
"""
import numpy as np
import pytest
import torch

from oracle import sdpa_decode_paged


def _torch_ref(q, k, v, scale=None):
    """torch float64 math path on contiguous (B, H, S, E) inputs, GQA by
    repeating key/value heads."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    g = qt.shape[1] // kt.shape[1]
    kt, vt = kt.repeat_interleave(g, 1), vt.repeat_interleave(g, 1)
    s = 1.0 / np.sqrt(q.shape[-1]) if scale is None else scale
    logits = (qt @ kt.transpose(-1, -2)) * s
    out = torch.softmax(logits, -1) @ vt
    return out.numpy(), torch.logsumexp(logits, -1).numpy()


def _paged(k, ps):
    """(B, Hkv, S, E) -> pool (B * S/ps, ps, Hkv, E) with identity table."""
    B, H, S, E = k.shape
    pool = k.transpose(0, 2, 1, 3).reshape(B * S // ps, ps, H, E)
    table = np.arange(B * S // ps).reshape(B, S // ps)
    return pool, table


@pytest.mark.parametrize("ps", [1, 4, 16])
def test_identity_layout_is_plain_attention(ps):
    rng = np.random.default_rng(1)
    B, Hq, Hkv, L, S, E = 2, 8, 2, 2, 48, 16
    q, k, v = rng.standard_normal((B, Hq, L, E)), rng.standard_normal((B, Hkv, S, E)), rng.standard_normal((B, Hkv, S, E))
    kp, table = _paged(k, ps)
    vp, _ = _paged(v, ps)
    o, l_ = sdpa_decode_paged(q, kp, vp, table, np.full(B, S))
    ro, rl = _torch_ref(q, k, v)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_, rl, rtol=0, atol=1e-12)


def test_page_shuffle_invariance_and_wrong_page():
    rng = np.random.default_rng(2)
    B, H, S, E, ps = 3, 2, 40, 8, 8
    q, k, v = rng.standard_normal((B, H, 1, E)), rng.standard_normal((B, H, S, E)), rng.standard_normal((B, H, S, E))
    kp, table = _paged(k, ps)
    vp, _ = _paged(v, ps)
    lens = np.array([40, 17, 1])
    o0, l0 = sdpa_decode_paged(q, kp, vp, table, lens)
    perm = rng.permutation(kp.shape[0])          # new position of each page
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    o1, l1 = sdpa_decode_paged(q, kp2, vp2, perm[table], lens)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)
    bad = table.copy()
    bad[0, 1] = table[1, 0]                      # row 0 reads row 1's first page
    o2, _ = sdpa_decode_paged(q, kp, vp, bad, lens)
    assert np.abs(o2[0] - o0[0]).max() > 1e-3


def test_unused_tokens_and_pages_are_not_read():
    rng = np.random.default_rng(3)
    H, E, ps = 2, 8, 8
    q = rng.standard_normal((1, H, 1, E))
    kp = rng.standard_normal((6, ps, H, E))
    vp = rng.standard_normal((6, ps, H, E))
    table = np.array([[4, 0, 5, 2]])
    n = 11                                       # page 4 whole, 3 tokens of page 0
    o0, l0 = sdpa_decode_paged(q, kp, vp, table, [n])
    kp[0, 3:], vp[0, 3:], kp[5], vp[5], kp[2], vp[2] = np.nan, np.nan, np.nan, np.nan, np.nan, np.nan
    o1, l1 = sdpa_decode_paged(q, kp, vp, table, [n])
    assert np.isfinite(o1).all() and np.isfinite(l1).all()
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)


def test_empty_row():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((2, 4, 1, 8))
    kp, vp = rng.standard_normal((3, 4, 2, 8)), rng.standard_normal((3, 4, 2, 8))
    o, l_ = sdpa_decode_paged(q, kp, vp, np.array([[0, 1], [2, 0]]), [0, 5])
    assert (o[0] == 0).all() and (l_[0] == -np.inf).all()
    assert np.isfinite(o[1]).all() and np.isfinite(l_[1]).all()


def test_equal_keys_closed_form():
    H, E, ps, n = 1, 4, 4, 7
    q = np.array([[[[0.5, -1.0, 2.0, 0.25]]]])
    kvec = np.array([1.0, 0.5, -0.5, 2.0])
    kp = np.tile(kvec, (3, ps, H, 1))
    vp = np.arange(3 * ps * H * 2, dtype=np.float64).reshape(3, ps, H, 2)
    table = np.array([[2, 0]])
    o, l_ = sdpa_decode_paged(q, kp, vp, table, [n])
    tokens = np.concatenate([vp[2], vp[0]])[:n, 0]          # (n, 2) in table order
    np.testing.assert_allclose(o[0, 0, 0], tokens.mean(axis=0), rtol=1e-14)
    np.testing.assert_allclose(l_[0, 0, 0], (q[0, 0, 0] @ kvec) / 2.0 + np.log(n), rtol=1e-14)
