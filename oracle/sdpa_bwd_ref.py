"""Plain float64 CPU oracle for the gradients of scaled dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path.

What it computes follows the exactref.ai page "scaled_dot_product_attention",
section "er.scaled_dot_product_attention.backward": for an output gradient
``grad`` (the shape of the forward's output) and the attention weights P of
the forward (same masks, scale and special-value rules as ``sdpa_ref``),

    dP   = grad V^T
    D_i  = sum_j P_ij dP_ij
    dS   = P * (dP - D)                     (D broadcast along each row)
    grad_value = P^T grad
    grad_query = scale * dS K
    grad_key   = scale * dS^T Q

where a key/value head shared by several query heads (``enable_gqa``;
query head h uses key/value head h // (Hq // Hkv)) sums the gradients of all
of them.  Non-finite values follow IEEE arithmetic: an excluded key has
P = 0, so an infinite dP under it makes D NaN (zero times infinity); a forward row that
is NaN spreads NaN to every gradient it feeds; a row that sees no key has
P = 0 everywhere and adds nothing.  The bias of a float mask is not
differentiated, and dropout must be 0.

Every value is computed in float64; numpy matmul, exp and sums serve as steps,
one row block of logits at a time, with no other blocking or reordering.

Pinned by tests/test_oracle_bwd_pins.py: central finite differences of the
forward oracle, torch's float64 autograd (the check the page itself names),
translation invariance of the keys, closed forms for constant values and a
zero scale, and the special-value rules above.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .sdpa_ref import ROW_BLOCK, _as_f64, _mask_to_bias, default_scale

__all__ = ["sdpa_backward", "sdpa_backward_packed", "attention_weights"]


def attention_weights(logits: np.ndarray) -> np.ndarray:
    """Row-wise softmax weights P of a block of logits (rows x S).

    exactref "Full specification": NaN or +inf anywhere in a row makes it
    NaN; a row without any finite logit gets all-zero weights; otherwise
    P_ij = exp(l_ij - m_i) / sum_j exp(l_ij - m_i)."""
    P = np.zeros_like(logits)
    with np.errstate(invalid="ignore", over="ignore", divide="ignore"):
        bad = np.isnan(logits).any(axis=1) | np.isposinf(logits).any(axis=1)
        has_finite = np.isfinite(logits).any(axis=1)
        for r in range(logits.shape[0]):
            if bad[r]:
                P[r] = np.nan
            elif has_finite[r]:
                e = np.exp(logits[r] - logits[r].max())
                P[r] = e / e.sum()
    return P


def sdpa_backward(
    query,
    key,
    value,
    grad,
    attn_mask=None,
    dropout_p: float = 0.0,
    is_causal: bool = False,
    scale: Optional[float] = None,
    enable_gqa: bool = False,
) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(grad_query, grad_key, grad_value) in float64 for the output gradient
    ``grad`` (B, Hq, L, Ev); the other arguments are the forward's
    (exactref "er.scaled_dot_product_attention.backward")."""
    if dropout_p != 0.0:
        raise ValueError("dropout_p must be 0: a random dropout has no deterministic result to check")
    q = _as_f64(query)
    k = _as_f64(key)
    v = _as_f64(value)
    g = _as_f64(grad)
    squeeze_head = q.ndim == 3
    if squeeze_head:
        q, k, v, g = q[:, None], k[:, None], v[:, None], g[:, None]
    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    Ev = v.shape[-1]
    if g.shape != (B, Hq, L, Ev):
        raise ValueError("grad must have the output's shape")
    if Hkv != Hq and (not enable_gqa or Hkv == 0 or Hq % Hkv != 0):
        raise ValueError("query heads must equal key/value heads, or be a multiple of them with enable_gqa")
    group = Hq // Hkv
    s = default_scale(E) if scale is None else float(scale)
    bias = _mask_to_bias(attn_mask, (B, Hq, L, S))

    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    with np.errstate(invalid="ignore", over="ignore"):
        for b in range(B):
            for h in range(Hq):
                kv = h // group  # contiguous grouping
                for r0 in range(0, L, ROW_BLOCK):
                    r1 = min(L, r0 + ROW_BLOCK)
                    qb = q[b, h, r0:r1]
                    logits = qb @ k[b, kv].T * s if E else np.zeros((r1 - r0, S))
                    if bias is not None:
                        logits = logits + bias[b, h, r0:r1]
                    if is_causal:
                        i = np.arange(r0, r1)[:, None]
                        j = np.arange(S)[None, :]
                        logits = np.where(j <= i, logits, -np.inf)
                    P = attention_weights(logits)
                    gb = g[b, h, r0:r1]
                    dP = gb @ v[b, kv].T
                    D = (P * dP).sum(axis=1, keepdims=True)
                    dS = P * (dP - D)
                    dv[b, kv] += P.T @ gb
                    dq[b, h, r0:r1] = s * (dS @ k[b, kv])
                    dk[b, kv] += s * (dS.T @ qb)
    if squeeze_head:
        return dq[:, 0], dk[:, 0], dv[:, 0]
    return dq, dk, dv


def sdpa_backward_packed(
    query,
    key,
    value,
    grad,
    seqlens: Sequence[int],
    causal: bool = False,
    scale: Optional[float] = None,
) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of block-diagonal attention over one packed batch (1, T, H, E)
    (xFormers tutorial, section 4 "Variable-length packed batch"): each
    segment's gradients are those of plain attention on its own tokens."""
    q, k, v, g = (_as_f64(x) for x in (query, key, value, grad))
    if q.ndim == 4:
        q, k, v, g = q[0], k[0], v[0], g[0]
    T, H, E = q.shape
    if sum(int(n) for n in seqlens) != T:
        raise ValueError("seqlens must sum to the packed length")
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    c = 0
    for n in seqlens:
        n = int(n)
        if n:
            sl = slice(c, c + n)
            a, b_, d = sdpa_backward(
                q[sl].transpose(1, 0, 2)[None], k[sl].transpose(1, 0, 2)[None], v[sl].transpose(1, 0, 2)[None],
                g[sl].transpose(1, 0, 2)[None], is_causal=causal, scale=scale)
            dq[sl], dk[sl], dv[sl] = a[0].transpose(1, 0, 2), b_[0].transpose(1, 0, 2), d[0].transpose(1, 0, 2)
        c += n
    return dq[None], dk[None], dv[None]
