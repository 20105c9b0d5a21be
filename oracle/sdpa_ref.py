"""Plain float64 CPU oracle for scaled dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (no kernels, headers, helpers, tables or constants).

What it computes follows the exactref.ai page "scaled_dot_product_attention"
(sections "Arguments" and "Full specification"):

    O = softmax(Q K^T * scale + mask) V      over the key axis
    lse_i = log(sum_j exp(l_ij))             natural log of each row's logits

where ``scale`` is 1/sqrt(E) unless given, and multiplies the raw dot
products once.  A boolean mask marks the keys a query may see (True = see);
a floating mask is a bias added after scaling, with -inf meaning the key is
excluded.  Under ``is_causal`` query i sees keys 0..i only.  With
``enable_gqa`` several consecutive query heads share one key/value head:
query head h uses key/value head h // (Hq // Hkv), the contiguous grouping
of the BMGHK layout (insureai360 xFormers tutorial, section 5
"Grouped-query attention").

Non-finite values, per the same "Full specification": one NaN or +inf
among a row's logits turns the whole row into NaN (its lse is NaN, or +inf
if the row has +inf but no NaN).  When none of a row's logits is finite,
every weight is zero, the output is those zero weights applied to V (0,
or NaN where V itself is not finite, since 0 * inf is NaN) and lse is
-inf.  With E = 0 every dot product is an empty sum (0), so only the mask
shapes the logits.

Block-diagonal (packed variable-length) attention follows the xFormers
tutorial, section 4 "Variable-length packed batch": each segment of a packed
sequence attends only to itself, optionally causally.

Every value is computed in float64.  A library primitive (numpy matmul, exp,
log, max) serves as a step; there is no blocking, fusion or reordering beyond
materialising one row block of logits at a time.

Pinned by tests/test_oracle_pins.py (worked examples printed on the pages,
closed forms, invariants, brute force in 50-digit arithmetic on tiny inputs,
and torch's float64 CPU math path as an independent library routine).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["default_scale", "sdpa", "sdpa_packed", "ROW_BLOCK"]

# Rows of logits materialised at once (memory bound only; no effect on values).
ROW_BLOCK = 256


def default_scale(E: int) -> float:
    """1/sqrt(E), the page's default for ``scale=None`` (exactref "Arguments").

    With E = 0 every dot product is 0 and the scale has nothing to scale;
    1.0 is returned as a placeholder."""
    if E == 0:
        return 1.0
    return 1.0 / math.sqrt(E)


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: upcast exactly, then to numpy
        import torch

        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _mask_to_bias(attn_mask, shape_bhls: Tuple[int, int, int, int]) -> Optional[np.ndarray]:
    """A bool mask (True keeps) becomes a 0 / -inf bias; a float mask is the bias.

    The two mask kinds of exactref "Arguments" (a boolean one marking the
    visible keys, a floating one added after scaling, -inf excluding the
    key).  The result is broadcast to (B, Hq, L, S)."""
    if attn_mask is None:
        return None
    if hasattr(attn_mask, "detach"):
        import torch

        if attn_mask.dtype == torch.bool:
            m = attn_mask.cpu().numpy()
        else:
            m = attn_mask.detach().to(torch.float64).cpu().numpy()
    else:
        m = np.asarray(attn_mask)
    if m.dtype == np.bool_:
        bias = np.where(m, 0.0, -np.inf)
    else:
        bias = m.astype(np.float64)
    return np.broadcast_to(bias, shape_bhls)


def _softmax_rows(logits: np.ndarray, vals: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax over the last axis of ``logits`` (rows x S) and the weighted sum
    with ``vals`` (S x Ev); returns (out rows x Ev, lse rows).

    exactref "Full specification": NaN or +inf anywhere in a row makes it
    NaN; a row without any finite logit gets all-zero weights and lse -inf;
    otherwise the weights are exp(l - max) / sum exp(l - max) and lse is
    max + log(sum)."""
    R = logits.shape[0]
    Ev = vals.shape[1]
    out = np.empty((R, Ev), dtype=np.float64)
    lse = np.empty((R,), dtype=np.float64)
    with np.errstate(invalid="ignore", over="ignore", divide="ignore"):
        has_nan = np.isnan(logits).any(axis=1)
        has_pinf = np.isposinf(logits).any(axis=1)
        finite = np.isfinite(logits)
        has_finite = finite.any(axis=1)
        for r in range(R):
            row = logits[r]
            if has_nan[r] or has_pinf[r]:
                out[r, :] = np.nan
                lse[r] = np.nan if has_nan[r] else np.inf
                continue
            if not has_finite[r]:
                # weight 0 on every key: 0 * V (NaN where V is non-finite)
                w = np.zeros_like(row)
                out[r, :] = w @ vals
                lse[r] = -np.inf
                continue
            m = row.max()
            p = np.exp(row - m)  # exp(-inf) = 0 for removed keys
            z = p.sum()
            out[r, :] = (p @ vals) / z
            lse[r] = m + math.log(z)
    return out, lse


def sdpa(
    query,
    key,
    value,
    attn_mask=None,
    dropout_p: float = 0.0,
    is_causal: bool = False,
    scale: Optional[float] = None,
    enable_gqa: bool = False,
) -> Tuple[np.ndarray, np.ndarray]:
    """softmax(Q K^T * scale + mask) V and its logsumexp, in float64.

    Shapes (exactref "Arguments"): query (B, Hq, L, E), key (B, Hkv, S, E),
    value (B, Hkv, S, Ev); a 3-D input (B, L, E) is treated as one head.
    Returns ``(out, lse)`` with out (B, Hq, L, Ev) and lse (B, Hq, L).

    ``dropout_p`` must be 0, else ``ValueError``: random dropout has no
    deterministic result to compare with (exactref "Special values and
    dropout").  Both ``attn_mask`` and
    ``is_causal`` may be given; each removes keys.
    """
    if dropout_p != 0.0:
        raise ValueError("dropout_p must be 0: a random dropout has no deterministic result to check")
    q = _as_f64(query)
    k = _as_f64(key)
    v = _as_f64(value)
    squeeze_head = q.ndim == 3
    if squeeze_head:
        q, k, v = q[:, None], k[:, None], v[:, None]
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("expected (B, H, L, E) inputs")
    B, Hq, L, E = q.shape
    Bk, Hkv, S, Ek = k.shape
    Bv, Hv, Sv, Ev = v.shape
    if Bk != B or Bv != B or Ek != E or Sv != S or Hv != Hkv:
        raise ValueError("query/key/value shapes do not agree")
    if Hkv != Hq:
        if not enable_gqa or Hkv == 0 or Hq % Hkv != 0:
            raise ValueError("query heads must equal key/value heads, or be a multiple of them with enable_gqa")
    group = Hq // Hkv
    s = default_scale(E) if scale is None else float(scale)
    bias = _mask_to_bias(attn_mask, (B, Hq, L, S))

    out = np.empty((B, Hq, L, Ev), dtype=np.float64)
    lse = np.empty((B, Hq, L), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kv = h // group  # contiguous grouping
            kh = k[b, kv]
            vh = v[b, kv]
            for r0 in range(0, L, ROW_BLOCK):
                r1 = min(L, r0 + ROW_BLOCK)
                if E == 0:
                    logits = np.zeros((r1 - r0, S), dtype=np.float64)
                else:
                    with np.errstate(invalid="ignore", over="ignore"):
                        logits = (q[b, h, r0:r1] @ kh.T) * s
                if bias is not None:
                    with np.errstate(invalid="ignore"):
                        logits = logits + bias[b, h, r0:r1]
                if is_causal:
                    i = np.arange(r0, r1)[:, None]
                    j = np.arange(S)[None, :]
                    logits = np.where(j <= i, logits, -np.inf)
                o, l_ = _softmax_rows(logits, vh)
                out[b, h, r0:r1] = o
                lse[b, h, r0:r1] = l_
    if squeeze_head:
        return out[:, 0], lse[:, 0]
    return out, lse


def sdpa_packed(
    query,
    key,
    value,
    seqlens: Sequence[int],
    causal: bool = False,
    scale: Optional[float] = None,
    heads: Optional[Sequence[int]] = None,
) -> Tuple[np.ndarray, np.ndarray]:
    """Block-diagonal attention over one packed batch without padding.

    Follows the xFormers tutorial, section 4 "Variable-length packed batch":
    inputs are (1, T, H, E) (BMHK, T = sum(seqlens)); segment s covers tokens
    [c_s, c_s + n_s) and attends only to keys of its own segment
    (``BlockDiagonalMask``), and with ``causal`` only to keys at or before its
    own position (``BlockDiagonalCausalMask``).  Returns out (1, T, H, Ev) and
    lse (H, T).  ``heads`` restricts the computation to some heads (the other
    entries are left NaN), for sampled checks of large inputs.
    """
    q = _as_f64(query)
    k = _as_f64(key)
    v = _as_f64(value)
    if q.ndim == 4:
        q, k, v = q[0], k[0], v[0]
    T, H, E = q.shape
    Ev = v.shape[-1]
    if sum(int(n) for n in seqlens) != T:
        raise ValueError("seqlens must sum to the packed length")
    out = np.full((1, T, H, Ev), np.nan, dtype=np.float64)
    lse = np.full((H, T), np.nan, dtype=np.float64)
    hs = range(H) if heads is None else heads
    c = 0
    for n in seqlens:
        n = int(n)
        if n == 0:
            continue
        for h in hs:
            # one segment, one head: plain attention on its own tokens
            o, l_ = sdpa(
                q[c : c + n, h][None, None],
                k[c : c + n, h][None, None],
                v[c : c + n, h][None, None],
                is_causal=causal,
                scale=scale,
            )
            out[0, c : c + n, h] = o[0, 0]
            lse[h, c : c + n] = l_[0, 0]
        c += n
    return out, lse
