"""Per-element error budgets for the attention forward and backward (test
infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only tests use it.

The exactref page "scaled_dot_product_attention" ("Full specification",
tolerance()) derives its tolerance from the error sources of a forward
computation: summing the dot products, multiplying by the scale, rounding
each logit, subtracting the row maximum, the exponential's few-ulp error,
summing the weights, dividing, and rounding the result to its dtype; and for
the logsumexp, the logarithm's ulps and the rounding of max + log.  Named
algorithms add their own sources, listed there too: FlashAttention rounds the
weights to bf16 / fp16 before multiplying them with V, rescales online and
multiplies by a reciprocal of the row sum.

``forward_budget`` turns that list into a first-order bound, element by
element, for the algorithm the GPU kernels implement, evaluated on the exact
(float64) quantities of the oracle:

* every weight w_ij = p_ij / Z_i carries a relative error eta_ij made of
  the logit error (an fp32 dot product of E terms, gamma_E * scale *
  sum_e |q_ie k_je|, plus fp32 roundings of the scaled score and the shift),
  the exponential's relative error (``exp_rel``: for 16-bit inputs the
  multi-function unit's 2^x or the FMA-pipe polynomial, both under 1e-4;
  for float32 expf, within 2 ulp) and, for 16-bit
  inputs, the rounding of P to the input dtype (the dtype's unit roundoff);
* out_ie = sum_j w_ij v_je is perturbed by sum_j w_ij eta_ij (|v_je| +
  |out_ie|) (numerator and row sum; a common rescale factor of the online
  recurrence cancels between them), by the fp32 accumulations of the value
  product and the row sum (gamma_S), and by the final rounding to the dtype;
* lse_i = m_i + log Z_i is perturbed by sum_j w_ij eta'_ij (eta' without the
  P rounding, since the row sum uses the fp32 weights), the logarithm and
  the fp32 rounding of the sum.

``backward_budget`` does the same for the gradients of the FlashAttention
backward: each recomputed weight inherits the logit error and the forward
logsumexp's budget; D_i = grad_i . out_i the forward output's budget; dS the
errors of dP, D and its cast; dQ, dK, dV the errors of their fp32 sums and the
final rounding.

A ``safety`` factor (default 2) covers the second-order terms.  The forward
budget is pinned in tests/test_budget_pins.py, the backward one in
tests/test_backward_budget_pins.py: an independent low-precision emulation
of the algorithm stays inside it on random inputs, and planted mistakes (a
scale off by 0.5 %, a dropped key, lse off by ulps of the dtype) leave it.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .sdpa_ref import _as_f64, _mask_to_bias, default_scale

__all__ = ["unit_roundoff", "forward_budget", "backward_budget"]

_U32 = 2.0 ** -24


def unit_roundoff(dtype_name: str) -> float:
    """Unit roundoff of round-to-nearest: half an ulp at 1 (p bits of
    precision, implicit bit included: 2^-p)."""
    return {"float32": 2.0 ** -24, "float16": 2.0 ** -11, "bfloat16": 2.0 ** -8}[dtype_name]


def _gamma(n: int, u: float) -> float:
    return n * u / (1.0 - n * u)


def forward_budget(
    query,
    key,
    value,
    *,
    dtype_name: str,
    is_causal: bool = False,
    scale: Optional[float] = None,
    attn_mask=None,
    enable_gqa: bool = False,
    exp_rel: Optional[float] = None,
    safety: float = 2.0,
) -> Tuple[np.ndarray, np.ndarray]:
    """(tol_out, tol_lse): per-element bounds on |computed - exact| for the
    forward of these inputs (the values as given, already in their dtype),
    shapes (B, Hq, L, Ev) and (B, Hq, L)."""
    q, k, v = _as_f64(query), _as_f64(key), _as_f64(value)
    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    Ev = v.shape[-1]
    group = Hq // Hkv
    s = default_scale(E) if scale is None else float(scale)
    bias = _mask_to_bias(attn_mask, (B, Hq, L, S))
    ud = unit_roundoff(dtype_name)
    if exp_rel is None:
        # 16-bit inputs take the tensor-core path (MUFU 2^x and a degree-3
        # FMA-pipe polynomial, relative error under 7.6e-5); float32 the
        # general kernels (expf, within 2 ulp).
        exp_rel = 1e-4 if dtype_name != "float32" else 4 * _U32
    p_round = ud if dtype_name != "float32" else 0.0  # P cast to the input dtype before P V
    gE, gS = _gamma(max(E, 1), _U32), _gamma(max(S, 1), _U32)
    tol_o = np.zeros((B, Hq, L, Ev))
    tol_l = np.zeros((B, Hq, L))
    with np.errstate(invalid="ignore", over="ignore", divide="ignore"):
        for b in range(B):
            for h in range(Hq):
                kv = h // group
                qa, ka, va = q[b, h], k[b, kv], v[b, kv]
                logits = (qa @ ka.T) * s if E else np.zeros((L, S))
                if bias is not None:
                    logits = logits + bias[b, h]
                if is_causal:
                    logits = np.where(np.arange(S)[None, :] <= np.arange(L)[:, None], logits, -np.inf)
                m = np.max(logits, axis=1, keepdims=True)
                fin = np.isfinite(m)
                m = np.where(fin, m, 0.0)
                p = np.exp(logits - m)
                Z = p.sum(axis=1, keepdims=True)
                w = np.where(Z > 0, p / np.where(Z > 0, Z, 1.0), 0.0)
                out = w @ va
                # relative error of each weight before normalisation
                dl = abs(s) * gE * (np.abs(qa) @ np.abs(ka).T) if E else np.zeros((L, S))
                dl = dl + _U32 * np.abs(np.where(np.isfinite(logits), logits, 0.0))
                dl = dl + _U32 * np.abs(np.where(np.isfinite(logits), logits - m, 0.0))
                eta_sum = dl + exp_rel                      # row-sum weights (fp32)
                eta_num = eta_sum + p_round                 # value-product weights (P rounded)
                absv = np.abs(va)
                abso = np.abs(out)
                t = (w * eta_num) @ absv + (w * eta_sum).sum(axis=1, keepdims=True) * abso
                t = t + gS * (w @ absv + abso) + ud * abso + 1e-30
                tol_o[b, h] = safety * t
                lse = (m + np.log(np.where(Z > 0, Z, 1.0)))[:, 0]
                tl = (w * eta_sum).sum(axis=1) + 4 * _U32 + 2 * _U32 * np.abs(lse)
                tol_l[b, h] = safety * tl
    return tol_o, tol_l


def backward_budget(
    query,
    key,
    value,
    grad,
    *,
    dtype_name: str,
    is_causal: bool = False,
    scale: Optional[float] = None,
    enable_gqa: bool = False,
    exp_rel: Optional[float] = None,
    safety: float = 2.0,
) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(tol_dq, tol_dk, tol_dv): per-element first-order bounds for the
    gradients as the backward kernels compute them.  The error sources are
    those the exactref backward section enumerates (recomputing the forward's
    weights, then summing dP, D and the three gradient products, rounding dS
    and rounding each result), specialised to the FlashAttention backward
    the kernels implement: weights rebuilt from the forward's fp32
    logsumexp, P and dS rounded to the input dtype before they are
    multiplied, and D_i = grad_i . out_i from the forward's output in the
    input dtype."""
    q, k, v, g = (_as_f64(x) for x in (query, key, value, grad))
    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    Ev = v.shape[-1]
    group = Hq // Hkv
    s = default_scale(E) if scale is None else float(scale)
    ud = unit_roundoff(dtype_name)
    if exp_rel is None:
        exp_rel = 1e-4 if dtype_name != "float32" else 4 * _U32
    cast = ud if dtype_name != "float32" else 0.0
    gE, gEv, gS, gL = (_gamma(max(n, 1), _U32) for n in (E, Ev, S, L * group))
    # the forward's own errors enter through its output (D) and its
    # logsumexp (every recomputed weight)
    tol_o, tol_l = forward_budget(q, k, v, dtype_name=dtype_name, is_causal=is_causal, scale=scale,
                                  enable_gqa=enable_gqa, exp_rel=exp_rel, safety=1.0)
    tdq = np.zeros_like(q)
    tdk = np.zeros_like(k)
    tdv = np.zeros_like(v)
    adk = np.zeros_like(k)  # sum of |terms| of dk, dv (for their accumulation errors)
    adv = np.zeros_like(v)
    dk_ex = np.zeros_like(k)
    dv_ex = np.zeros_like(v)
    with np.errstate(invalid="ignore", over="ignore", divide="ignore"):
        for b in range(B):
            for h in range(Hq):
                kv = h // group
                qa, ka, va, ga = q[b, h], k[b, kv], v[b, kv], g[b, h]
                logits = (qa @ ka.T) * s if E else np.zeros((L, S))
                if is_causal:
                    logits = np.where(np.arange(S)[None, :] <= np.arange(L)[:, None], logits, -np.inf)
                m = np.max(logits, axis=1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0.0)
                p = np.exp(logits - m)
                Z = p.sum(axis=1, keepdims=True)
                P = np.where(Z > 0, p / np.where(Z > 0, Z, 1.0), 0.0)
                out = P @ va
                # relative error of each recomputed weight: the logit's, the
                # forward logsumexp's (its budget), the subtraction and exp;
                # the cast before P^T grad comes on top for dV
                dl = abs(s) * gE * (np.abs(qa) @ np.abs(ka).T) if E else np.zeros((L, S))
                dl = dl + 2 * _U32 * np.abs(np.where(np.isfinite(logits), logits, 0.0))
                lse = m + np.log(np.where(Z > 0, Z, 1.0))
                eta = dl + exp_rel + tol_l[b, h][:, None] + 2 * _U32 * (1 + np.abs(lse))
                dP = ga @ va.T
                adP = np.abs(ga) @ np.abs(va).T
                D = (ga * out).sum(axis=1, keepdims=True)
                # D from the forward's output in the input dtype (its budget
                # includes the rounding) and the fp32 dot product
                eD = (np.abs(ga) * tol_o[b, h]).sum(axis=1, keepdims=True)
                eD = eD + gEv * (np.abs(ga) * np.abs(out)).sum(axis=1, keepdims=True)
                dS = P * (dP - D)
                edS = P * eta * np.abs(dP - D) + P * (gEv * adP + eD) + cast * np.abs(dS)
                # dq = scale dS K
                dq = s * (dS @ ka)
                tdq[b, h] = abs(s) * (edS @ np.abs(ka) + gS * (np.abs(dS) @ np.abs(ka))) + ud * np.abs(dq)
                # dk, dv summed over the group's query heads
                adk[b, kv] += abs(s) * (np.abs(dS).T @ np.abs(qa))
                tdk[b, kv] += abs(s) * (edS.T @ np.abs(qa))
                dk_ex[b, kv] += s * (dS.T @ qa)
                adv[b, kv] += P.T @ np.abs(ga)
                tdv[b, kv] += ((P * (eta + cast)).T @ np.abs(ga))
                dv_ex[b, kv] += P.T @ ga
        tdk = tdk + gL * adk + ud * np.abs(dk_ex)
        tdv = tdv + gL * adv + ud * np.abs(dv_ex)
    return safety * tdq + 1e-30, safety * tdk + 1e-30, safety * tdv + 1e-30
