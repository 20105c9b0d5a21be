"""Seeded synthetic workloads for scaled dot-product attention.

This module is shared by the tests, the smoke check and the benchmark, and by
both sides of every parity check (the float64 oracle and the CUDA library).  It
holds only shapes, seeds and random-number generation: none of the attention
arithmetic.

Inputs are iid N(0, 1) drawn in float32 by ``torch.randn`` with a CPU
``torch.Generator`` seeded per tensor, then rounded once to the workload's
dtype.  Large tensors are drawn in chunks along their leading axis, chunk ``i``
from its own seed, so any slice can be regenerated on the CPU without
generating the rest.

The five workloads restate the configurations the method is measured on:
fp32 small case (worked-example scale), bf16 causal prefill, fp16 packed
variable-length block-diagonal causal attention, bf16 grouped-query decode and
fp16 causal prefill with head_dim 96 at scale 1/sqrt(96) and 1/96 (the
double-scaling case of the hourtab.com xFormers post).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

DTYPES = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "fp32" | "fp16" | "bf16"
    B: int
    Hq: int
    Hkv: int
    L: int
    S: int
    E: int
    Ev: int
    mask: str  # "none" | "causal" | "block_diag" | "block_diag_causal"
    seed: int
    layout: str = "bhle"  # "bhle" (B, H, L, E) or "packed" (1, T, H, E)
    scale: Optional[float] = None
    varlen_lo: int = 0
    varlen_hi: int = 0

    @property
    def torch_dtype(self) -> torch.dtype:
        return DTYPES[self.dtype]


# The five workloads.  Names state what each is, with its sizes.
WORKLOADS = {
    "fp32_b1_h2_l64_e16": Workload("fp32_b1_h2_l64_e16", "fp32", 1, 2, 2, 64, 64, 16, 16, "none", 0),
    "fp32_b1_h2_l64_e16_causal": Workload("fp32_b1_h2_l64_e16_causal", "fp32", 1, 2, 2, 64, 64, 16, 16, "causal", 0),
    "bf16_causal_b4_h16_l2048_e128": Workload(
        "bf16_causal_b4_h16_l2048_e128", "bf16", 4, 16, 16, 2048, 2048, 128, 128, "causal", 2
    ),
    "fp16_varlen_t32768_h8_e64": Workload(
        "fp16_varlen_t32768_h8_e64", "fp16", 1, 8, 8, 32768, 32768, 64, 64, "block_diag_causal", 3,
        layout="packed", varlen_lo=8, varlen_hi=4096,
    ),
    "bf16_gqa_decode_b64_hq32_hkv8_s16384_e128": Workload(
        "bf16_gqa_decode_b64_hq32_hkv8_s16384_e128", "bf16", 64, 32, 8, 1, 16384, 128, 128, "none", 4
    ),
    "fp16_causal_b1_h64_l2048_e96": Workload(
        "fp16_causal_b1_h64_l2048_e96", "fp16", 1, 64, 64, 2048, 2048, 96, 96, "causal", 5
    ),
    "fp16_causal_b1_h64_l2048_e96_scale1_96": Workload(
        "fp16_causal_b1_h64_l2048_e96_scale1_96", "fp16", 1, 64, 64, 2048, 2048, 96, 96, "causal", 5,
        scale=1.0 / 96.0,
    ),
}

# The workload the benchmark times by default: bf16 causal prefill.
HEADLINE = "bf16_causal_b4_h16_l2048_e128"


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn(shape: Sequence[int], seed: int, dtype: torch.dtype) -> torch.Tensor:
    """iid N(0,1) in float32 from ``seed``, rounded once to ``dtype`` (CPU)."""
    x = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    return x.to(dtype)


def chunk_seed(seed: int, index: int) -> int:
    """Seed of chunk ``index`` of a tensor drawn in chunks."""
    return (int(seed) * 1_000_003 + 7919 * int(index) + 17) % (2**62)


def randn_chunk(shape: Sequence[int], seed: int, index: int, dtype: torch.dtype) -> torch.Tensor:
    """Chunk ``index`` (along the leading axis) of a tensor drawn by chunks:
    its shape is ``shape[1:]``."""
    return randn(tuple(shape[1:]), chunk_seed(seed, index), dtype)


def randn_chunked(shape: Sequence[int], seed: int, dtype: torch.dtype, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole tensor drawn by chunks along its leading axis; ``out`` (any
    device) receives it chunk by chunk when given."""
    if out is None:
        out = torch.empty(tuple(shape), dtype=dtype)
    for i in range(shape[0]):
        out[i].copy_(randn_chunk(shape, seed, i, dtype))
    return out


def tensor_seeds(w: Workload) -> Tuple[int, int, int]:
    """Seeds of Q, K and V for a workload."""
    return (w.seed * 3 + 0, w.seed * 3 + 1, w.seed * 3 + 2)


def varlen_seqlens(total: int, lo: int, hi: int, seed: int) -> List[int]:
    """Segment lengths drawn uniformly from the integers [lo, hi] until they
    reach ``total``; the last one is cut to fit (so it may be shorter than lo)."""
    rng = np.random.default_rng(seed)
    out: List[int] = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return out


def cu_seqlens_of(seqlens: Sequence[int]) -> List[int]:
    cu = [0]
    for n in seqlens:
        cu.append(cu[-1] + int(n))
    return cu


def shapes(w: Workload) -> Tuple[Tuple[int, ...], Tuple[int, ...], Tuple[int, ...]]:
    """Shapes of Q, K, V: (B, H, L, E) or, packed, (1, T, H, E)."""
    if w.layout == "packed":
        return (1, w.L, w.Hq, w.E), (1, w.S, w.Hkv, w.E), (1, w.S, w.Hkv, w.Ev)
    return (w.B, w.Hq, w.L, w.E), (w.B, w.Hkv, w.S, w.E), (w.B, w.Hkv, w.S, w.Ev)


def make_inputs(w: Workload, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V of a workload on ``device``, drawn on the CPU by chunks along
    the leading axis (batch for BHLE, the single packed batch otherwise)."""
    qs, ks, vs = shapes(w)
    sq, sk, sv = tensor_seeds(w)
    out = []
    for shp, sd in ((qs, sq), (ks, sk), (vs, sv)):
        t = torch.empty(shp, dtype=w.torch_dtype, device=device)
        randn_chunked(shp, sd, w.torch_dtype, out=t)
        out.append(t)
    return out[0], out[1], out[2]


def make_slice(w: Workload, which: str, b: int) -> torch.Tensor:
    """Batch entry ``b`` of Q, K or V regenerated on the CPU (BHLE layout)."""
    qs, ks, vs = shapes(w)
    sq, sk, sv = tensor_seeds(w)
    shp, sd = {"q": (qs, sq), "k": (ks, sk), "v": (vs, sv)}[which]
    return randn_chunk(shp, sd, b, w.torch_dtype)


def workload_seqlens(w: Workload) -> Optional[List[int]]:
    if w.layout != "packed":
        return None
    return varlen_seqlens(w.L, w.varlen_lo, w.varlen_hi, w.seed)


def kept_pairs(w: Workload, seqlens: Optional[Sequence[int]] = None) -> int:
    """Number of (query, key) pairs the mask keeps: the unit of work.

    Causal keeps j <= i (L(L+1)/2 pairs per head when L = S); block-diagonal
    keeps pairs inside one segment; block-diagonal causal both."""
    if w.layout == "packed":
        sl = seqlens if seqlens is not None else workload_seqlens(w)
        if w.mask == "block_diag_causal":
            per_head = sum(n * (n + 1) // 2 for n in sl)
        else:
            per_head = sum(n * n for n in sl)
        return per_head * w.Hq
    if w.mask == "causal":
        per = sum(min(i + 1, w.S) for i in range(w.L))
    else:
        per = w.L * w.S
    return per * w.B * w.Hq


def flops(w: Workload, seqlens: Optional[Sequence[int]] = None) -> int:
    """Algorithmic flops: 2*E (scores) + 2*Ev (weighted sum) per kept pair."""
    return kept_pairs(w, seqlens) * (2 * w.E + 2 * w.Ev)


def kv_bytes(w: Workload) -> int:
    """K and V bytes one call must read (decode's unit of work)."""
    el = torch.tensor([], dtype=w.torch_dtype).element_size()
    return w.B * w.Hkv * w.S * (w.E + w.Ev) * el
