"""Float64 CPU oracle for decode attention over a paged key/value cache.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only tests, the smoke
check and the benchmark's CPU legs use it; it shares no code with the CUDA
path.

A paged cache keeps each sequence's keys and values in fixed-size pages of a
shared pool, found through a per-sequence block table.  The hourtab.com
xFormers retainer post (its "Related retainer posts") names the engines that
use one and their classic failure: pages read past what was allocated for a
sequence give garbage attention with no error.  The pages define no further
semantics, so this oracle takes the plain reading: the keys (values) of
batch row b are the first ``seq_lens[b]`` tokens of its pages
``block_table[b, 0], block_table[b, 1], ...`` taken in table order, and the
result is ordinary attention of that row's queries over them with no mask
(exactref "scaled_dot_product_attention", "Full specification": a row with
no key gets output 0 and lse -inf).  Query head h reads key/value head
h // (Hq / Hkv).

Pool layout: k_pages (num_pages, page_size, Hkv, E), v_pages
(num_pages, page_size, Hkv, Ev); block_table (B, max_pages) integers;
seq_lens (B,) integers.  Pinned by tests/test_oracle_paged_pins.py.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .sdpa_ref import _as_f64, sdpa

__all__ = ["gather_pages", "sdpa_decode_paged"]


def gather_pages(pages, block_table, seq_lens, b: int) -> np.ndarray:
    """The first seq_lens[b] tokens of row b's pages, in table order, as
    (Hkv, n, features)."""
    pool = _as_f64(pages)
    page_size = pool.shape[1]
    n = int(np.asarray(seq_lens)[b])
    if n == 0:
        return np.zeros((pool.shape[2], 0, pool.shape[3]))
    n_pages = -(-n // page_size)
    table = np.asarray(block_table)[b, :n_pages].astype(np.int64)
    if (table < 0).any() or (table >= pool.shape[0]).any():
        raise IndexError("block table entry outside the page pool")
    tokens = np.concatenate([pool[pg] for pg in table], axis=0)[:n]  # (n, Hkv, F)
    return np.ascontiguousarray(tokens.transpose(1, 0, 2))


def sdpa_decode_paged(query, k_pages, v_pages, block_table, seq_lens,
                      scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of query (B, Hq, L, E) over each row's paged keys and
    values.  Returns out (B, Hq, L, Ev) and lse (B, Hq, L)."""
    q = _as_f64(query)
    k_pages, v_pages = _as_f64(k_pages), _as_f64(v_pages)
    B, Hq, L, E = q.shape
    Ev = v_pages.shape[-1]
    out = np.empty((B, Hq, L, Ev))
    lse = np.empty((B, Hq, L))
    for b in range(B):
        kb = gather_pages(k_pages, block_table, seq_lens, b)
        vb = gather_pages(v_pages, block_table, seq_lens, b)
        o, l_ = sdpa(q[b:b + 1], kb[None], vb[None], scale=scale, enable_gqa=True)
        out[b], lse[b] = o[0], l_[0]
    return out, lse
