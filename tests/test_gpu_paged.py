"""Parity of the paged-cache decode (sdpa_decode_paged through the C ABI) with
the float64 oracle (oracle/paged_ref.py) on the same seeded inputs.

Tolerances as for the contiguous decode: bf16/fp16 max |diff| <= 2e-2 on O
and <= 1e-2 on lse (fp32 dot products and sums over up to 2^15 keys, one
rounding of O to the dtype); an empty row must give exactly O = 0 and
lse = -inf.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import gather_pages, sdpa as ref_sdpa, sdpa_decode_paged as ref_paged

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


def _close(out, lse, ro, rl, what):
    o = out.double().cpu().numpy()
    l_ = lse.double().cpu().numpy()
    assert o.shape == ro.shape and l_.shape == rl.shape
    fin = np.isfinite(rl)
    assert np.array_equal(l_[~fin], rl[~fin]), f"{what}: non-finite lse differ"
    assert np.abs(o - ro).max(initial=0.0) <= 2e-2, f"{what}: max |dO| = {np.abs(o - ro).max():.3e}"
    assert np.abs(l_[fin] - rl[fin]).max(initial=0.0) <= 1e-2, f"{what}: lse"


def _problem(dt, B, Hq, Hkv, L, E, ps, max_pages, num_pages, lens, layout, seed):
    """Seeded query and pools; each row's table a random draw of distinct pages."""
    q = W.randn((B, Hq, L, E), seed, dt)
    shape = (num_pages, ps, Hkv, E) if layout == "token_major" else (num_pages, Hkv, ps, E)
    kp, vp = W.randn(shape, seed + 1, dt), W.randn(shape, seed + 2, dt)
    rng = np.random.default_rng(seed)
    table = np.stack([rng.permutation(num_pages)[:max_pages] for _ in range(B)]).astype(np.int32)
    return q, kp, vp, table, np.asarray(lens, dtype=np.int32)


def _oracle(q, kp, vp, table, lens, layout, scale=None):
    if layout == "head_major":  # the oracle takes token-major pools
        kp, vp = kp.transpose(1, 2), vp.transpose(1, 2)
    return ref_paged(q, kp, vp, table, lens, scale=scale)


def _run(q, kp, vp, table, lens, layout, scale=None):
    from scaled_dot_product_15_b200 import api, sdpa_decode_paged

    out, lse = sdpa_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), torch.from_numpy(table).to(DEV),
                                 torch.from_numpy(lens).to(DEV), scale, pages_layout=layout)
    torch.cuda.synchronize()
    assert api.take_device_error() == 0
    assert api.last_launch_count() in (1, 2)
    return out, lse


CASES = [
    # dtype, B, Hq, Hkv, L, E, page_size, max_pages, num_pages, seq_lens, layout
    (torch.bfloat16, 3, 32, 8, 1, 128, 16, 40, 200, [640, 1, 333], "token_major"),
    (torch.float16, 2, 8, 8, 2, 64, 1, 300, 700, [300, 0], "token_major"),
    (torch.bfloat16, 2, 8, 2, 2, 256, 256, 8, 20, [2048, 1500], "head_major"),
    (torch.float16, 4, 32, 8, 1, 128, 64, 64, 300, [4096, 4095, 65, 64], "token_major"),
    (torch.bfloat16, 1, 32, 8, 1, 128, 16, 1300, 1400, [20000], "head_major"),
    (torch.bfloat16, 2, 4, 1, 1, 64, 2, 600, 1300, [1199, 7], "token_major"),
    (torch.float16, 2, 8, 1, 1, 256, 4, 300, 700, [1197, 3], "head_major"),     # small pages, 8 rows per head
    (torch.bfloat16, 3, 32, 8, 1, 128, 4, 400, 1300, [1600, 5, 999], "token_major"),
    (torch.bfloat16, 2, 16, 2, 1, 128, 8, 200, 450, [1595, 8], "token_major"),  # smallest grouped page, 8 rows
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c[1:9]) + f"-{c[10]}")
def test_paged_decode(case):
    dt, B, Hq, Hkv, L, E, ps, max_pages, num_pages, lens, layout = case
    q, kp, vp, table, lens = _problem(dt, B, Hq, Hkv, L, E, ps, max_pages, num_pages, lens, layout, 611)
    out, lse = _run(q, kp, vp, table, lens, layout)
    ro, rl = _oracle(q, kp, vp, table, lens, layout)
    _close(out, lse, ro, rl, str(case))
    for b, n in enumerate(lens):
        if n == 0:
            assert (out[b] == 0).all() and torch.isneginf(lse[b]).all()


def test_shared_prefix_pages_and_scale():
    """Two rows reading the same prefix pages (prefix sharing), explicit scale."""
    dt = torch.bfloat16
    q, kp, vp, table, lens = _problem(dt, 2, 16, 4, 1, 128, 32, 20, 64, [600, 630], "token_major", 612)
    table[1, :10] = table[0, :10]
    out, lse = _run(q, kp, vp, table, lens, "token_major", scale=0.05)
    ro, rl = _oracle(q, kp, vp, table, lens, "token_major", scale=0.05)
    _close(out, lse, ro, rl, "shared prefix")


def test_identity_pages_match_contiguous_decode():
    """A contiguous cache cut into pages in order gives sdpa()'s result."""
    from scaled_dot_product_15_b200 import sdpa

    dt, B, Hq, Hkv, S, E, ps = torch.bfloat16, 4, 32, 8, 3072, 128, 16
    q, k, v = W.randn((B, Hq, 1, E), 613, dt), W.randn((B, Hkv, S, E), 614, dt), W.randn((B, Hkv, S, E), 615, dt)
    kp = k.transpose(1, 2).reshape(B * S // ps, ps, Hkv, E)
    vp = v.transpose(1, 2).reshape(B * S // ps, ps, Hkv, E)
    table = np.arange(B * S // ps, dtype=np.int32).reshape(B, S // ps)
    out, lse = _run(q, kp, vp, table, np.full(B, S, dtype=np.int32), "token_major")
    o2, l2 = sdpa(q.to(DEV), k.to(DEV), v.to(DEV), enable_gqa=True)
    assert torch.equal(out, o2) or (out.float() - o2.float()).abs().max() <= 4e-3
    assert (lse - l2).abs().max() <= 1e-4


def test_table_and_lengths_read_on_device_in_a_graph():
    """Block table and lengths are device data: a captured call replays with
    new contents."""
    from scaled_dot_product_15_b200 import sdpa_decode_paged

    dt = torch.bfloat16
    q, kp, vp, table, lens = _problem(dt, 2, 32, 8, 1, 128, 16, 64, 256, [1000, 200], "token_major", 616)
    qd, kd, vd = q.to(DEV), kp.to(DEV), vp.to(DEV)
    td, ld = torch.from_numpy(table).to(DEV), torch.from_numpy(lens).to(DEV)
    out, lse = sdpa_decode_paged(qd, kd, vd, td, ld)  # allocates outputs and workspace outside the graph
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sdpa_decode_paged(qd, kd, vd, td, ld, out=out, lse=lse)
    table2 = np.roll(table, 3, axis=1).copy()
    lens2 = np.array([17, 1024], dtype=np.int32)
    td.copy_(torch.from_numpy(table2))
    ld.copy_(torch.from_numpy(lens2))
    g.replay()
    torch.cuda.synchronize()
    ro, rl = _oracle(q, kp, vp, table2, lens2, "token_major")
    _close(out, lse, ro, rl, "graph replay")
    del g


def test_device_side_checks_report_and_stay_in_bounds():
    """A table entry outside the pool drops that page (code 32); a length past
    the table is clamped (code 31).  Both are found by the kernel's own
    checks before any access."""
    from scaled_dot_product_15_b200 import api

    dt = torch.bfloat16
    q, kp, vp, table, lens = _problem(dt, 2, 8, 2, 1, 128, 16, 8, 40, [100, 50], "token_major", 617)
    bad = table.copy()
    bad[0, 2] = 40                                   # one past the pool
    from scaled_dot_product_15_b200 import sdpa_decode_paged

    out, lse = sdpa_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), torch.from_numpy(bad).to(DEV),
                                 torch.from_numpy(lens).to(DEV))
    torch.cuda.synchronize()
    assert api.take_device_error() == 32
    # expected: row 0 without page 2's tokens (32..47)
    kb = gather_pages(kp, table, lens, 0)
    vb = gather_pages(vp, table, lens, 0)
    keep = np.r_[0:32, 48:100]
    ro, rl = ref_sdpa(q[0:1], kb[None][:, :, keep], vb[None][:, :, keep], enable_gqa=True)
    _close(out[0:1], lse[0:1], ro, rl, "dropped page")
    out, lse = sdpa_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), torch.from_numpy(table).to(DEV),
                                 torch.tensor([100, 9999], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert api.take_device_error() == 31
    ro, rl = _oracle(q, kp, vp, table, np.array([100, 8 * 16]), "token_major")
    _close(out, lse, ro, rl, "clamped length")
