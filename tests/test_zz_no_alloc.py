"""The allocation-free decode entry point, sdpa_decode_fwd_noalloc().

It is meant for callers that cannot allocate device memory when they call
(a runtime that reserves all its memory up front, or a plugin interface that
passes only inputs and outputs), so it keeps the decode kernels' scratch in a
fixed array inside the library instead of a caller workspace.  These checks
call it through the C ABI and compare it, twice in a row, with sdpa_fwd() on
the same inputs, within the tolerances of the parity tests (bf16: 2e-2 on O,
1e-2 on lse).  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

O_TOL, L_TOL = 2e-2, 1e-2


@pytest.fixture(scope="module")
def lib():
    import os

    from scaled_dot_product_15_b200 import api, build

    if not os.path.exists(api.LIB_PATH):
        build.build()
    assert torch.cuda.is_available(), "these tests need a GPU"
    return api.load_library()


def _strides(t):
    from scaled_dot_product_15_b200 import api

    return api._i64x4(t.stride())


def _noalloc(lib, q, k, v, out, lse, scale=None):
    from scaled_dot_product_15_b200 import api

    B, Hq, L, E = q.shape
    _, Hkv, S, _ = k.shape
    Ev = v.shape[-1]
    code = {torch.float16: api.SDPA_F16, torch.bfloat16: api.SDPA_BF16}[q.dtype]
    return lib.sdpa_decode_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
        B, Hq, Hkv, L, S, E, Ev, _strides(q), _strides(k), _strides(v), _strides(out),
        0 if scale is None else 1, 0.0 if scale is None else float(scale), code,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize(
    "B,Hq,Hkv,L,S,E,dt",
    [
        (64, 32, 8, 1, 16384, 128, torch.bfloat16),   # the decode workload's shape
        (3, 8, 2, 2, 3000, 64, torch.float16),
        (1, 4, 1, 1, 777, 256, torch.bfloat16),
    ],
)
def test_noalloc_matches_sdpa_fwd_twice(lib, B, Hq, Hkv, L, S, E, dt):
    from scaled_dot_product_15_b200 import api, sdpa

    g = torch.Generator(device="cuda")
    g.manual_seed(B * 100 + S)
    q = torch.randn(B, Hq, L, E, device="cuda", generator=g).to(dt)
    k = torch.randn(B, Hkv, S, E, device="cuda", generator=g).to(dt)
    v = torch.randn(B, Hkv, S, E, device="cuda", generator=g).to(dt)
    ref_o, ref_l = sdpa(q, k, v, enable_gqa=Hq != Hkv)
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        st = _noalloc(lib, q, k, v, out, lse)
        assert st == api.SDPA_OK, lib.sdpa_status_string(st)
        torch.cuda.synchronize()
        eo = (out.float() - ref_o.float()).abs().max().item()
        el = (lse - ref_l).abs().max().item()
        assert eo <= O_TOL and el <= L_TOL, (call, eo, el)


def test_noalloc_rejects_oversized_and_unsupported(lib):
    from scaled_dot_product_15_b200 import api

    # 64 x 8 x 65536 keys needs 64 chunks x 2048 rows x 129 floats = 67.6 MB of
    # scratch, more than the 32 MiB array: refused before any launch.
    B, Hq, Hkv, S, E = 64, 32, 8, 65536, 128
    need = lib.sdpa_fwd_workspace_size(B, Hq, Hkv, 1, S, E, E, api.MASK_NONE, api.SDPA_BF16)
    assert need > 32 * 1024 * 1024
    q = torch.zeros(B, Hq, 1, E, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, S, E, device="cuda", dtype=torch.bfloat16)
    out = torch.zeros_like(q)
    lse = torch.zeros(B, Hq, 1, device="cuda")
    assert _noalloc(lib, q, k, k, out, lse) == api.SDPA_ERR_WORKSPACE
    del k
    # head size 96 is not a decode-kernel shape
    q = torch.zeros(1, 4, 1, 96, device="cuda", dtype=torch.float16)
    k = torch.zeros(1, 1, 64, 96, device="cuda", dtype=torch.float16)
    out = torch.zeros_like(q)
    lse = torch.zeros(1, 4, 1, device="cuda")
    assert _noalloc(lib, q, k, k, out, lse) == api.SDPA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
