"""CPU checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from scaled_dot_product_15_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdpa15.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sdpa_\w+)\s*\(", src)))


def test_header_declares_bound_symbols():
    assert _declared() == sorted(api.exported_symbols())


def test_library_exports_every_declared_symbol():
    lib = api.load_library()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sdpa_\w+)$", out, flags=re.M))
    assert set(_declared()) <= exported


def test_status_strings_and_version():
    lib = api.load_library()
    assert lib.sdpa_abi_version() == 2
    for s in range(5):
        assert lib.sdpa_status_string(s)
    assert lib.sdpa_status_string(99) == b"unknown status"


def _call(**kw):
    lib = api.load_library()
    a = dict(B=1, Hq=2, Hkv=2, L=8, S=8, E=64, Ev=64, mask=0, dtype=api.SDPA_BF16, scale=None,
             cu=None, n_seqs=0, maxlen=0, bias=None, ws=None, ws_bytes=0)
    a.update(kw)
    fake = 0x10000  # never dereferenced: every case below fails on the host
    st = api._i64x4((a["Hq"] * a["L"] * a["E"], a["L"] * a["E"], a["E"], 1))
    sv = api._i64x4((a["Hkv"] * a["S"] * a["Ev"], a["S"] * a["Ev"], a["Ev"], 1))
    sk = api._i64x4((a["Hkv"] * a["S"] * a["E"], a["S"] * a["E"], a["E"], 1))
    so = api._i64x4((a["Hq"] * a["L"] * a["Ev"], a["L"] * a["Ev"], a["Ev"], 1))
    if "qstride" in kw:
        st = api._i64x4(kw["qstride"])
    ptr = kw.get("ptr", fake)
    return lib.sdpa_fwd(ptr, fake, fake, fake, fake, a["B"], a["Hq"], a["Hkv"], a["L"], a["S"], a["E"], a["Ev"],
                        st, sk, sv, so, 0 if a["scale"] is None else 1, a["scale"] or 0.0, a["mask"], a["cu"],
                        a["n_seqs"], a["maxlen"], a["bias"], api._i64x4((0, 0, 0, 0)), a["dtype"], a["ws"],
                        a["ws_bytes"], None)


def test_host_side_rejections():
    assert _call(Hq=3, Hkv=2) == api.SDPA_ERR_INVALID          # Hq not a multiple of Hkv
    assert _call(dtype=7) == api.SDPA_ERR_INVALID               # unknown dtype
    assert _call(mask=9) == api.SDPA_ERR_INVALID                # unknown mask
    assert _call(E=0, Ev=0) == api.SDPA_ERR_UNSUPPORTED         # Ev = 0: no output features
    assert _call(E=512) == api.SDPA_ERR_UNSUPPORTED
    assert _call(qstride=(1, 1, 1, 2)) == api.SDPA_ERR_INVALID  # feature stride must be 1
    assert _call(mask=api.MASK_BLOCK_DIAG, B=2) == api.SDPA_ERR_INVALID
    assert _call(mask=api.MASK_BLOCK_DIAG) == api.SDPA_ERR_INVALID  # no cu_seqlens
    assert _call(mask=api.MASK_FLOAT_BIAS) == api.SDPA_ERR_INVALID  # no bias
    assert _call(mask=api.MASK_BOOL) == api.SDPA_ERR_INVALID       # no byte mask
    assert _call(mask=6) == api.SDPA_ERR_INVALID                    # unknown mask kind
    assert _call(scale=float("nan")) == api.SDPA_ERR_INVALID
    assert _call(ptr=None) == api.SDPA_ERR_INVALID
    assert _call(B=0) == api.SDPA_OK                            # empty problem: nothing to do
    assert _call(L=0) == api.SDPA_OK


def test_no_gpu_means_unsupported_not_a_crash():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _call() == api.SDPA_ERR_UNSUPPORTED


def test_workspace_size_is_deterministic():
    lib = api.load_library()
    args = (64, 32, 8, 1, 16384, 128, 128, api.MASK_NONE, api.SDPA_BF16)
    n = lib.sdpa_fwd_workspace_size(*args)
    assert n > 0 and n == lib.sdpa_fwd_workspace_size(*args)
    assert n % 4 == 0
    assert lib.sdpa_fwd_workspace_size(4, 16, 16, 2048, 2048, 128, 128, api.MASK_CAUSAL, api.SDPA_BF16) == 0
    assert lib.sdpa_fwd_workspace_size(1, 3, 2, 1, 10, 64, 64, 0, api.SDPA_BF16) == 0  # invalid


def _plan(B, Hq, Hkv, L, S, E, Ev, mask, dtype, align=0):
    lib = api.load_library()
    st = lambda H, n, e: api._i64x4((H * n * e, n * e, e, 1))
    base = 0x100000 + align
    return lib.sdpa_fwd_plan(B, Hq, Hkv, L, S, E, Ev, st(Hq, L, E), st(Hkv, S, E), st(Hkv, S, Ev),
                             st(Hq, L, Ev), mask, dtype, base, base, base, base)


def test_dispatch_plan():
    assert _plan(1, 2, 2, 64, 64, 16, 16, 0, api.SDPA_F32) == 3              # fp32: SIMT
    assert _plan(64, 32, 8, 1, 16384, 128, 128, 0, api.SDPA_BF16) == 2       # GQA decode
    assert _plan(64, 32, 8, 1, 16384, 128, 128, 0, api.SDPA_BF16, align=2) == 3  # unaligned
    assert _plan(1, 2, 2, 64, 64, 48, 48, api.MASK_FLOAT_BIAS, api.SDPA_F16) == 3
    assert _plan(1, 2, 2, 256, 256, 128, 128, api.MASK_BOOL, api.SDPA_BF16) == 3  # bool masks: general kernels
    assert _plan(1, 3, 2, 64, 64, 64, 64, 0, api.SDPA_F16) == -api.SDPA_ERR_INVALID


def _bwd(**kw):
    lib = api.load_library()
    a = dict(B=1, Hq=2, Hkv=2, L=8, S=8, E=64, Ev=64, mask=0, dtype=api.SDPA_BF16, ws=None, ws_bytes=0,
             scale=None)
    a.update(kw)
    fake = 0x10000  # never dereferenced: every case below fails on the host
    sq = api._i64x4((a["Hq"] * a["L"] * a["E"], a["L"] * a["E"], a["E"], 1))
    sk = api._i64x4((a["Hkv"] * a["S"] * a["E"], a["S"] * a["E"], a["E"], 1))
    sv = api._i64x4((a["Hkv"] * a["S"] * a["Ev"], a["S"] * a["Ev"], a["Ev"], 1))
    so = api._i64x4((a["Hq"] * a["L"] * a["Ev"], a["L"] * a["Ev"], a["Ev"], 1))
    sdq = api._i64x4(kw.get("dqstride", (a["Hq"] * a["L"] * a["E"], a["L"] * a["E"], a["E"], 1)))
    ptr = kw.get("ptr", fake)
    return lib.sdpa_bwd(fake, fake, fake, fake, fake, fake, ptr, fake, fake,
                        a["B"], a["Hq"], a["Hkv"], a["L"], a["S"], a["E"], a["Ev"],
                        sq, sk, sv, so, so, sdq, sk, sv, 0 if a["scale"] is None else 1, a["scale"] or 0.0,
                        a["mask"], None, 0, 0, None, api._i64x4((0, 0, 0, 0)), a["dtype"], a["ws"],
                        a["ws_bytes"], None)


def test_backward_host_side_rejections_and_workspace():
    lib = api.load_library()
    assert lib.sdpa_bwd_workspace_size(4, 16, 16, 2048, 2048, 128, 128, api.MASK_CAUSAL, api.SDPA_BF16) == 4 * 16 * 2048 * 4
    assert lib.sdpa_bwd_workspace_size(1, 3, 2, 8, 8, 64, 64, 0, api.SDPA_BF16) == 0  # invalid shape
    assert lib.sdpa_bwd_workspace_size(1, 2, 2, 3, 8, 64, 64, 0, api.SDPA_BF16) == 256  # rounded up
    assert _bwd(Hq=3, Hkv=2) == api.SDPA_ERR_INVALID
    assert _bwd(E=300) == api.SDPA_ERR_UNSUPPORTED
    assert _bwd(dqstride=(1, 1, 1, 2)) == api.SDPA_ERR_INVALID     # a gradient's feature stride
    assert _bwd(scale=float("inf")) == api.SDPA_ERR_INVALID
    assert _bwd(ptr=None) == api.SDPA_ERR_INVALID                   # missing dq
    assert _bwd() == api.SDPA_ERR_WORKSPACE                         # D needs workspace
    import torch

    if not torch.cuda.is_available():  # with a GPU this would launch on fake pointers
        assert _bwd(ws=0x10100, ws_bytes=256) == api.SDPA_ERR_UNSUPPORTED
    assert _bwd(ws=0x10180, ws_bytes=256) == api.SDPA_ERR_WORKSPACE  # not 256-byte aligned
    assert _bwd(B=0) == api.SDPA_OK


def _paged(B=2, Hq=8, Hkv=2, L=1, E=128, Ev=128, num_pages=16, page_size=16, max_pages=4, dtype=api.SDPA_BF16,
           kstride=None, scale=None, ptr=0x100000, table=0x200000):
    lib = api.load_library()
    qs = api._i64x4((Hq * L * E, L * E, E, 1))
    ks = api._i64x4(kstride or (page_size * Hkv * E, E, Hkv * E, 1))  # token-major pool
    os_ = api._i64x4((Hq * L * Ev, L * Ev, Ev, 1))
    return lib.sdpa_decode_paged(ptr, ptr, ptr, table, table, ptr, ptr, B, Hq, Hkv, L, E, Ev, num_pages, page_size,
                                 max_pages, qs, ks, ks, os_, 0 if scale is None else 1, scale or 0.0, dtype,
                                 None, 0, None)


def test_paged_decode_host_side_rejections_and_workspace():
    assert _paged(Hq=3, Hkv=2) == api.SDPA_ERR_INVALID           # Hq not a multiple of Hkv
    assert _paged(page_size=24) == api.SDPA_ERR_UNSUPPORTED      # not a power of two
    assert _paged(page_size=0) == api.SDPA_ERR_INVALID
    assert _paged(max_pages=0) == api.SDPA_ERR_INVALID
    assert _paged(num_pages=0) == api.SDPA_ERR_INVALID
    assert _paged(dtype=api.SDPA_F32) == api.SDPA_ERR_UNSUPPORTED  # 16-bit only
    assert _paged(E=96, Ev=96) == api.SDPA_ERR_UNSUPPORTED       # E in {64, 128, 256}
    assert _paged(Hq=16, Hkv=1) == api.SDPA_ERR_UNSUPPORTED      # more than 8 rows per key/value head
    assert _paged(kstride=(1, 1, 1, 2)) == api.SDPA_ERR_INVALID  # feature stride must be 1
    assert _paged(kstride=(16, 8, 4, 1)) == api.SDPA_ERR_UNSUPPORTED  # rows not 16-byte aligned
    assert _paged(scale=float("inf")) == api.SDPA_ERR_INVALID
    assert _paged(ptr=None) == api.SDPA_ERR_INVALID
    assert _paged(table=None) == api.SDPA_ERR_INVALID
    assert _paged(B=0, ptr=None, table=None) == api.SDPA_OK       # empty problem
    lib = api.load_library()
    n = lib.sdpa_decode_paged_workspace_size(64, 32, 8, 1, 128, 128, 16, 1024, api.SDPA_BF16)
    assert n > 0 and n == lib.sdpa_fwd_workspace_size(64, 32, 8, 1, 16384, 128, 128, api.MASK_NONE, api.SDPA_BF16)
    assert lib.sdpa_decode_paged_workspace_size(64, 32, 8, 1, 128, 128, 24, 1024, api.SDPA_BF16) == 0
    assert _paged(B=64, Hq=32, Hkv=8, max_pages=1024, num_pages=65536) == api.SDPA_ERR_WORKSPACE  # needs scratch


def test_paged_decode_without_gpu_is_unsupported():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _paged() == api.SDPA_ERR_UNSUPPORTED


def test_mask_arguments_are_marshalled_without_conversion_of_bool_masks():
    import torch

    m = torch.rand(5, 7) > 0.5
    kind, t, st = api._mask_arg(m, torch.device("cpu"), 2, 3, 5, 7)
    assert kind == api.MASK_BOOL and t.dtype == torch.bool and t.data_ptr() == m.data_ptr()
    assert tuple(st) == (0, 0, 7, 1) and t.shape == (2, 3, 5, 7)      # broadcast, byte strides
    f = torch.randn(2, 1, 5, 7, dtype=torch.float16)
    kind, t, st = api._mask_arg(f, torch.device("cpu"), 2, 3, 5, 7)
    assert kind == api.MASK_FLOAT_BIAS and t.dtype == torch.float32
    assert tuple(st) == (35, 0, 7, 1)
