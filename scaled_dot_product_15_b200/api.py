"""Thin Python binding of the C ABI in include/sdpa15.h.

Argument marshalling only: shapes, strides, pointers and the stream are read
from torch tensors and passed to ``sdpa_fwd``; every step of the attention
runs in the library's CUDA kernels.  torch provides device memory (outputs and
the workspace) and the current stream.  There is no fallback: if the library
is missing or the device is not a B200 the call raises.

Mask arguments are passed in the library's formats: a boolean mask (True
where the key is visible) as its bytes, a floating mask as float32 (cast
when it has another dtype) -- the two mask kinds of the exactref page's
"Arguments".
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libsdpa15.so")

SDPA_OK, SDPA_ERR_INVALID, SDPA_ERR_UNSUPPORTED, SDPA_ERR_CUDA, SDPA_ERR_WORKSPACE = range(5)
SDPA_F32, SDPA_F16, SDPA_BF16 = 0, 1, 2
MASK_NONE, MASK_CAUSAL, MASK_BLOCK_DIAG, MASK_BLOCK_DIAG_CAUSAL, MASK_FLOAT_BIAS, MASK_BOOL = range(6)
PLAN_NAMES = {1: "prefill_tcgen05", 2: "decode_split", 3: "simt"}

_DTYPE_CODE = {torch.float32: SDPA_F32, torch.float16: SDPA_F16, torch.bfloat16: SDPA_BF16}

# Every symbol include/sdpa15.h declares, with its ctypes signature.
_I64x4 = ctypes.POINTER(ctypes.c_int64)
_SIGNATURES = {
    "sdpa_abi_version": (ctypes.c_int, []),
    "sdpa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sdpa_fwd_workspace_size": (ctypes.c_size_t, [ctypes.c_int] * 9),
    "sdpa_fwd": (
        ctypes.c_int,
        [ctypes.c_void_p] * 5
        + [ctypes.c_int] * 7
        + [_I64x4] * 4
        + [ctypes.c_int, ctypes.c_float]
        + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        + [ctypes.c_void_p, _I64x4]
        + [ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    ),
    "sdpa_fwd_plan": (
        ctypes.c_int,
        [ctypes.c_int] * 7 + [_I64x4] * 4 + [ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 4,
    ),
    "sdpa_bwd_workspace_size": (ctypes.c_size_t, [ctypes.c_int] * 9),
    "sdpa_bwd": (
        ctypes.c_int,
        [ctypes.c_void_p] * 9
        + [ctypes.c_int] * 7
        + [_I64x4] * 8
        + [ctypes.c_int, ctypes.c_float]
        + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        + [ctypes.c_void_p, _I64x4]
        + [ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    ),
    "sdpa_bwd_plan": (
        ctypes.c_int,
        [ctypes.c_int] * 7 + [_I64x4] * 7 + [ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 7,
    ),
    "sdpa_last_launch_count": (ctypes.c_int, []),
    "sdpa_take_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int)]),
    "sdpa_decode_fwd_noalloc": (
        ctypes.c_int,
        [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [_I64x4] * 4
        + [ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p],
    ),
    "sdpa_decode_paged_workspace_size": (ctypes.c_size_t, [ctypes.c_int] * 9),
    "sdpa_decode_paged": (
        ctypes.c_int,
        [ctypes.c_void_p] * 7 + [ctypes.c_int] * 9 + [_I64x4] * 4
        + [ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    ),
}

_lib = None
_lib_lock = threading.Lock()


class SdpaError(RuntimeError):
    pass


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise SdpaError(
                f"CUDA library not built: {path} is missing "
                "(run python -m scaled_dot_product_15_b200.build)"
            )
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def exported_symbols() -> Sequence[str]:
    return tuple(_SIGNATURES)


def _i64x4(vals) -> ctypes.Array:
    return (ctypes.c_int64 * 4)(*[int(x) for x in vals])


def _check(status: int, what: str) -> None:
    if status != SDPA_OK:
        msg = load_library().sdpa_status_string(status).decode()
        raise SdpaError(f"{what}: {msg} (status {status})")


_ws_cache = {}


def _workspace(device: torch.device, nbytes: int) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    key = (device.type, device.index)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _strides(t: torch.Tensor, layout: str):
    s = t.stride()
    if layout == "bhle":
        return (s[0], s[1], s[2], s[3])
    if layout == "bmhk":
        return (s[0], s[2], s[1], s[3])
    raise ValueError(f"unknown layout {layout!r}")


def _dims(t: torch.Tensor, layout: str):
    if layout == "bhle":
        return t.shape[0], t.shape[1], t.shape[2], t.shape[3]  # B, H, seq, feat
    return t.shape[0], t.shape[2], t.shape[1], t.shape[3]


def _mask_arg(attn_mask: torch.Tensor, dev, B: int, Hq: int, L: int, S: int):
    """(mask kind, tensor, strides) of an attn_mask for the C ABI: a bool
    mask goes as bytes (MASK_BOOL, no copy beyond the move to the device), a
    float mask as float32 (MASK_FLOAT_BIAS); both broadcast to (B, Hq, L, S)
    with zero strides."""
    m = attn_mask.to(dev)
    if m.dtype == torch.bool:
        kind = MASK_BOOL
    else:
        kind = MASK_FLOAT_BIAS
        if m.dtype != torch.float32:
            m = m.to(torch.float32)
    m = m.expand(B, Hq, L, S)
    return kind, m, _i64x4(m.stride())


def sdpa(
    query: torch.Tensor,
    key: torch.Tensor,
    value: torch.Tensor,
    attn_mask: Optional[torch.Tensor] = None,
    dropout_p: float = 0.0,
    is_causal: bool = False,
    scale: Optional[float] = None,
    enable_gqa: bool = False,
    *,
    layout: str = "bhle",
    cu_seqlens: Optional[torch.Tensor] = None,
    max_seqlen: Optional[int] = None,
    out: Optional[torch.Tensor] = None,
    lse: Optional[torch.Tensor] = None,
) -> Tuple[torch.Tensor, torch.Tensor]:
    """softmax(Q K^T * scale + mask) V and the per-row logsumexp, on a B200.

    ``layout="bhle"``: tensors are (B, H, L, E); ``"bmhk"``: (B, L, H, E), the
    xFormers layout; ``"bmghk"``: the xFormers grouped layout (B, L, G, H, E)
    with key/value broadcast over H (see _sdpa_bmghk).  With ``cu_seqlens`` (int32, on the device, n+1 cumulative
    segment starts) the inputs are one packed batch (1, T, H, E) attended
    block-diagonally, causally within each segment when ``is_causal``.
    Returns ``(out, lse)``: out in the query's layout with Ev features, lse
    float32 of shape (B, Hq, L).
    """
    if dropout_p != 0.0:
        raise ValueError("dropout_p must be 0: a random dropout has no deterministic result to check")
    if layout == "bmghk":
        return _sdpa_bmghk(query, key, value, attn_mask, is_causal, scale, out, lse)
    lib = load_library()
    if query.dim() != 4 or key.dim() != 4 or value.dim() != 4:
        raise ValueError("query, key and value must be 4-D")
    if not (query.dtype == key.dtype == value.dtype):
        raise ValueError("query, key and value must share a dtype")
    if query.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {query.dtype}")
    if not (query.is_cuda and key.is_cuda and value.is_cuda):
        raise ValueError("inputs must be CUDA tensors")
    if cu_seqlens is not None and layout == "bhle":
        layout = "bmhk"  # packed batches are (1, T, H, E)
    B, Hq, L, E = _dims(query, layout)
    Bk, Hkv, S, Ek = _dims(key, layout)
    Bv, Hv, Sv, Ev = _dims(value, layout)
    if Bk != B or Bv != B or Ek != E or Sv != S or Hv != Hkv:
        raise ValueError("query/key/value shapes do not agree")
    if Hq != Hkv and not enable_gqa:
        raise ValueError("query heads differ from key/value heads: pass enable_gqa=True")
    if cu_seqlens is not None and attn_mask is not None:
        raise ValueError("attn_mask cannot be combined with cu_seqlens")
    if is_causal and attn_mask is not None:
        raise ValueError("pass either attn_mask or is_causal, not both")
    dev = query.device
    dcode = _DTYPE_CODE[query.dtype]

    if out is None:
        if layout == "bhle":
            out = torch.empty((B, Hq, L, Ev), dtype=query.dtype, device=dev)
        else:
            out = torch.empty((B, L, Hq, Ev), dtype=query.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    if not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be a contiguous float32 tensor")

    mask_kind = MASK_NONE
    bias_t = None
    bias_str = _i64x4((0, 0, 0, 0))
    cu_ptr, n_seqs, maxlen = None, 0, 0
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        mask_kind = MASK_BLOCK_DIAG_CAUSAL if is_causal else MASK_BLOCK_DIAG
        n_seqs = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        maxlen = int(max_seqlen)
        cu_ptr = cu_seqlens.data_ptr()
    elif is_causal:
        mask_kind = MASK_CAUSAL
    elif attn_mask is not None:
        mask_kind, bias_t, bias_str = _mask_arg(attn_mask, dev, B, Hq, L, S)

    qs, ks, vs, os_ = (_i64x4(_strides(t, layout)) for t in (query, key, value, out))
    ws_bytes = lib.sdpa_fwd_workspace_size(B, Hq, Hkv, L, S, E, Ev, mask_kind, dcode)
    ws = _workspace(dev, ws_bytes)
    ws_ptr = None
    if ws is not None:
        base = ws.data_ptr()
        ws_ptr = (base + 255) // 256 * 256
    stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        status = lib.sdpa_fwd(
            query.data_ptr(), key.data_ptr(), value.data_ptr(), out.data_ptr(), lse.data_ptr(),
            B, Hq, Hkv, L, S, E, Ev, qs, ks, vs, os_,
            0 if scale is None else 1, 0.0 if scale is None else float(scale),
            mask_kind, cu_ptr, n_seqs, maxlen,
            None if bias_t is None else bias_t.data_ptr(), bias_str,
            dcode, ws_ptr, ws_bytes, stream,
        )
    _check(status, "sdpa_fwd")
    return out, lse


def sdpa_backward(
    query: torch.Tensor,
    key: torch.Tensor,
    value: torch.Tensor,
    out: torch.Tensor,
    lse: torch.Tensor,
    grad: torch.Tensor,
    attn_mask: Optional[torch.Tensor] = None,
    dropout_p: float = 0.0,
    is_causal: bool = False,
    scale: Optional[float] = None,
    enable_gqa: bool = False,
    *,
    layout: str = "bhle",
    cu_seqlens: Optional[torch.Tensor] = None,
    max_seqlen: Optional[int] = None,
) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(grad_query, grad_key, grad_value) for the output gradient ``grad``,
    given the forward's inputs and its outputs ``out`` and ``lse`` (as sdpa()
    returned them); the other arguments are sdpa()'s."""
    if dropout_p != 0.0:
        raise ValueError("dropout_p must be 0: a random dropout has no deterministic result to check")
    lib = load_library()
    for t in (query, key, value, out, grad):
        if t.dim() != 4 or not t.is_cuda:
            raise ValueError("query, key, value, out and grad must be 4-D CUDA tensors")
    if not (query.dtype == key.dtype == value.dtype == out.dtype == grad.dtype):
        raise ValueError("query, key, value, out and grad must share a dtype")
    if query.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {query.dtype}")
    if cu_seqlens is not None and layout == "bhle":
        layout = "bmhk"
    B, Hq, L, E = _dims(query, layout)
    _, Hkv, S, _ = _dims(key, layout)
    Ev = _dims(value, layout)[3]
    if Hq != Hkv and not enable_gqa:
        raise ValueError("query heads differ from key/value heads: pass enable_gqa=True")
    if tuple(grad.shape) != tuple(out.shape):
        raise ValueError("grad must have the output's shape")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, L):
        raise ValueError("lse must be the forward's contiguous float32 (B, Hq, L) logsumexp")
    if is_causal and attn_mask is not None:
        raise ValueError("pass either attn_mask or is_causal, not both")
    dev = query.device
    dcode = _DTYPE_CODE[query.dtype]
    mask_kind = MASK_NONE
    bias_t, bias_str = None, _i64x4((0, 0, 0, 0))
    cu_ptr, n_seqs, maxlen = None, 0, 0
    if cu_seqlens is not None:
        if attn_mask is not None:
            raise ValueError("attn_mask cannot be combined with cu_seqlens")
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        mask_kind = MASK_BLOCK_DIAG_CAUSAL if is_causal else MASK_BLOCK_DIAG
        cu_ptr, n_seqs, maxlen = cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, int(max_seqlen)
    elif is_causal:
        mask_kind = MASK_CAUSAL
    elif attn_mask is not None:
        mask_kind, bias_t, bias_str = _mask_arg(attn_mask, dev, B, Hq, L, S)
    dq, dk, dv = torch.empty_like(query), torch.empty_like(key), torch.empty_like(value)
    strides = [_i64x4(_strides(t, layout)) for t in (query, key, value, out, grad, dq, dk, dv)]
    ws_bytes = lib.sdpa_bwd_workspace_size(B, Hq, Hkv, L, S, E, Ev, mask_kind, dcode)
    ws = _workspace(dev, ws_bytes)
    ws_ptr = None if ws is None else (ws.data_ptr() + 255) // 256 * 256
    stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        status = lib.sdpa_bwd(
            query.data_ptr(), key.data_ptr(), value.data_ptr(), out.data_ptr(), lse.data_ptr(),
            grad.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
            B, Hq, Hkv, L, S, E, Ev, *strides,
            0 if scale is None else 1, 0.0 if scale is None else float(scale),
            mask_kind, cu_ptr, n_seqs, maxlen,
            None if bias_t is None else bias_t.data_ptr(), bias_str,
            dcode, ws_ptr, ws_bytes, stream,
        )
    _check(status, "sdpa_bwd")
    return dq, dk, dv


def backward_plan(query, key, value, grad, *, layout="bhle", mask_kind=MASK_NONE) -> str:
    """Name of the kernel family sdpa_backward() would run for these tensors
    (gradients laid out like their inputs)."""
    lib = load_library()
    B, Hq, L, E = _dims(query, layout)
    _, Hkv, S, _ = _dims(key, layout)
    Ev = _dims(value, layout)[3]
    st = [_i64x4(_strides(t, layout)) for t in (query, key, value, grad, query, key, value)]
    r = lib.sdpa_bwd_plan(B, Hq, Hkv, L, S, E, Ev, *st, mask_kind, _DTYPE_CODE[query.dtype],
                          query.data_ptr(), key.data_ptr(), value.data_ptr(), grad.data_ptr(),
                          query.data_ptr(), key.data_ptr(), value.data_ptr())
    if r < 0:
        _check(-r, "sdpa_bwd_plan")
    return {1: "backward_tcgen05", 3: "backward_simt"}[r]


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, query, key, value, is_causal, scale, enable_gqa, layout, cu_seqlens, max_seqlen):
        out, lse = sdpa(query, key, value, is_causal=is_causal, scale=scale, enable_gqa=enable_gqa,
                        layout=layout, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen)
        ctx.save_for_backward(query, key, value, out, lse)
        ctx.args = (is_causal, scale, enable_gqa, layout, cu_seqlens, max_seqlen)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, grad_out, grad_lse):
        query, key, value, out, lse = ctx.saved_tensors
        is_causal, scale, enable_gqa, layout, cu_seqlens, max_seqlen = ctx.args
        dq, dk, dv = sdpa_backward(query, key, value, out, lse, grad_out.contiguous(), is_causal=is_causal,
                                   scale=scale, enable_gqa=enable_gqa, layout=layout, cu_seqlens=cu_seqlens,
                                   max_seqlen=max_seqlen)
        return dq, dk, dv, None, None, None, None, None, None


def attention(query, key, value, is_causal=False, scale=None, enable_gqa=False, *, layout="bhle",
              cu_seqlens=None, max_seqlen=None) -> torch.Tensor:
    """sdpa() as a differentiable op: returns the output; its backward runs
    sdpa_backward() (the logsumexp is kept for it, not differentiated)."""
    return _Attention.apply(query, key, value, is_causal, scale, enable_gqa, layout, cu_seqlens, max_seqlen)[0]


def _sdpa_bmghk(query, key, value, attn_mask, is_causal, scale, out, lse):
    """The xFormers BMGHK layout (insureai360 tutorial, section 5
    "Grouped-query attention"): query (B, M, G, H, K); key and value
    (B, M, G, H, K) with the H axis a broadcast (stride 0) or of extent 1, so
    that query head (g, h) reads key/value group g.  Views only: the query's
    (G, H) axes merge into G*H heads and the key/value's H axis is dropped,
    which is exactly the contiguous GQA grouping the kernels implement.
    Returns out (B, M, G, H, Kv) and lse (B, G, H, M)."""
    for t in (query, key, value):
        if t.dim() != 5:
            raise ValueError("bmghk tensors must be 5-D")
    B, M, G, H, K = query.shape
    if query.stride(2) != H * query.stride(3):
        raise ValueError("the query's G and H axes must be mergeable (stride_G == H * stride_H)")
    if key.shape[2] != G or value.shape[2] != G:
        raise ValueError("key/value must have the query's G axis")
    q4 = query.reshape(B, M, G * H, K) if query.is_contiguous() else query.view(B, M, G * H, K)
    k4 = key[:, :, :, 0, :]
    v4 = value[:, :, :, 0, :]
    o4 = None if out is None else out.view(B, M, G * H, value.shape[-1])
    l3 = None if lse is None else lse.view(B, G * H, M)
    o, l = sdpa(q4, k4, v4, attn_mask=attn_mask, is_causal=is_causal, scale=scale, enable_gqa=H > 1,
                layout="bmhk", out=o4, lse=l3)
    return o.view(B, M, G, H, value.shape[-1]), l.view(B, G, H, M)


def plan(query, key, value, *, layout="bhle", mask_kind=MASK_NONE, out=None) -> str:
    """Name of the kernel family sdpa() would run for these tensors."""
    lib = load_library()
    B, Hq, L, E = _dims(query, layout)
    _, Hkv, S, _ = _dims(key, layout)
    Ev = _dims(value, layout)[3]
    if out is None:
        shape = (B, Hq, L, Ev) if layout == "bhle" else (B, L, Hq, Ev)
        out = torch.empty(shape, dtype=query.dtype, device=query.device)
    r = lib.sdpa_fwd_plan(
        B, Hq, Hkv, L, S, E, Ev,
        *(_i64x4(_strides(t, layout)) for t in (query, key, value, out)),
        mask_kind, _DTYPE_CODE[query.dtype],
        query.data_ptr(), key.data_ptr(), value.data_ptr(), out.data_ptr(),
    )
    if r < 0:
        _check(-r, "sdpa_fwd_plan")
    return PLAN_NAMES[r]


def sdpa_decode_paged(
    query: torch.Tensor,
    k_pages: torch.Tensor,
    v_pages: torch.Tensor,
    block_table: torch.Tensor,
    seq_lens: torch.Tensor,
    scale: Optional[float] = None,
    *,
    pages_layout: str = "token_major",
    out: Optional[torch.Tensor] = None,
    lse: Optional[torch.Tensor] = None,
) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode attention of query (B, Hq, L, E) over a paged key/value cache.

    Row b's keys and values are the first ``seq_lens[b]`` tokens of pages
    ``block_table[b, 0], block_table[b, 1], ...`` of the pools (see
    sdpa_decode_paged in include/sdpa15.h).  ``pages_layout="token_major"``:
    pools (num_pages, page_size, Hkv, E); ``"head_major"``: (num_pages, Hkv,
    page_size, E).  block_table (B, max_pages) and seq_lens (B,) are int32 on
    the device.  Returns ``(out, lse)``: out (B, Hq, L, Ev), lse float32
    (B, Hq, L).  Query heads are grouped over key/value heads (Hq a multiple
    of Hkv).
    """
    lib = load_library()
    if query.dim() != 4 or k_pages.dim() != 4 or v_pages.dim() != 4:
        raise ValueError("query and the page pools must be 4-D")
    if not (query.dtype == k_pages.dtype == v_pages.dtype) or query.dtype not in _DTYPE_CODE:
        raise ValueError("query and the page pools must share a supported dtype")
    for t, name in ((block_table, "block_table"), (seq_lens, "seq_lens")):
        if t.dtype != torch.int32 or not t.is_cuda:
            raise ValueError(f"{name} must be an int32 CUDA tensor")
    if not (query.is_cuda and k_pages.is_cuda and v_pages.is_cuda):
        raise ValueError("inputs must be CUDA tensors")
    B, Hq, L, E = query.shape
    if pages_layout == "token_major":
        num_pages, page_size, Hkv, Ek = k_pages.shape
        perm = (0, 2, 1, 3)
    elif pages_layout == "head_major":
        num_pages, Hkv, page_size, Ek = k_pages.shape
        perm = (0, 1, 2, 3)
    else:
        raise ValueError(f"unknown pages_layout {pages_layout!r}")
    Ev = v_pages.shape[-1]
    if Ek != E or tuple(v_pages.shape[:3]) != tuple(k_pages.shape[:3]):
        raise ValueError("query and page pool shapes do not agree")
    if Hkv == 0 or Hq % Hkv != 0:
        raise ValueError("query heads must be a multiple of key/value heads")
    if block_table.dim() != 2 or block_table.shape[0] != B or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous (B, max_pages) tensor")
    if seq_lens.shape != (B,) or not seq_lens.is_contiguous():
        raise ValueError("seq_lens must be a contiguous (B,) tensor")
    max_pages = block_table.shape[1]
    dev = query.device
    dcode = _DTYPE_CODE[query.dtype]
    if out is None:
        out = torch.empty((B, Hq, L, Ev), dtype=query.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    if not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be a contiguous float32 tensor")
    ks_, vs_ = (tuple(t.stride(d) for d in perm) for t in (k_pages, v_pages))
    qs, os_ = _i64x4(query.stride()), _i64x4(out.stride())
    ws_bytes = lib.sdpa_decode_paged_workspace_size(B, Hq, Hkv, L, E, Ev, page_size, max_pages, dcode)
    ws = _workspace(dev, ws_bytes)
    ws_ptr = None if ws is None else (ws.data_ptr() + 255) // 256 * 256
    stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        status = lib.sdpa_decode_paged(
            query.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
            seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(),
            B, Hq, Hkv, L, E, Ev, num_pages, page_size, max_pages,
            qs, _i64x4(ks_), _i64x4(vs_), os_,
            0 if scale is None else 1, 0.0 if scale is None else float(scale),
            dcode, ws_ptr, ws_bytes, stream,
        )
    _check(status, "sdpa_decode_paged")
    return out, lse


def take_device_error() -> int:
    """Device-side error word (0 = none; below 30: a kernel gave up on a
    wait; 31 / 32: a paged decode's seq_lens / block table check), cleared."""
    code = ctypes.c_int(0)
    _check(load_library().sdpa_take_device_error(ctypes.byref(code)), "sdpa_take_device_error")
    return code.value


def last_launch_count() -> int:
    return load_library().sdpa_last_launch_count()


def default_scale(E: int) -> float:
    return 1.0 / math.sqrt(E)


class PreparedCall:
    """sdpa() with its arguments marshalled once, for repeated launches on the
    same tensors (benchmarks, decode loops).  Calling it enqueues the kernels
    on the current stream and returns the number of kernels launched."""

    def __init__(self, query, key, value, *, is_causal=False, scale=None, enable_gqa=False,
                 layout="bhle", cu_seqlens=None, max_seqlen=None, out=None, lse=None):
        # One ordinary call validates everything and allocates the outputs.
        self.out, self.lse = sdpa(query, key, value, is_causal=is_causal, scale=scale, enable_gqa=enable_gqa,
                                  layout=layout, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen, out=out, lse=lse)
        self._lib = load_library()
        if cu_seqlens is not None and layout == "bhle":
            layout = "bmhk"
        B, Hq, L, E = _dims(query, layout)
        _, Hkv, S, _ = _dims(key, layout)
        Ev = _dims(value, layout)[3]
        mask_kind = MASK_NONE
        cu_ptr, n_seqs, maxlen = None, 0, 0
        if cu_seqlens is not None:
            mask_kind = MASK_BLOCK_DIAG_CAUSAL if is_causal else MASK_BLOCK_DIAG
            cu_ptr, n_seqs, maxlen = cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, int(max_seqlen)
        elif is_causal:
            mask_kind = MASK_CAUSAL
        dcode = _DTYPE_CODE[query.dtype]
        ws_bytes = self._lib.sdpa_fwd_workspace_size(B, Hq, Hkv, L, S, E, Ev, mask_kind, dcode)
        ws = _workspace(query.device, ws_bytes)
        ws_ptr = None if ws is None else (ws.data_ptr() + 255) // 256 * 256
        self._keep = (query, key, value, cu_seqlens, ws)
        self.device = query.device
        self._args = (
            query.data_ptr(), key.data_ptr(), value.data_ptr(), self.out.data_ptr(), self.lse.data_ptr(),
            B, Hq, Hkv, L, S, E, Ev,
            *(_i64x4(_strides(t, layout)) for t in (query, key, value, self.out)),
            0 if scale is None else 1, 0.0 if scale is None else float(scale),
            mask_kind, cu_ptr, n_seqs, maxlen, None, _i64x4((0, 0, 0, 0)),
            dcode, ws_ptr, ws_bytes,
        )
        self.plan = plan(query, key, value, layout=layout, mask_kind=mask_kind, out=self.out)

    def __call__(self, stream=None) -> int:
        s = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        st = self._lib.sdpa_fwd(*self._args, s)
        if st != SDPA_OK:
            _check(st, "sdpa_fwd")
        return self._lib.sdpa_last_launch_count()
