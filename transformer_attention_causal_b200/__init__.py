"""B200-native causal (MHA / GQA / MQA) scaled-dot-product attention.

The compute lives in ``libb200attn.so`` (CUDA C++ for sm_100a behind the C ABI
declared in ``include/b200attn.h``).  This package only marshals arguments:
torch supplies device memory and the current stream; every step of the
attention runs in the library's kernels.

    prefill(q, k, v, scale=..., causal=True)        q [B,H,T,d], k/v [B,Hkv,T,d]
    cached(q, k_hist, v_hist, start_pos=..., scale=...)
                                                    q [B,H,Tnew,d], k/v [B,Hkv,S_cap,d]
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import AttnError

__all__ = ["prefill", "prefill_backward", "cached", "cached_paged", "kv_append_rope",
           "cached_workspace_size", "prefill_backward_workspace_size",
           "cached_paged_workspace_size", "prefill_plan", "cached_plan", "device_status",
           "set_wait_timeout_ns", "AttnError"]


def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return _lib.F32
    if t.dtype == torch.bfloat16:
        return _lib.BF16
    if t.dtype == torch.float16:
        return _lib.F16
    raise TypeError(f"unsupported dtype {t.dtype}: expected float32, bfloat16 or float16")


def _code_of(dtype) -> int:
    torch = _torch()
    return {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16, torch.float16: _lib.F16}[dtype]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _on_device(device):
    """Context that makes `device` current for the call: the library launches
    on the current device, the stream handle comes from `device`."""
    return _torch().cuda.device(device)


def _require_cuda(device):
    if device.type != "cuda":
        raise ValueError("tensors must live on a CUDA device")


def _check(*tensors):
    """Every given tensor is contiguous and all sit on one CUDA device, which
    is returned.  The C ABI sees raw pointers only, so a tensor on another
    device (or a strided view) would be read or written out of bounds."""
    device = None
    for t in tensors:
        if t is None:
            continue
        if device is None:
            device = t.device
            _require_cuda(device)
        elif t.device != device:
            raise ValueError(f"all tensors must sit on one device ({device} and {t.device})")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return device


def _same_dtype(ref, names_tensors):
    """Tensors that the library reads or writes with `ref`'s element type."""
    for name, t in names_tensors:
        if t is not None and t.dtype != ref.dtype:
            raise TypeError(f"{name} is {t.dtype}, expected {ref.dtype} like q")


def _shape_is(name, t, shape):
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_lse(lse, shape):
    torch = _torch()
    if lse is not None:
        if lse.dtype != torch.float32:
            raise TypeError("lse must be float32")
        _shape_is("lse", lse, shape)


def _dims4(name, t):
    if t.dim() != 4:
        raise ValueError(f"{name} must be 4-dimensional, got {t.dim()} dimensions")


def prefill(q, k, v, *, scale: float, causal: bool = True, out=None, lse=None, stream=None,
            window: int = 0):
    """Full-sequence attention.  q [B,H,T,d]; k, v [B,Hkv,T,d]; returns O [B,H,T,d].
    ``lse`` (optional float32 [B,H,T]) receives the log-sum-exp of each row.
    ``window`` w > 0: local attention, row p sees keys p - w < j <= p (causal)."""
    device = _check(q, k, v, out, lse)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dims4(name, t)
    B, H, T, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, T, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    code = _dtype_code(q)
    _same_dtype(q, (("k", k), ("v", v), ("out", out)))
    _shape_is("out", out, q.shape)
    _check_lse(lse, (B, H, T))
    if window and not causal:
        raise ValueError("a local window is causal")
    with _on_device(device):
        if out is None:
            out = q.new_empty(q.shape)
        if window:
            st = _lib.load().attn_prefill_local(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                                code, B, H, Hkv, T, d, float(scale), int(window),
                                                _stream_handle(stream, device))
            if st != _lib.OK:
                raise AttnError(st, "attn_prefill_local")
            return out
        st = _lib.load().attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), code,
                                      B, H, Hkv, T, d, float(scale), int(bool(causal)),
                                      _stream_handle(stream, device))
    if st != _lib.OK:
        raise AttnError(st, "attn_prefill")
    return out


def prefill_backward_workspace_size(dtype, B, H, Hkv, T, d) -> int:
    return int(_lib.load().attn_prefill_backward_workspace_size(_code_of(dtype), B, H, Hkv, T, d))


def prefill_backward(q, k, v, out, lse, dout, *, scale: float, causal: bool = True, dq=None,
                     dk=None, dv=None, workspace=None, stream=None, window: int = 0):
    """Gradients of full-sequence attention.  q, out, dout [B,H,T,d]; k, v
    [B,Hkv,T,d]; lse float32 [B,H,T] as written by ``prefill`` for the same
    inputs (and the same ``window``: w > 0 is local attention).  Returns
    (dq, dk, dv); dk and dv are summed over the query heads that share each
    K/V head."""
    torch = _torch()
    device = _check(q, k, v, out, lse, dout, dq, dk, dv, workspace)
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _dims4(name, t)
    B, H, T, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, T, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, Hkv, T, d] matching q")
    if tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("out and dout must match q")
    if lse is None or lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, T):
        raise ValueError("lse must be float32 [B, H, T]")
    code = _dtype_code(q)
    _same_dtype(q, (("k", k), ("v", v), ("out", out), ("dout", dout), ("dq", dq), ("dk", dk),
                    ("dv", dv)))
    _shape_is("dq", dq, q.shape)
    _shape_is("dk", dk, k.shape)
    _shape_is("dv", dv, k.shape)
    if window and not causal:
        raise ValueError("a local window is causal")
    with _on_device(device):
        dq = q.new_empty(q.shape) if dq is None else dq
        dk = k.new_empty(k.shape) if dk is None else dk
        dv = v.new_empty(v.shape) if dv is None else dv
        need = prefill_backward_workspace_size(q.dtype, B, H, Hkv, T, d)
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        if window:
            st = _lib.load().attn_prefill_backward_local(
                _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                _ptr(dv), code, B, H, Hkv, T, d, float(scale), int(window), _ptr(workspace),
                ws_bytes, _stream_handle(stream, device))
            if st != _lib.OK:
                raise AttnError(st, "attn_prefill_backward_local")
            return dq, dk, dv
        st = _lib.load().attn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                               _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), code,
                                               B, H, Hkv, T, d, float(scale), int(bool(causal)),
                                               _ptr(workspace), ws_bytes,
                                               _stream_handle(stream, device))
    if st != _lib.OK:
        raise AttnError(st, "attn_prefill_backward")
    return dq, dk, dv


def cached_workspace_size(dtype, B, H, Hkv, Tnew, S, d, start_pos, window: int = 0) -> int:
    if window:
        return int(_lib.load().attn_cached_local_workspace_size(_code_of(dtype), B, H, Hkv, Tnew,
                                                                 S, d, start_pos, window))
    return int(_lib.load().attn_cached_workspace_size(_code_of(dtype), B, H, Hkv, Tnew, S, d,
                                                       start_pos))


def cached(q, k_hist, v_hist, *, start_pos: int, scale: float, S: int | None = None, out=None,
           lse=None, workspace=None, stream=None, window: int = 0):
    """New tokens at ``start_pos`` against a K/V history that already holds them.
    q [B,H,Tnew,d]; k_hist, v_hist [B,Hkv,S_cap,d] (first S rows valid, default
    S = S_cap).  ``workspace`` (uint8 CUDA tensor) is allocated here when not given."""
    device = _check(q, k_hist, v_hist, out, lse, workspace)
    for name, t in (("q", q), ("k_hist", k_hist), ("v_hist", v_hist)):
        _dims4(name, t)
    B, H, Tnew, d = q.shape
    Hkv, S_cap = k_hist.shape[1], k_hist.shape[2]
    if tuple(v_hist.shape) != tuple(k_hist.shape) or k_hist.shape[0] != B or k_hist.shape[3] != d:
        raise ValueError("k_hist and v_hist must be [B, Hkv, S_cap, d] matching q")
    code = _dtype_code(q)
    _same_dtype(q, (("k_hist", k_hist), ("v_hist", v_hist), ("out", out)))
    _shape_is("out", out, q.shape)
    _check_lse(lse, (B, H, Tnew))
    S = S_cap if S is None else int(S)
    with _on_device(device):
        if out is None:
            out = q.new_empty(q.shape)
        need = cached_workspace_size(q.dtype, B, H, Hkv, Tnew, S, d, start_pos, window)
        if workspace is None and need > 0:
            workspace = _torch().empty(need, dtype=_torch().uint8, device=device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        if window:
            st = _lib.load().attn_cached_local(_ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(out),
                                               _ptr(lse), code, B, H, Hkv, Tnew, S, S_cap, d,
                                               int(start_pos), float(scale), int(window),
                                               _ptr(workspace), ws_bytes,
                                               _stream_handle(stream, device))
            if st != _lib.OK:
                raise AttnError(st, "attn_cached_local")
            return out
        st = _lib.load().attn_cached(_ptr(q), _ptr(k_hist), _ptr(v_hist), _ptr(out), _ptr(lse),
                                     code, B, H, Hkv, Tnew, S, S_cap, d, int(start_pos),
                                     float(scale), _ptr(workspace), ws_bytes,
                                     _stream_handle(stream, device))
    if st != _lib.OK:
        raise AttnError(st, "attn_cached")
    return out


def cached_paged_workspace_size(dtype, B, H, Hkv, Tnew, d, max_kv_len) -> int:
    return int(_lib.load().attn_cached_paged_workspace_size(_code_of(dtype), B, H, Hkv, Tnew, d,
                                                             max_kv_len))


def cached_paged(q, k_pages, v_pages, page_table, kv_lens, *, max_kv_len: int, scale: float,
                 out=None, lse=None, workspace=None, stream=None):
    """New tokens of each sequence against its paged K/V history.
    q [B,H,Tnew,d]; k_pages, v_pages [num_pages, Hkv, page_size, d];
    page_table int32 [B, max_pages]; kv_lens int32 [B] (each sequence's length,
    new tokens included; all <= max_kv_len)."""
    torch = _torch()
    device = _check(q, k_pages, v_pages, page_table, kv_lens, out, lse, workspace)
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        _dims4(name, t)
    B, H, Tnew, d = q.shape
    num_pages, Hkv, page_size = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if tuple(v_pages.shape) != tuple(k_pages.shape) or k_pages.shape[3] != d:
        raise ValueError("k_pages and v_pages must be [num_pages, Hkv, page_size, d] matching q")
    if page_table.dtype != torch.int32 or kv_lens.dtype != torch.int32:
        raise TypeError("page_table and kv_lens must be int32")
    if page_table.dim() != 2 or page_table.shape[0] != B or tuple(kv_lens.shape) != (B,):
        raise ValueError("page_table must be [B, max_pages] and kv_lens [B]")
    code = _dtype_code(q)
    _same_dtype(q, (("k_pages", k_pages), ("v_pages", v_pages), ("out", out)))
    _shape_is("out", out, q.shape)
    _check_lse(lse, (B, H, Tnew))
    with _on_device(device):
        if out is None:
            out = q.new_empty(q.shape)
        need = cached_paged_workspace_size(q.dtype, B, H, Hkv, Tnew, d, max_kv_len)
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = _lib.load().attn_cached_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(out),
                                           _ptr(lse), code, B, H, Hkv, Tnew, d, _ptr(page_table),
                                           page_table.shape[1], num_pages, page_size,
                                           _ptr(kv_lens), int(max_kv_len), float(scale),
                                           _ptr(workspace), ws_bytes,
                                           _stream_handle(stream, device))
    if st != _lib.OK:
        raise AttnError(st, "attn_cached_paged")
    return out


def kv_append_rope(k_new, v_new, k_cache, v_cache, *, start_pos: int, rope_base: float = 10000.0,
                   stream=None):
    """Write the new tokens' K (rotated with NeoX RoPE at positions
    start_pos + t; rope_base <= 0: unrotated) and V into the caches.
    k_new, v_new [B, Hkv, Tnew, d]; k_cache, v_cache [B, Hkv, S_cap, d]."""
    device = _check(k_new, v_new, k_cache, v_cache)
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dims4(name, t)
    B, Hkv, Tnew, d = k_new.shape
    S_cap = k_cache.shape[2]
    if tuple(v_new.shape) != tuple(k_new.shape) or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or tuple(k_cache.shape[:2]) != (B, Hkv) or k_cache.shape[3] != d:
        raise ValueError("expected k_new, v_new [B, Hkv, Tnew, d] and caches [B, Hkv, S_cap, d]")
    if not (k_new.dtype == v_new.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("all four tensors must share one dtype")
    code = _dtype_code(k_new)
    with _on_device(device):
        st = _lib.load().attn_kv_append_rope(_ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                             _ptr(v_cache), code, B, Hkv, Tnew, S_cap, d,
                                             int(start_pos), float(rope_base),
                                             _stream_handle(stream, device))
    if st != _lib.OK:
        raise AttnError(st, "attn_kv_append_rope")
    return k_cache, v_cache


def prefill_plan(dtype, B, H, Hkv, T, d, causal=True) -> str:
    k = _lib.load().attn_prefill_plan(_code_of(dtype), B, H, Hkv, T, d, int(bool(causal)))
    return _lib.KERNEL_NAMES[k]


def cached_plan(dtype, B, H, Hkv, Tnew, S, S_cap, d, start_pos) -> str:
    k = _lib.load().attn_cached_plan(_code_of(dtype), B, H, Hkv, Tnew, S, S_cap, d, start_pos)
    return _lib.KERNEL_NAMES[k]


def device_status(stream=None, reset: bool = True) -> int:
    """Synchronise the stream and return (and by default clear) the device
    status word: 0 = OK, 5 = a bounded device-side wait ran out."""
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(_lib.load().attn_device_status(ctypes.c_void_p(s.cuda_stream), int(bool(reset))))


def set_wait_timeout_ns(ns: int) -> None:
    _lib.load().attn_set_wait_timeout_ns(int(ns))
