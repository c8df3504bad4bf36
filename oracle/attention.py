"""ctypes front end of the fp64 C oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY — see the package docstring.  The arithmetic lives in
the C file; this module only compiles it with gcc, marshals arrays and returns
numpy float64 results.  The definition it follows is written out, with its
sources, at the top of ``attn_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD_DIR, "liboracle.so")

# dtype codes shared with attn_oracle.c
_F32, _BF16, _F16, _F64 = 0, 1, 2, 3

_lock = threading.Lock()
_handle = None


def library_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE double: no fast-math, no FMA
    contraction) into ``oracle/_build/liboracle.so``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_attention.restype = ctypes.c_int
    lib.oracle_attention.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64,
                                     i64, i64, i64, dbl, ctypes.c_int, vp, i64, vp, vp,
                                     vp, ctypes.c_int]
    lib.oracle_attention_window.restype = ctypes.c_int
    lib.oracle_attention_window.argtypes = [vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64,
                                            i64, i64, i64, dbl, ctypes.c_int, i64, vp, i64, vp,
                                            vp, vp, ctypes.c_int]
    lib.oracle_widen_bf16.restype = dbl
    lib.oracle_widen_bf16.argtypes = [ctypes.c_uint16]
    lib.oracle_widen_f16.restype = dbl
    lib.oracle_widen_f16.argtypes = [ctypes.c_uint16]
    lib.oracle_num_cores.restype = ctypes.c_int
    lib.oracle_rope_append.restype = ctypes.c_int
    lib.oracle_rope_append.argtypes = [vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, dbl, vp, vp]
    return lib


def _lib():
    global _handle
    with _lock:
        if _handle is None:
            _handle = _bind(build())
    return _handle


def num_cores() -> int:
    return int(_lib().oracle_num_cores())


def _as_raw(x):
    """Return (contiguous numpy array of raw storage, dtype code).

    Accepts numpy arrays (float32/float64/float16) or CPU torch tensors
    (float32/bfloat16/float16/float64).  bf16/f16 travel as their raw 16-bit
    patterns; the C side widens them exactly."""
    try:
        import torch  # noqa: WPS433 (optional)
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), _BF16
        if x.dtype == torch.float16:
            return x.view(torch.int16).numpy().view(np.uint16), _F16
        if x.dtype == torch.float32:
            return x.numpy(), _F32
        if x.dtype == torch.float64:
            return x.numpy(), _F64
        raise TypeError(f"unsupported torch dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, _F32
    if x.dtype == np.float64:
        return x, _F64
    if x.dtype == np.float16:
        return x.view(np.uint16), _F16
    raise TypeError(f"unsupported numpy dtype {x.dtype}")


def attention(q, k, v, *, scale: float, causal: bool = True, start_pos: int = 0,
              S: int | None = None, rows=None, want_lse: bool = False,
              want_probs: bool = False, nthreads: int = 0, window: int = 0, _lib_handle=None):
    """fp64 attention rows.

    q: [B, H, Tq, d]; k, v: [B, Hkv, S_cap, d] (first ``S`` rows valid; default
    S = S_cap).  Query row i sits at absolute position ``start_pos + i``.
    ``window`` w > 0 keeps only keys p - w < j <= p (a local window).
    ``rows``: optional iterable of flat row ids ``(b*H + h)*Tq + i``; the
    result then has one row per id, in that order.

    Returns ``out`` ([B, H, Tq, d] float64, or [len(rows), d]), plus ``lse``
    and/or ``probs`` ([..., S]) when asked, as a tuple in that order.
    """
    qa, code = _as_raw(q)
    ka, kcode = _as_raw(k)
    va, vcode = _as_raw(v)
    if not (code == kcode == vcode):
        raise TypeError("q, k, v must share one dtype")
    if qa.ndim != 4 or ka.ndim != 4 or va.shape != ka.shape:
        raise ValueError("expected q [B,H,Tq,d] and k, v [B,Hkv,S_cap,d]")
    B, H, Tq, d = qa.shape
    Bk, Hkv, S_cap, dk = ka.shape
    if Bk != B or dk != d:
        raise ValueError("batch or head_dim mismatch")
    S = S_cap if S is None else int(S)
    if rows is None:
        rows_arr = None
        nrows = B * H * Tq
        out_shape = (B, H, Tq, d)
    else:
        rows_arr = np.ascontiguousarray(np.asarray(list(rows) if not isinstance(rows, np.ndarray)
                                                   else rows, dtype=np.int64))
        nrows = int(rows_arr.shape[0])
        out_shape = (nrows, d)
    out = np.zeros((nrows, d), dtype=np.float64)
    lse = np.zeros((nrows,), dtype=np.float64) if want_lse else None
    probs = np.zeros((nrows, S), dtype=np.float64) if want_probs else None
    ptr = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    lib = _lib() if _lib_handle is None else _lib_handle
    rc = lib.oracle_attention_window(
        ptr(qa), ptr(ka), ptr(va), code, B, H, Hkv, Tq, S, S_cap, d, int(start_pos),
        float(scale), int(bool(causal)), int(window), ptr(rows_arr), nrows, ptr(out), ptr(lse),
        ptr(probs), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attention rejected its arguments (code {rc})")
    res = [out.reshape(out_shape)]
    if want_lse:
        res.append(lse.reshape(out_shape[:-1]))
    if want_probs:
        res.append(probs.reshape(out_shape[:-1] + (S,)))
    return res[0] if len(res) == 1 else tuple(res)


def widen_bits(bits: np.ndarray, kind: str, _lib_handle=None) -> np.ndarray:
    """Widen raw 16-bit patterns (``kind`` = 'bf16' or 'f16') to float64 with
    the oracle's own bit-level conversion."""
    lib = _lib() if _lib_handle is None else _lib_handle
    fn = lib.oracle_widen_bf16 if kind == "bf16" else lib.oracle_widen_f16
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([fn(int(b)) for b in flat], dtype=np.float64).reshape(np.shape(bits))


def load_variant(path: str):
    """Bind another build of ``attn_oracle.c`` (the tests compile deliberately
    broken copies to show that the pins catch them).  Returns an object with
    ``attention`` and ``widen_bits`` bound to that build."""
    import types

    handle = _bind(path)
    return types.SimpleNamespace(
        attention=lambda *a, **kw: attention(*a, _lib_handle=handle, **kw),
        widen_bits=lambda *a, **kw: widen_bits(*a, _lib_handle=handle, **kw),
        rope_append=lambda *a, **kw: rope_append(*a, _lib_handle=handle, **kw),
    )


def rope_append(k_new, v_new, *, start_pos: int, base: float, _lib_handle=None):
    """fp64 rows that a KV-cache append writes: K rotated with NeoX RoPE at
    positions start_pos + t (base <= 0: no rotation), V unchanged.
    k_new, v_new: [B, Hkv, Tnew, d].  Returns (k_rows, v_rows) float64."""
    ka, code = _as_raw(k_new)
    va, vcode = _as_raw(v_new)
    if code != vcode or ka.shape != va.shape or ka.ndim != 4:
        raise ValueError("k_new and v_new must be [B, Hkv, Tnew, d] of one dtype")
    B, Hkv, Tnew, d = ka.shape
    k_out = np.zeros(ka.shape, dtype=np.float64)
    v_out = np.zeros(ka.shape, dtype=np.float64)
    lib = _lib() if _lib_handle is None else _lib_handle
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.oracle_rope_append(ptr(ka), ptr(va), code, B, Hkv, Tnew, d, int(start_pos),
                                float(base), ptr(k_out), ptr(v_out))
    if rc != 0:
        raise ValueError(f"oracle_rope_append rejected its arguments (code {rc})")
    return k_out, v_out
