"""ctypes loader for libb200attn.so (declarations in include/b200attn.h).

The library is built in-tree (``python -m transformer_attention_causal_b200.build``
or ``__graft_entry__.build()``).  If it is missing, every call raises: there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libb200attn.so")

# attn_status_t
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(6)
# attn_dtype_t
F32, BF16, F16 = 0, 1, 2
# attn_kernel_t
KERNEL_NONE, KERNEL_SIMT, KERNEL_TCGEN05, KERNEL_SPLITKV = 0, 1, 2, 3
KERNEL_NAMES = {KERNEL_NONE: "none", KERNEL_SIMT: "simt", KERNEL_TCGEN05: "tcgen05",
                KERNEL_SPLITKV: "splitkv", -1: "rejected"}

EXPORTS = ("attn_prefill", "attn_cached", "attn_prefill_local", "attn_cached_local",
           "attn_cached_local_workspace_size", "attn_cached_paged", "attn_cached_paged_workspace_size",
           "attn_prefill_backward", "attn_prefill_backward_local",
           "attn_prefill_backward_workspace_size",
           "attn_kv_append_rope", "attn_cached_workspace_size", "attn_prefill_plan",
           "attn_cached_plan", "attn_status_string", "attn_device_status",
           "attn_set_wait_timeout_ns", "attn_test_set_flags", "attn_version")

_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m transformer_attention_causal_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(LIB_PATH)
            i64, vp, c_int, f32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.attn_prefill.restype = c_int
            lib.attn_prefill.argtypes = [vp, vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64, f32,
                                         c_int, vp]
            lib.attn_cached.restype = c_int
            lib.attn_cached.argtypes = [vp, vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64, i64,
                                        i64, i64, f32, vp, ctypes.c_size_t, vp]
            lib.attn_cached_workspace_size.restype = ctypes.c_size_t
            lib.attn_cached_workspace_size.argtypes = [c_int, i64, i64, i64, i64, i64, i64, i64]
            lib.attn_prefill_plan.restype = c_int
            lib.attn_prefill_plan.argtypes = [c_int, i64, i64, i64, i64, i64, c_int]
            lib.attn_cached_plan.restype = c_int
            lib.attn_cached_plan.argtypes = [c_int, i64, i64, i64, i64, i64, i64, i64, i64]
            lib.attn_status_string.restype = ctypes.c_char_p
            lib.attn_status_string.argtypes = [c_int]
            lib.attn_device_status.restype = c_int
            lib.attn_device_status.argtypes = [vp, c_int]
            lib.attn_set_wait_timeout_ns.restype = None
            lib.attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
            lib.attn_kv_append_rope.restype = c_int
            lib.attn_kv_append_rope.argtypes = [vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64,
                                                i64, f32, vp]
            lib.attn_prefill_local.restype = c_int
            lib.attn_prefill_local.argtypes = [vp, vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64,
                                               f32, i64, vp]
            lib.attn_cached_local.restype = c_int
            lib.attn_cached_local.argtypes = [vp, vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64,
                                              i64, i64, i64, f32, i64, vp, ctypes.c_size_t, vp]
            lib.attn_cached_local_workspace_size.restype = ctypes.c_size_t
            lib.attn_cached_local_workspace_size.argtypes = [c_int, i64, i64, i64, i64, i64, i64,
                                                             i64, i64]
            lib.attn_cached_paged.restype = c_int
            lib.attn_cached_paged.argtypes = [vp, vp, vp, vp, vp, c_int, i64, i64, i64, i64, i64,
                                              vp, i64, i64, i64, vp, i64, f32, vp,
                                              ctypes.c_size_t, vp]
            lib.attn_cached_paged_workspace_size.restype = ctypes.c_size_t
            lib.attn_cached_paged_workspace_size.argtypes = [c_int, i64, i64, i64, i64, i64, i64]
            lib.attn_prefill_backward.restype = c_int
            lib.attn_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, c_int, i64, i64,
                                                  i64, i64, i64, f32, c_int, vp, ctypes.c_size_t,
                                                  vp]
            lib.attn_prefill_backward_local.restype = c_int
            lib.attn_prefill_backward_local.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, c_int, i64,
                                                        i64, i64, i64, i64, f32, i64, vp,
                                                        ctypes.c_size_t, vp]
            lib.attn_prefill_backward_workspace_size.restype = ctypes.c_size_t
            lib.attn_prefill_backward_workspace_size.argtypes = [c_int, i64, i64, i64, i64, i64]
            lib.attn_test_set_flags.restype = None
            lib.attn_test_set_flags.argtypes = [ctypes.c_uint32]
            lib.attn_version.restype = c_int
            lib.attn_version.argtypes = []
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().attn_status_string(int(status)).decode()
