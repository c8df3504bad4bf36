"""The Python binding's argument checks, on CPU.

The C ABI receives raw pointers and cannot see a buffer's size, type or
device, so the binding must reject every mismatch before it calls the
library: a wrong-typed K, a too-small output or row statistic, or a tensor on
another device would otherwise turn into an out-of-bounds device access.
These tests run on meta tensors (no memory, no GPU) with the library replaced
by a recorder, and check that each mismatch raises before any library call
while a well-formed call reaches the library with the expected arguments.
"""
import contextlib

import pytest
import torch

import transformer_attention_causal_b200 as attn
from transformer_attention_causal_b200 import _lib

META = "meta"


class FakeLib:
    """Records compute calls; workspace queries report 0 bytes."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("workspace_size"):
            return lambda *a: 0

        def call(*args):
            self.calls.append((name, args))
            return _lib.OK

        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(_lib, "load", lambda: lib)
    # meta tensors stand in for device tensors: no device check, no stream
    monkeypatch.setattr(attn, "_require_cuda", lambda device: None)
    monkeypatch.setattr(attn, "_on_device", lambda device: contextlib.nullcontext())
    monkeypatch.setattr(attn, "_stream_handle", lambda stream, device: None)
    return lib


def t(*shape, dtype=torch.bfloat16, device=META):
    return torch.empty(shape, dtype=dtype, device=device)


B, H, HKV, T, D = 2, 8, 2, 64, 64


def qkv(dtype=torch.bfloat16):
    return t(B, H, T, D, dtype=dtype), t(B, HKV, T, D, dtype=dtype), t(B, HKV, T, D, dtype=dtype)


# ---------------------------------------------------------------- prefill

def test_prefill_well_formed_call_reaches_the_library(fake):
    q, k, v = qkv()
    out = attn.prefill(q, k, v, scale=0.125, lse=t(B, H, T, dtype=torch.float32))
    assert [c[0] for c in fake.calls] == ["attn_prefill"]
    assert tuple(out.shape) == tuple(q.shape) and out.dtype == q.dtype
    args = fake.calls[0][1]
    assert args[5:11] == (_lib.BF16, B, H, HKV, T, D)


@pytest.mark.parametrize("case", ["k_dtype", "v_dtype", "out_dtype", "out_shape", "lse_dtype",
                                  "lse_shape", "k_device", "out_device", "strided", "q_dims",
                                  "kv_shape", "window_not_causal", "int_dtype"])
def test_prefill_rejects_mismatch_before_any_call(fake, case):
    q, k, v = qkv()
    kw = {}
    if case == "k_dtype":
        k = t(B, HKV, T, D, dtype=torch.float32)
    elif case == "v_dtype":
        v = t(B, HKV, T, D, dtype=torch.float16)
    elif case == "out_dtype":
        kw["out"] = t(B, H, T, D, dtype=torch.float16)
    elif case == "out_shape":
        kw["out"] = t(B, H, T - 1, D)
    elif case == "lse_dtype":
        kw["lse"] = t(B, H, T, dtype=torch.bfloat16)
    elif case == "lse_shape":
        kw["lse"] = t(B, H, T + 1, dtype=torch.float32)
    elif case == "k_device":
        k = t(B, HKV, T, D, device="cpu")
    elif case == "out_device":
        kw["out"] = t(B, H, T, D, device="cpu")
    elif case == "strided":
        k = t(B, HKV, D, T).transpose(2, 3)
    elif case == "q_dims":
        q = t(B * H, T, D)
    elif case == "kv_shape":
        v = t(B, HKV, T, D + 16)
    elif case == "window_not_causal":
        kw.update(window=16, causal=False)
    elif case == "int_dtype":
        q, k, v = (x.to(torch.int16) for x in (q, k, v))
    with pytest.raises((ValueError, TypeError)):
        attn.prefill(q, k, v, scale=0.125, **kw)
    assert fake.calls == []


def test_prefill_rejects_a_host_tensor(monkeypatch):
    """Without the test stand-ins: a CPU tensor is refused outright."""
    lib = FakeLib()
    monkeypatch.setattr(_lib, "load", lambda: lib)
    q, k, v = (torch.empty(x.shape, dtype=x.dtype) for x in qkv())
    with pytest.raises(ValueError, match="CUDA"):
        attn.prefill(q, k, v, scale=0.125)
    assert lib.calls == []


# ---------------------------------------------------------------- cached

def cache_args(S_cap=256, Tnew=1, dtype=torch.bfloat16):
    return (t(B, H, Tnew, D, dtype=dtype), t(B, HKV, S_cap, D, dtype=dtype),
            t(B, HKV, S_cap, D, dtype=dtype))


def test_cached_well_formed_call_reaches_the_library(fake):
    q, k, v = cache_args()
    attn.cached(q, k, v, start_pos=255, scale=0.125, lse=t(B, H, 1, dtype=torch.float32))
    assert [c[0] for c in fake.calls] == ["attn_cached"]


@pytest.mark.parametrize("case", ["k_dtype", "out_shape", "out_dtype", "lse_shape", "ws_device",
                                  "v_device", "kv_batch"])
def test_cached_rejects_mismatch_before_any_call(fake, case):
    q, k, v = cache_args()
    kw = {}
    if case == "k_dtype":
        k = t(B, HKV, 256, D, dtype=torch.float16)
    elif case == "out_shape":
        kw["out"] = t(B, H, 2, D)
    elif case == "out_dtype":
        kw["out"] = t(B, H, 1, D, dtype=torch.float32)
    elif case == "lse_shape":
        kw["lse"] = t(B, H, dtype=torch.float32)
    elif case == "ws_device":
        kw["workspace"] = t(1024, dtype=torch.uint8, device="cpu")
    elif case == "v_device":
        v = t(B, HKV, 256, D, device="cpu")
    elif case == "kv_batch":
        k, v = t(B + 1, HKV, 256, D), t(B + 1, HKV, 256, D)
    with pytest.raises((ValueError, TypeError)):
        attn.cached(q, k, v, start_pos=255, scale=0.125, **kw)
    assert fake.calls == []


# ---------------------------------------------------------------- paged

def paged_args(dtype=torch.float16):
    q = t(B, H, 4, D, dtype=dtype)
    kp, vp = t(16, HKV, 64, D, dtype=dtype), t(16, HKV, 64, D, dtype=dtype)
    table, lens = t(B, 8, dtype=torch.int32), t(B, dtype=torch.int32)
    return q, kp, vp, table, lens


def test_cached_paged_well_formed_call_reaches_the_library(fake):
    attn.cached_paged(*paged_args(), max_kv_len=512, scale=0.1)
    assert [c[0] for c in fake.calls] == ["attn_cached_paged"]


@pytest.mark.parametrize("case", ["k_dtype", "out_shape", "table_device", "lens_dtype",
                                  "lse_dtype"])
def test_cached_paged_rejects_mismatch_before_any_call(fake, case):
    q, kp, vp, table, lens = paged_args()
    kw = {}
    if case == "k_dtype":
        kp = t(16, HKV, 64, D, dtype=torch.bfloat16)
    elif case == "out_shape":
        kw["out"] = t(B, H, 3, D, dtype=torch.float16)
    elif case == "table_device":
        table = t(B, 8, dtype=torch.int32, device="cpu")
    elif case == "lens_dtype":
        lens = t(B, dtype=torch.int64)
    elif case == "lse_dtype":
        kw["lse"] = t(B, H, 4, dtype=torch.float16)
    with pytest.raises((ValueError, TypeError)):
        attn.cached_paged(q, kp, vp, table, lens, max_kv_len=512, scale=0.1, **kw)
    assert fake.calls == []


# ---------------------------------------------------------------- backward

def bwd_args(dtype=torch.bfloat16):
    q, k, v = qkv(dtype)
    return q, k, v, t(B, H, T, D, dtype=dtype), t(B, H, T, dtype=torch.float32), \
        t(B, H, T, D, dtype=dtype)


def test_backward_well_formed_call_reaches_the_library(fake):
    dq, dk, dv = attn.prefill_backward(*bwd_args(), scale=0.125)
    assert [c[0] for c in fake.calls] == ["attn_prefill_backward"]
    assert tuple(dk.shape) == (B, HKV, T, D) and tuple(dq.shape) == (B, H, T, D)


@pytest.mark.parametrize("case", ["o_dtype", "dout_dtype", "k_dtype", "dq_shape", "dk_shape",
                                  "dv_dtype", "lse_dtype", "dq_device"])
def test_backward_rejects_mismatch_before_any_call(fake, case):
    q, k, v, o, lse, dout = bwd_args()
    kw = {}
    if case == "o_dtype":
        o = t(B, H, T, D, dtype=torch.float16)
    elif case == "dout_dtype":
        dout = t(B, H, T, D, dtype=torch.float32)
    elif case == "k_dtype":
        k = t(B, HKV, T, D, dtype=torch.float16)
    elif case == "dq_shape":
        kw["dq"] = t(B, HKV, T, D)
    elif case == "dk_shape":
        kw["dk"] = t(B, H, T, D)
    elif case == "dv_dtype":
        kw["dv"] = t(B, HKV, T, D, dtype=torch.float32)
    elif case == "lse_dtype":
        lse = t(B, H, T, dtype=torch.bfloat16)
    elif case == "dq_device":
        kw["dq"] = t(B, H, T, D, device="cpu")
    with pytest.raises((ValueError, TypeError)):
        attn.prefill_backward(q, k, v, o, lse, dout, scale=0.125, **kw)
    assert fake.calls == []


# ---------------------------------------------------------------- append

def test_append_rejects_mismatch_before_any_call(fake):
    kn, vn = t(B, HKV, 4, D), t(B, HKV, 4, D)
    kc, vc = t(B, HKV, 64, D), t(B, HKV, 64, D)
    attn.kv_append_rope(kn, vn, kc, vc, start_pos=3)
    assert [c[0] for c in fake.calls] == ["attn_kv_append_rope"]
    fake.calls.clear()
    for bad in ((kn, vn, kc, t(B, HKV, 64, D, dtype=torch.float16)),
                (kn, vn, kc, t(B, HKV, 64, D, device="cpu")),
                (kn, t(B, HKV, 5, D), kc, vc),
                (kn, vn, t(B, HKV, 64, D + 8), vc)):
        with pytest.raises((ValueError, TypeError)):
            attn.kv_append_rope(*bad, start_pos=3)
    assert fake.calls == []
