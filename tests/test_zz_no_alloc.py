"""attn_cached_noalloc: the cached entry point for callers that may not
allocate device memory (plugins handed only their input/output buffers by a
host framework that owns the allocator; serving loops that forbid allocation
once warm).  Its split-KV partials live in a fixed 16 MiB library-owned device
array instead of a caller workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from transformer_attention_causal_b200 import _lib, inputs

BF16 = 1
SCRATCH_BYTES = 16 << 20


def noalloc_fn():
    lib = _lib.load()
    fn = lib.attn_cached_noalloc
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, i64, i64, i64, i64,
                   ctypes.c_float, vp]
    return lib, fn


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Checked before any device work (host only): a decode whose partials
    need more than the 16 MiB array returns ATTN_ERR_WORKSPACE."""
    lib, fn = noalloc_fn()
    # the split plan decides the partials' size: search for a decode that needs more
    S = 1 << 20
    found = None
    for d, H, Hkv, Tnew in ((128, 32, 4, 1), (128, 16, 2, 1), (256, 16, 4, 1), (64, 32, 4, 2)):
        for B in (20, 37, 50, 74, 100, 150, 200, 300):
            need = lib.attn_cached_workspace_size(BF16, B, H, Hkv, Tnew, S, d, S - Tnew)
            if need > SCRATCH_BYTES:
                found = (B, H, Hkv, Tnew, d)
                break
        if found:
            break
    assert found, "no decode shape found whose partials exceed the scratch array"
    B, H, Hkv, Tnew, d = found
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the call is rejected first
    rc = fn(fake, fake, fake, fake, None, BF16, B, H, Hkv, Tnew, S, S, d, S - Tnew, 0.1, None)
    assert rc == _lib.ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_cached_on_two_calls_in_a_row():
    """Two calls in a row (different inputs): each must match the regular
    workspace entry point and, independently of the GPU, the fp64 oracle on
    the same seeded inputs; the second call must not see the first's data."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_attention_causal_b200 as attn
    from oracle import attention as oracle_attention
    from transformer_attention_causal_b200.build import build

    build()
    lib, fn = noalloc_fn()
    B, H, Hkv, Tnew, S, d = 8, 32, 8, 1, 8192, 128
    start = S - Tnew
    scale = 1.0 / math.sqrt(d)
    need = lib.attn_cached_workspace_size(BF16, B, H, Hkv, Tnew, S, d, start)
    assert 0 < need <= SCRATCH_BYTES  # this problem does use the scratch array
    stream = torch.cuda.current_stream()
    for seed in (21, 22):  # two calls in a row: the second must not see the first's data
        q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, torch.bfloat16, seed=seed)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        ref = attn.cached(qd, kd, vd, start_pos=start, scale=scale)
        out = torch.full_like(qd, float("nan"))
        rc = fn(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()),
                ctypes.c_void_p(vd.data_ptr()), ctypes.c_void_p(out.data_ptr()), None, BF16, B, H,
                Hkv, Tnew, S, S, d, start, scale, ctypes.c_void_p(stream.cuda_stream))
        assert rc == _lib.OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        # the 16-bit tolerance used throughout the tests, against the existing
        # entry point and against the fp64 oracle (every row of the call)
        err = np.abs(got - ref.double().cpu().numpy())
        assert np.all(np.isfinite(err))
        assert err.max() <= 1.5e-2 and err.mean() <= 2e-3, (seed, err.max(), err.mean())
        exact = oracle_attention(q, k, v, scale=scale, causal=True, start_pos=start)
        err = np.abs(got - exact)
        assert err.max() <= 1.5e-2 and err.mean() <= 2e-3, (seed, err.max(), err.mean())
    assert attn.device_status() == 0


@pytest.mark.gpu
def test_noalloc_chunked_prefill_pieces_match_the_oracle():
    """A chunked prefill whose 16 units are cut into pieces of their key range:
    the pieces' partials go to the fixed array too.  Two calls in a row, each
    against the fp64 oracle on every row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import transformer_attention_causal_b200 as attn
    from oracle import attention as oracle_attention
    from transformer_attention_causal_b200.build import build

    build()
    lib, fn = noalloc_fn()
    B, H, Hkv, Tnew, S, d = 2, 8, 1, 256, 2048, 128
    start = S - Tnew
    scale = 1.0 / math.sqrt(d)
    need = lib.attn_cached_workspace_size(BF16, B, H, Hkv, Tnew, S, d, start)
    assert 0 < need <= SCRATCH_BYTES  # pieces, and they fit the array
    stream = torch.cuda.current_stream()
    for seed in (31, 32):
        q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, torch.bfloat16, seed=seed)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        out = torch.full_like(qd, float("nan"))
        rc = fn(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()),
                ctypes.c_void_p(vd.data_ptr()), ctypes.c_void_p(out.data_ptr()), None, BF16, B, H,
                Hkv, Tnew, S, S, d, start, scale, ctypes.c_void_p(stream.cuda_stream))
        assert rc == _lib.OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        exact = oracle_attention(q, k, v, scale=scale, causal=True, start_pos=start)
        err = np.abs(got - exact)
        assert np.all(np.isfinite(err))
        assert err.max() <= 1.5e-2 and err.mean() <= 2e-3, (seed, err.max(), err.mean())
    assert attn.device_status() == 0
