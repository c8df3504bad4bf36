"""Device-side failure detection without a GPU fault (needs a B200).

Every wait inside the kernels is bounded.  The test hook makes the TMA
producers issue no copies, so the consumers' waits run out after a short
limit: the kernels must record ATTN_ERR_DEVICE_TIMEOUT, exit cleanly (TMEM
freed, no copy left in flight) and leave the context usable, which the normal
calls afterwards check against the oracle.  No fault, trap or hang is
provoked: nothing waits without a bound.
"""
import math

import numpy as np
import pytest
import torch

import transformer_attention_causal_b200 as attn
from oracle import attention as oracle
from oracle import attention_backward as oracle_backward
from transformer_attention_causal_b200 import _lib, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from transformer_attention_causal_b200.build import build

    build()


def test_bounded_waits_report_a_timeout_and_leave_the_context_usable():
    lib = _lib.load()
    scale = 1 / math.sqrt(128)
    pq, pk, pv = inputs.qkv(1, 4, 2, 256, 256, 128, torch.bfloat16, seed=31)
    dq, dk, dv = inputs.qkv(2, 8, 2, 1, 1000, 128, torch.bfloat16, seed=32)
    assert attn.prefill_plan(torch.bfloat16, 1, 4, 2, 256, 128) == "tcgen05"
    assert attn.cached_plan(torch.bfloat16, 2, 8, 2, 1, 1000, 1000, 128, 999) == "splitkv"
    pq, pk, pv, dq, dk, dv = (t.cuda() for t in (pq, pk, pv, dq, dk, dv))
    assert attn.device_status(reset=True) == _lib.OK
    # a head size of 80 (the second 64-column chunk partly filled) too
    sq, sk, sv = (t.cuda() for t in inputs.qkv(1, 3, 3, 300, 300, 80, torch.bfloat16, seed=33))
    try:
        attn.set_wait_timeout_ns(20_000_000)  # 20 ms
        lib.attn_test_set_flags(1)
        attn.prefill(pq, pk, pv, scale=scale)
        assert attn.device_status(reset=True) == _lib.ERR_DEVICE_TIMEOUT
        attn.prefill(sq, sk, sv, scale=1 / math.sqrt(80))
        assert attn.device_status(reset=True) == _lib.ERR_DEVICE_TIMEOUT
        attn.cached(dq, dk, dv, start_pos=999, scale=scale)
        assert attn.device_status(reset=True) == _lib.ERR_DEVICE_TIMEOUT
    finally:
        lib.attn_test_set_flags(0)
        attn.set_wait_timeout_ns(0)
    # the context is intact: normal calls run and match the oracle
    out = attn.prefill(pq, pk, pv, scale=scale).float().cpu().numpy()
    ref = oracle(pq.cpu(), pk.cpu(), pv.cpu(), scale=scale, causal=True)
    err = np.abs(out - ref)
    assert err.max() <= 1.5e-2 and err.mean() <= 2e-3
    out = attn.cached(dq, dk, dv, start_pos=999, scale=scale).float().cpu().numpy()
    ref = oracle(dq.cpu(), dk.cpu(), dv.cpu(), scale=scale, causal=True, start_pos=999)
    err = np.abs(out - ref)
    assert err.max() <= 1.5e-2 and err.mean() <= 2e-3
    out = attn.prefill(sq, sk, sv, scale=1 / math.sqrt(80)).float().cpu().numpy()
    ref = oracle(sq.cpu(), sk.cpu(), sv.cpu(), scale=1 / math.sqrt(80), causal=True)
    err = np.abs(out - ref)
    assert err.max() <= 1.5e-2 and err.mean() <= 2e-3
    assert attn.device_status() == _lib.OK


@pytest.mark.parametrize("window", [0, 100])
def test_backward_waits_report_a_timeout_and_leave_the_context_usable(window):
    """Both backward kernels (dK/dV and dQ) under the no-copy hook."""
    lib = _lib.load()
    scale = 1 / math.sqrt(128)
    B, H, Hkv, T, d = 1, 4, 2, 300, 128
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, torch.bfloat16, seed=33)
    dout = inputs.upstream(B, H, T, d, torch.bfloat16, seed=33)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    o = attn.prefill(qg, kg, vg, scale=scale, lse=lse, window=window)
    assert attn.device_status(reset=True) == _lib.OK
    try:
        attn.set_wait_timeout_ns(20_000_000)  # 20 ms
        lib.attn_test_set_flags(1)
        attn.prefill_backward(qg, kg, vg, o, lse, dog, scale=scale, window=window)
        assert attn.device_status(reset=True) == _lib.ERR_DEVICE_TIMEOUT
    finally:
        lib.attn_test_set_flags(0)
        attn.set_wait_timeout_ns(0)
    grads = attn.prefill_backward(qg, kg, vg, o, lse, dog, scale=scale, window=window)
    torch.cuda.synchronize()
    ref = oracle_backward(q, k, v, dout, scale=scale, causal=True, window=window)
    for g, r in zip(grads, ref):
        g = g.double().cpu().numpy()
        assert np.linalg.norm(g - r) <= 2 * 2.0 ** -8 * np.linalg.norm(r)
    assert attn.device_status() == _lib.OK
