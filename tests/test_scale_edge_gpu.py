"""Degenerate and negative scales on every kernel family (needs a B200).

scale = 0 makes every visible key weigh the same (the oracle's closed form:
each row is the mean of the values it sees); a negative scale is ordinary
attention on -Q.  Masked keys must still carry exactly zero weight.
Tolerances as everywhere: float32 normwise 1e-5, 16-bit max abs 1.5e-2 and
mean abs 2e-3; the backward as in test_backward_gpu.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import transformer_attention_causal_b200 as attn
from transformer_attention_causal_b200 import inputs

pytestmark = pytest.mark.gpu

BF16, F16, F32 = torch.bfloat16, torch.float16, torch.float32


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from transformer_attention_causal_b200.build import build

    build()
    torch.cuda.init()
    yield
    assert attn.device_status() == 0


def check(got, ref, dtype):
    got = got.to(torch.float64).cpu().numpy()
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    if dtype == F32:
        assert err.max() <= 1e-5 * max(1.0, np.abs(ref).max())
    else:
        assert err.max() <= 1.5e-2, f"max abs error {err.max():.3e}"
        assert err.mean() <= 2e-3, f"mean abs error {err.mean():.3e}"


SCALES = [0.0, -0.09]

PREFILL = [
    # dtype, B, H, Hkv, T, d, kernel
    (BF16, 1, 4, 2, 300, 128, "tcgen05"),
    (F16, 1, 2, 2, 257, 80, "tcgen05"),
    (F32, 1, 2, 1, 100, 64, "simt"),
]


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("case", PREFILL, ids=lambda c: "-".join(map(str, c)))
def test_prefill(case, scale):
    dtype, B, H, Hkv, T, d, kernel = case
    assert attn.prefill_plan(dtype, B, H, Hkv, T, d) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=11)
    got = attn.prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale)
    check(got, oracle.attention(q, k, v, scale=scale, causal=True), dtype)


@pytest.mark.parametrize("scale", SCALES)
def test_windowed_prefill(scale):
    q, k, v = inputs.qkv(1, 4, 2, 400, 400, 128, BF16, seed=12)
    got = attn.prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, window=100)
    check(got, oracle.attention(q, k, v, scale=scale, causal=True, window=100), BF16)


CACHED = [
    # dtype, B, H, Hkv, Tnew, start_pos, S, d, kernel
    (BF16, 2, 8, 2, 1, 999, 1000, 128, "splitkv"),
    (F16, 2, 8, 1, 200, 300, 500, 128, "tcgen05"),
    (BF16, 1, 8, 2, 130, 1000, 1130, 64, "tcgen05"),   # 8 units, each cut into 2 pieces of its keys
]


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("case", CACHED, ids=lambda c: "-".join(map(str, c)))
def test_cached(case, scale):
    dtype, B, H, Hkv, Tnew, st, S, d, kernel = case
    assert attn.cached_plan(dtype, B, H, Hkv, Tnew, S, S, d, st) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, dtype, seed=13)
    got = attn.cached(q.cuda(), k.cuda(), v.cuda(), start_pos=st, scale=scale)
    check(got, oracle.attention(q, k, v, scale=scale, causal=True, start_pos=st), dtype)


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("dtype,d", [(BF16, 128), (F32, 64)])
def test_backward(dtype, d, scale):
    B, H, Hkv, T = 1, 4, 2, 200
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=14)
    dout = inputs.upstream(B, H, T, d, dtype, seed=14)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    o = attn.prefill(qg, kg, vg, scale=scale, lse=lse)
    grads = attn.prefill_backward(qg, kg, vg, o, lse, dout.cuda(), scale=scale)
    ref = oracle.attention_backward(q, k, v, dout, scale=scale)
    u = 2.0 ** -8 if dtype == BF16 else 5e-6
    for g, r in zip(grads, ref):
        g = g.double().cpu().numpy()
        assert np.all(np.isfinite(g))
        nr = np.linalg.norm(r)
        if nr == 0:
            assert np.abs(g).max() <= 1e-4
        else:
            assert np.linalg.norm(g - r) <= 2 * u * nr
