"""Backward pass: CUDA path vs the fp64 oracle (needs a B200).

The forward runs first on the GPU (it writes O and the row statistic lse the
backward rebuilds probabilities from, "Causal Multi-Head Self-Attention",
Two exact full-sequence algorithms); the oracle's gradients come from q, k, v
and dO alone.

Tolerance, from the rounding the CUDA path performs (u = 2^-8 for bf16, 2^-11
for f16): P and dS are rounded once to the input type for the tensor cores,
the saved O once (so D = dO.O carries one more), and each gradient once on
output; each of these contributes about u/(2 sqrt 3) relative RMS error, in
total about 1.2 u = 5e-3 (bf16) normwise.  The bound is 2u normwise (the
Frobenius norm of the error over that of the gradient, per tensor) and 5u of
the tensor's largest magnitude for any single element.  float32 runs on the
CUDA-core kernels with fp32 throughout: u = 5e-6 there (bound 1e-5 normwise,
as for the float32 forward).
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
UNIT = {BF16: 2.0 ** -8, F16: 2.0 ** -11, F32: 5e-6}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from transformer_attention_causal_b200.build import build

    build()
    torch.cuda.init()
    yield
    assert attn.device_status() == 0


def run_gpu(q, k, v, dout, scale, causal):
    qg, kg, vg, dg = (t.cuda() for t in (q, k, v, dout))
    B, H, T, _ = q.shape
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    o = attn.prefill(qg, kg, vg, scale=scale, causal=causal, lse=lse)
    dq, dk, dv = attn.prefill_backward(qg, kg, vg, o, lse, dg, scale=scale, causal=causal)
    torch.cuda.synchronize()
    return dq.cpu(), dk.cpu(), dv.cpu()


def check(name, got, ref, dtype):
    got = got.to(torch.float64).numpy()
    assert np.all(np.isfinite(got)), name
    u = UNIT[dtype]
    err = got - ref
    scale = np.abs(ref).max()
    if scale == 0:
        assert np.abs(got).max() <= 1e-4, name
        return
    normwise = np.linalg.norm(err) / np.linalg.norm(ref)
    assert normwise <= 2 * u, f"{name}: normwise error {normwise:.3e}"
    assert np.abs(err).max() <= 5 * u * scale, f"{name}: max error {np.abs(err).max():.3e} of {scale:.3e}"


CASES = [
    # dtype, B, H, Hkv, T, d, causal
    (BF16, 1, 2, 1, 300, 128, True),     # GQA pair, ragged last tile
    (BF16, 2, 4, 4, 257, 64, True),      # MHA, d = 64, a one-row last tile
    (F16, 1, 8, 2, 384, 128, True),      # G = 4, whole tiles
    (BF16, 1, 2, 2, 200, 80, True),      # d = 80 (a zero-filled half chunk)
    (BF16, 1, 4, 1, 129, 96, False),     # MQA, full attention
    (F16, 2, 2, 1, 100, 128, True),      # one partial tile
    (BF16, 1, 6, 3, 1000, 128, True),    # many tiles
    (F16, 1, 2, 2, 700, 112, False),     # full attention, d = 112
    # CUDA-core kernels: float32, and 16-bit head sizes outside the tensor-core set
    (F32, 1, 4, 2, 130, 64, True),
    (F32, 2, 2, 1, 77, 40, False),
    (F32, 1, 2, 2, 200, 256, True),
    (BF16, 1, 2, 2, 150, 48, True),
    (F16, 1, 4, 1, 100, 200, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(case):
    dtype, B, H, Hkv, T, d, causal = case
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=T + d)
    dout = inputs.upstream(B, H, T, d, dtype, seed=T + d)
    scale = 1 / math.sqrt(d)
    got = run_gpu(q, k, v, dout, scale, causal)
    ref = oracle.attention_backward(q, k, v, dout, scale=scale, causal=causal)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        check(name, g, r, dtype)


WINDOWED = [
    # dtype, B, H, Hkv, T, d, window
    (BF16, 1, 4, 2, 500, 128, 32),       # the pages' window of 32
    (F16, 1, 2, 1, 700, 64, 300),        # a window spanning several tiles
    (BF16, 1, 2, 2, 1000, 80, 128),      # window = one tile
    (F32, 1, 2, 1, 150, 64, 20),         # CUDA-core kernels
    (BF16, 1, 2, 2, 200, 48, 50),
]


@pytest.mark.parametrize("case", WINDOWED, ids=lambda c: "-".join(map(str, c)))
def test_windowed_backward_matches_oracle(case):
    dtype, B, H, Hkv, T, d, w = case
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=T + w)
    dout = inputs.upstream(B, H, T, d, dtype, seed=T + w)
    scale = 1 / math.sqrt(d)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    o = attn.prefill(qg, kg, vg, scale=scale, window=w, lse=lse)
    got = attn.prefill_backward(qg, kg, vg, o, lse, dout.cuda(), scale=scale, window=w)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(q, k, v, dout, scale=scale, window=w)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        check(name, g.cpu(), r, dtype)


def test_single_position():
    # one key: dq = dk = 0 and dv = the summed upstream rows (up to rounding)
    q, k, v = inputs.qkv(1, 4, 2, 1, 1, 64, BF16, seed=5)
    dout = inputs.upstream(1, 4, 1, 64, BF16, seed=5)
    dq, dk, dv = run_gpu(q, k, v, dout, 0.125, True)
    assert dq.abs().max() <= 1e-4 and dk.abs().max() <= 1e-4
    ref = oracle.attention_backward(q, k, v, dout, scale=0.125)[2]
    check("dv", dv, ref, BF16)


def test_zero_heads_zero_the_key_gradients():
    k = torch.randn(1, 2, 64, 64, device="cuda").to(BF16)
    dk = torch.full_like(k, 3.0)
    dv = torch.full_like(k, 3.0)
    q = torch.empty((1, 0, 64, 64), dtype=BF16, device="cuda")
    lse = torch.empty((1, 0, 64), dtype=torch.float32, device="cuda")
    attn.prefill_backward(q, k, k, q, lse, q, scale=0.1, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert dk.abs().max() == 0 and dv.abs().max() == 0


def test_full_size_group_of_the_benchmark_workload():
    """GQA 16/8, d = 128, T = 4096, bf16, B = 8 (the benchmark's backward
    workload), in its launch configuration; the oracle recomputes every
    gradient of two (batch, K/V head) groups in full."""
    B, H, Hkv, T, d = 8, 16, 8, 4096, 128
    G = H // Hkv
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=0)
    dout = inputs.upstream(B, H, T, d, BF16, seed=0)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = run_gpu(q, k, v, dout, scale, True)
    for b, kvh in ((0, 0), (B - 1, Hkv - 1)):
        hs = slice(kvh * G, (kvh + 1) * G)
        ref = oracle.attention_backward(q[b:b + 1, hs], k[b:b + 1, kvh:kvh + 1],
                                        v[b:b + 1, kvh:kvh + 1], dout[b:b + 1, hs], scale=scale)
        check("dq", dq[b:b + 1, hs], ref[0], BF16)
        check("dk", dk[b:b + 1, kvh:kvh + 1], ref[1], BF16)
        check("dv", dv[b:b + 1, kvh:kvh + 1], ref[2], BF16)


def test_full_size_backward_sampled_heads_and_sums():
    """The backward workload at full size (B=8, 16 query / 8 K/V heads,
    T=4096, d=128, bf16), whose key and query tiles are worked through in
    several groups of heads: dQ of three (b, h) slices and dK, dV of one
    (b, K/V head) against the oracle on those heads alone (a head's dQ needs
    only its own rows; a K/V head's dK and dV only its G query heads), and for
    every (b, K/V head) the sums that hold at any size: sum_j dV_j = sum of
    dO over its query heads (each probability row sums to 1) and
    sum_j dK_j = 0 (shifting every key leaves each softmax row unchanged)."""
    B, H, Hkv, T, d = 8, 16, 8, 4096, 128
    G = H // Hkv
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=9)
    dout = inputs.upstream(B, H, T, d, BF16, seed=9)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = run_gpu(q, k, v, dout, scale, True)
    u = UNIT[BF16]
    for b, h in ((0, 0), (3, 9), (7, 15)):
        kvh = h // G
        ref, _, _ = oracle.attention_backward(q[b:b + 1, h:h + 1], k[b:b + 1, kvh:kvh + 1],
                                              v[b:b + 1, kvh:kvh + 1], dout[b:b + 1, h:h + 1],
                                              scale=scale, causal=True)
        check(f"dq[{b},{h}]", dq[b:b + 1, h:h + 1], ref, BF16)
    b, kvh = 5, 6
    _, ref_dk, ref_dv = oracle.attention_backward(q[b:b + 1, kvh * G:(kvh + 1) * G],
                                                  k[b:b + 1, kvh:kvh + 1], v[b:b + 1, kvh:kvh + 1],
                                                  dout[b:b + 1, kvh * G:(kvh + 1) * G],
                                                  scale=scale, causal=True)
    check("dk[5,6]", dk[b:b + 1, kvh:kvh + 1], ref_dk, BF16)
    check("dv[5,6]", dv[b:b + 1, kvh:kvh + 1], ref_dv, BF16)
    dv64, dk64 = dv.double(), dk.double()
    do_sum = dout.double().reshape(B, Hkv, G, T, d).sum(dim=(2, 3))        # [B, Hkv, d]
    dv_sum = dv64.sum(dim=2)
    assert torch.all((dv_sum - do_sum).abs() <= 8 * u * do_sum.abs().amax(dim=-1, keepdim=True) + 1e-2)
    dk_scale = dk64.abs().sum(dim=2)
    assert torch.all(dk64.sum(dim=2).abs() <= 8 * u * dk_scale + 1e-3)
