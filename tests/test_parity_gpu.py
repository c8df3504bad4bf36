"""CUDA path vs the fp64 oracle on identical seeded inputs (needs a B200).

Tolerances (stated with the workloads this library targets):
  * float32 inputs: normwise relative error per (b, h) slice,
        max|gpu - oracle| / max|oracle| <= 1e-5;
  * bf16 / fp16 inputs (the oracle runs on the same rounded values, widened
    exactly): max abs error <= 1.5e-2 and mean abs error <= 2e-3 over all
    compared elements.

Small cases cover every kernel family at sizes that span several tiles with a
ragged tail; the full-size workloads run in the configuration the benchmark
times and are checked on sampled rows the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import transformer_attention_causal_b200 as attn
from oracle import attention as oracle
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


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    if dtype == F32:
        ref2 = ref.reshape(ref.shape[0], -1) if ref.ndim > 1 else ref.reshape(1, -1)
        err2 = err.reshape(ref2.shape)
        denom = np.maximum(np.abs(ref2).max(axis=1), 1e-30)
        rel = err2.max(axis=1) / denom
        assert rel.max() <= 1e-5, f"{what}: normwise relative error {rel.max():.3e} > 1e-5"
    else:
        assert err.max() <= 1.5e-2, f"{what}: max abs error {err.max():.3e} > 1.5e-2"
        assert err.mean() <= 2e-3, f"{what}: mean abs error {err.mean():.3e} > 2e-3"


def to_dev(*ts):
    return [t.cuda() for t in ts]


def gpu_prefill(q, k, v, scale, causal=True, want_lse=False):
    qd, kd, vd = to_dev(q, k, v)
    lse = torch.empty(q.shape[:3], dtype=F32, device="cuda") if want_lse else None
    out = attn.prefill(qd, kd, vd, scale=scale, causal=causal, lse=lse)
    torch.cuda.synchronize()
    return (out.cpu(), lse.cpu()) if want_lse else out.cpu()


def gpu_cached(q, k, v, start_pos, scale, S=None, want_lse=False):
    qd, kd, vd = to_dev(q, k, v)
    lse = torch.empty(q.shape[:3], dtype=F32, device="cuda") if want_lse else None
    out = attn.cached(qd, kd, vd, start_pos=start_pos, scale=scale, S=S, lse=lse)
    torch.cuda.synchronize()
    return (out.cpu(), lse.cpu()) if want_lse else out.cpu()


def f64(t):
    return t.to(torch.float64).numpy()


# ------------------------------------------------------------------ small: prefill

PREFILL_CASES = [
    # dtype, B, H, Hkv, T, d, causal, expected kernel
    (F32, 1, 2, 1, 16, 8, True, "simt"),          # the tiny float32 workload
    (F32, 2, 4, 2, 70, 40, True, "simt"),
    (F32, 1, 3, 1, 33, 64, False, "simt"),
    (BF16, 2, 4, 2, 300, 128, True, "tcgen05"),    # G = 2: two heads per CTA, ragged tail
    (BF16, 1, 3, 3, 333, 80, True, "tcgen05"),     # MHA: two row tiles per CTA, odd tile count
    (F16, 2, 8, 1, 260, 64, True, "tcgen05"),      # MQA, head size 64
    (BF16, 1, 2, 1, 200, 96, False, "tcgen05"),    # non-causal
    (F16, 1, 4, 4, 129, 112, True, "tcgen05"),
    (BF16, 1, 2, 2, 1, 128, True, "tcgen05"),      # single token
    (BF16, 1, 2, 1, 128, 128, True, "tcgen05"),    # exactly one tile
    (BF16, 1, 2, 1, 512, 64, True, "tcgen05"),     # whole tiles only
    (BF16, 2, 4, 2, 50, 40, True, "simt"),         # 16-bit, head size the tensor-core kernel skips
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "-".join(map(str, c)))
def test_prefill_small(case):
    dtype, B, H, Hkv, T, d, causal, kernel = case
    assert attn.prefill_plan(dtype, B, H, Hkv, T, d, causal) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=11)
    scale = 1.0 / math.sqrt(d)
    got, lse = gpu_prefill(q, k, v, scale, causal, want_lse=True)
    ref, ref_lse = oracle(q, k, v, scale=scale, causal=causal, want_lse=True)
    assert_close(f64(got).reshape(B * H, -1), ref.reshape(B * H, -1), dtype, str(case))
    np.testing.assert_allclose(f64(lse), ref_lse, rtol=0, atol=2e-3 if dtype != F32 else 1e-5)


def test_tiny_float32_workload_exact_tolerance():
    """B=1, H=2, Hkv=1, T=16, d=8, scale 1/sqrt(8), seed 0: normwise 1e-5."""
    q, k, v = inputs.qkv(1, 2, 1, 16, 16, 8, F32, seed=0)
    got = gpu_prefill(q, k, v, 1 / math.sqrt(8))
    ref = oracle(q, k, v, scale=1 / math.sqrt(8), causal=True)
    assert_close(f64(got).reshape(2, -1), ref.reshape(2, -1), F32)


@pytest.mark.parametrize("dtype", [F32, BF16])
def test_worked_example_through_the_abi(dtype):
    """Multi-query attention, annotated §2.1: q=(1,0), keys (1,0),(0,1),(1,1),
    values 1,2,3, unscaled -> 2.0.  Run as one cached query at position 2, and
    as a causal prefill whose rows give 1, (e+2)/(e+1), 2."""
    e = math.e
    k = torch.tensor([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]], dtype=F32)
    v = torch.tensor([[1.0, 0.0], [2.0, 0.0], [3.0, 0.0]], dtype=F32)
    # head size 2 is padded to 8 with zeros (zeros change neither the dot
    # products nor the first output column)
    kp = torch.zeros((1, 1, 3, 8)); kp[0, 0, :, :2] = k
    vp = torch.zeros((1, 1, 3, 8)); vp[0, 0, :, :2] = v
    q1 = torch.zeros((1, 1, 1, 8)); q1[0, 0, 0, 0] = 1.0
    out = gpu_cached(q1.to(dtype), kp.to(dtype), vp.to(dtype), start_pos=2, scale=1.0)
    tol = 1e-6 if dtype == F32 else 1e-2
    assert abs(float(out[0, 0, 0, 0]) - 2.0) <= tol
    q3 = torch.zeros((1, 1, 3, 8)); q3[0, 0, :, 0] = 1.0
    out = gpu_prefill(q3.to(dtype), kp.to(dtype), vp.to(dtype), scale=1.0)
    np.testing.assert_allclose(f64(out)[0, 0, :, 0], [1.0, (e + 2) / (e + 1), 2.0], atol=tol)


# ------------------------------------------------------------------ small: cached

CACHED_CASES = [
    # dtype, B, H, Hkv, Tnew, start_pos, S, S_cap, d, expected kernel
    (BF16, 3, 8, 2, 1, 999, 1000, 1000, 128, "splitkv"),    # GQA decode, G = 4
    (F16, 2, 8, 1, 1, 776, 777, 777, 128, "splitkv"),       # MQA decode, G = 8
    (BF16, 2, 4, 4, 3, 497, 500, 500, 64, "splitkv"),       # MHA, 3 new tokens
    (BF16, 1, 4, 1, 4, 2900, 3000, 3100, 128, "splitkv"),   # history past the last query
    (F16, 2, 16, 2, 1, 4099, 4100, 4100, 256, "splitkv"),   # head size 256
    (BF16, 2, 4, 4, 2, 1500, 1502, 1600, 256, "splitkv"),   # head size 256, two rows per K/V head
    (BF16, 1, 4, 1, 1, 19999, 20000, 20000, 128, "splitkv"),  # one long sequence: many splits
    (BF16, 2, 4, 2, 1, 0, 1, 1, 128, "splitkv"),            # first token
    (F16, 2, 16, 1, 1, 1999, 2000, 2048, 64, "splitkv"),    # 16 rows per K/V head at d = 64
    (BF16, 2, 8, 8, 1, 1299, 1300, 1300, 80, "splitkv"),    # MHA decode, d = 80 (a part-filled chunk)
    (F16, 1, 8, 2, 3, 997, 1000, 1024, 96, "splitkv"),      # d = 96, 12 rows per K/V head
    (BF16, 2, 16, 2, 1, 2047, 2048, 2048, 112, "splitkv"),  # d = 112, 8 rows
    (BF16, 1, 4, 1, 4, 4999, 5003, 5003, 80, "splitkv"),    # d = 80, 16 rows, several splits
    (F16, 2, 8, 1, 200, 300, 500, 520, 128, "tcgen05"),     # MQA chunked prefill
    (BF16, 1, 4, 2, 64, 37, 101, 101, 80, "tcgen05"),       # unaligned start
    (BF16, 1, 2, 2, 100, 400, 600, 640, 64, "tcgen05"),     # history past the last query
    # chunked prefills whose units are fewer than half the SMs: each unit is
    # cut into pieces of its key range, merged by a second kernel
    (F16, 2, 8, 1, 256, 1792, 2048, 2048, 128, "tcgen05"),   # 16 units, 3 pieces each
    (BF16, 1, 4, 4, 300, 1100, 1400, 1400, 80, "tcgen05"),   # MHA, an empty second slot, 2 pieces
    (BF16, 1, 8, 2, 130, 1000, 1130, 1152, 64, "tcgen05"),   # d = 64, unaligned start, 2 pieces
    (BF16, 1, 2, 1, 64, 4000, 4064, 4096, 112, "tcgen05"),   # one unit in 4 pieces
    (F32, 2, 4, 2, 5, 60, 70, 72, 32, "simt"),
    (BF16, 1, 4, 2, 3, 20, 30, 30, 40, "simt"),
]


@pytest.mark.parametrize("case", CACHED_CASES, ids=lambda c: "-".join(map(str, c)))
def test_cached_small(case):
    dtype, B, H, Hkv, Tnew, start, S, S_cap, d, kernel = case
    assert attn.cached_plan(dtype, B, H, Hkv, Tnew, S, S_cap, d, start) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, dtype, seed=5, S_cap=S_cap)
    scale = 1.0 / math.sqrt(d)
    got, lse = gpu_cached(q, k, v, start, scale, S=S, want_lse=True)
    ref, ref_lse = oracle(q, k, v, scale=scale, causal=True, start_pos=start, S=S, want_lse=True)
    assert_close(f64(got).reshape(B * H, -1), ref.reshape(B * H, -1), dtype, str(case))
    np.testing.assert_allclose(f64(lse), ref_lse, rtol=0, atol=2e-3 if dtype != F32 else 1e-5)


# ------------------------------------------------------------------ invariants on the GPU

def test_outputs_are_deterministic_and_inputs_untouched():
    for dtype, (B, H, Hkv, T, d) in [(BF16, (2, 4, 2, 300, 128)), (F32, (1, 2, 1, 40, 16))]:
        q, k, v = to_dev(*inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=3))
        q0, k0, v0 = q.clone(), k.clone(), v.clone()
        a = attn.prefill(q, k, v, scale=0.1)
        b = attn.prefill(q, k, v, scale=0.1)
        torch.cuda.synchronize()
        assert torch.equal(a, b)
        assert torch.equal(q, q0) and torch.equal(k, k0) and torch.equal(v, v0)
    q, k, v = to_dev(*inputs.qkv(4, 8, 2, 1, 3000, 128, BF16, seed=4))
    a = attn.cached(q, k, v, start_pos=2999, scale=0.1)
    b = attn.cached(q, k, v, start_pos=2999, scale=0.1)
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype,d", [(BF16, 128), (F16, 80), (F32, 16)])
def test_future_tokens_do_not_change_earlier_rows(dtype, d):
    """Perturbing Q, K, V after position i leaves row i bit-for-bit unchanged."""
    B, H, Hkv, T = 1, 4, 2, 300
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=8)
    base = gpu_prefill(q, k, v, 0.1)
    for i in (0, 127, 128, 200, 298):
        q2, k2, v2 = q.clone(), k.clone(), v.clone()
        q2[:, :, i + 1:] = -q2[:, :, i + 1:]
        k2[:, :, i + 1:] = k2[:, :, i + 1:] * 3
        v2[:, :, i + 1:] = v2[:, :, i + 1:] + 1
        pert = gpu_prefill(q2, k2, v2, 0.1)
        assert torch.equal(pert[:, :, : i + 1], base[:, :, : i + 1]), f"row {i}"


def test_gqa_equals_mha_on_repeated_heads():
    B, H, Hkv, T, d = 2, 8, 2, 260, 128
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=9)
    gqa = gpu_prefill(q, k, v, 0.09)
    rep = H // Hkv
    mha = gpu_prefill(q, k.repeat_interleave(rep, 1).contiguous(),
                      v.repeat_interleave(rep, 1).contiguous(), 0.09)
    assert (gqa.float() - mha.float()).abs().max() <= 1e-2


def test_cached_rows_match_prefill_rows():
    B, H, Hkv, T, d = 2, 8, 2, 400, 128
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=10)
    full = gpu_prefill(q, k, v, 0.09)
    for Tnew in (1, 2, 150):
        start = T - Tnew
        part = gpu_cached(q[:, :, start:].contiguous(), k, v, start, 0.09)
        assert (part.float() - full[:, :, start:].float()).abs().max() <= 1e-2, Tnew


def test_rows_with_large_logits():
    """Scores scaled up 50x: the running maximum moves a lot and the lazy
    rescale path of the tensor-core kernel must fire."""
    B, H, Hkv, T, d = 1, 2, 1, 384, 128
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=12)
    # make later keys score higher so the maximum keeps rising
    ramp = torch.linspace(0.5, 4.0, T).reshape(1, 1, T, 1)
    k = (k.float() * ramp).to(BF16)
    scale = 50.0 / math.sqrt(d)
    got = gpu_prefill(q, k, v, scale)
    ref = oracle(q, k, v, scale=scale, causal=True)
    assert_close(f64(got).reshape(B * H, -1), ref.reshape(B * H, -1), BF16)


@pytest.mark.parametrize("case", [
    # B, H, Hkv, Tnew, start_pos, S, kernel
    (2, 8, 2, 1, 1499, 1500, "splitkv"),     # decode: the MMA kernel's lazy rescale
    (1, 4, 1, 4, 996, 1000, "splitkv"),      # several new rows per K/V head
    (1, 4, 2, 200, 500, 700, "tcgen05"),     # chunked prefill
], ids=lambda c: "-".join(map(str, c)))
def test_cached_rows_with_large_logits(case):
    """Cached attention with the scores scaled up 50x and keys growing along
    the sequence, so the running maximum keeps rising from split to split and
    tile to tile."""
    B, H, Hkv, Tnew, st, S, kernel = case
    d = 128
    assert attn.cached_plan(BF16, B, H, Hkv, Tnew, S, S, d, st) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, BF16, seed=13)
    ramp = torch.linspace(0.5, 4.0, S).reshape(1, 1, S, 1)
    k = (k.float() * ramp).to(BF16)
    scale = 50.0 / math.sqrt(d)
    got = gpu_cached(q, k, v, st, scale)
    ref = oracle(q, k, v, scale=scale, causal=True, start_pos=st)
    assert_close(f64(got).reshape(B * H, -1), ref.reshape(B * H, -1), BF16)


def test_empty_problem_leaves_output_untouched():
    q = torch.zeros((0, 4, 8, 64), dtype=BF16, device="cuda")
    out = attn.prefill(q, q.new_zeros((0, 2, 8, 64)), q.new_zeros((0, 2, 8, 64)), scale=0.1)
    assert out.shape == q.shape


def test_rejected_call_leaves_output_untouched():
    q, k, v = to_dev(*inputs.qkv(1, 4, 2, 1, 4096, 128, BF16, seed=1))
    out = torch.full_like(q, 7.0)
    need = attn.cached_workspace_size(BF16, 1, 4, 2, 1, 4096, 128, 4095)
    if need:
        ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
        with pytest.raises(attn.AttnError):
            attn.cached(q, k, v, start_pos=4095, scale=0.1, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)
    with pytest.raises(attn.AttnError):
        attn.cached(q, k, v, start_pos=4096, scale=0.1, out=out)  # start_pos + Tnew > S
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


# ------------------------------------------------------------------ full-size workloads

def sample_rows(B, H, T, n, seed):
    """Flat row ids: tile edges and the last row of every sampled slice, plus
    seeded random rows."""
    g = np.random.default_rng(seed)
    rows = set()
    for _ in range(n):
        b, h = int(g.integers(B)), int(g.integers(H))
        for i in {0, min(127, T - 1), min(128, T - 1), T - 1, int(g.integers(T))}:
            rows.add((b * H + h) * T + i)
    return sorted(rows)


FULL = {
    "bitnet3b_mha_prefill_bf16": dict(kind="prefill", dtype=BF16, B=1, H=32, Hkv=32, T=2048, d=80),
    "gqa16x8_prefill_bf16": dict(kind="prefill", dtype=BF16, B=8, H=16, Hkv=8, T=4096, d=128),
    "gqa_decode_bf16": dict(kind="cached", dtype=BF16, B=64, H=32, Hkv=8, Tnew=1, start=8191,
                            S=8192, d=128),
    "mqa_chunked_prefill_f16": dict(kind="cached", dtype=F16, B=32, H=8, Hkv=1, Tnew=512,
                                    start=3584, S=4096, d=128),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_workload_sampled_rows(name):
    c = FULL[name]
    d, dtype = c["d"], c["dtype"]
    scale = 1.0 / math.sqrt(d)
    if c["kind"] == "prefill":
        B, H, Hkv, T = c["B"], c["H"], c["Hkv"], c["T"]
        q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=0)
        got = gpu_prefill(q, k, v, scale)
        rows = sample_rows(B, H, T, 12, 1)
        ref = oracle(q, k, v, scale=scale, causal=True, rows=rows)
        Tq = T
        start = 0
    else:
        B, H, Hkv, Tq, start, S = c["B"], c["H"], c["Hkv"], c["Tnew"], c["start"], c["S"]
        q, k, v = inputs.qkv(B, H, Hkv, Tq, S, d, dtype, seed=0)
        got = gpu_cached(q, k, v, start, scale)
        rows = sample_rows(B, H, Tq, 16, 2)
        ref = oracle(q, k, v, scale=scale, causal=True, start_pos=start, rows=rows)
    flat = f64(got).reshape(-1, d)
    assert np.all(np.isfinite(flat))
    assert_close(flat[rows], ref, dtype, name)
