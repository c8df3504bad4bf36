"""Local (sliding-window) attention: CUDA path vs the fp64 oracle (needs a B200).

Every kernel family takes the window: the tcgen05 prefill (rows whose window
starts in a later key tile, tiles masked at both edges, tiles below every
window skipped), the split-KV decode kernels (the split plan starts at the
first row's window) and the CUDA-core kernel.  Tolerances as everywhere:
float32 normwise 1e-5 per (b, h) slice; 16-bit max abs 1.5e-2, mean abs 2e-3.
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
        g = err.reshape(-1, err.shape[-2] * err.shape[-1])
        r = np.abs(ref).reshape(g.shape).max(axis=1)
        assert (g.max(axis=1) / r).max() <= 1e-5
    else:
        assert err.max() <= 1.5e-2, f"max abs error {err.max():.3e}"
        assert err.mean() <= 2e-3, f"mean abs error {err.mean():.3e}"


PREFILL = [
    # dtype, B, H, Hkv, T, d, window, kernel
    (BF16, 1, 4, 2, 1000, 128, 32, "tcgen05"),     # the pages' window of 32; GQA slot pairs
    (BF16, 1, 4, 4, 777, 80, 100, "tcgen05"),      # MHA row-tile pairs, d = 80
    (F16, 2, 2, 1, 1500, 64, 300, "tcgen05"),      # MQA, a window spanning several tiles
    (BF16, 1, 2, 2, 1024, 128, 128, "tcgen05"),    # window = one tile
    (BF16, 1, 4, 4, 2048, 128, 120, "tcgen05"),    # MHA, each second slot's window starts a tile later
    (BF16, 1, 2, 2, 1024, 128, 136, "tcgen05"),    # only rows 0-6 of a second slot see its first tile
    (BF16, 1, 2, 1, 600, 128, 1, "tcgen05"),       # only the own position
    (F32, 1, 4, 2, 300, 48, 17, "simt"),
    (BF16, 1, 2, 2, 200, 40, 50, "simt"),
]


@pytest.mark.parametrize("case", PREFILL, ids=lambda c: "-".join(map(str, c)))
def test_prefill_window_matches_oracle(case):
    dtype, B, H, Hkv, T, d, w, kernel = case
    assert attn.prefill_plan(dtype, B, H, Hkv, T, d) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, dtype, seed=T + w)
    scale = 1 / math.sqrt(d)
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    got = attn.prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, window=w, lse=lse)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.attention(q, k, v, scale=scale, causal=True, window=w, want_lse=True)
    check(got, ref, dtype)
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= (1e-4 if dtype == F32 else 2e-3)


def test_a_window_covering_everything_is_plain_causal():
    q, k, v = (t.cuda() for t in inputs.qkv(1, 4, 2, 700, 700, 128, BF16, seed=3))
    a = attn.prefill(q, k, v, scale=0.1, window=700)
    b = attn.prefill(q, k, v, scale=0.1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


CACHED = [
    # dtype, B, H, Hkv, Tnew, start_pos, S, d, window, kernel
    (BF16, 2, 8, 2, 1, 4095, 4096, 128, 32, "splitkv"),      # decode, window of 32
    (BF16, 2, 32, 8, 1, 8191, 8192, 128, 1024, "splitkv"),   # GQA decode, several splits
    (F16, 2, 4, 1, 4, 3000, 3004, 128, 100, "splitkv"),      # 4 new tokens: per-row edges
    (BF16, 1, 4, 4, 2, 2000, 2002, 256, 700, "splitkv"),     # d = 256
    (BF16, 2, 8, 8, 1, 3000, 3001, 80, 500, "splitkv"),      # MHA decode, d = 80
    (F16, 1, 8, 2, 2, 1500, 1502, 112, 129, "splitkv"),      # d = 112, per-row edges
    (F16, 2, 8, 1, 200, 300, 500, 128, 64, "tcgen05"),       # chunked prefill with a window
    (F32, 1, 4, 2, 5, 60, 70, 32, 9, "simt"),
]


@pytest.mark.parametrize("case", CACHED, ids=lambda c: "-".join(map(str, c)))
def test_cached_window_matches_oracle(case):
    dtype, B, H, Hkv, Tnew, st, S, d, w, kernel = case
    assert attn.cached_plan(dtype, B, H, Hkv, Tnew, S, S, d, st) == kernel
    q, k, v = inputs.qkv(B, H, Hkv, Tnew, S, d, dtype, seed=S + w)
    scale = 1 / math.sqrt(d)
    got = attn.cached(q.cuda(), k.cuda(), v.cuda(), start_pos=st, scale=scale, window=w)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, scale=scale, causal=True, start_pos=st, window=w)
    check(got, ref, dtype)


def test_window_workspace_covers_only_the_window():
    full = attn.cached_workspace_size(BF16, 64, 32, 8, 1, 8192, 128, 8191)
    local = attn.cached_workspace_size(BF16, 64, 32, 8, 1, 8192, 128, 8191, window=256)
    assert local <= full


def test_full_size_windowed_prefill_sampled_rows():
    """The benchmark's windowed workload: GQA 32/8, d = 128, T = 8192,
    window 2048, bf16, B = 2 (sampled rows)."""
    B, H, Hkv, T, d, w = 2, 32, 8, 8192, 128, 2048
    q, k, v = inputs.qkv(B, H, Hkv, T, T, d, BF16, seed=0)
    got = attn.prefill(q.cuda(), k.cuda(), v.cuda(), scale=1 / math.sqrt(d), window=w).cpu()
    rng = np.random.default_rng(0)
    rows = np.sort(np.concatenate([rng.choice(B * H * T, 48, replace=False),
                                   [0, 127, 128, 2047, 2048, 2049, 8191, B * H * T - 1]]))
    ref = oracle.attention(q, k, v, scale=1 / math.sqrt(d), causal=True, window=w, rows=rows)
    flat = got.reshape(B * H * T, d)[torch.as_tensor(rows)]
    check(flat.reshape(1, len(rows), d), ref.reshape(1, len(rows), d), BF16)


@pytest.mark.parametrize("kind", ["prefill", "decode"])
def test_window_with_large_logits(kind):
    """Scores scaled up 50x with keys growing along the sequence: within a
    window the running maximum keeps rising, and the keys that leave the
    window are the small ones."""
    d, w = 128, 300
    if kind == "prefill":
        B, H, Hkv, T, S, st = 1, 4, 2, 900, 900, 0
    else:
        B, H, Hkv, T, S, st = 2, 8, 2, 1, 2000, 1999
    q, k, v = inputs.qkv(B, H, Hkv, T, S, d, BF16, seed=21)
    ramp = torch.linspace(0.5, 4.0, S).reshape(1, 1, S, 1)
    k = (k.float() * ramp).to(BF16)
    scale = 50.0 / math.sqrt(d)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    if kind == "prefill":
        got = attn.prefill(qd, kd, vd, scale=scale, window=w)
    else:
        got = attn.cached(qd, kd, vd, start_pos=st, scale=scale, window=w)
    ref = oracle.attention(q, k, v, scale=scale, causal=True, start_pos=st, window=w)
    check(got, ref, BF16)
