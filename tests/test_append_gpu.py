"""KV-cache append with RoPE on K: CUDA path vs the fp64 oracle (needs a B200).

The kernel rotates in fp32 from an angle reduced in fp64 and rounds once to
the cache dtype.  The exact rotation rounded to nearest sits within half a
unit in the last place (ulp) of the cache dtype; the fp32 arithmetic adds a
few fp32 ulps of the pair's size on top, which can move an element across a
rounding boundary.  So, for bf16 / fp16 caches: every element within one ulp
of the oracle (the ulp at the oracle's value) and at least 99.9% of them
equal to the oracle rounded to nearest; float32 caches: per-row normwise
relative error <= 2e-6.  V rows, and K rows without a base, are copied
bit for bit; cache rows outside [start_pos, start_pos + Tnew) keep their bits.
"""
import numpy as np
import pytest
import torch

import transformer_attention_causal_b200 as attn
import oracle
from transformer_attention_causal_b200 import inputs

pytestmark = pytest.mark.gpu

BF16, F16, F32 = torch.bfloat16, torch.float16, torch.float32
MANT = {BF16: 7, F16: 10}            # explicit mantissa bits
MIN_EXP = {BF16: -126, F16: -14}     # smallest normal exponent


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from transformer_attention_causal_b200.build import build

    build()
    torch.cuda.init()
    yield
    assert attn.device_status() == 0


def ulp(x, dtype):
    """Spacing of the dtype's representable numbers at |x|."""
    _, e = np.frexp(np.abs(x))                # |x| = m * 2^e, m in [0.5, 1)
    e = np.where(x == 0, MIN_EXP[dtype], np.maximum(e - 1, MIN_EXP[dtype]))
    return np.ldexp(1.0, e - MANT[dtype])


def make_case(B, Hkv, Tnew, S_cap, d, dtype, seed):
    k_new = inputs.normal((B, Hkv, Tnew, d), seed, 0, dtype)
    v_new = inputs.normal((B, Hkv, Tnew, d), seed, 1, dtype)
    k_cache = inputs.normal((B, Hkv, S_cap, d), seed, 2, dtype)
    v_cache = inputs.normal((B, Hkv, S_cap, d), seed, 3, dtype)
    return k_new, v_new, k_cache, v_cache


def check_rows(got, ref, dtype, what):
    got = got.to(torch.float64).numpy()
    assert np.all(np.isfinite(got)), what
    if dtype == F32:
        g = got.reshape(-1, got.shape[-1])
        r = ref.reshape(g.shape)
        rel = np.abs(g - r).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)
        assert rel.max() <= 2e-6, f"{what}: normwise relative error {rel.max():.3e}"
        return
    err = np.abs(got - ref)
    bound = ulp(ref, dtype)
    assert np.all(err <= bound), f"{what}: {int((err > bound).sum())} elements beyond one ulp"
    nearest = torch.from_numpy(ref).to(dtype).to(torch.float64).numpy()
    off = np.count_nonzero(got != nearest)
    assert off <= 1e-3 * got.size, f"{what}: {off} of {got.size} not rounded to nearest"


CASES = [
    # B, Hkv, Tnew, S_cap, d, start_pos, base, dtype
    (2, 3, 37, 64, 128, 0, 10000.0, BF16),     # prefill-style append from position 0
    (2, 2, 5, 600, 64, 500, 10000.0, F16),
    (3, 4, 1, 8192, 128, 8191, 10000.0, BF16),  # one decode token at the last slot
    (1, 2, 3, 100003, 256, 100000, 1e6, BF16),  # large positions: angle reduction
    (2, 1, 16, 40, 8, 3, 10000.0, BF16),        # smallest bf16 head
    (2, 8, 7, 50, 80, 40, 10000.0, F16),        # head size of the 3B model
    (2, 3, 9, 20, 12, 11, 500.0, F32),
    (1, 2, 4, 4200, 96, 4096, 10000.0, F32),
]


@pytest.mark.parametrize("B,Hkv,Tnew,S_cap,d,start_pos,base,dtype", CASES)
def test_append_matches_oracle(B, Hkv, Tnew, S_cap, d, start_pos, base, dtype):
    k_new, v_new, k_cache, v_cache = make_case(B, Hkv, Tnew, S_cap, d, dtype, seed=S_cap + d)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    attn.kv_append_rope(k_new.cuda(), v_new.cuda(), kc, vc, start_pos=start_pos, rope_base=base)
    torch.cuda.synchronize()
    kc, vc = kc.cpu(), vc.cpu()
    ref_k, _ = oracle.rope_append(k_new, v_new, start_pos=start_pos, base=base)
    rows = slice(start_pos, start_pos + Tnew)
    check_rows(kc[:, :, rows], ref_k, dtype, "K rows")
    assert torch.equal(vc[:, :, rows], v_new), "V rows are not a bitwise copy"
    # rows outside the appended range keep their bits
    keep = torch.ones(S_cap, dtype=torch.bool)
    keep[rows] = False
    assert torch.equal(kc[:, :, keep], k_cache[:, :, keep])
    assert torch.equal(vc[:, :, keep], v_cache[:, :, keep])


@pytest.mark.parametrize("dtype", [BF16, F16, F32])
def test_append_without_a_base_copies_bits(dtype):
    k_new, v_new, k_cache, v_cache = make_case(2, 3, 6, 32, 64, dtype, seed=7)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    attn.kv_append_rope(k_new.cuda(), v_new.cuda(), kc, vc, start_pos=20, rope_base=0.0)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu()[:, :, 20:26], k_new)
    assert torch.equal(vc.cpu()[:, :, 20:26], v_new)
    assert torch.equal(kc.cpu()[:, :, :20], k_cache[:, :, :20])


def test_position_zero_leaves_keys_unrotated():
    """cos 0 = 1 and sin 0 = 0 exactly: the first token's K is copied as is."""
    k_new, v_new, k_cache, v_cache = make_case(1, 2, 1, 8, 128, BF16, seed=9)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    attn.kv_append_rope(k_new.cuda(), v_new.cuda(), kc, vc, start_pos=0)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu()[:, :, :1], k_new)


@pytest.mark.parametrize("dtype", [BF16, F16])
def test_append_then_attend(dtype):
    """Decode step as a model runs it: append the new token's K/V at
    start_pos, then attend over the cache.  The oracle builds its own cache
    from its own rotated rows (rounded to the cache dtype) and attends over
    that; the outputs agree within the attention tolerance."""
    B, H, Hkv, d, S_cap, start_pos, Tnew = 2, 8, 2, 128, 1024, 700, 3
    scale = d ** -0.5
    q = inputs.normal((B, H, Tnew, d), 32, 0, dtype)
    k_new, v_new, k_cache, v_cache = make_case(B, Hkv, Tnew, S_cap, d, dtype, seed=31)
    kc, vc = k_cache.cuda(), v_cache.cuda()
    attn.kv_append_rope(k_new.cuda(), v_new.cuda(), kc, vc, start_pos=start_pos)
    S = start_pos + Tnew
    o = attn.cached(q.cuda(), kc, vc, start_pos=start_pos, scale=scale, S=S)
    torch.cuda.synchronize()
    ref_k, _ = oracle.rope_append(k_new, v_new, start_pos=start_pos, base=10000.0)
    k_ref = k_cache.clone()
    k_ref[:, :, start_pos:S] = torch.from_numpy(ref_k).to(dtype)
    v_ref = v_cache.clone()
    v_ref[:, :, start_pos:S] = v_new
    ref_o = oracle.attention(q, k_ref, v_ref, scale=scale, causal=True, start_pos=start_pos,
                             S=S)
    err = np.abs(o.cpu().to(torch.float64).numpy() - ref_o)
    assert err.max() <= 1.5e-2 and err.mean() <= 2e-3
