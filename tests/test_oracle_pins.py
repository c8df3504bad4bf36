"""Pins for the fp64 oracle, against facts that do not come from the oracle.

CPU only.  Each test names what fixes the expected value: the worked example
printed on the "Multi-query attention, annotated" page (§2.1), closed forms of
the softmax, invariants stated by the pages (rows sum to one, masked
probabilities are exactly zero, the future does not leak, GQA equals MHA on
repeated K/V heads, cached rows equal prefill rows), exhaustive checks of the
exact widening against library conversions, and an independent library
routine (torch float64 softmax + matmul) on tiny shapes.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import attention, widen_bits
from transformer_attention_causal_b200 import inputs

E = math.e


def _worked_example_tensors(g):
    q = torch.tensor(g["q"], dtype=torch.float64).reshape(1, 1, 1, 2)
    k = torch.tensor([g["k0"], g["k1"], g["k2"]], dtype=torch.float64).reshape(1, 1, 3, 2)
    v = torch.tensor([[x, 0.0] for x in g["v"]], dtype=torch.float64).reshape(1, 1, 3, 2)
    return q, k, v


# ---------------------------------------------------------------- worked example

def test_worked_example_printed_values(golden_dir):
    """Multi-query attention, annotated §2.1: scores (1,0,1), shares
    0.422/0.155/0.422, output 2.0 — run as one cached query at position 2."""
    g = read_golden(os.path.join(golden_dir, "worked_example_mqa.txt"))
    q, k, v = _worked_example_tensors(g)
    out, lse, probs = attention(q, k, v, scale=g["scale"][0], causal=True, start_pos=2,
                                want_lse=True, want_probs=True)
    assert np.round(probs[0, 0, 0], 3).tolist() == g["weights_3dp"]
    assert round(out[0, 0, 0, 0], 3) == g["output_3dp"][0]
    assert out[0, 0, 0, 1] == 0.0
    # lse = ln(sum_j e^{s_j}) with the printed scores
    assert lse[0, 0, 0] == pytest.approx(math.log(sum(math.exp(s) for s in g["scores"])), abs=1e-15)


def test_worked_example_closed_form(golden_dir):
    """Exact shares e/(2e+1), 1/(2e+1); output (4e+2)/(2e+1) = 2 exactly."""
    g = read_golden(os.path.join(golden_dir, "worked_example_mqa.txt"))
    q, k, v = _worked_example_tensors(g)
    out, probs = attention(q, k, v, scale=1.0, causal=True, start_pos=2, want_probs=True)
    np.testing.assert_allclose(probs[0, 0, 0], [E / (2 * E + 1), 1 / (2 * E + 1), E / (2 * E + 1)],
                               rtol=0, atol=1e-15)
    assert abs(out[0, 0, 0, 0] - 2.0) < 1e-15


def test_worked_example_as_prefill(golden_dir):
    """Same keys/values as a causal prefill with every query = (1,0):
    row 0 sees key 0 only -> 1; row 1 -> (e+2)/(e+1); row 2 -> 2."""
    g = read_golden(os.path.join(golden_dir, "worked_example_mqa.txt"))
    _, k, v = _worked_example_tensors(g)
    q = torch.tensor([[1.0, 0.0]] * 3, dtype=torch.float64).reshape(1, 1, 3, 2)
    out = attention(q, k, v, scale=1.0, causal=True)
    np.testing.assert_allclose(out[0, 0, :, 0], [1.0, (E + 2) / (E + 1), 2.0], rtol=0, atol=1e-15)


# ---------------------------------------------------------------- closed forms

def _rand(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64).to(dtype)


def test_first_row_sees_only_key_zero():
    """Causal row 0 has one visible key: O = V[0] exactly, lse = its score."""
    q, k, v = _rand((2, 4, 5, 8), 1), _rand((2, 2, 5, 8), 2), _rand((2, 2, 5, 8), 3)
    out, lse = attention(q, k, v, scale=0.3, causal=True, want_lse=True)
    for b, h in itertools.product(range(2), range(4)):
        np.testing.assert_array_equal(out[b, h, 0], v[b, h // 2, 0].numpy())
        s = 0.3 * float(np.dot(q[b, h, 0].numpy(), k[b, h // 2, 0].numpy()))
        assert lse[b, h, 0] == pytest.approx(s, rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("start_pos,Tq,S", [(0, 7, 7), (5, 3, 8), (2, 2, 10)])
def test_zero_keys_give_causal_prefix_mean(start_pos, Tq, S):
    """K = 0 makes every visible score 0: O_i = mean(V[0..p_i]), lse = ln(p_i+1),
    with p_i = start_pos + i; keys past p_i are present but masked."""
    q = _rand((1, 2, Tq, 4), 4)
    k = torch.zeros((1, 1, S, 4), dtype=torch.float64)
    v = _rand((1, 1, S, 4), 5)
    out, lse = attention(q, k, v, scale=0.7, causal=True, start_pos=start_pos, want_lse=True)
    for i in range(Tq):
        p = start_pos + i
        expect = v[0, 0, : p + 1].numpy().mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(out[0, h, i], expect, rtol=1e-13, atol=1e-14)
            assert lse[0, h, i] == pytest.approx(math.log(p + 1), rel=1e-14)


def test_scale_zero_gives_prefix_mean():
    q, k, v = _rand((1, 1, 6, 3), 6), _rand((1, 1, 6, 3), 7), _rand((1, 1, 6, 3), 8)
    out = attention(q, k, v, scale=0.0, causal=True)
    for i in range(6):
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, : i + 1].numpy().mean(axis=0),
                                   rtol=1e-13, atol=1e-14)


def test_noncausal_zero_keys_give_full_mean():
    q, v = _rand((1, 1, 4, 3), 9), _rand((1, 1, 9, 3), 10)
    k = torch.zeros((1, 1, 9, 3), dtype=torch.float64)
    out = attention(q, k, v, scale=1.0, causal=False)
    for i in range(4):
        np.testing.assert_allclose(out[0, 0, i], v[0, 0].numpy().mean(axis=0), rtol=1e-13, atol=1e-14)


def test_constant_values_pass_through():
    """V = c on every visible row: the weights sum to one, so O = c."""
    q, k = _rand((2, 2, 9, 5), 11), _rand((2, 2, 9, 5), 12)
    v = torch.full((2, 2, 9, 5), 3.25, dtype=torch.float64)
    out = attention(q, k, v, scale=0.5, causal=True)
    np.testing.assert_allclose(out, 3.25, rtol=1e-14)


@pytest.mark.parametrize("a,scale", [(1.0, 1.0), (2.0, 0.25), (-3.0, 0.6)])
def test_two_keys_are_a_logistic(a, scale):
    """q = (a, 0), k0 = (1, 0), k1 = (0, 1): weight of key 0 is
    1 / (1 + exp(-a*scale)); pins both the scale and the sign of the exponent."""
    q = torch.tensor([a, 0.0], dtype=torch.float64).reshape(1, 1, 1, 2)
    k = torch.tensor([[1.0, 0.0], [0.0, 1.0]], dtype=torch.float64).reshape(1, 1, 2, 2)
    v = torch.tensor([[1.0, 0.0], [0.0, 1.0]], dtype=torch.float64).reshape(1, 1, 2, 2)
    out = attention(q, k, v, scale=scale, causal=False)
    w0 = 1.0 / (1.0 + math.exp(-a * scale))
    np.testing.assert_allclose(out[0, 0, 0], [w0, 1 - w0], rtol=1e-14)


def test_gqa_head_mapping_is_h_over_group():
    """V[b, kvh] = kvh + 1 everywhere: every query head h reads K/V head
    h // (H/Hkv) (repeat_interleave order), so O[b, h] = h // g + 1."""
    B, H, Hkv, T, d = 2, 8, 2, 6, 4
    g = H // Hkv
    q, k = _rand((B, H, T, d), 13), _rand((B, Hkv, T, d), 14)
    v = torch.zeros((B, Hkv, T, d), dtype=torch.float64)
    for kvh in range(Hkv):
        v[:, kvh] = kvh + 1
    out = attention(q, k, v, scale=0.4, causal=True)
    for h in range(H):
        np.testing.assert_allclose(out[:, h], h // g + 1, rtol=1e-14)


def test_dominant_key_selects_its_value():
    """One key aligned with the query and far larger than the others: the
    softmax tends to one-hot and O tends to that key's value row."""
    d = 6
    q = _rand((1, 1, 1, d), 15)
    k = _rand((1, 1, 7, d), 16) * 0.1
    k[0, 0, 4] = q[0, 0, 0] * 60.0
    v = _rand((1, 1, 7, d), 17)
    out = attention(q, k, v, scale=1.0, causal=False)
    np.testing.assert_allclose(out[0, 0, 0], v[0, 0, 4].numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants

def test_rows_sum_to_one_and_masked_are_exactly_zero():
    q, k, v = _rand((2, 4, 6, 8), 18), _rand((2, 2, 11, 8), 19), _rand((2, 2, 11, 8), 20)
    out, probs = attention(q, k, v, scale=0.35, causal=True, start_pos=3, S=11, want_probs=True)
    np.testing.assert_allclose(probs.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    for i in range(6):
        p = 3 + i
        assert np.all(probs[:, :, i, p + 1:] == 0.0)
        assert np.all(probs[:, :, i, : p + 1] > 0.0)


def test_future_tokens_do_not_change_earlier_rows():
    """Perturbing every position after i leaves row i bit-for-bit unchanged."""
    T = 9
    q, k, v = _rand((1, 2, T, 8), 21), _rand((1, 1, T, 8), 22), _rand((1, 1, T, 8), 23)
    base = attention(q, k, v, scale=0.35, causal=True)
    for i in range(T - 1):
        q2, k2, v2 = q.clone(), k.clone(), v.clone()
        q2[:, :, i + 1:] += 5.0
        k2[:, :, i + 1:] *= -3.0
        v2[:, :, i + 1:] += 7.0
        pert = attention(q2, k2, v2, scale=0.35, causal=True)
        np.testing.assert_array_equal(pert[:, :, : i + 1], base[:, :, : i + 1])


def test_gqa_equals_mha_on_repeated_heads():
    B, H, Hkv, T, d = 2, 6, 3, 7, 5
    q, k, v = _rand((B, H, T, d), 24), _rand((B, Hkv, T, d), 25), _rand((B, Hkv, T, d), 26)
    gqa = attention(q, k, v, scale=0.45, causal=True)
    rep = H // Hkv
    mha = attention(q, k.repeat_interleave(rep, dim=1), v.repeat_interleave(rep, dim=1),
                    scale=0.45, causal=True)
    np.testing.assert_array_equal(gqa, mha)


def test_cached_rows_equal_prefill_rows():
    """New tokens at start_pos against the full history reproduce the matching
    rows of the full causal prefill (same visible keys, same arithmetic)."""
    B, H, Hkv, T, d, Tnew = 2, 4, 2, 12, 8, 5
    q, k, v = _rand((B, H, T, d), 27), _rand((B, Hkv, T, d), 28), _rand((B, Hkv, T, d), 29)
    full = attention(q, k, v, scale=0.35, causal=True)
    start = T - Tnew
    cached = attention(q[:, :, start:], k, v, scale=0.35, causal=True, start_pos=start)
    np.testing.assert_array_equal(cached, full[:, :, start:])


def test_history_past_the_last_query_is_ignored():
    """Keys beyond start_pos + Tnew - 1 are masked even though they exist."""
    q = _rand((1, 2, 3, 4), 30)
    k, v = _rand((1, 1, 12, 4), 31), _rand((1, 1, 12, 4), 32)
    long = attention(q, k, v, scale=0.5, causal=True, start_pos=4, S=12)
    short = attention(q, k[:, :, :7].contiguous(), v[:, :, :7].contiguous(), scale=0.5,
                      causal=True, start_pos=4, S=7)
    np.testing.assert_array_equal(long, short)


def test_batches_are_isolated():
    q, k, v = _rand((3, 2, 5, 4), 33), _rand((3, 2, 5, 4), 34), _rand((3, 2, 5, 4), 35)
    base = attention(q, k, v, scale=0.5, causal=True)
    k2, v2 = k.clone(), v.clone()
    k2[1] += 4.0
    v2[1] -= 2.0
    pert = attention(q, k2, v2, scale=0.5, causal=True)
    np.testing.assert_array_equal(pert[0], base[0])
    np.testing.assert_array_equal(pert[2], base[2])
    assert not np.array_equal(pert[1], base[1])


def test_noncausal_is_invariant_to_key_order():
    q, k, v = _rand((1, 2, 4, 6), 36), _rand((1, 2, 10, 6), 37), _rand((1, 2, 10, 6), 38)
    perm = torch.randperm(10, generator=torch.Generator().manual_seed(0))
    a = attention(q, k, v, scale=0.4, causal=False)
    b = attention(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), scale=0.4, causal=False)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_row_subset_matches_full_result():
    q, k, v = _rand((2, 4, 6, 8), 39), _rand((2, 2, 6, 8), 40), _rand((2, 2, 6, 8), 41)
    full, lse = attention(q, k, v, scale=0.35, causal=True, want_lse=True)
    rows = [0, 7, 13, 47, 30]
    sub, sub_lse = attention(q, k, v, scale=0.35, causal=True, rows=rows, want_lse=True)
    flat = full.reshape(-1, 8)
    np.testing.assert_array_equal(sub, flat[rows])
    np.testing.assert_array_equal(sub_lse, lse.reshape(-1)[rows])


# ---------------------------------------------------------------- library routine

def _torch_reference(q, k, v, scale, causal, start_pos):
    """softmax(q k^T * scale + causal bias) @ v in float64 with torch library
    ops; K/V heads expanded with repeat_interleave ("Grouped-Query Attention"
    §5.1-5.2).  The bias hides key j from query i when j > start_pos + i."""
    rep = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    scores = torch.matmul(q, k.transpose(-2, -1)) * scale
    if causal:
        Tq, S = q.shape[-2], k.shape[-2]
        qpos = torch.arange(Tq).unsqueeze(1) + start_pos
        kpos = torch.arange(S).unsqueeze(0)
        bias = torch.zeros((Tq, S), dtype=torch.float64).masked_fill(kpos > qpos, float("-inf"))
        scores = scores + bias
    return torch.matmul(torch.softmax(scores, dim=-1), v)


def test_tiny_shapes_against_torch_float64():
    """Every tiny shape up to the (2, 9, 32)-sized batch of the "Grouped-Query
    Attention" parity check, causal and not, against the library routine."""
    seed = 100
    for B, (H, Hkv), T, d, causal in itertools.product(
            (1, 2), ((1, 1), (2, 1), (2, 2), (4, 2), (4, 1)), (1, 2, 5, 9), (1, 3, 8, 32),
            (True, False)):
        seed += 1
        q, k, v = _rand((B, H, T, d), seed), _rand((B, Hkv, T, d), seed + 1000), \
            _rand((B, Hkv, T, d), seed + 2000)
        got = attention(q, k, v, scale=1 / math.sqrt(d), causal=causal)
        ref = _torch_reference(q, k, v, 1 / math.sqrt(d), causal, 0).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_cached_shapes_against_torch_float64():
    for start_pos, Tnew, (H, Hkv) in itertools.product((0, 3, 8), (1, 2, 4), ((4, 1), (4, 2))):
        S = start_pos + Tnew
        q = _rand((2, H, Tnew, 8), start_pos * 7 + Tnew)
        k = _rand((2, Hkv, S, 8), 500 + start_pos)
        v = _rand((2, Hkv, S, 8), 900 + Tnew)
        got = attention(q, k, v, scale=0.3, causal=True, start_pos=start_pos)
        ref = _torch_reference(q, k, v, 0.3, True, start_pos).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- exact widening

def test_bf16_widening_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ours = widen_bits(bits, "bf16")
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(lib)
    np.testing.assert_array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan], lib[~nan])


def test_f16_widening_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ours = widen_bits(bits, "f16")
    lib = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(lib)
    np.testing.assert_array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan], lib[~nan])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
def test_low_precision_inputs_equal_their_exact_float64_values(dtype):
    """The oracle on rounded inputs equals the oracle on those same values
    given as float64 (the widening is exact, nothing else changes)."""
    q, k, v = inputs.qkv(1, 4, 2, 7, 7, 16, dtype, seed=3)
    a = attention(q, k, v, scale=0.25, causal=True)
    b = attention(q.double(), k.double(), v.double(), scale=0.25, causal=True)
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- argument checks

def test_malformed_arguments_are_rejected():
    q, k, v = _rand((1, 3, 2, 4), 1), _rand((1, 2, 2, 4), 2), _rand((1, 2, 2, 4), 3)
    with pytest.raises(ValueError):
        attention(q, k, v, scale=1.0)  # H % Hkv != 0
    q = _rand((1, 2, 2, 4), 1)
    with pytest.raises(ValueError):
        attention(q, k, v, scale=1.0, S=3)  # S > S_cap
    with pytest.raises(ValueError):
        attention(q, k, v, scale=1.0, rows=[4])  # row id out of range
