"""Pins for the oracle's backward pass (CPU).

The gradients are fixed by facts that do not retype the Jacobian formula:
centered finite differences of the C oracle's forward (the check the pages
name for every input of attention, "Causal Multi-Head Self-Attention",
Test coverage); fp64 autograd of a materialised forward written with torch
primitives; the single-key closed form (the output is the value row, so Q and
K get no gradient); invariants (a shift of every key leaves each softmax row
unchanged, so the key gradients sum to zero; every probability row sums to
one, so the value gradients sum to the summed upstream rows); exactly zero
gradient through masked scores ("Causal Multi-Head Self-Attention", Causal
mask); and permutation equivariance of non-causal attention.

Every pin takes the backward implementation as its ``bwd`` argument so that
test_oracle_backward_mutants.py can run the same pins against broken copies.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.backward import attention_backward


@pytest.fixture
def bwd():
    return attention_backward


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _loss(q, k, v, dout, scale, causal, window):
    out = oracle.attention(q, k, v, scale=scale, causal=causal, window=window)
    return float((out * dout.numpy()).sum())


FD_CASES = [
    # B, H, Hkv, T, d, causal, window, scale
    (1, 2, 1, 5, 3, True, 0, 0.8),
    (2, 4, 2, 4, 2, True, 0, 1.3),
    (1, 2, 2, 6, 3, False, 0, 0.6),
    (1, 3, 1, 7, 2, True, 3, 0.9),
]


@pytest.mark.parametrize("case", FD_CASES, ids=lambda c: "-".join(map(str, c)))
def test_centered_finite_differences(case, bwd):
    B, H, Hkv, T, d, causal, window, scale = case
    q, k, v = _rand((B, H, T, d), 1), _rand((B, Hkv, T, d), 2), _rand((B, Hkv, T, d), 3)
    dout = _rand((B, H, T, d), 4)
    dq, dk, dv = bwd(q, k, v, dout, scale=scale, causal=causal, window=window)
    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        flat = x.view(-1)
        num = np.zeros(flat.numel())
        for e in range(flat.numel()):
            keep = float(flat[e])
            flat[e] = keep + eps
            lp = _loss(q, k, v, dout, scale, causal, window)
            flat[e] = keep - eps
            lm = _loss(q, k, v, dout, scale, causal, window)
            flat[e] = keep
            num[e] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g.reshape(-1), num, rtol=1e-6, atol=1e-8, err_msg=name)


def _autograd(q, k, v, dout, scale, causal, window):
    """Gradients of a materialised forward built from torch primitives."""
    q, k, v = (t.clone().requires_grad_(True) for t in (q, k, v))
    B, H, T, d = q.shape
    G = H // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)
    vv = v.repeat_interleave(G, dim=1)
    s = scale * torch.einsum("bhid,bhjd->bhij", q, kk)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = torch.ones(T, T, dtype=torch.bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    p = torch.softmax(s.masked_fill(~allowed, float("-inf")), dim=-1)
    out = torch.einsum("bhij,bhjd->bhid", p, vv)
    (out * dout).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("case", [
    (2, 6, 2, 33, 8, True, 0, 0.35),
    (1, 4, 4, 40, 16, False, 0, 0.25),
    (2, 8, 1, 37, 5, True, 0, 1.1),
    (1, 4, 2, 50, 8, True, 7, 0.5),
], ids=lambda c: "-".join(map(str, c)))
def test_matches_fp64_autograd_of_a_materialised_forward(case, bwd):
    B, H, Hkv, T, d, causal, window, scale = case
    q, k, v = _rand((B, H, T, d), 5), _rand((B, Hkv, T, d), 6), _rand((B, Hkv, T, d), 7)
    dout = _rand((B, H, T, d), 8)
    got = bwd(q, k, v, dout, scale=scale, causal=causal, window=window)
    ref = _autograd(q, k, v, dout, scale, causal, window)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-12)


def test_single_position_closed_form(bwd):
    # one key: every row's output is that key's value row whatever Q and K are
    q, k, v = _rand((2, 4, 1, 6), 9), _rand((2, 2, 1, 6), 10), _rand((2, 2, 1, 6), 11)
    dout = _rand((2, 4, 1, 6), 12)
    dq, dk, dv = bwd(q, k, v, dout, scale=0.4)
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(dk, 0.0)
    want = dout.numpy().reshape(2, 2, 2, 1, 6).sum(axis=2)
    np.testing.assert_allclose(dv, want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("causal,window", [(True, 0), (False, 0), (True, 9)])
def test_gradient_sums(causal, window, bwd):
    B, H, Hkv, T, d = 2, 6, 3, 45, 7
    q, k, v = _rand((B, H, T, d), 13), _rand((B, Hkv, T, d), 14), _rand((B, Hkv, T, d), 15)
    dout = _rand((B, H, T, d), 16)
    dq, dk, dv = bwd(q, k, v, dout, scale=0.3, causal=causal, window=window)
    # adding one vector to every key shifts each score row by a constant
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    # rows of P sum to one: sum_j dV_j = sum over the group's heads and rows of dO
    want = dout.numpy().reshape(B, Hkv, H // Hkv, T, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), want, rtol=1e-12, atol=1e-11)


def test_masked_scores_carry_no_gradient(bwd):
    B, H, Hkv, T, d = 1, 4, 2, 30, 6
    q, k, v = _rand((B, H, T, d), 17), _rand((B, Hkv, T, d), 18), _rand((B, Hkv, T, d), 19)
    dout = _rand((B, H, T, d), 20)
    dq, dk, dv = bwd(q, k, v, dout, scale=0.5)
    j0 = 12
    # keys at or after j0 are read only by rows at or after j0
    dout2, q2 = dout.clone(), q.clone()
    dout2[:, :, :j0] = _rand((B, H, j0, d), 21)
    q2[:, :, :j0] = _rand((B, H, j0, d), 22)
    _, dk2, dv2 = bwd(q2, k, v, dout2, scale=0.5)
    np.testing.assert_allclose(dk2[:, :, j0:], dk[:, :, j0:], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(dv2[:, :, j0:], dv[:, :, j0:], rtol=1e-13, atol=1e-14)
    # rows before j0 never see keys at or after j0
    k3, v3 = k.clone(), v.clone()
    k3[:, :, j0:] = _rand((B, Hkv, T - j0, d), 23)
    v3[:, :, j0:] = _rand((B, Hkv, T - j0, d), 24)
    dq3, dk3, dv3 = bwd(q, k3, v3, dout, scale=0.5)
    np.testing.assert_allclose(dq3[:, :, :j0], dq[:, :, :j0], rtol=1e-13, atol=1e-14)
    # the last key only takes gradient from the last row
    last = T - 1
    dout4 = dout.clone()
    dout4[:, :, :last] = 0
    q4 = q.clone()
    q4[:, :, :last] = 0
    _, dk4, dv4 = bwd(q4, k, v, dout4, scale=0.5)
    np.testing.assert_allclose(dk4[:, :, last], dk[:, :, last], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv4[:, :, last], dv[:, :, last], rtol=1e-12, atol=1e-14)


def test_non_causal_permutation_equivariance(bwd):
    B, H, Hkv, T, d = 1, 2, 1, 19, 5
    q, k, v = _rand((B, H, T, d), 25), _rand((B, Hkv, T, d), 26), _rand((B, Hkv, T, d), 27)
    dout = _rand((B, H, T, d), 28)
    perm = torch.as_tensor(np.random.default_rng(0).permutation(T))
    dq, dk, dv = bwd(q, k, v, dout, scale=0.6, causal=False)
    dqp, dkp, dvp = bwd(q, k[:, :, perm], v[:, :, perm], dout, scale=0.6, causal=False)
    np.testing.assert_allclose(dqp, dq, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dkp, dk[:, :, perm.numpy()], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dvp, dv[:, :, perm.numpy()], rtol=1e-12, atol=1e-13)
