"""Pins for the oracle's local window (CPU).

Fixed by cases that do not retype the mask: a window of one key returns the
query's own value row; a window at least as long as the history is plain
causal attention; with K = 0 every visible key weighs the same, so each row is
the mean of the last min(w, p + 1) values (which pins both window edges) and
lse = ln(min(w, p + 1)); a brute-force softmax over the banded score matrix
(numpy, written here) on small shapes; and the window-32 configuration of the
pages ("Multi-query attention, annotated" §4.1: the current position and the
previous 31) on a long row.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def test_window_of_one_returns_the_own_value():
    q, k, v = _rand((1, 2, 6, 4), 1), _rand((1, 1, 6, 4), 2), _rand((1, 1, 6, 4), 3)
    out, lse = attention(q, k, v, scale=0.7, window=1, want_lse=True)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], v[0, 0].numpy(), rtol=0, atol=1e-15)
        s_self = 0.7 * (q[0, h] * k[0, 0]).sum(-1).numpy()
        np.testing.assert_allclose(lse[0, h], s_self, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("w", [9, 10, 50])
def test_a_window_covering_the_history_is_plain_causal(w):
    q, k, v = _rand((2, 2, 9, 4), 4), _rand((2, 2, 9, 4), 5), _rand((2, 2, 9, 4), 6)
    a = attention(q, k, v, scale=0.5, window=w)
    b = attention(q, k, v, scale=0.5)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("w,start", [(3, 0), (4, 5), (32, 40)])
def test_uniform_scores_average_the_window(w, start):
    Tq, d = 12, 3
    S = start + Tq
    q = _rand((1, 1, Tq, d), 7)
    k = torch.zeros((1, 1, S, d), dtype=torch.float64)
    v = _rand((1, 1, S, d), 8)
    out, lse = attention(q, k, v, scale=1.0, start_pos=start, window=w, want_lse=True)
    for i in range(Tq):
        p = start + i
        lo = max(0, p - w + 1)
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, lo:p + 1].mean(0).numpy(), rtol=1e-12)
        np.testing.assert_allclose(lse[0, 0, i], math.log(p + 1 - lo), rtol=1e-12)


@pytest.mark.parametrize("B,H,Hkv,Tq,S,w", [(1, 2, 1, 7, 7, 3), (2, 4, 2, 5, 11, 4)])
def test_brute_force_banded_softmax(B, H, Hkv, Tq, S, w):
    q, k, v = _rand((B, H, Tq, 5), 9), _rand((B, Hkv, S, 5), 10), _rand((B, Hkv, S, 5), 11)
    start = S - Tq
    got = attention(q, k, v, scale=0.4, start_pos=start, window=w)
    g = H // Hkv
    for b in range(B):
        for h in range(H):
            kk, vv = k[b, h // g].numpy(), v[b, h // g].numpy()
            for i in range(Tq):
                p = start + i
                js = [j for j in range(S) if p - w < j <= p]
                sc = np.array([0.4 * float(np.dot(q[b, h, i].numpy(), kk[j])) for j in js])
                e = np.exp(sc - sc.max())
                ref = (e[:, None] * vv[js]).sum(0) / e.sum()
                np.testing.assert_allclose(got[b, h, i], ref, rtol=1e-12, atol=1e-13)


def test_the_pages_window_of_32():
    """Last query of a 200-token sequence with w = 32 sees positions 168..199
    only: moving any earlier value changes nothing, moving one inside does."""
    q, k, v = _rand((1, 1, 1, 8), 12), _rand((1, 1, 200, 8), 13), _rand((1, 1, 200, 8), 14)
    base = attention(q, k, v, scale=0.3, start_pos=199, window=32)
    v2 = v.clone()
    v2[0, 0, :168] += 5.0
    np.testing.assert_array_equal(attention(q, k, v2, scale=0.3, start_pos=199, window=32), base)
    v2[0, 0, 168] += 5.0
    assert not np.allclose(attention(q, k, v2, scale=0.3, start_pos=199, window=32), base)
