"""Pins for the oracle's paged cache (CPU).

The gather is checked against a paged cache built here independently, by
reshaping a contiguous history (so a transposed page layout, a wrong page
index or a wrong row within a page shows up), plus invariants: the physical
placement of pages does not matter, one page holding the whole history is the
contiguous case, and each sequence's own length places its new tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import paged as paged_mod


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def pages_from_contiguous(k, page_size, perm):
    """k [B, Hkv, S, d] -> pages [B * S / page_size, Hkv, page_size, d] with
    sequence b's logical page i stored at physical page perm[b * n + i]."""
    B, Hkv, S, d = k.shape
    n = S // page_size
    blocks = k.reshape(B, Hkv, n, page_size, d).permute(0, 2, 1, 3, 4).reshape(B * n, Hkv, page_size, d)
    pages = torch.empty_like(blocks)
    pages[torch.as_tensor(perm)] = blocks
    table = torch.as_tensor(perm, dtype=torch.int64).reshape(B, n)
    return pages, table


@pytest.mark.parametrize("page_size", [1, 2, 4, 8])
def test_gather_inverts_an_independent_paging(page_size):
    B, Hkv, S, d = 2, 3, 16, 4
    k = _rand((B, Hkv, S, d), 1)
    perm = np.random.default_rng(page_size).permutation(B * S // page_size)
    pages, table = pages_from_contiguous(k, page_size, perm)
    for b in range(B):
        for L in (1, 7, S):
            got = oracle.gather_pages(pages, table[b], L)
            np.testing.assert_array_equal(got.numpy(), k[b, :, :L].numpy())


def test_paged_attention_equals_contiguous_cached_attention():
    B, H, Hkv, S, d, Tnew, P = 2, 4, 2, 24, 8, 3, 8
    q = _rand((B, H, Tnew, d), 2)
    k, v = _rand((B, Hkv, S, d), 3), _rand((B, Hkv, S, d), 4)
    perm = np.random.default_rng(5).permutation(B * S // P)
    kp, table = pages_from_contiguous(k, P, perm)
    vp, _ = pages_from_contiguous(v, P, perm)
    lens = [S, 13]
    got = oracle.paged_attention(q, kp, vp, table, lens, scale=0.3)
    for b, L in enumerate(lens):
        ref = oracle.attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], scale=0.3, causal=True,
                               start_pos=L - Tnew, S=L)
        np.testing.assert_allclose(got[b:b + 1], ref, rtol=0, atol=1e-15)


def test_physical_placement_does_not_matter():
    B, H, Hkv, S, d, Tnew, P = 1, 2, 1, 32, 4, 2, 8
    q = _rand((B, H, Tnew, d), 6)
    k, v = _rand((B, Hkv, S, d), 7), _rand((B, Hkv, S, d), 8)
    outs = []
    for seed in (0, 1, 2):
        perm = np.random.default_rng(seed).permutation(S // P)
        kp, table = pages_from_contiguous(k, P, perm)
        vp, _ = pages_from_contiguous(v, P, perm)
        outs.append(oracle.paged_attention(q, kp, vp, table, [S], scale=0.5))
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_new_tokens_sit_at_the_end_of_each_sequence():
    """K = 0 makes every visible key weigh the same: the last new token of a
    sequence of length L averages all L values; the first averages L - Tnew + 1."""
    B, H, Hkv, S, d, Tnew, P = 2, 2, 1, 16, 4, 3, 4
    q = _rand((B, H, Tnew, d), 9)
    k = torch.zeros((B, Hkv, S, d), dtype=torch.float64)
    v = _rand((B, Hkv, S, d), 10)
    perm = np.arange(B * S // P)
    kp, table = pages_from_contiguous(k, P, perm)
    vp, _ = pages_from_contiguous(v, P, perm)
    lens = [16, 9]
    out = oracle.paged_attention(q, kp, vp, table, lens, scale=1.0)
    for b, L in enumerate(lens):
        for t in range(Tnew):
            n_vis = L - Tnew + t + 1
            np.testing.assert_allclose(out[b, 0, t], v[b, 0, :n_vis].mean(0).numpy(), rtol=1e-12)


def test_a_transposed_page_layout_is_caught(monkeypatch):
    """Planted mistake (on the CPU): reading pages as [num_pages, page_size,
    Hkv, d] must fail the independent-paging pin."""
    def wrong(pages, row, length):
        page_size = pages.shape[2]
        flat = pages.reshape(pages.shape[0], page_size, pages.shape[1], pages.shape[3])
        rows = [flat[int(row[j // page_size]), j % page_size] for j in range(length)]
        return torch.stack(rows, dim=1)
    monkeypatch.setattr(oracle, "gather_pages", wrong)
    with pytest.raises(AssertionError):
        test_gather_inverts_an_independent_paging(4)


def test_an_off_by_one_page_index_is_caught(monkeypatch):
    real = paged_mod.gather_pages

    def wrong(pages, row, length):
        shifted = torch.roll(torch.as_tensor(row), 1)
        return real(pages, shifted, length)
    monkeypatch.setattr(paged_mod, "gather_pages", wrong)
    with pytest.raises(AssertionError):
        test_paged_attention_equals_contiguous_cached_attention()
