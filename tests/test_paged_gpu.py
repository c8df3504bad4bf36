"""Cached attention over a paged K/V cache: CUDA path vs the fp64 oracle
(needs a B200).

Pages are built from a seeded contiguous history with a seeded permutation of
physical pages (plus pages no sequence uses); sequences have their own
lengths.  Tolerance as for every 16-bit path: max abs error <= 1.5e-2 and mean
abs error <= 2e-3 against the oracle on the same rounded inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import transformer_attention_causal_b200 as attn
from transformer_attention_causal_b200 import inputs

pytestmark = pytest.mark.gpu

BF16, F16 = torch.bfloat16, torch.float16
DEVICE_INDEX = 6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from transformer_attention_causal_b200.build import build

    build()
    torch.cuda.init()
    yield
    assert attn.device_status() == 0


def make_paged(B, H, Hkv, Tnew, d, lens, page_size, dtype, seed, spare_pages=3):
    """q, pages and table; sequence b's logical page i sits at a seeded
    physical page.  Returns CPU tensors."""
    max_len = max(lens)
    max_pages = (max_len + page_size - 1) // page_size
    q = inputs.normal((B, H, Tnew, d), seed, 0, dtype)
    k = inputs.normal((B, Hkv, max_pages * page_size, d), seed, 1, dtype)
    v = inputs.normal((B, Hkv, max_pages * page_size, d), seed, 2, dtype)
    num_pages = B * max_pages + spare_pages
    perm = np.random.default_rng(seed).permutation(num_pages)[:B * max_pages]
    k_pages = torch.zeros((num_pages, Hkv, page_size, d), dtype=dtype)
    v_pages = torch.zeros_like(k_pages)
    for b in range(B):
        for i in range(max_pages):
            ph = perm[b * max_pages + i]
            k_pages[ph] = k[b, :, i * page_size:(i + 1) * page_size]
            v_pages[ph] = v[b, :, i * page_size:(i + 1) * page_size]
    table = torch.as_tensor(perm.reshape(B, max_pages), dtype=torch.int32)
    kv_lens = torch.as_tensor(lens, dtype=torch.int32)
    return q, k_pages, v_pages, table, kv_lens


def run_gpu(q, k_pages, v_pages, table, kv_lens, scale, max_kv_len=None, lse=False):
    dev = [t.cuda() for t in (q, k_pages, v_pages, table, kv_lens)]
    lse_t = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda") if lse else None
    out = attn.cached_paged(*dev, max_kv_len=int(max_kv_len or int(kv_lens.max())), scale=scale,
                            lse=lse_t)
    torch.cuda.synchronize()
    return (out.cpu(), lse_t.cpu() if lse else None)


def check(got, ref):
    err = np.abs(got.to(torch.float64).numpy() - ref)
    assert np.all(np.isfinite(got.float().numpy()))
    assert err.max() <= 1.5e-2, f"max abs error {err.max():.3e}"
    assert err.mean() <= 2e-3, f"mean abs error {err.mean():.3e}"


CASES = [
    # B, H, Hkv, Tnew, d, lens, page_size, dtype
    (3, 8, 2, 1, 128, [1000, 37, 517], 16, BF16),      # decode, small pages, ragged lengths
    (2, 32, 8, 1, 128, [4096, 2049], 64, BF16),        # GQA 4:1 decode
    (2, 16, 4, 4, 128, [700, 1500], 256, F16),         # 4 new tokens per sequence
    (2, 8, 1, 1, 64, [333, 64], 8, BF16),              # MQA, d = 64, the smallest pages
    (2, 4, 4, 2, 256, [900, 129], 32, F16),            # d = 256
    (3, 8, 8, 1, 80, [700, 129, 2048], 64, BF16),      # MHA decode, d = 80
    (2, 8, 2, 2, 96, [333, 1000], 16, F16),            # d = 96, 8 rows per K/V head
    (4, 8, 8, 1, 128, [1, 5, 128, 129], 128, BF16),    # lengths at page edges, a single token
    # chunked prefill (many new rows per K/V head): the tensor-core kernel
    # copying whole pages, one to sixteen copies per 128-key tile
    (2, 8, 1, 200, 128, [1000, 450], 64, F16),         # MQA, two pages per tile
    (2, 16, 4, 300, 128, [800, 300], 128, BF16),       # a page per tile; a sequence of only new tokens
    (1, 8, 2, 129, 64, [2000], 256, BF16),             # pages longer than a tile, d = 64
    (2, 4, 4, 64, 80, [129, 1000], 16, F16),           # MHA, d = 80
    (3, 8, 2, 100, 96, [100, 357, 1024], 8, BF16),     # the smallest pages
]


@pytest.mark.parametrize("B,H,Hkv,Tnew,d,lens,page_size,dtype", CASES)
def test_paged_matches_oracle(B, H, Hkv, Tnew, d, lens, page_size, dtype):
    q, kp, vp, table, kv_lens = make_paged(B, H, Hkv, Tnew, d, lens, page_size, dtype,
                                           seed=sum(lens) + page_size)
    scale = 1 / math.sqrt(d)
    got, lse = run_gpu(q, kp, vp, table, kv_lens, scale, lse=True)
    ref, ref_lse = oracle.paged_attention(q, kp, vp, table, lens, scale=scale, want_lse=True)
    check(got, ref)
    assert np.abs(lse.numpy() - ref_lse).max() <= 2e-3


def test_a_larger_length_bound_changes_nothing():
    """max_kv_len only plans the split: any bound >= every length gives the
    same numbers as the tight one."""
    q, kp, vp, table, kv_lens = make_paged(2, 8, 2, 1, 128, [300, 900], 16, BF16, seed=3)
    a, _ = run_gpu(q, kp, vp, table, kv_lens, 0.1, max_kv_len=900)
    pages = table.shape[1] * 16
    b, _ = run_gpu(q, kp, vp, table, kv_lens, 0.1, max_kv_len=pages)
    check(a, b.to(torch.float64).numpy())


def test_paged_equals_contiguous_cached_on_the_same_history():
    """One sequence length for all: the contiguous entry point on the gathered
    history agrees with the paged one."""
    B, H, Hkv, Tnew, d, L, P = 2, 16, 4, 1, 128, 2048, 64
    q, kp, vp, table, kv_lens = make_paged(B, H, Hkv, Tnew, d, [L] * B, P, BF16, seed=4)
    got, _ = run_gpu(q, kp, vp, table, kv_lens, 0.088)
    k = torch.stack([oracle.gather_pages(kp, table[b], L) for b in range(B)])
    v = torch.stack([oracle.gather_pages(vp, table[b], L) for b in range(B)])
    ref = attn.cached(q.cuda(), k.cuda(), v.cuda(), start_pos=L - Tnew, scale=0.088).cpu()
    check(got, ref.to(torch.float64).numpy())


@pytest.mark.parametrize("what", ["page", "length"])
def test_out_of_range_entries_are_reported_not_followed(what):
    """A page id past the pool, or a length past the bound, is caught by the
    kernel's own range check: recorded as ATTN_ERR_DEVICE_INDEX, clamped, and
    no load leaves the pools."""
    q, kp, vp, table, kv_lens = make_paged(2, 8, 2, 1, 128, [200, 100], 16, BF16, seed=5)
    if what == "page":
        table[1, 2] = kp.shape[0] + 7
        bound = 200
    else:
        kv_lens[0] = 250
        bound = 200
    run_gpu(q, kp, vp, table, kv_lens, 0.1, max_kv_len=bound)
    assert attn.device_status() == DEVICE_INDEX
    assert attn.device_status() == 0


def test_out_of_range_page_in_chunked_prefill_is_reported():
    q, kp, vp, table, kv_lens = make_paged(2, 8, 2, 150, 128, [300, 200], 16, BF16, seed=6)
    table[1, 3] = kp.shape[0] + 5
    run_gpu(q, kp, vp, table, kv_lens, 0.1)
    assert attn.device_status() == DEVICE_INDEX
    assert attn.device_status() == 0


def test_full_size_decode_sampled_rows():
    """The benchmark's paged decode workload: B = 64, 32 query heads over 8 K/V
    heads, d = 128, bf16, 64-token pages, one new token per sequence; lengths
    8192 for every sequence.  Rows of four sequences are checked."""
    B, H, Hkv, d, L, P = 64, 32, 8, 128, 8192, 64
    q, kp, vp, table, kv_lens = make_paged(B, H, Hkv, 1, d, [L] * B, P, BF16, seed=6,
                                           spare_pages=0)
    got, _ = run_gpu(q, kp, vp, table, kv_lens, 1 / math.sqrt(d))
    for b in (0, 17, 42, 63):
        ref = oracle.paged_attention(q[b:b + 1], kp, vp, table[b:b + 1], [L],
                                     scale=1 / math.sqrt(d))
        check(got[b:b + 1], ref)


def poison_tails(k_pages, v_pages, table, lens):
    """Fill every page row that no sequence reads (the rows of a sequence's
    last page past its length) with NaN, +inf and -inf in turn: a pool from
    torch.empty or a recycled page may hold any bit pattern there."""
    P = k_pages.shape[2]
    bad = [float("nan"), float("inf"), float("-inf")]
    for b, L in enumerate(lens):
        for j in range(L, table.shape[1] * P):
            ph, r = int(table[b, j // P]), j % P
            k_pages[ph, :, r] = bad[j % 3]
            v_pages[ph, :, r] = bad[(j + 1) % 3]


NAN_TAIL_CASES = [
    # chunked prefill on the tensor-core kernel (whole pages copied)
    (2, 8, 1, 200, 128, [1000, 450], 64, F16),
    (2, 16, 4, 300, 128, [777, 301], 128, BF16),
    (1, 8, 2, 129, 64, [2001], 256, BF16),
    (3, 8, 2, 100, 96, [100, 357, 1027], 8, BF16),
    (2, 4, 4, 64, 80, [129, 1000], 16, F16),
    # the split-KV decode kernels
    (3, 8, 2, 1, 128, [1000, 37, 517], 16, BF16),
    (2, 4, 4, 2, 256, [900, 129], 32, F16),
]


@pytest.mark.parametrize("B,H,Hkv,Tnew,d,lens,page_size,dtype", NAN_TAIL_CASES)
def test_unused_page_rows_holding_nan_or_inf_change_nothing(B, H, Hkv, Tnew, d, lens, page_size,
                                                             dtype):
    """Paging changes only where K/V live ("Causal Multi-Head Self-Attention",
    Algorithm and cache boundaries): rows past a sequence's length are not part
    of it, whatever they hold."""
    q, kp, vp, table, kv_lens = make_paged(B, H, Hkv, Tnew, d, lens, page_size, dtype,
                                           seed=7 + sum(lens))
    poison_tails(kp, vp, table, lens)
    scale = 1 / math.sqrt(d)
    got, lse = run_gpu(q, kp, vp, table, kv_lens, scale, lse=True)
    ref, ref_lse = oracle.paged_attention(q, kp, vp, table, lens, scale=scale, want_lse=True)
    check(got, ref)
    assert np.abs(lse.numpy() - ref_lse).max() <= 2e-3
