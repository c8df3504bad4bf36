"""Paged K/V cache for the fp64 oracle: the logical history of each sequence
gathered out of its pages, then ordinary cached attention on it.

TEST INFRASTRUCTURE ONLY (see the package docstring).  A paged cache changes
where keys and values live, not what is computed ("Causal Multi-Head
Self-Attention", Algorithm and cache boundaries: paging controls where K/V
state lives, paged decode reads a logical-to-physical page table;
attention_cached.go, CausalAttentionPackedBlocks: blocks laid out head-major,
[kv head][token within block][d]).  So the oracle is the gather written out
plus ``attention`` per sequence.

Layout: pages [num_pages, Hkv, page_size, d]; token j of sequence b is row
j % page_size of physical page page_table[b, j // page_size].  Sequence b holds
kv_lens[b] tokens; its Tnew new queries sit at positions kv_lens[b] - Tnew ...
"""
from __future__ import annotations

import numpy as np
import torch

from .attention import attention


def gather_pages(pages, page_table_row, length: int):
    """[Hkv, length, d] history of one sequence, in logical token order."""
    pages = pages if isinstance(pages, torch.Tensor) else torch.as_tensor(pages)
    page_size = pages.shape[2]
    rows = []
    for j in range(length):
        phys = int(page_table_row[j // page_size])
        rows.append(pages[phys, :, j % page_size, :])   # [Hkv, d]
    if not rows:
        return pages.new_zeros((pages.shape[1], 0, pages.shape[3]))
    return torch.stack(rows, dim=1)                      # [Hkv, length, d]


def paged_attention(q, k_pages, v_pages, page_table, kv_lens, *, scale: float,
                    want_lse: bool = False):
    """fp64 rows [B, H, Tnew, d] (and lse [B, H, Tnew] when asked)."""
    B, H, Tnew, d = q.shape
    outs, lses = [], []
    for b in range(B):
        L = int(kv_lens[b])
        if L < Tnew:
            raise ValueError("each sequence must hold its new tokens")
        k = gather_pages(k_pages, page_table[b], L).unsqueeze(0).contiguous()
        v = gather_pages(v_pages, page_table[b], L).unsqueeze(0).contiguous()
        res = attention(q[b:b + 1].contiguous(), k, v, scale=scale, causal=True,
                        start_pos=L - Tnew, want_lse=want_lse)
        if want_lse:
            outs.append(res[0])
            lses.append(res[1])
        else:
            outs.append(res)
    out = np.concatenate(outs, axis=0)
    return (out, np.concatenate(lses, axis=0)) if want_lse else out
