"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no attention arithmetic: it only draws i.i.d. N(0, 1)
numbers and rounds them to the requested dtype.

Recipe.  A tensor of shape [B, Hx, L, d] is filled one (b, hx) slice at a time.
Slice (b, hx) of stream ``stream`` (0 = Q, 1 = K, 2 = V, 3 = the upstream
gradient dO of the backward pass, others free) is
``torch.randn((L, d), generator=torch.Generator().manual_seed(slice_seed))`` in
float32, then cast to the dtype with round-to-nearest-even, where
``slice_seed = splitmix64(seed, stream, b, hx) >> 1``.  Because every slice
has its own seed, any slice can be regenerated alone (the oracle checks sampled
rows of full-size workloads that way) and slices can be drawn in parallel.

splitmix64 is the finaliser published by Steele, Lea and Flood ("Fast
splittable pseudorandom number generators", 2014), applied to a 64-bit key
folded from (seed, stream, b, hx).
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import torch

_MASK = (1 << 64) - 1
Q_STREAM, K_STREAM, V_STREAM, DO_STREAM = 0, 1, 2, 3


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK
    return x ^ (x >> 31)


def slice_seed(seed: int, stream: int, b: int, hx: int) -> int:
    key = _splitmix64(seed & _MASK)
    key = _splitmix64(key ^ (stream & 0xFFFF))
    key = _splitmix64(key ^ ((b & 0xFFFFFFFF) << 16))
    key = _splitmix64(key ^ ((hx & 0xFFFFFFFF) << 8))
    return key >> 1


def normal_slice(seed: int, stream: int, b: int, hx: int, L: int, d: int,
                 dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(slice_seed(seed, stream, b, hx))
    return torch.randn((L, d), generator=g, dtype=torch.float32).to(dtype)


def normal(shape, seed: int, stream: int, dtype: torch.dtype, workers: int = 8) -> torch.Tensor:
    """[B, Hx, L, d] tensor on the CPU, filled slice by slice as described above."""
    B, Hx, L, d = (int(s) for s in shape)
    out = torch.empty((B, Hx, L, d), dtype=dtype)

    def fill(idx: int) -> None:
        b, hx = divmod(idx, Hx)
        out[b, hx].copy_(normal_slice(seed, stream, b, hx, L, d, dtype))

    n = B * Hx
    if n <= 1 or workers <= 1:
        for idx in range(n):
            fill(idx)
    else:
        with ThreadPoolExecutor(max_workers=workers) as pool:
            list(pool.map(fill, range(n)))
    return out


def qkv(B: int, H: int, Hkv: int, Tq: int, S: int, d: int, dtype: torch.dtype,
        seed: int = 0, S_cap: int | None = None):
    """Q [B, H, Tq, d] and K, V [B, Hkv, S_cap, d] (first S rows drawn; rows
    S..S_cap-1, if any, are zero) on the CPU."""
    q = normal((B, H, Tq, d), seed, Q_STREAM, dtype)
    k = normal((B, Hkv, S, d), seed, K_STREAM, dtype)
    v = normal((B, Hkv, S, d), seed, V_STREAM, dtype)
    if S_cap is not None and S_cap > S:
        pad = torch.zeros((B, Hkv, S_cap - S, d), dtype=dtype)
        k = torch.cat([k, pad], dim=2)
        v = torch.cat([v, pad], dim=2)
    return q, k, v


def upstream(B: int, H: int, T: int, d: int, dtype: torch.dtype, seed: int = 0) -> torch.Tensor:
    """dO [B, H, T, d] on the CPU: the gradient fed into the backward pass."""
    return normal((B, H, T, d), seed, DO_STREAM, dtype)
