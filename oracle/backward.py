"""fp64 gradients of full-sequence causal attention (the backward pass).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What it computes ("Causal Multi-Head Self-Attention", Two exact
full-sequence algorithms; Causal mask): for the context O = softmax(S) V of
every head, S = scale * Q K^T with the causal (and optional local-window) mask,
and an upstream gradient dO of the context, the vector-Jacobian product gives
dQ, dK and dV.  The pages fix two facts used here: a context upstream produces
query, key and value gradients, and a masked (future) score carries exactly
zero gradient.  The Flash backward there recomputes each probability from Q, K
and saved row statistics; the oracle instead materialises the full
probability matrix with a plain two-pass softmax, which is the same real
number, and applies the softmax Jacobian by its definition:

    P      = softmax over the visible keys of each row (0 on masked keys)
    dV     = P^T dO
    dP     = dO V^T
    dS_ij  = P_ij (dP_ij - sum_k P_ik dP_ik)      (J^T g of the softmax row)
    dQ     = scale * dS K
    dK     = scale * dS^T Q

Grouped-query attention ("Grouped-Query Attention" §5.1): query head h reads
K/V head h // G, so dK and dV of a K/V head are the sums over its G query
heads.  Inputs are widened exactly to float64 (bf16/f16/f32 -> f64 is exact);
every step is float64 numpy.  Parity pinned by centered finite differences of
the C oracle's forward, by fp64 autograd of a materialised forward, by closed
forms and by invariants (tests/test_oracle_backward_pins.py).
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def visible_mask(T: int, causal: bool, window: int = 0) -> np.ndarray:
    """[T, T] boolean: row i may read key j (j <= i when causal; with a local
    window w > 0 also j > i - w)."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = np.ones((T, T), dtype=bool)
    if causal:
        vis &= j <= i
    if window > 0:
        vis &= j > i - window
    return vis


def probabilities(q_bh: np.ndarray, k_bh: np.ndarray, scale: float, vis: np.ndarray) -> np.ndarray:
    """Row softmax of scale * q k^T over the visible keys, two passes
    (maximum, then exponentials and their sum); exactly 0 on masked keys."""
    s = scale * (q_bh @ k_bh.T)
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    w = np.where(vis, np.exp(s - m), 0.0)
    return w / w.sum(axis=1, keepdims=True)


def attention_backward(q, k, v, dout, *, scale: float, causal: bool = True, window: int = 0):
    """fp64 (dq, dk, dv) for q, dout [B, H, T, d] and k, v [B, Hkv, T, d].

    Returns float64 arrays of the input shapes; dk and dv are summed over the
    query heads that share each K/V head."""
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(dout)
    if Q.ndim != 4 or K.shape != V.shape or dO.shape != Q.shape:
        raise ValueError("expected q, dout [B,H,T,d] and k, v [B,Hkv,T,d]")
    B, H, T, d = Q.shape
    Hkv = K.shape[1]
    if K.shape[0] != B or K.shape[2] != T or K.shape[3] != d or Hkv == 0 or H % Hkv:
        raise ValueError("k, v must be [B, Hkv, T, d] with Hkv dividing H")
    G = H // Hkv
    vis = visible_mask(T, causal, window)
    dq = np.zeros_like(Q)
    dk = np.zeros_like(K)
    dv = np.zeros_like(V)
    for b in range(B):
        for h in range(H):
            kvh = h // G
            P = probabilities(Q[b, h], K[b, kvh], scale, vis)
            dP = dO[b, h] @ V[b, kvh].T
            rho = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - rho)
            dq[b, h] = scale * (dS @ K[b, kvh])
            dk[b, kvh] += scale * (dS.T @ Q[b, h])
            dv[b, kvh] += P.T @ dO[b, h]
    return dq, dk, dv
