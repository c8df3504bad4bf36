"""Coefficients of the FMA-pipe exp2 used for part of the softmax exponentials.

    python transformer_attention_causal_b200/csrc/gen_exp2_poly.py

Method (a standard range reduction, coefficients fitted here):
  2^x = 2^j * 2^f,  j = round-to-nearest(x),  f = x - j in [-1/2, 1/2].
  j is obtained by adding 1.5 * 2^23 in float32 (the sum's low mantissa bits
  then hold j) and subtracting it again; 2^j is applied by adding j << 23 to
  the bit pattern of p(f).
  p is a degree-N polynomial fitted to 2^f on [-1/2, 1/2] by weighted least
  squares on Chebyshev nodes, weights 1/2^f (so the fit minimises relative
  error), followed by a few Lawson reweighting passes toward the minimax
  (equal-ripple) solution; the constant term is then fixed to 1 exactly so
  that p(0) = 1 and 2^j is exact for integer x.

The script prints the coefficients (float32, as C literals) and the maximum
relative error of the float32 Horner evaluation against 2^x in float64.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int, nodes: int = 4000, lawson: int = 60):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    # p(f) = 1 + f * q(f): fit q so that the constant term is exactly 1
    A = np.stack([f ** (i + 1) for i in range(degree)], axis=1)
    rhs = target - 1.0
    w = 1.0 / target                                       # relative error
    lw = np.ones_like(f)
    for _ in range(lawson):
        sw = np.sqrt(w * w * lw)
        c, *_ = np.linalg.lstsq(A * sw[:, None], rhs * sw, rcond=None)
        err = np.abs((A @ c - rhs) * w)
        lw = lw * (err + 1e-30)
        lw /= lw.sum()
    return np.concatenate([[1.0], c]).astype(np.float32)


def eval_f32(coef: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The device algorithm, step by step in float32."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)                           # 1.5 * 2^23
    t = (x + big).astype(np.float32)
    j = (t - big).astype(np.float32)
    fr = (x - j).astype(np.float32)
    p = np.float32(coef[-1])
    for c in coef[-2::-1]:
        p = (p * fr + np.float32(c)).astype(np.float32)    # one rounding per step, like FFMA
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def max_rel_error(coef, lo=-126.0, hi=16.0, n=2_000_001):
    x = np.linspace(lo, hi, n, dtype=np.float64).astype(np.float32)
    got = eval_f32(coef, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got - ref) / ref))


if __name__ == "__main__":
    for deg in (3, 4):
        c = fit(deg)
        print(f"degree {deg}: " + ", ".join(f"{v:.9e}f" for v in c),
              f" max rel err {max_rel_error(c):.3e}")
