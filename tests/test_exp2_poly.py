"""The FMA-pipe exp2 of the prefill kernel against its error bound (CPU).

The kernel's constants must be the ones gen_exp2_poly.py fits, and the
algorithm evaluated step by step in float32 must stay within 1.1e-4 relative
of 2^x over [-126, 16] and be exact at integers (p(0) = 1)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "transformer_attention_causal_b200", "csrc")


def load_gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly",
                                                  os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def kernel_coefficients():
    text = open(os.path.join(CSRC, "prefill_tcgen05.cuh")).read()
    vals = {k: float(v) for k, v in re.findall(r"(kC[123])\s*=\s*([0-9.eE+-]+)f", text)}
    return np.array([1.0, vals["kC1"], vals["kC2"], vals["kC3"]], dtype=np.float32)


def test_kernel_uses_the_fitted_coefficients():
    gen = load_gen()
    np.testing.assert_allclose(kernel_coefficients(), gen.fit(3), rtol=1e-7)


def test_error_bound_over_the_softmax_range():
    gen = load_gen()
    assert gen.max_rel_error(kernel_coefficients()) <= 1.1e-4


def test_exact_at_integers_and_clamped_below():
    gen = load_gen()
    c = kernel_coefficients()
    ints = np.arange(-126, 17, dtype=np.float32)
    np.testing.assert_array_equal(gen.eval_f32(c, ints), np.exp2(ints.astype(np.float64)))
    assert gen.eval_f32(c, np.array([-300.0], dtype=np.float32))[0] == np.float32(2.0 ** -126)
