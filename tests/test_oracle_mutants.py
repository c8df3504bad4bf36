"""The oracle's pins catch plausible mistakes.

Each case compiles a copy of ``oracle/attn_oracle.c`` with one deliberate
mistake planted in it (on the CPU, into a temporary directory) and runs every
pin of ``test_oracle_pins.py``, ``test_oracle_rope_pins.py`` and
``test_oracle_window_pins.py`` against that
copy: at least one pin must fail.
The unmodified oracle passes all of them (that file's own run).
"""
import inspect
import os
import subprocess

import pytest

import test_oracle_pins as pins
import test_oracle_rope_pins as rope_pins
import test_oracle_window_pins as window_pins
from oracle.attention import load_variant

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "attn_oracle.c")

# (name, [(exact text in attn_oracle.c, replacement), ...])
MUTANTS = [
    ("scale dropped", [("s[j] = J->scale * dot;", "s[j] = dot;")]),
    ("mask includes diagonal off by one", [("if (J->causal && j > p) return 0;",
                                           "if (J->causal && j >= p) return 0;")]),
    ("mask one position too wide", [("if (J->causal && j > p) return 0;",
                                     "if (J->causal && j > p + 1) return 0;")]),
    ("window one key too wide", [("j <= p - J->window) return 0;", "j < p - J->window) return 0;")]),
    ("window ignored", [("if (J->window > 0 && j <= p - J->window) return 0;", "")]),
    ("GQA head taken modulo", [("int64_t kvh = h / g;", "int64_t kvh = h % J->Hkv;")]),
    ("start_pos ignored", [("int64_t p = J->start_pos + i;", "int64_t p = i;")]),
    ("exponent sign flipped", [("w[j] = exp(s[j] - M);", "w[j] = exp(M - s[j]);")]),
    ("weights not normalised", [("double pj = w[j] / L;", "double pj = w[j];")]),
    ("keys read as values", [("o[t] += pj * load_elem(J->v,", "o[t] += pj * load_elem(J->k,")]),
    ("queries read as keys", [("load_elem(J->k, J->dtype, (kv_base + j) * d + t);",
                               "load_elem(J->q, J->dtype, q_off + t);")]),
    ("lse without the max", [("J->lse[slot] = M + log(L);", "J->lse[slot] = log(L);")]),
    ("bf16 widened with a wrong shift", [("(uint32_t)bits << 16", "(uint32_t)bits << 15")]),
    ("f16 exponent bias off by one", [("e - 25);", "e - 24);")]),
    ("f16 subnormals scaled wrongly", [("ldexp((double)frac, -24)", "ldexp((double)frac, -25)")]),
    ("batch stride ignored for K/V", [("int64_t kv_base = (b * J->Hkv + kvh) * J->S_cap;",
                                       "int64_t kv_base = kvh * J->S_cap;")]),
    ("RoPE partner adjacent", [("load_elem(k_new, dtype, row + i + h);",
                                "load_elem(k_new, dtype, row + (i ^ 1));")]),
    ("RoPE rotation reversed", [("k_out[row + i] = x0 * cos(a) - x1 * sin(a);",
                                 "k_out[row + i] = x0 * cos(a) + x1 * sin(a);"),
                                ("k_out[row + i + h] = x1 * cos(a) + x0 * sin(a);",
                                 "k_out[row + i + h] = x1 * cos(a) - x0 * sin(a);")]),
    ("RoPE frequency exponent halved", [("pow(base, -2.0 * (double)i / (double)d)",
                                         "pow(base, -1.0 * (double)i / (double)d)")]),
    ("RoPE position ignores start_pos", [("const double pos = (double)(start_pos + t);",
                                          "const double pos = (double)t;")]),
]


def _pin_calls(golden_dir):
    """Every test function of the pin modules, with its parameter sets."""
    calls = []
    members = inspect.getmembers(pins, inspect.isfunction) + \
        inspect.getmembers(rope_pins, inspect.isfunction) + \
        inspect.getmembers(window_pins, inspect.isfunction)
    for name, fn in members:
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        sig = inspect.signature(fn).parameters
        if params:
            m = params[0]
            argnames = [a.strip() for a in m.args[0].split(",")]
            for values in m.args[1]:
                values = values if isinstance(values, (tuple, list)) else (values,)
                calls.append((name, fn, dict(zip(argnames, values))))
        elif "golden_dir" in sig:
            calls.append((name, fn, {"golden_dir": golden_dir}))
        else:
            calls.append((name, fn, {}))
    return calls


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, edits, tmp_path, golden_dir, monkeypatch):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-shared", "-fPIC", "-pthread",
                    str(path), "-o", str(lib), "-lm"], check=True)
    variant = load_variant(str(lib))
    monkeypatch.setattr(pins, "attention", variant.attention)
    monkeypatch.setattr(pins, "widen_bits", variant.widen_bits)
    monkeypatch.setattr(rope_pins, "rope_append", variant.rope_append)
    monkeypatch.setattr(window_pins, "attention", variant.attention)
    failed = []
    for test_name, fn, kwargs in _pin_calls(golden_dir):
        try:
            fn(**kwargs)
        except Exception:  # noqa: BLE001 - any failure counts
            failed.append(test_name)
    assert failed, f"no pin caught the planted mistake: {name}"
