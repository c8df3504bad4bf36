"""The backward pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/backward.py`` (a text
substitution, executed on the CPU as a separate module) and runs every pin of
``test_oracle_backward_pins.py`` against the copy: at least one must fail.
"""
import inspect
import os

import pytest

import test_oracle_backward_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "backward.py")

MUTANTS = [
    ("softmax Jacobian without the row term", [("dS = P * (dP - rho)", "dS = P * dP")]),
    ("softmax Jacobian sign flipped", [("dS = P * (dP - rho)", "dS = P * (rho - dP)")]),
    ("row term summed over the wrong axis", [("rho = (P * dP).sum(axis=1,", "rho = (P * dP).sum(axis=0,")]),
    ("dQ without the scale", [("dq[b, h] = scale * (dS @ K[b, kvh])", "dq[b, h] = dS @ K[b, kvh]")]),
    ("dK from P instead of dS", [("dk[b, kvh] += scale * (dS.T @ Q[b, h])",
                                  "dk[b, kvh] += scale * (P.T @ Q[b, h])")]),
    ("dV with P untransposed", [("dv[b, kvh] += P.T @ dO[b, h]", "dv[b, kvh] += P @ dO[b, h]")]),
    ("dP from keys instead of values", [("dP = dO[b, h] @ V[b, kvh].T", "dP = dO[b, h] @ K[b, kvh].T")]),
    ("GQA heads overwrite instead of summing", [("dk[b, kvh] += ", "dk[b, kvh] = "),
                                                ("dv[b, kvh] += ", "dv[b, kvh] = ")]),
    ("K/V head taken modulo", [("kvh = h // G", "kvh = h % Hkv")]),
    ("mask admits the next key", [("vis &= j <= i", "vis &= j <= i + 1")]),
    ("window one key too wide", [("vis &= j > i - window", "vis &= j >= i - window")]),
    ("probabilities not normalised", [("return w / w.sum(axis=1, keepdims=True)", "return w")]),
    ("scores without the scale", [("s = scale * (q_bh @ k_bh.T)", "s = q_bh @ k_bh.T")]),
]


def _variant(subs):
    src = open(SRC).read()
    for old, new in subs:
        assert old in src, f"mutant anchor not found: {old!r}"
        src = src.replace(old, new)
    ns = {"__name__": "oracle_backward_mutant"}
    exec(compile(src, "oracle_backward_mutant", "exec"), ns)
    return ns["attention_backward"]


def _pin_calls():
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            yield name, fn, {}
            continue
        argnames = [a.strip() for a in params[0].args[0].split(",")]
        for values in params[0].args[1]:
            values = values if len(argnames) > 1 else (values,)
            yield name, fn, dict(zip(argnames, values))


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_pin_fails_on_the_mutant(mutant):
    _, subs = mutant
    bwd = _variant(subs)
    for name, fn, kw in _pin_calls():
        try:
            fn(bwd=bwd, **kw)
        except Exception:   # noqa: BLE001 (an assertion or a shape error both expose it)
            return
    pytest.fail("no backward pin failed on the planted mistake")


def test_the_unmodified_copy_passes_every_pin():
    bwd = _variant([])
    for _, fn, kw in _pin_calls():
        fn(bwd=bwd, **kw)
