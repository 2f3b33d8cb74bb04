"""The oracle pins catch plausible mistakes.

Each case plants one mistake in a private copy of the C oracle (compiled to a
temporary library on the CPU), swaps it in for the real oracle library, and
checks that at least one pin of tests/test_oracle_pins.py then fails. The real
oracle is never modified.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as oracle_build
from tests import test_oracle_pins as pins

# (name, original text, planted mistake, pins expected to notice)
MUTANTS = [
    ("sink scaled by 1/sqrt(d)",
     "exp(sink - m);", "exp(sink * scale - m);",
     [lambda: pins.test_zero_query_constant_value_closed_form(0),
      lambda: pins.test_sink_equals_virtual_zero_value_key(0)]),
    ("sink missing from the denominator",
     "double den = isinf(sink) && sink < 0 ? 0.0 : exp(sink - m);", "double den = 0.0;",
     [lambda: pins.test_sink_equals_virtual_zero_value_key(0),
      lambda: pins.test_window_one_closed_form()]),
    ("window admits one key too many",
     "int64_t lo = window > 0 ? (i - window + 1 > 0 ? i - window + 1 : 0) : 0;",
     "int64_t lo = window > 0 ? (i - window > 0 ? i - window : 0) : 0;",
     [lambda: pins.test_zero_query_constant_value_closed_form(4),
      lambda: pins.test_window_one_closed_form()]),
    ("rotation sign flipped",
     "y[k] = x1 * c - x2 * s;", "y[k] = x1 * c + x2 * s;",
     [pins.test_rope_unit_vectors_closed_form]),
    ("interleaved pairing instead of half-split",
     "double x1 = x[k], x2 = x[k + HALF];", "double x1 = x[2 * (k % 16) + (k / 16) * 32], "
     "x2 = x[2 * (k % 16) + 1 + (k / 16) * 32];",
     [pins.test_rope_unit_vectors_closed_form]),
    ("frequency exponent -k/d",
     "return pow(ROPE_THETA, -2.0 * (double)k / (double)D);",
     "return pow(ROPE_THETA, -1.0 * (double)k / (double)D);",
     [pins.test_rope_unit_vectors_closed_form]),
    ("kv head h % 8 instead of h / 8",
     "int h = g * GROUP + hh;\n            oracle_rope(q_rows",
     "int h = hh * NKV + g;\n            oracle_rope(q_rows",
     [lambda: pins.test_no_sink_no_rotation_equals_sdpa(0)]),
    ("scores not scaled",
     "s[j - lo] = dot * scale;", "s[j - lo] = dot;",
     [lambda: pins.test_no_sink_no_rotation_equals_sdpa(0), pins.test_window_one_closed_form]),
    ("causal bound excludes the query itself",
     "attend_row(qr, kr, vg, (int64_t)NKV * D, lo, i, sinks[h], s, out + (r * NQ + h) * D);",
     "attend_row(qr, kr, vg, (int64_t)NKV * D, lo, i - 1, sinks[h], s, out + (r * NQ + h) * D);",
     [pins.test_window_one_closed_form]),
]


def _build_mutant(src_text: str, tmpdir: str) -> str:
    c = os.path.join(tmpdir, "mutant.c")
    so = os.path.join(tmpdir, "libmutant.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", c, "-o", so,
                           "-lm"])
    return so


@pytest.mark.parametrize("name,orig,mutated,checks", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, orig, mutated, checks):
    src = open(oracle_build.SRC).read()
    assert src.count(orig) == 1, "mutation anchor not found: " + orig
    real = oracle._load()
    with tempfile.TemporaryDirectory() as tmp:
        lib = ctypes.CDLL(_build_mutant(src.replace(orig, mutated), tmp))
        for fn in ("oracle_rope_rows", "oracle_prefill", "oracle_prefill_rows", "oracle_decode"):
            getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        caught = []
        oracle._lib = lib
        try:
            for check in checks:
                try:
                    check()
                    caught.append(False)
                except AssertionError:
                    caught.append(True)
        finally:
            oracle._lib = real
    assert any(caught), "no pin noticed the planted mistake: %s" % name
