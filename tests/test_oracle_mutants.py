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
     "int h = g * GROUP + hh;\n            rotate(q_rows",
     "int h = hh * NKV + g;\n            rotate(q_rows",
     [lambda: pins.test_no_sink_no_rotation_equals_sdpa(0)]),
    ("scores not scaled",
     "s[j - lo] = dot * scale;", "s[j - lo] = dot;",
     [lambda: pins.test_no_sink_no_rotation_equals_sdpa(0), pins.test_window_one_closed_form]),
    ("YaRN blend weights swapped (interpolate the high frequencies)",
     "f[k] = inv_freq(k) / factor * ramp + inv_freq(k) * (1.0 - ramp);",
     "f[k] = inv_freq(k) / factor * (1.0 - ramp) + inv_freq(k) * ramp;",
     [pins.test_yarn_bands_and_attention_factor]),
    ("YaRN attention factor left out",
     "const double mscale = factor <= 1.0 ? 1.0 : 0.1 * log(factor) + 1.0;",
     "const double mscale = 1.0;",
     [pins.test_yarn_bands_and_attention_factor,
      pins.test_yarn_attention_scales_logits_by_mscale_squared]),
    ("YaRN correction pairs swapped between the betas",
     "double lo = yarn_pair_for_turns(beta_fast, original);",
     "double lo = yarn_pair_for_turns(beta_slow * 2.0, original);",
     [pins.test_yarn_ramp_is_linear_in_the_pair_index]),
    ("YaRN frequency ramp over turns instead of pair index",
     "double ramp = ((double)k - lo) / (hi - lo);",
     "double ramp = (original * inv_freq(k) / TWO_PI - beta_fast) / (beta_slow - beta_fast);",
     [pins.test_yarn_ramp_is_linear_in_the_pair_index]),
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
        for fn in ("oracle_rope_rows", "oracle_rope_yarn", "oracle_prefill", "oracle_prefill_rows",
                   "oracle_decode"):
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
