"""The CPU oracle against hand-derived examples, brute force, library routines and
the invariants of the method; plus planted mistakes that the pins must catch.

Each planted mistake is a textual edit of a temporary copy of oracle/oracle.c,
built on the CPU; the real oracle source is never modified.  Mistakes in the
Python composition of the FFN step (up-projection, GELU, the next linear's codes)
are planted by overriding that one method on a separate oracle instance.
"""
import os
import tempfile
import types

import pytest

import oracle as oracle_pkg
from oracle import Oracle
from oracle import build as oracle_build

import oracle_pins as P


@pytest.mark.parametrize("check", P.GOLDEN_CHECKS, ids=lambda c: c.__name__)
def test_golden(oracle, golden, check):
    assert check(oracle, golden) == []


@pytest.mark.parametrize("check", [c for c in P.ALL_CHECKS if c not in P.GOLDEN_CHECKS],
                         ids=lambda c: c.__name__)
def test_property(oracle, check):
    assert check(oracle) == []


# (description, [(text in oracle.c, replacement), ...])
MUTANTS = [
    ("reciprocal multiply instead of division",
     [("float t = v / s;", "float t = v * (1.0f / s);")]),
    ("round half away from zero", [("float r = rintf(t);", "float r = roundf(t);")]),
    ("no clamp at +qmax", [("if (r > qmax) r = qmax;", "")]),
    ("channel scale not folded into activations",
     [("xp[k] = oracle_bf16_to_float(x[(size_t)m * K + k]) * ck;",
       "xp[k] = oracle_bf16_to_float(x[(size_t)m * K + k]);")]),
    ("clip ratio ignored", [("float clip = alpha[(size_t)step * S + sid] * amax;",
                             "float clip = amax;")]),
    ("clip table indexed [stream][step]",
     [("float clip = alpha[(size_t)step * S + sid] * amax;",
       "float clip = alpha[(size_t)sid * T + step] * amax;")]),
    ("signed maximum instead of absolute", [("      float a = fabsf(xp[k]);", "      float a = xp[k];")]),
    ("weight qmax 8", [("const float qmax = 7.0f;", "const float qmax = 8.0f;")]),
    ("high nibble holds the even k (pack and unpack)",
     [("return (uint8_t)(((unsigned)lo & 0xFu) | (((unsigned)hi & 0xFu) << 4));",
       "return (uint8_t)(((unsigned)hi & 0xFu) | (((unsigned)lo & 0xFu) << 4));"),
      ("int v = high ? (byte >> 4) & 0xF : byte & 0xF;",
       "int v = high ? byte & 0xF : (byte >> 4) & 0xF;")]),
    ("nibble sign extension wrong", [("return v >= 8 ? v - 16 : v;", "return v >= 8 ? 16 - v : v;")]),
    ("weight nibble off by one",
     [("int w = unpack_nibble(qw[(size_t)n * (K / 2) + k / 2], k & 1);",
       "int w = unpack_nibble(qw[(size_t)n * (K / 2) + k / 2], (k + 1) & 1);")]),
    ("bias dropped", [("if (bias) v += (double)bias[n];", "")]),
    ("output compensation indexed [stream][step]",
     [("if (beta) v += (double)beta[((size_t)step * S + sid) * N + n];",
       "if (beta) v += (double)beta[((size_t)sid * T + step) * N + n];")]),
    ("accumulator transposed",
     [("(double)acc[(size_t)m * N + n];", "(double)acc[(size_t)n * M + m];")]),
    ("token and channel scales swapped",
     [("double v = (double)s_tok[m] * (double)s_w[n]", "double v = (double)s_tok[n] * (double)s_w[m]")]),
    ("bf16 rounding half away from zero",
     [("double r = nearbyint(ldexp(a, 8 - e));", "double r = round(ldexp(a, 8 - e));")]),
    ("channel scale inverted", [("if (a > 0.0f && b > 0.0f) ck = sqrtf(a / b);",
                                 "if (a > 0.0f && b > 0.0f) ck = sqrtf(b / a);")]),
    ("static path: channel scale not folded into activations",
     [("xp[k] = ck * oracle_bf16_to_float(x[(size_t)m * K + k]);",
       "xp[k] = oracle_bf16_to_float(x[(size_t)m * K + k]);")]),
    ("static clip multiplies by the gain",
     [("float clip = g > 0.0f ? thr[step] / g : 0.0f;",
       "float clip = g > 0.0f ? thr[step] * g : 0.0f;")]),
    ("static gain table indexed [stream][step]",
     [("float g = gain[(size_t)step * S + sid];", "float g = gain[(size_t)sid * T + step];")]),
    ("static threshold of step 0 for every step",
     [("float clip = g > 0.0f ? thr[step] / g : 0.0f;",
       "float clip = g > 0.0f ? thr[0] / g : 0.0f;")]),
    ("GELU distribution function at the wrong scale",
     [("erfc(-v / sqrt(2.0))", "erfc(-v / 2.0)")]),
    ("GELU with the upper tail 1 - Phi", [("erfc(-v / sqrt(2.0))", "erfc(v / sqrt(2.0))")]),
    ("GELU without the one half", [("v * 0.5 * erfc", "v * erfc")]),
    ("GELU as v * erf without the leading one",
     [("return v * 0.5 * erfc(-v / sqrt(2.0));", "return v * 0.5 * erf(v / sqrt(2.0));")]),
    ("GELU skipped before the bf16 rounding",
     [("h[i] = oracle_double_to_bf16(oracle_gelu(a));", "h[i] = oracle_double_to_bf16(a);")]),
    ("no clamp at -qmax", [("if (r < -qmax) r = -qmax;", "")]),
    ("zero scale divides by zero", [("if (s == 0.0f) return 0;", "")]),
    ("activation scale divided by 2^(b-1) instead of qmax",
     [("float clip = alpha[(size_t)step * S + sid] * amax;\n    float s = clip / qmax;",
       "float clip = alpha[(size_t)step * S + sid] * amax;\n    float s = clip / (qmax + 1.0f);")]),
    ("clip ratio of stream 0 for every row",
     [("float clip = alpha[(size_t)step * S + sid] * amax;",
       "float clip = alpha[(size_t)step * S] * amax;")]),
    ("x' rounded to bf16 before quantization",
     [("xp[k] = oracle_bf16_to_float(x[(size_t)m * K + k]) * ck;",
       "xp[k] = oracle_bf16_to_float(oracle_double_to_bf16("
       "oracle_bf16_to_float(x[(size_t)m * K + k]) * ck));")]),
    ("static scale without the division by qmax",
     [("float clip = g > 0.0f ? thr[step] / g : 0.0f;\n    float s = clip / qmax;",
       "float clip = g > 0.0f ? thr[step] / g : 0.0f;\n    float s = clip;")]),
    ("weight scale from the signed maximum",
     [("      float a = fabsf(wp[k]);", "      float a = wp[k];")]),
    ("GEMM drops the last k",
     [("for (int k = 0; k < K; ++k) {\n        int w = unpack_nibble",
       "for (int k = 0; k < K - 1; ++k) {\n        int w = unpack_nibble")]),
    ("compensation of stream 0 for every row",
     [("if (beta) v += (double)beta[((size_t)step * S + sid) * N + n];",
       "if (beta) v += (double)beta[((size_t)step * S) * N + n];")]),
    ("4-bit activation codes always from the low nibble",
     [("  return unpack_nibble(b, k & 1);", "  return unpack_nibble(b, 0);")]),
    ("bf16 rounding truncates", [("double r = nearbyint(ldexp(a, 8 - e));",
                                 "double r = trunc(ldexp(a, 8 - e));")]),
    ("channel scale without the square root",
     [("if (a > 0.0f && b > 0.0f) ck = sqrtf(a / b);", "if (a > 0.0f && b > 0.0f) ck = a / b;")]),
    ("cinv equal to c", [("cinv[k] = 1.0f / ck;", "cinv[k] = ck;")]),
    ("scale as alpha * (amax / qmax)",
     [("float clip = alpha[(size_t)step * S + sid] * amax;\n    float s = clip / qmax;",
       "float clip = alpha[(size_t)step * S + sid] * amax;\n"
       "    float s = alpha[(size_t)step * S + sid] * (amax / qmax);")]),
    ("static: a non-positive gain keeps the threshold",
     [("float clip = g > 0.0f ? thr[step] / g : 0.0f;",
       "float clip = g > 0.0f ? thr[step] / g : thr[step];")]),
]


@pytest.fixture(scope="module")
def mutant_dir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("desc,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(golden, mutant_dir, desc, edits):
    src = open(oracle_build.SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"edit site not unique or missing: {old!r}"
        src = src.replace(old, new)
    tag = "".join(ch if ch.isalnum() else "_" for ch in desc)
    c_path = os.path.join(mutant_dir, f"{tag}.c")
    with open(c_path, "w") as f:
        f.write(src)
    # the mutant includes "oracle.h" from the real source directory
    so = oracle_build.build(c_path, os.path.join(mutant_dir, f"{tag}.so"),
                            extra=("-I", os.path.dirname(oracle_build.SRC)))
    mutant = Oracle(oracle_pkg.load(so))
    fails = P.all_failures(mutant, golden)
    assert fails, f"planted mistake '{desc}' passed every pin"


# Mistakes in composing the FFN step: each replaces Oracle.linear_gelu_quant_static
# on one instance with a wrong composition of the oracle's own (correct) parts.
def _codes_of_y(o, x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias, cinv_n, thr_n,
                gain_n, bits_n):
    y = o.linear(x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias)[0]
    codes, s = o.act_quant_static(y, cinv_n, sid, thr_n, gain_n, step, bits_n)
    return codes, s, o.gelu_bf16(y), y


def _next_channel_scale_dropped(o, x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias,
                                cinv_n, thr_n, gain_n, bits_n):
    y = o.linear(x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias)[0]
    h = o.gelu_bf16(y)
    codes, s = o.act_quant_static(h, None, sid, thr_n, gain_n, step, bits_n)
    return codes, s, h, y


def _next_codes_4_bit(o, x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias, cinv_n,
                      thr_n, gain_n, bits_n):
    y = o.linear(x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias)[0]
    h = o.gelu_bf16(y)
    codes, s = o.act_quant_static(h, cinv_n, sid, thr_n, gain_n, step, 4)
    return codes, s, h, y


@pytest.mark.parametrize("wrong", [_codes_of_y, _next_channel_scale_dropped, _next_codes_4_bit],
                         ids=lambda f: f.__name__.strip("_"))
def test_planted_composition_mistake_is_caught(golden, wrong):
    mutant = Oracle()
    mutant.linear_gelu_quant_static = types.MethodType(wrong, mutant)
    assert P.all_failures(mutant, golden), f"{wrong.__name__} passed every pin"
