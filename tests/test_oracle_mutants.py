"""The oracle's pins catch plausible mistakes (CPU).

Each case copies oracle/fp8_oracle.c, plants one mistake of the kind a
restatement of the definition could make (a wrong tie rule, a dropped sign, a
transposed index, a missing term), builds the copy and runs every pin of
tests/test_oracle.py against it.  At least one pin must fail.  An unmodified
copy must pass all of them, so that a failure means the pins noticed the
mistake, not that the harness is broken.  Every planted mistake keeps all
memory accesses inside their arrays.
"""
import inspect
import os
import re
import sys

import pytest

import oracle

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import test_oracle  # noqa: E402

SRC = os.path.join(os.path.dirname(oracle.__file__), "fp8_oracle.c")

# (what the mistake is, pattern, replacement, None for a plain text
# replacement of every occurrence or the count of a regex substitution, 0 = all)
MUTANTS = [
    ("encode: ties away from zero",
     "n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "n = fl + 1.0;", None),
    ("encode: ties toward zero",
     "n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "n = fl;", None),
    ("encode: saturates to the NaN code",
     "return sign | 0x7E;", "return sign | 0x7F;", None),
    ("encode: a negative value rounding to zero loses its sign",
     "if (r == 0.0)\n        return sign;", "if (r == 0.0)\n        return 0x00;", None),
    ("encode: subnormal spacing one binade too fine",
     "quantum = ldexp(1.0, -9);", "quantum = ldexp(1.0, -10);", None),
    ("encode: normal spacing one binade too coarse",
     "quantum = ldexp(1.0, (e - 1) - 3);", "quantum = ldexp(1.0, (e - 1) - 2);", None),
    ("decode: exponent bias 8",
     "mag = ldexp(1.0 + (double)m / 8.0, e - 7);", "mag = ldexp(1.0 + (double)m / 8.0, e - 8);", None),
    ("decode: subnormals read as normals",
     "mag = ldexp((double)m, -9);", "mag = ldexp(1.0 + (double)m / 8.0, -7);", None),
    ("scale: amax times the rounded reciprocal of 448",
     "volatile float s = amax / 448.0f;", "volatile float s = amax * (1.0f / 448.0f);", None),
    ("code: x times the rounded reciprocal of s",
     "volatile float ratio = x / s;", "volatile float ratio = x * (1.0f / s);", None),
    ("amax: signed maximum instead of the largest magnitude",
     r"if \(fabsf\(v\) > amax\)\s*amax = fabsf\(v\);", "if (v > amax) amax = v;", 0),
    ("row-wise scales stored [rows, cols/128]",
     "s[g * rows + r] = sc;", "s[r * groups + g] = sc;", None),
    ("column-wise codes written untransposed",
     "qT[c * rows + r] =", "qT[r * cols + c] =", None),
    ("weight scales stored transposed",
     "s[nb * kb_count + kb] = sc;", "s[kb * nb_count + nb] = sc;", None),
    ("weight amax over the block's first row only",
     r"for \(int i = 0; i < GROUP; \+\+i\)(\s*)for \(int j = 0; j < GROUP; \+\+j\) \{(\s*)float v",
     r"for (int i = 0; i < 1; ++i)\1for (int j = 0; j < GROUP; ++j) {\2float v", 1),
    ("slab sum drops its last product",
     "k < (t + 1) * GROUP; ++k", "k < (t + 1) * GROUP - 1; ++k", None),
    ("bound: signed instead of absolute sum",
     "abs_acc += fabs(c) * p_abs;", "abs_acc += c * p;", None),
    ("promotion: the first slab's scales for every slab",
     "double c = (double)sa[t * sa_stride] * (double)sb[t * sb_stride];",
     "double c = (double)sa[0] * (double)sb[0];", None),
    ("fprop: activation scales read as [M, K/128]",
     "sx + m, M,", "sx + m * kb_count, 1,", None),
    ("dgrad: weight codes read untransposed",
     "wt[k * N + n] = orc_e4m3_decode(wq[n * K + k]);",
     "wt[k * N + n] = orc_e4m3_decode(wq[k * N + n]);", None),
    ("dgrad: weight scale read as [K/128, N/128]",
     "sw + k / GROUP,\n                         kb_count,",
     "sw + (k / GROUP) * (N / GROUP),\n                         1,", None),
    ("wgrad: both outer-product scales from dY",
     "sdyT + n, N, sxT + k, K,", "sdyT + n, N, sdyT + n, N,", None),
    ("bf16 rounding: ties away from zero",
     "up = fmod(below, 2.0) == 1.0;", "up = 1;", None),
    ("bf16 rounding: the side of a midpoint ignored",
     "up = (lo > 0.0) == (hi > 0.0);", "up = fmod(below, 2.0) == 1.0;", None),
    ("bf16 rounding: no subnormal spacing",
     "int lead = ex - 1 < -126 ? -126 : ex - 1;", "int lead = ex - 1;", None),
    ("silu: the double quotient for every g (no small-g series)",
     "if (fabs(g) < 0x1p-30)\n        return bf16_round_split(g / 2.0, g * g / 4.0);\n", "", None),
    ("silu: e^g instead of e^-g",
     "return orc_bf16_from_double(g / (1.0 + exp(-g)));", "return orc_bf16_from_double(g / (1.0 + exp(g)));", None),
    ("swiglu: gate and up swapped",
     "double s = (double)orc_bf16_to_float(orc_silu_bf16(gate[j]));\n            h[r * ffn + j] = orc_bf16_from_double(s * (double)uf);",
     "double s = (double)orc_bf16_to_float(orc_silu_bf16(up[j]));\n            h[r * ffn + j] = orc_bf16_from_double(s * (double)gf);", None),
    ("swiglu: silu not rounded to bfloat16 before the product",
     "double s = (double)orc_bf16_to_float(orc_silu_bf16(gate[j]));",
     "double s = (double)gf / (1.0 + exp(-(double)gf));", None),
    ("main-gradient accumulation drops the running value",
     "dw_out[i * K + k] = v + dw_out[i * K + k];", "dw_out[i * K + k] = 0.0 * v + dw_out[i * K + k];", None),
    ("main-gradient accumulation reads the running value of output position i, not row n",
     "double v = dw_in[n * K + k];", "double v = dw_in[i * K + k];", None),
    ("main-gradient accumulation subtracts the product",
     "dw_out[i * K + k] = v + dw_out[i * K + k];", "dw_out[i * K + k] = v - dw_out[i * K + k];", None),
    ("rmsnorm: mean over cols - 1",
     "double ms = sum / (double)cols + (double)eps;", "double ms = sum / (double)(cols - 1) + (double)eps;", None),
    ("rmsnorm: eps left out",
     "double ms = sum / (double)cols + (double)eps;", "double ms = sum / (double)cols;", None),
    ("rmsnorm: r from float32 square root and division",
     "r[i] = (float)(1.0 / sqrt(ms));", "r[i] = 1.0f / sqrtf((float)ms);", None),
    ("rmsnorm: gamma applied before the first bfloat16 rounding",
     "double b = (double)orc_bf16_to_float(orc_bf16_from_double((double)t));", "double b = (double)t;", None),
    ("rmsnorm: x divided by 1/r instead of multiplied by r",
     "volatile float t = xf * r[i];", "volatile float t = xf / (1.0f / r[i]);", None),
]


def _pins():
    out = []
    for name, fn in vars(test_oracle).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        params = list(inspect.signature(fn).parameters)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not params:
            out.append((name, fn, {}))
            continue
        assert len(marks) == 1 and len(params) == 1, name
        argname, values = marks[0].args
        for v in values:
            out.append((f"{name}[{v}]", fn, {argname: v}))
    return out


def _plant(source, pattern, replacement, regex_count):
    if regex_count is not None:
        mutated, n = re.subn(pattern, replacement, source, count=regex_count)
    else:
        n = source.count(pattern)
        mutated = source.replace(pattern, replacement)
    assert n >= 1, f"pattern not found: {pattern!r}"
    return mutated


def _failing_pins(lib_path, stop_at_first):
    failed = []
    with oracle.library(lib_path):
        for name, fn, kwargs in _pins():
            try:
                fn(**kwargs)
            except Exception:             # noqa: BLE001 - any failure is a detection
                failed.append(name)
                if stop_at_first:
                    break
    return failed


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unmodified_copy_passes_every_pin(source, tmp_path):
    src = tmp_path / "copy.c"
    src.write_text(source)
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / "libcopy.so"))
    assert _failing_pins(lib, stop_at_first=False) == []


@pytest.mark.parametrize("what,pattern,replacement,regex_count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(source, tmp_path, what, pattern, replacement, regex_count):
    src = tmp_path / "mutant.c"
    src.write_text(_plant(source, pattern, replacement, regex_count))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / "libmutant.so"))
    assert _failing_pins(lib, stop_at_first=True), f"no pin noticed: {what}"
