"""The oracle's pins catch plausible mistakes.

Each case plants one slip in a copy of ``oracle/quik_oracle.c`` (a dropped
term, a wrong divisor, index or operand, a swapped nibble, a different
rounding rule), rebuilds that copy and runs the pin file that covers the
function: the pins must fail.  CPU only; the real oracle is untouched.
"""
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "quik_oracle.c")

DENSE, NORM, SPARSE = "test_oracle_pins.py", "test_oracle_rmsnorm_pins.py", "test_oracle_sparse24_pins.py"
EXACT = "test_oracle_rmsnorm_exact_sum.py"

# (name, function whose body is changed, or None for a unique line anywhere,
#  old text, new text, pin file)
MUTATIONS = [
    # dense quantiser and layer
    ("divisor 8", "oracle_quantize_rows", "float s = amax / (float)qmax;",
     "float s = amax / (float)(qmax + 1);", DENSE),
    ("round half away from zero", None, "float r = rintf(v / s);", "float r = roundf(v / s);", DENSE),
    ("nibbles swapped", "oracle_quantize_rows",
     "(uint8_t)((codes[2 * i] & 0xF) | ((codes[2 * i + 1] & 0xF) << 4))",
     "(uint8_t)((codes[2 * i + 1] & 0xF) | ((codes[2 * i] & 0xF) << 4))", DENSE),
    ("bias dropped", None, "y += half_to_double(bias[n]);", "y += 0.0;", DENSE),
    ("no reorder", "oracle_quantize_rows", "xr[j] = half_to_float(X[r * K + perm[j]]);",
     "xr[j] = half_to_float(X[r * K + j]);", DENSE),
    ("outlier column off by one", "oracle_quantize_rows",
     "o16[r * k_o + i] = X[r * K + perm[Ki + i]];",
     "o16[r * k_o + i] = X[r * K + perm[Ki + i - (i > 0)]];", DENSE),
    ("group scale index", None, "(double)sx[m * G + g] * (double)sw[n * G + g]",
     "(double)sx[m * G] * (double)sw[n * G + g]", DENSE),
    ("outlier operand reversed", None,
     "half_to_double(xo[m * k_o + i]) * half_to_double(wo[n * k_o + i])",
     "half_to_double(xo[m * k_o + (k_o - 1 - i)]) * half_to_double(wo[n * k_o + i])", DENSE),
    ("INT8 divisor 128", "oracle_quantize_rows", "float s = amax / 127.0f;",
     "float s = amax / 128.0f;", DENSE),
    ("signed absmax", "oracle_quantize_rows",
     "if (fabsf(xr[j]) > amax) amax = fabsf(xr[j]);", "if (xr[j] > amax) amax = xr[j];", DENSE),
    ("nibble decoded unsigned", None,
     "return nib >= 8 ? (int)nib - 16 : (int)nib;", "return (int)nib;", DENSE),
    ("outliers in the absmax", "oracle_quantize_rows",
     "for (int64_t j = g * gs; j < (g + 1) * gs; ++j)\n                        if (fabsf",
     "for (int64_t j = g * gs; j < (g + 1) * gs + (group ? 0 : k_o); ++j)\n"
     "                        if (fabsf", DENSE),
    # RMS norm folded into the quantiser
    ("norm: squares over the INT4 channels only", "oracle_rmsnorm_quantize_rows",
     "for (int64_t k = 0; k < K; ++k) {\n                double h = half_to_double(X[r * K + k]);",
     "for (int64_t k = 0; k < Ki; ++k) {\n                double h = half_to_double(X[r * K + perm[k]]);",
     NORM),
    ("norm: mean over K_i", "oracle_rmsnorm_quantize_rows",
     "ss / (double)K + (double)eps", "ss / (double)(Ki > 0 ? Ki : K) + (double)eps", NORM),
    ("norm: eps outside the root", "oracle_rmsnorm_quantize_rows",
     "1.0 / sqrt(ss / (double)K + (double)eps)", "1.0 / (sqrt(ss / (double)K) + (double)eps)", NORM),
    ("norm: gamma not reordered", "oracle_rmsnorm_quantize_rows",
     "half_to_double(gamma[c])", "half_to_double(gamma[j])", NORM),
    ("norm: scale without the row factor", "oracle_rmsnorm_quantize_rows",
     "scale[r * G + g] = (float)((double)s * rf);", "scale[r * G + g] = s;", NORM),
    ("norm: FP16 outliers without the row factor", "oracle_rmsnorm_quantize_rows",
     "double_to_half((double)z[Ki + i] * rf)", "double_to_half((double)z[Ki + i])", NORM),
    ("norm: INT8 outlier scale without the row factor", "oracle_rmsnorm_quantize_rows",
     "o_scale[r] = (float)((double)s * rf);", "o_scale[r] = s;", NORM),
    ("norm: squares summed in fp64, in order", "oracle_rmsnorm_quantize_rows",
     "double ss = ldexp((double)S, -48);",
     "double ss = 0.0;\n            for (int64_t k2 = 0; k2 < K; ++k2) {\n"
     "                double h2 = half_to_double(X[r * K + k2]);\n                ss += h2 * h2;\n"
     "            }", EXACT),
    ("norm: squares summed in fp64, reversed", "oracle_rmsnorm_quantize_rows",
     "double ss = ldexp((double)S, -48);",
     "double ss = 0.0;\n            for (int64_t k2 = K - 1; k2 >= 0; --k2) {\n"
     "                double h2 = half_to_double(X[r * K + k2]);\n                ss += h2 * h2;\n"
     "            }", EXACT),
    ("norm: exact sum truncated to 64 bits", "oracle_rmsnorm_quantize_rows",
     "double ss = ldexp((double)S, -48);", "double ss = ldexp((double)(uint64_t)S, -48);", EXACT),
    # 2:4-sparse weights
    ("2:4: ties to the higher position", "oracle_prune24_quantize_rows",
     "if (fabsf(g[i]) > fabsf(g[a])) a = i;", "if (fabsf(g[i]) >= fabsf(g[a])) a = i;", SPARSE),
    ("2:4: keeps the smallest", "oracle_prune24_quantize_rows",
     "if (fabsf(g[i]) > fabsf(g[a])) a = i;", "if (fabsf(g[i]) < fabsf(g[a])) a = i;", SPARSE),
    ("2:4: pair nibble order", "oracle_prune24_quantize_rows",
     "uint8_t nib = (uint8_t)(i0 | (i1 << 2));", "uint8_t nib = (uint8_t)(i1 | (i0 << 2));", SPARSE),
    ("2:4: code nibble order", "oracle_prune24_quantize_rows",
     "(uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4))", "(uint8_t)((q1 & 0xF) | ((q0 & 0xF) << 4))", SPARSE),
    ("2:4: divisor 8", "oracle_prune24_quantize_rows", "float s = amax / 7.0f;",
     "float s = amax / 8.0f;", SPARSE),
    ("2:4: expansion swaps the positions", "oracle_unpack24",
     "int pos[2] = {(int)(4 * t + i0), (int)(4 * t + i1)};",
     "int pos[2] = {(int)(4 * t + i1), (int)(4 * t + i0)};", SPARSE),
]


def _function_span(text, name):
    start = text.index(f"int {name}(")
    nxt = [m.start() for m in re.finditer(r"\n/\*\n \* oracle_", text) if m.start() > start]
    return start, (nxt[0] if nxt else len(text))


def _mutate(text, func, old, new):
    lo, hi = _function_span(text, func) if func else (0, len(text))
    body = text[lo:hi]
    assert body.count(old) == 1, f"mutation site not unique: {old!r}"
    return text[:lo] + body.replace(old, new) + text[hi:]


@pytest.mark.parametrize("name,func,old,new,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, func, old, new, pins):
    work = tmp_path / "copy"
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), work / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", ".pytest_cache"))
    src = (work / "oracle" / "quik_oracle.c")
    src.write_text(_mutate(src.read_text(), func, old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join("tests", pins)], cwd=work, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode != 0, f"the pins in {pins} pass with the mistake '{name}' planted"


def test_unmutated_copy_passes(tmp_path):
    """The harness itself: an unchanged copy passes every pin file."""
    work = tmp_path / "copy"
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), work / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", ".pytest_cache"))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join("tests", DENSE), os.path.join("tests", NORM),
                        os.path.join("tests", SPARSE), os.path.join("tests", EXACT)], cwd=work, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
