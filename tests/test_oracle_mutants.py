"""The oracle's pins must catch plausible mistakes.

Each case plants one small mistake in a temporary copy of
``oracle/aria_oracle.c`` (a wrong bias, rounding rule, index, sign, dropped
term or transposed order), compiles it, and runs the oracle pin suite
(``test_oracle_fp16.py``, ``test_oracle_quant.py``, ``test_oracle_gemm.py``)
against it through ``ARIA_ORACLE_LIB``: the suite must fail. The unmodified
copy, built the same way, must pass. CPU only.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "aria_oracle.c")
PINS = [os.path.join(ROOT, "tests", f) for f in
        ("test_oracle_fp16.py", "test_oracle_quant.py", "test_oracle_gemm.py")]
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

# (name, exact text in aria_oracle.c, replacement)
MUTANTS = [
    ("fp16 decode exponent bias", "v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
    ("fp16 encode ties away from zero", "double r = nearbyint(ldexp(ax, 11 - E));",
     "double r = floor(ldexp(ax, 11 - E) + 0.5);"),
    ("fp16 overflow threshold", "if (ax >= 65520.0)", "if (ax >= 65504.0)"),
    ("fp16 subnormal truncated", "double r = nearbyint(ax * ldexp(1.0, 24));", "double r = floor(ax * ldexp(1.0, 24));"),
    ("int8 scale divisor", "float s = a / 127.0f;", "float s = a / 128.0f;"),
    ("int8 codes truncated", "float r = nearbyintf(quot);", "float r = truncf(quot);"),
    ("int8 quotient by reciprocal", "float quot = h2f(x[k]) / s;", "float quot = h2f(x[k]) * (1.0f / s);"),
    ("act quant scale of row 0", "quant_row_i8(X + m * K, K, Xq + m * K, sx + m);",
     "quant_row_i8(X + m * K, K, Xq + m * K, sx + 0 * m);"),
    ("q4 scale divisor", "orc_float_to_half(a / 7.0f)", "orc_float_to_half(a / 8.0f)"),
    ("q4 nibble order", "if ((k & 1) == 0)", "if ((k & 1) == 1)"),
    ("q4 code offset", "uint8_t nib = (uint8_t)(q + 8);", "uint8_t nib = (uint8_t)(q + 7);"),
    ("q4 scale kept in fp32", "float sf = h2f(s16);", "float sf = a / 7.0f;"),
    ("q4 dequant group index", "out[n * K + k] = (double)(nib - 8) * orc_half_to_double(S[n * G + k / 32]);",
     "out[n * K + k] = (double)(nib - 8) * orc_half_to_double(S[n * G + k / 64]);"),
    ("int GEMM reversed k", "acc += (int64_t)x[k] * (int64_t)w[k];", "acc += (int64_t)x[k] * (int64_t)w[K - 1 - k];"),
    ("int GEMM negative overflow unflagged", "if (acc > INT32_MAX || acc < INT32_MIN)", "if (acc > INT32_MAX)"),
    ("W8A8 s_w dropped", "double y = (double)C[i * N + n] * smx * (double)sw[n];", "double y = (double)C[i * N + n] * smx;"),
    ("bias dropped", "y += orc_half_to_double(bias[n]);", "y += 0.0 * orc_half_to_double(bias[n]);"),
    ("steering sign", "y += (double)alpha * (double)v[n];", "y -= (double)alpha * (double)v[n];"),
    ("q8 reference scale dropped", "y += orc_half_to_double(x[k]) * ((double)Wq[n * K + k] * s);",
     "y += orc_half_to_double(x[k]) * (double)Wq[n * K + k];"),
    ("q4 reference code offset", "double w = (double)(nib - 8) * orc_half_to_double(S[n * G + k / 32]);",
     "double w = (double)(nib - 7) * orc_half_to_double(S[n * G + k / 32]);"),
    ("q4 clamp at 8", "if (r > 7.0f) r = 7.0f;", "if (r > 8.0f) r = 8.0f;"),
    ("q4 clamp at -8", "if (r < -7.0f) r = -7.0f;", "if (r < -8.0f) r = -8.0f;"),
    ("W8A8 output rounded through fp32", "Y[i * N + n] = orc_double_to_half(epi_terms(n, bias, v, alpha, y));",
     "Y[i * N + n] = orc_double_to_half((double)(float)epi_terms(n, bias, v, alpha, y));"),
    ("fp16 NaN encoded as infinity", "return (uint16_t)(sign | 0x7e00);", "return (uint16_t)(sign | 0x7c00);"),
    ("q4 zero scale not special", "if (sf != 0.0f) {", "if (sf != -1.0f) {"),
    ("W8A8 token scale of the output row", "double smx = (double)sx[pick(rows, i)];",
     "double smx = (double)sx[i];"),
    ("fp16 reference reads W transposed", "y += orc_half_to_double(x[k]) * orc_half_to_double(w[k]);",
     "y += orc_half_to_double(x[k]) * orc_half_to_double(W[k * N + n]);"),
    ("fp16 reference drops the last k", "y += orc_half_to_double(x[k]) * orc_half_to_double(w[k]);",
     "y += orc_half_to_double(x[k]) * orc_half_to_double(w[k]) * (double)(k + 1 < K);"),
    ("fp16 reference weight row of the token", "const uint16_t *w = W + n * K;",
     "const uint16_t *w = W + (n % 8) * K;"),
]


def _run_pins(tmp_path, src_text):
    c = tmp_path / "oracle_copy.c"
    c.write_text(src_text)
    so = tmp_path / "liboracle_copy.so"
    subprocess.check_call(["gcc", *CFLAGS, str(c), "-o", str(so), "-lm"])
    env = dict(os.environ, ARIA_ORACLE_LIB=str(so))
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return res


def test_unmodified_copy_passes(tmp_path):
    res = _run_pins(tmp_path, open(SRC).read())
    assert res.returncode == 0, res.stdout[-2000:]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old}"
    res = _run_pins(tmp_path, src.replace(old, new))
    assert res.returncode != 0, f"pins did not catch: {name}\n{res.stdout[-1500:]}"
