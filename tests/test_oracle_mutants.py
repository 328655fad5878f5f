"""Plant plausible mistakes in a copy of the oracle and show the pins catch them.

Each mutant is oracle.c with one textual change, compiled to a temporary
shared object on the CPU.  Every mutant must fail at least one check of
``tests/oracle_pins.py``; a mutant that passes them all would mean the pins
leave that part of the oracle unchecked."""
import os

import pytest

import oracle
from tests import oracle_pins as P

MUTANTS = [
    ("divisor 128 instead of 127", "float s = amax / 127.0f;", "float s = amax / 128.0f;"),
    ("ties away from zero", "float r = nearbyintf(t);", "float r = roundf(t);"),
    ("truncation instead of rounding", "float r = nearbyintf(t);", "float r = truncf(t);"),
    ("signed max instead of absmax", "float a = fabsf(v[k]);", "float a = v[k];"),
    ("multiply by reciprocal of 127 per element", "float t = v[k] / s;", "float t = v[k] * (127.0f / amax);"),
    ("no upper clamp", "if (r > 127.0f) r = 127.0f;", ""),
    ("lower clamp at -128", "if (r < -127.0f) r = -127.0f;", "if (r < -128.0f) r = -128.0f;"),
    ("wrong reduction index", "s += (int64_t)ar[k] * (int64_t)br[k];",
     "s += (int64_t)ar[k] * (int64_t)br[j->K - 1 - k];"),
    ("transposed weight", "const int8_t* br = j->b + n * j->K;", "const int8_t* br = j->b + n;"),
    ("16-bit accumulator", "int64_t s = 0;", "int16_t s = 0;"),
    ("per-channel scale used twice", "t = t * scale_a[m];", "t = t * scale_w[n];"),
    ("dropped bias", "float y = t + b;", "float y = t;"),
    ("subtracted bias", "float y = t + b;", "float y = t - b;"),
    ("bf16 ties always up", "else round_up = (int)(kept & 1u);", "else round_up = 1;"),
    ("bf16 truncation", "if (dropped > 0x8000u) round_up = 1;", "if (dropped > 0xffffu) round_up = 1;"),
    ("bf16 widening shift", "uint32_t u = ((uint32_t)h) << 16;", "uint32_t u = ((uint32_t)h) << 15;"),
    ("zero test on absmax instead of scale", "if (s == 0.0f) { q[k] = 0; continue; }",
     "if (amax == 0.0f) { q[k] = 0; continue; }"),
    # fp8 e4m3 variant
    ("e4m3 divisor 447", "float sc = peak / 448.0f;", "float sc = peak / 447.0f;"),
    ("e4m3 exponent bias 8", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3 subnormal exponent -7", "if (e == 0) v = ldexp((double)m / 8.0, -6);",
     "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    ("e4m3 four mantissa bits", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 16.0, e - 7);"),
    ("e4m3 sign dropped", "return sign ? -v : v;", "return v;"),
    ("e4m3 ties to odd", "else best = ((c & 1) == 0) ? c : (uint8_t)(c - 1);",
     "else best = ((c & 1) == 1) ? c : (uint8_t)(c - 1);"),
    ("e4m3 ties up", "else best = ((c & 1) == 0) ? c : (uint8_t)(c - 1);", "else best = c;"),
    ("e4m3 rounds down", "if (a > mid) best = c;", "if (a > hi) best = c;"),
    ("e4m3 signed peak", "peak = fmaxf(peak, fabsf(v[k]));", "peak = fmaxf(peak, v[k]);"),
    ("e4m3 gemm transposed weight", "s += lut[a[m * K + k]] * lut[b[n * K + k]];",
     "s += lut[a[m * K + k]] * lut[b[k * N + n]];"),
    ("e4m3 gemm wrong reduction index", "s += lut[a[m * K + k]] * lut[b[n * K + k]];",
     "s += lut[a[m * K + k]] * lut[b[n * K + (K - 1 - k)]];"),
    ("e4m3 epilogue scale_w twice", "d *= scale_a[m];", "d *= scale_w[n];"),
    ("e4m3 epilogue dropped bias", "oracle_f32_to_bf16_rne(d + bn);", "oracle_f32_to_bf16_rne(d);"),
    # GELU before a linear layer, and its exp
    ("gelu cubic coefficient 0.04471", "static const float GELU_C1 = 0.044715f;",
     "static const float GELU_C1 = 0.04471f;"),
    ("gelu without the cubic term", "float inner = h + GELU_C1 * h3;", "float inner = h;"),
    ("gelu wrong sign in exp", "float x = -2.0f * u;", "float x = 2.0f * u;"),
    ("gelu 1 - e", "oracle_recip(1.0f + oracle_expf(x))", "oracle_recip(1.0f - oracle_expf(x))"),
    ("reciprocal without the residual step", "    y = fmaf(y, fmaf(-d, y, 1.0f), y);\n", ""),
    ("reciprocal initial value a factor 4 off", "uint32_t yb = 0x7EF311C3u - b;",
     "uint32_t yb = 0x7DF311C3u - b;"),
    ("exp without the low part of ln2", "r = fmaf(-k, LN2_LO, r);", ""),
    ("exp Taylor term r^7 dropped", "float p = 1.0f / 5040.0f;", "float p = 0.0f;"),
    ("exp scale off by one", "uint32_t bits = (uint32_t)((int32_t)k + 127) << 23;",
     "uint32_t bits = (uint32_t)((int32_t)k + 128) << 23;"),
]


def _fails_some_check(orc) -> list:
    failed = []
    for check in P.ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, RuntimeError, ValueError, OverflowError, FloatingPointError):
            failed.append(check.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    mpath = os.path.join(tmp_path, "mutant.c")
    with open(mpath, "w") as fh:
        fh.write(src.replace(old, new))
    lib = oracle.build(force=True, src=mpath, out=os.path.join(tmp_path, "mutant.so"))
    failed = _fails_some_check(oracle.Oracle(lib))
    assert failed, f"mutant '{name}' passes every pin"
