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
    # GELU before a linear layer (binary64) and the binary64 -> bf16 rounding
    ("gelu cubic coefficient 0.04471", "static const double GELU_C1 = 0.044715;",
     "static const double GELU_C1 = 0.04471;"),
    ("gelu sqrt(2)/pi for sqrt(2/pi)", "static const double GELU_C0 = 0.79788456080286535587989211986876373695;",
     "static const double GELU_C0 = 0.45015815807855303477759959550337001681;"),
    ("gelu without the cubic term", "double inner = h + GELU_C1 * h3;", "double inner = h;"),
    ("gelu wrong sign in exp", "double e = exp(-2.0 * u);", "double e = exp(2.0 * u);"),
    ("gelu sigmoid(u) for sigmoid(2u)", "double e = exp(-2.0 * u);", "double e = exp(-u);"),
    ("gelu 1 - e", "return h / (1.0 + e);", "return h / (1.0 - e);"),
    ("gelu halved twice", "return h / (1.0 + e);", "return 0.5 * h / (1.0 + e);"),
    ("bf16 from binary64 through binary32 (double rounding)", "double n = nearbyint(ldexp(a, 7 - E));",
     "double n = nearbyint(ldexp((double)(float)a, 7 - E));"),
    ("bf16 from binary64 ties away from zero", "double n = nearbyint(ldexp(a, 7 - E));",
     "double n = round(ldexp(a, 7 - E));"),
    ("bf16 from binary64 truncated", "double n = nearbyint(ldexp(a, 7 - E));",
     "double n = trunc(ldexp(a, 7 - E));"),
    ("bf16 from binary64 subnormal spacing 2^-134", "if (E < -126) E = -126;", "if (E < -127) E = -127;"),
    ("bf16 from binary64 loses the sign", "uint16_t sign = signbit(d) ? 0x8000u : 0x0000u;",
     "uint16_t sign = 0x0000u;"),
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
