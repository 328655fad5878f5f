"""Checks that pin the CPU oracle to things other than itself.

Each ``check_*`` takes an oracle instance and raises AssertionError if the
oracle disagrees with what the paper's method and the mathematics fix:
hand-worked fixtures under ``tests/golden/``, library routines (numpy's
float32 division and rint, numpy's int64 matmul, torch's bf16 rounding),
exact rational arithmetic, closed forms and invariants.  The same checks
are run against deliberately broken copies of the oracle to show that a
plausible mistake anywhere in it fails at least one of them.

Method: "Realizing Native INT8 Compute for Diffusion Transformers on
Consumer GPUs" (arXiv 2606.14598), abstract -- per-token activation
quantization, per-channel weight quantization, int8 x int8 -> int32 GEMM,
per-token x per-channel dequantization plus bias in the epilogue, bf16 out.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

U32 = 2.0 ** -24   # binary32 unit roundoff
U16 = 2.0 ** -8    # bf16 unit roundoff (8 significant bits)


# ------------------------------------------------------------- helpers


def bf16_bits(values) -> np.ndarray:
    """Exact bf16 bit patterns of values that torch can represent exactly."""
    t = torch.tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    assert (t.float().numpy() == np.asarray(values, np.float32)).all(), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_float(bits) -> np.ndarray:
    t = torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16).copy()).view(torch.bfloat16)
    return t.float().numpy()


def read_rows(name: str):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.split() for p in line.split("|")]
            rows.append(parts)
    return rows


def parse_num(tok: str) -> float:
    """A decimal, or a*2^b for exact powers of two (e.g. subnormals)."""
    if "*2^" in tok:
        a, b = tok.split("*2^")
        return float(a) * 2.0 ** int(b)
    return float(tok)


def read_keyed(name: str) -> dict:
    out: dict = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out.setdefault(key, []).append([float(v) for v in vals])
    return out


def numpy_quantize(x: np.ndarray):
    """The quantizer through numpy's float32 routines (library cross-check)."""
    x = x.astype(np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = (amax / np.float32(127.0)).astype(np.float32)
    q = np.zeros(x.shape, np.int8)
    nz = amax > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x[nz] / s[nz, None]).astype(np.float32)
    q[nz] = np.clip(np.rint(t), -127, 127).astype(np.int8)
    return q, s


def edge_rows(K: int, rng: np.random.Generator) -> np.ndarray:
    """bf16 rows that exercise the quantizer's special cases."""
    rows = []
    z = np.zeros(K, np.float32)
    rows.append(z.copy())                                  # all zero
    r = z.copy(); r[K // 3] = -3.0; rows.append(r)         # single non-zero, negative
    r = -z; rows.append(r)                                 # all -0
    r = rng.standard_normal(K).astype(np.float32) * np.float32(2.0 ** -130); rows.append(r)  # subnormal
    r = np.full(K, 0.5, np.float32); r[0] = 127.0; rows.append(r)          # ties at .5
    r = (np.arange(K, dtype=np.float32) % 255 - 127) + np.float32(0.5)    # many ties
    r[1] = 127.0; rows.append(np.clip(r, -127, 127))
    r = rng.standard_normal(K).astype(np.float32) * np.float32(1e4); rows.append(r)  # large
    return bits_to_float(torch.tensor(np.stack(rows)).to(torch.bfloat16).view(torch.int16).numpy()
                         .view(np.uint16))


def to_bits(x: np.ndarray) -> np.ndarray:
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------- bf16


def check_bf16_widen(orc) -> None:
    """bf16 -> f32 equals torch's conversion on every non-NaN bit pattern."""
    pats = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    mine = orc.bf16_bits_to_f32(pats)
    ref = bits_to_float(pats)
    ok = np.isnan(ref) | (mine.view(np.uint32) == ref.view(np.uint32))
    assert ok.all(), "bf16 widening differs from torch"


def check_bf16_round(orc) -> None:
    """f32 -> bf16 RNE equals torch's conversion, ties and overflow included."""
    rng = np.random.default_rng(11)
    hi = rng.integers(0, 65536, 4000).astype(np.uint32) << 16
    lows = np.array([0, 1, 0x7fff, 0x8000, 0x8001, 0xffff], np.uint32)
    u = (hi[:, None] | lows[None, :]).reshape(-1)
    f = u.view(np.float32)
    f = f[~np.isnan(f)]
    extra = np.array([3.3895314e38, 3.4028235e38, -3.4028235e38, 1e-45, -0.0, 0.0, np.inf, -np.inf],
                     np.float32)
    f = np.concatenate([f, extra])
    mine = orc.f32_to_bf16_bits(f)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (mine == ref).all(), f"bf16 rounding differs from torch at {np.flatnonzero(mine != ref)[:5]}"


# ------------------------------------------------------------ quantizer


def check_quant_golden(orc) -> None:
    """Hand-worked rows (tests/golden/quant_act_rows.txt)."""
    for xs, qs, ss in read_rows("quant_act_rows.txt"):
        x = np.array([float(v) for v in xs], np.float32)
        q, s = orc.quantize_act(bf16_bits(x)[None, :])
        want = np.array([int(v) for v in qs], np.int8)
        assert (q[0] == want).all(), f"codes {q[0]} != {want} for {x}"
        if ss[0] != "-":
            assert s[0] == np.float32(float(ss[0])), f"scale {s[0]} != {ss[0]}"


def check_weight_golden(orc) -> None:
    """Hand-worked fp32 weight rows (tests/golden/quant_weight_rows.txt)."""
    for ws, qs, ss in read_rows("quant_weight_rows.txt"):
        w = np.array([parse_num(v) for v in ws], np.float32)
        assert (w.astype(np.float64) == np.array([parse_num(v) for v in ws])).all(), "not exact in fp32"
        q, s = orc.quantize_weight(w[None, :])
        assert (q[0] == np.array([int(v) for v in qs], np.int8)).all(), f"codes {q[0]} for {w}"
        assert s[0] == np.float32(parse_num(ss[0]))


def check_quant_vs_numpy(orc) -> None:
    """Quantizer equals the same rule through numpy float32 division + rint."""
    rng = np.random.default_rng(5)
    K = 200
    x = np.concatenate([edge_rows(K, rng),
                        bits_to_float(to_bits(rng.standard_normal((40, K)).astype(np.float32)))])
    q, s = orc.quantize_act(to_bits(x))
    q2, s2 = numpy_quantize(x)
    assert (s.view(np.uint32) == s2.view(np.uint32)).all(), "scales differ from numpy"
    assert (q == q2).all(), "codes differ from numpy"
    w = rng.standard_normal((30, 96)).astype(np.float32) * np.float32(0.02)
    wq, sw = orc.quantize_weight(w)
    wq2, sw2 = numpy_quantize(w)
    assert (sw.view(np.uint32) == sw2.view(np.uint32)).all() and (wq == wq2).all()


def check_quant_invariants(orc) -> None:
    """Properties any per-token absmax quantizer with round-to-nearest has."""
    rng = np.random.default_rng(6)
    K = 300
    x = bits_to_float(to_bits(rng.standard_normal((64, K)).astype(np.float32)
                              * np.float32(3.0) ** rng.integers(-3, 4, (64, 1)).astype(np.float32)))
    q, s = orc.quantize_act(to_bits(x))
    amax = np.abs(x).max(axis=1)
    # the largest |x| of every row maps to +-127 with the sign of x
    arg = np.abs(x).argmax(axis=1)
    assert (np.abs(q).max(axis=1) == 127).all()
    assert (q[np.arange(64), arg] == np.sign(x[np.arange(64), arg]) * 127).all()
    # round to nearest: |q*s - x| <= s/2 (plus the rounding of s and of x/s)
    err = np.abs(q.astype(np.float64) * s[:, None].astype(np.float64) - x.astype(np.float64))
    assert (err <= s[:, None] * (0.5 + 1e-4)).all(), "reconstruction error above half a step"
    # scale s is absmax/127 to within one binary32 rounding
    assert np.allclose(s.astype(np.float64), amax.astype(np.float64) / 127.0, rtol=2 * U32, atol=0)
    # exact power-of-two scaling: same codes, scale times 2^j
    for j in (-5, 7):
        q2, s2 = orc.quantize_act(to_bits(x * np.float32(2.0 ** j)))
        assert (q2 == q).all() and (s2 == s * np.float32(2.0 ** j)).all()
    # negation: codes negate, scale unchanged
    q3, s3 = orc.quantize_act(to_bits(-x))
    assert (q3 == -q).all() and (s3 == s).all()
    # row independence: permuting tokens permutes results
    perm = rng.permutation(64)
    q4, s4 = orc.quantize_act(to_bits(x[perm]))
    assert (q4 == q[perm]).all() and (s4 == s[perm]).all()


# ----------------------------------------------------------------- GEMM


def check_gemm_vs_numpy(orc) -> None:
    """Exact accumulator equals numpy's int64 matmul (and a Python brute force)."""
    rng = np.random.default_rng(7)
    for M, N, K in [(1, 1, 1), (5, 3, 7), (33, 17, 96), (70, 40, 272)]:
        a = rng.integers(-127, 128, (M, K), dtype=np.int8)
        b = rng.integers(-127, 128, (N, K), dtype=np.int8)
        acc = orc.gemm_i64(a, b, nthreads=3)
        assert (acc == a.astype(np.int64) @ b.astype(np.int64).T).all()
    a = rng.integers(-127, 128, (3, 5), dtype=np.int8)
    b = rng.integers(-127, 128, (4, 5), dtype=np.int8)
    acc = orc.gemm_i64(a, b)
    for m in range(3):
        for n in range(4):
            assert acc[m, n] == sum(int(a[m, k]) * int(b[n, k]) for k in range(5))


def check_gemm_closed_forms(orc) -> None:
    """Identity and one-hot weights; worst-case all-+-127 rows at K = 12288."""
    rng = np.random.default_rng(8)
    K = 48
    xq = rng.integers(-127, 128, (9, K), dtype=np.int8)
    eye = (np.eye(K, dtype=np.int64) * 127).astype(np.int8)
    assert (orc.gemm_i64(xq, eye) == 127 * xq.astype(np.int64)).all()
    cols = rng.integers(0, K, 20)
    onehot = np.zeros((20, K), np.int8)
    onehot[np.arange(20), cols] = 1
    assert (orc.gemm_i64(xq, onehot) == xq[:, cols].astype(np.int64)).all()
    K = 12288
    x = np.stack([np.full(K, 127, np.int8), np.full(K, -127, np.int8)])
    acc = orc.gemm_i64(x, x)
    big = K * 127 * 127
    assert big == 198193152 and big < 2 ** 31
    assert (acc == np.array([[big, -big], [-big, big]])).all()


def check_gemm_invariants(orc) -> None:
    rng = np.random.default_rng(9)
    a = rng.integers(-127, 128, (12, 64), dtype=np.int8)
    b = rng.integers(-127, 128, (10, 64), dtype=np.int8)
    acc = orc.gemm_i64(a, b)
    pm, pn = rng.permutation(12), rng.permutation(10)
    assert (orc.gemm_i64(a[pm], b[pn]) == acc[pm][:, pn]).all()
    assert (orc.gemm_i64(-a, b) == -acc).all()
    pk = rng.permutation(64)   # permuting the reduction index changes nothing
    assert (orc.gemm_i64(a[:, pk], b[:, pk]) == acc).all()


# ------------------------------------------------------------- epilogue


def _exact_y(acc, sa, sw, bias_f) -> list:
    return [[Fraction(int(acc[m, n])) * Fraction(float(sa[m])) * Fraction(float(sw[n]))
             + Fraction(float(bias_f[n])) for n in range(acc.shape[1])] for m in range(acc.shape[0])]


def check_epilogue_exact_bound(orc) -> None:
    """bf16 output within the binary32 + bf16 rounding bound of the exact value."""
    rng = np.random.default_rng(10)
    M, N = 24, 20
    acc = rng.integers(-200_000_000, 200_000_000, (M, N)).astype(np.int64)
    acc[0, :] = 0
    sa = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), M)).astype(np.float32)
    sw = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), N)).astype(np.float32)
    bias = to_bits(rng.standard_normal(N).astype(np.float32) * np.float32(0.1))
    bias_f = bits_to_float(bias)
    out = bits_to_float(orc.epilogue(acc, sa, sw, bias))
    y = _exact_y(acc, sa, sw, bias_f)
    for m in range(M):
        for n in range(N):
            prod = abs(float(Fraction(int(acc[m, n])) * Fraction(float(sa[m])) * Fraction(float(sw[n]))))
            ye = float(y[m][n])
            bound = U16 * abs(ye) + 4 * U32 * (prod + abs(float(bias_f[n]))) + 1e-38
            assert abs(float(out[m, n]) - ye) <= bound, (m, n, out[m, n], ye)
    # a zero accumulator gives the bias exactly
    assert (out[0] == bias_f).all()
    # the fp64 recomputation agrees with the exact value to binary64 precision
    y64 = orc.epilogue_f64(acc, sa, sw, bias)
    for m in range(M):
        for n in range(N):
            assert abs(y64[m, n] - float(y[m][n])) <= 4 * 2.0 ** -53 * (abs(float(y[m][n])) + 1.0)


def check_epilogue_bias_optional(orc) -> None:
    rng = np.random.default_rng(12)
    acc = rng.integers(-10 ** 6, 10 ** 6, (5, 8)).astype(np.int64)
    sa = np.full(5, 0.01, np.float32)
    sw = np.full(8, 0.02, np.float32)
    zero = np.zeros(8, np.uint16)
    assert (orc.epilogue(acc, sa, sw, None) == orc.epilogue(acc, sa, sw, zero)).all()


def check_hand_linear(orc) -> None:
    """The worked example of tests/golden/hand_linear_2x4x2.txt, step by step."""
    g = read_keyed("hand_linear_2x4x2.txt")
    x = bf16_bits(np.array(g["x"], np.float32))
    wq = np.array(g["wq"], np.int8)
    sw = np.array(g["scale_w"][0], np.float32)
    bias = bf16_bits(np.array(g["bias"][0], np.float32))
    out, xq, sa, acc = orc.linear(x, wq, sw, bias)
    assert (xq == np.array(g["xq"], np.int8)).all()
    assert (sa == np.array(g["scale_a"][0], np.float32)).all()
    assert (acc == np.array(g["acc"], np.int64)).all()
    assert (bits_to_float(out) == np.array(g["out"], np.float32)).all(), bits_to_float(out)


def check_linear_identity_weight(orc) -> None:
    """Identity weight (127 * I, scale 1/127), zero bias: out ~ X within the
    quantization step of each token."""
    rng = np.random.default_rng(13)
    K = 64
    x = to_bits(rng.standard_normal((16, K)).astype(np.float32))
    xf = bits_to_float(x).astype(np.float64)
    wq = (np.eye(K) * 127).astype(np.int8)
    sw = np.full(K, np.float32(1.0) / np.float32(127.0), np.float32)
    out, xq, sa, acc = orc.linear(x, wq, sw, np.zeros(K, np.uint16))
    y = bits_to_float(out).astype(np.float64)
    step = sa.astype(np.float64)[:, None]
    assert (np.abs(y - xf) <= 0.5 * step * (1 + 1e-3) + U16 * np.abs(xf) + 1e-30).all()


def check_linear_composition(orc) -> None:
    """The whole layer equals its three steps run one after another."""
    rng = np.random.default_rng(14)
    x = to_bits(rng.standard_normal((20, 80)).astype(np.float32))
    wq = rng.integers(-127, 128, (24, 80), dtype=np.int8)
    sw = np.exp(rng.uniform(-9, -2, 24)).astype(np.float32)
    bias = to_bits(rng.standard_normal(24).astype(np.float32))
    out, xq, sa, acc = orc.linear(x, wq, sw, bias)
    q2, s2 = orc.quantize_act(x)
    a2 = orc.gemm_i64(q2, wq)
    assert (q2 == xq).all() and (s2 == sa).all() and (a2 == acc).all()
    assert (orc.epilogue(a2, s2, sw, bias) == out).all()


ALL_CHECKS = [
    check_bf16_widen, check_bf16_round,
    check_quant_golden, check_weight_golden, check_quant_vs_numpy, check_quant_invariants,
    check_gemm_vs_numpy, check_gemm_closed_forms, check_gemm_invariants,
    check_epilogue_exact_bound, check_epilogue_bias_optional,
    check_hand_linear, check_linear_identity_weight, check_linear_composition,
]


# ------------------------------------------------------------ fp8 e4m3


def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def check_e4m3_decode(orc) -> None:
    """E4M3 code -> value equals torch's float8_e4m3fn on all 256 codes."""
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])


def check_e4m3_encode(orc) -> None:
    """value -> E4M3 (RNE) equals torch's conversion, at every midpoint too."""
    vals = orc.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))          # non-negative finite codes
    mids = 0.5 * (vals[:-1] + vals[1:])
    rng = np.random.default_rng(21)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
                        rng.uniform(0, 448, 3000), rng.uniform(0, 2.0 ** -5, 500)]).astype(np.float32)
    x = np.concatenate([x, -x])
    x = x[np.abs(x) <= 448]
    assert np.array_equal(orc.f32_to_e4m3(x), _torch_e4m3(x))


def check_fp8_quant_golden(orc) -> None:
    """Hand-worked rows (tests/golden/quant_fp8_rows.txt)."""
    for xs, qs, ss in read_rows("quant_fp8_rows.txt"):
        x = np.array([float(v) for v in xs], np.float32)
        q, s = orc.quantize_act_fp8(bf16_bits(x)[None, :])
        want = np.array([int(v, 16) for v in qs], np.uint8)
        assert (q[0] == want).all(), f"codes {q[0]} != {want} for {x}"
        assert s[0] == np.float32(float(ss[0]))


def numpy_quantize_fp8(x: np.ndarray):
    """The FP8 quantizer through numpy float32 division and torch's E4M3 conversion."""
    x = x.astype(np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = (amax / np.float32(448.0)).astype(np.float32)
    q = np.zeros(x.shape, np.uint8)
    nz = s > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x[nz] / s[nz, None]).astype(np.float32)
    q[nz] = _torch_e4m3(np.clip(t, -448, 448))
    return q, s


def check_fp8_quant_vs_library(orc) -> None:
    rng = np.random.default_rng(22)
    K = 160
    x = np.concatenate([edge_rows(K, rng), bits_to_float(to_bits(rng.standard_normal((30, K)).astype(np.float32)))])
    q, s = orc.quantize_act_fp8(to_bits(x))
    q2, s2 = numpy_quantize_fp8(x)
    # -0 codes: the library keeps the sign of a negative quotient that rounds to zero
    assert (s.view(np.uint32) == s2.view(np.uint32)).all()
    assert (q == q2).all(), np.argwhere(q != q2)[:5]
    w = (rng.standard_normal((20, 64)) * 0.02).astype(np.float32)
    wq, sw = orc.quantize_weight_fp8(w)
    wq2, sw2 = numpy_quantize_fp8(w)
    assert (sw.view(np.uint32) == sw2.view(np.uint32)).all() and (wq == wq2).all()


def check_fp8_quant_invariants(orc) -> None:
    rng = np.random.default_rng(23)
    x = bits_to_float(to_bits(rng.standard_normal((32, 200)).astype(np.float32) * 5))
    q, s = orc.quantize_act_fp8(to_bits(x))
    arg = np.abs(x).argmax(axis=1)
    top = q[np.arange(32), arg]
    assert ((top == 0x7E) | (top == 0xFE)).all(), "the row absmax must map to +-448"
    vals = orc.e4m3_to_f64(q)
    # E4M3 keeps 4 significant bits: relative rounding <= 2^-4 (normals) of |x/s|
    rel = np.abs(vals * s[:, None] - x) / np.maximum(np.abs(x), 1e-30)
    big = np.abs(x / s[:, None]) >= 2.0 ** -6
    assert (rel[big] <= 2.0 ** -4 * (1 + 1e-6)).all()
    q2, s2 = orc.quantize_act_fp8(to_bits(x * np.float32(8.0)))
    assert (q2 == q).all() and (s2 == s * np.float32(8.0)).all()
    q3, _ = orc.quantize_act_fp8(to_bits(-x))
    assert ((q3 ^ q) == 0x80)[x != 0].all()


def check_fp8_gemm(orc) -> None:
    """The FP8 accumulator equals numpy's float64 matmul of the decoded codes;
    diagonal 1.0 weights select the activations."""
    rng = np.random.default_rng(24)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    a = rng.choice(finite, (9, 48))
    b = rng.choice(finite, (7, 48))
    acc = orc.gemm_fp8(a, b)
    ref = orc.e4m3_to_f64(a) @ orc.e4m3_to_f64(b).T
    assert np.allclose(acc, ref, rtol=1e-12, atol=1e-12)
    ref2 = torch.from_numpy(a).view(torch.float8_e4m3fn).double().numpy() @ \
        torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy().T
    assert np.allclose(acc, ref2, rtol=1e-12, atol=1e-12)
    eye = np.zeros((48, 48), np.uint8)
    eye[np.arange(48), np.arange(48)] = 0x38
    assert np.array_equal(orc.gemm_fp8(a, eye), orc.e4m3_to_f64(a))


def check_fp8_epilogue(orc) -> None:
    """bf16 output within the binary32 + bf16 rounding bound of the exact value."""
    rng = np.random.default_rng(25)
    M, N = 12, 16
    acc = rng.standard_normal((M, N)) * 1e5
    acc[0, :] = 0.0
    sa = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), M)).astype(np.float32)
    sw = np.exp(rng.uniform(np.log(1e-4), np.log(1e-1), N)).astype(np.float32)
    bias = to_bits(rng.standard_normal(N).astype(np.float32) * np.float32(0.1))
    bf = bits_to_float(bias)
    out = bits_to_float(orc.epilogue_fp8(acc, sa, sw, bias))
    for m in range(M):
        for n in range(N):
            exact = Fraction(float(acc[m, n])) * Fraction(float(sa[m])) * Fraction(float(sw[n])) + Fraction(float(bf[n]))
            ye = float(exact)
            prod = abs(float(acc[m, n]) * float(sa[m]) * float(sw[n]))
            assert abs(float(out[m, n]) - ye) <= U16 * abs(ye) + 5 * U32 * (prod + abs(float(bf[n]))) + 1e-38
    assert (out[0] == bf).all()


ALL_CHECKS += [check_e4m3_decode, check_e4m3_encode, check_fp8_quant_golden, check_fp8_quant_vs_library,
               check_fp8_quant_invariants, check_fp8_gemm, check_fp8_epilogue]


# ------------------------------------------------- GELU before a linear layer
#
# GELU is the library's reading of the producer of the down-projection's
# input (the pages name no activation): the tanh form of Hendrycks & Gimpel,
# gelu(h) = 0.5 h (1 + tanh(u)), u = sqrt(2/pi) (h + 0.044715 h^3), rounded
# once to bf16.  The oracle evaluates it in binary64 (as h / (1 + exp(-2u)),
# the same function) and rounds that once to bf16; these checks hold it to
# the exact function.


def _bf16_positive_grid():
    """All non-negative finite bf16 values in increasing order (bit patterns
    0x0000..0x7F7F), as float64 (exact)."""
    bits = np.arange(0x7F80, dtype=np.uint32)
    return (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64), bits.astype(np.uint16)


_BF16_MAX = float(np.array([0x7F7F0000], np.uint32).view(np.float32)[0])


def nearest_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float64 values by the definition of rounding to
    nearest, ties to even: bracket |x| between adjacent bf16 values by a
    search over all of them, compare it with their exact midpoint (a sum of
    two bf16 values halved is exact in binary64), and on a tie take the even
    bit pattern; beyond the midpoint of the largest finite value and 2^128,
    infinity."""
    x = np.asarray(x, np.float64)
    grid, gbits = _bf16_positive_grid()
    a = np.abs(x)
    out = np.zeros(x.shape, np.uint16)
    i = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, len(grid) - 1)   # grid[i] <= a
    lo, hi = grid[i], grid[np.minimum(i + 1, len(grid) - 1)]
    mid = 0.5 * (lo + hi)
    up = (a > mid) | ((a == mid) & (gbits[i] & 1 == 1))
    b = np.where(up, gbits[np.minimum(i + 1, len(grid) - 1)], gbits[i]).astype(np.uint16)
    top = 0.5 * (_BF16_MAX + 2.0 ** 128)                     # ties go to the even 2^128 = inf
    b = np.where(a >= top, np.uint16(0x7F80), b)
    b = np.where(np.isinf(a), np.uint16(0x7F80), b)
    out[...] = b | np.where(np.signbit(x), np.uint16(0x8000), np.uint16(0))
    nan = np.isnan(x)
    out[nan] = 0x7FC0 | (out[nan] & 0x8000)
    return out


def check_f64_to_bf16(orc) -> None:
    """The binary64 -> bf16 rounding against nearest_bf16_bits on random
    values over the whole range (subnormal bf16 results and overflow
    included), every kind of midpoint between adjacent bf16 values exactly
    (ties to even) and one binary64 ulp either side of it (a route through
    binary32 rounds those twice and fails), zeros, infinities."""
    rng = np.random.default_rng(41)
    mags = np.exp2(rng.uniform(-140, 129, 40000))
    vals = mags * np.where(rng.random(40000) < 0.5, -1.0, 1.0)
    grid, _ = _bf16_positive_grid()
    idx = rng.integers(0, len(grid) - 1, 20000)
    idx = np.concatenate([idx, np.arange(0, 300), np.arange(len(grid) - 300, len(grid) - 1)])
    mids = 0.5 * (grid[idx] + grid[idx + 1])
    near = np.concatenate([mids, np.nextafter(mids, np.inf), np.nextafter(mids, 0.0)])
    near = np.concatenate([near, -near])
    top = 0.5 * (_BF16_MAX + 2.0 ** 128)
    special = np.array([0.0, -0.0, np.inf, -np.inf, _BF16_MAX, top, np.nextafter(top, 0.0), 1e300, 2.0 ** -134,
                        np.nextafter(2.0 ** -134, 1.0), 2.0 ** -135, 1e-300])
    x = np.concatenate([vals, near, special])
    got = orc.f64_to_bf16_bits(x)
    want = nearest_bf16_bits(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]).hex(), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]


_EXACT_GELU_CACHE = None


def exact_gelu_table():
    """For every finite bf16 input h (bit patterns 0x0000..0x7F7F and their
    negatives): (bits of h, exact bf16 rounding of gelu(h), relative
    distance of gelu(h) from the nearest bf16 rounding boundary), with gelu
    evaluated in 60-digit decimal arithmetic (sqrt(2/pi) to 60 digits,
    0.044715 exact, the decimal module's correctly rounded exp), i.e. the
    exact function to far below any binary64 error; rounded to bf16 by
    comparison with exact midpoints.  Independent of the oracle (cached)."""
    global _EXACT_GELU_CACHE
    if _EXACT_GELU_CACHE is not None:
        return _EXACT_GELU_CACHE
    from decimal import Decimal, localcontext
    grid, gbits = _bf16_positive_grid()
    hbits, gout, dist = [], [], []
    with localcontext() as ctx:
        ctx.prec = 60
        ctx.Emin = -999999999
        ctx.Emax = 999999999
        pi = Decimal("3.14159265358979323846264338327950288419716939937510582097494459230781640628620899")
        c0 = (Decimal(2) / pi).sqrt()
        c1 = Decimal("0.044715")
        for sign in (0, 1):
            for j in range(len(grid)):
                h = Decimal(float(grid[j])) * (-1 if sign else 1)
                u = c0 * (h + c1 * h * h * h)
                x = -2 * u
                if x > 4000:              # |gelu| < 2^128 e^-4000: far below the least bf16 subnormal
                    g = Decimal(0)
                elif x < -4000:           # 1 + e^x = 1 to 1700 digits: gelu = h to far below bf16
                    g = h
                else:
                    g = h / (1 + x.exp())
                hbits.append(int(gbits[j]) | (0x8000 if sign else 0))
                a = abs(g)
                # bracket |g| by the bf16 grid (float(a) is the nearest double; then exact comparison)
                af = float(a)
                i = int(np.searchsorted(grid, af, side="right")) - 1
                i = max(0, min(i, len(grid) - 2))
                while i > 0 and Decimal(float(grid[i])) > a:
                    i -= 1
                while i + 1 < len(grid) and Decimal(float(grid[i + 1])) <= a:
                    i += 1
                if i + 1 >= len(grid):    # at or above the largest finite value
                    top = (Decimal(_BF16_MAX) + Decimal(2) ** 128) / 2
                    b, dd = (0x7F80 if a >= top else int(gbits[-1])), 1.0
                else:
                    lo, hi = Decimal(float(grid[i])), Decimal(float(grid[i + 1]))
                    mid = (lo + hi) / 2
                    if a > mid or (a == mid and gbits[i] & 1):
                        b = int(gbits[i + 1])
                    else:
                        b = int(gbits[i])
                    dd = float(abs(a - mid) / mid) if a != 0 else 1.0
                if g < 0 or (g == 0 and sign):
                    b |= 0x8000
                gout.append(b)
                dist.append(dd)
    _EXACT_GELU_CACHE = (np.array(hbits, np.uint16), np.array(gout, np.uint16), np.array(dist))
    return _EXACT_GELU_CACHE


NEAR_TIE = 2.0 ** -40   # binary64 evaluation error of gelu is far below this (relative)


def check_gelu_exact(orc) -> None:
    """bf16_rne(gelu(h)) equals the correctly rounded bf16 value of the exact
    tanh-form GELU on every finite bf16 input, except where the exact value
    lies within 2^-40 (relative) of a bf16 rounding boundary, where a binary64
    evaluation cannot tell the side.  Those inputs are exactly the 256 with
    0 < |h| < 2^-125 and an odd last bit: there gelu(h) = h/2 + 0.3989 h^2
    + ..., h/2 is the midpoint of two bf16 values, and the h^2 term lies some
    2^-130 below binary64's resolution of h/2, so the binary64 value is h/2
    exactly and rounds to even (the exact value would round toward +inf).
    The oracle gives that, checked as the closed form bf16_rne(h/2)."""
    hb, want, dist = exact_gelu_table()
    got = orc.gelu(hb[None, :])[0]
    near = dist < NEAR_TIE
    mag = hb & np.uint16(0x7FFF)
    tiny_odd = (mag > 0) & (mag < 0x0100) & (hb & 1 == 1)       # 0 < |h| < 2^-125, odd last bit
    assert np.array_equal(near, tiny_odd), [hex(int(h)) for h in hb[near != tiny_odd][:10]]
    bad = np.flatnonzero((got != want) & ~near)
    assert bad.size == 0, [(hex(int(hb[i])), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]
    hv = (hb[near].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(got[near], nearest_bf16_bits(hv / 2))


def check_gelu_f64_vs_torch(orc) -> None:
    """The binary64 GELU against torch's float64 tanh GELU (its own tanh):
    relative difference below 2^-47 where torch's 0.5 h (1 + tanh(u)) is
    well conditioned (h >= -2); everywhere within |h| 2^-50 absolute, the
    error of 1 + tanh(u) in torch's form, which cancels for negative h.  Closed forms:
    gelu(0) = 0; bf16 gelu(h) = h for bf16 h >= 4 (1 + exp(-2u) < 1 + 2^-15);
    bf16 gelu(h) = -0 for h <= -11 (|gelu| below the least bf16 subnormal);
    bf16 gelu(h) = h / 2 for 2^-125 <= |h| <= 2^-20 (gelu(h) = h/2 + 0.4 h^2 + ...)."""
    h = np.concatenate([np.linspace(-20, 20, 400001), np.linspace(-1e-3, 1e-3, 20001),
                        np.geomspace(1e-30, 1e4, 20000), -np.geomspace(1e-30, 1e4, 20000)])
    mine = orc.gelu_f64(h)
    ref = torch.nn.functional.gelu(torch.from_numpy(h), approximate="tanh").numpy()
    good = h >= -2
    rel = np.abs(mine[good] - ref[good]) / np.maximum(np.abs(ref[good]), 1e-300)
    assert rel.max() < 2.0 ** -47, float(rel.max())
    assert (np.abs(mine - ref) <= np.abs(h) * 2.0 ** -50).all()
    assert orc.gelu_f64(np.array([0.0]))[0] == 0.0
    grid, gbits = _bf16_positive_grid()
    big = gbits[grid >= 4.0]
    assert np.array_equal(orc.gelu(big[None, :])[0], big)
    neg = gbits[grid >= 11.0] | np.uint16(0x8000)
    assert (orc.gelu(neg[None, :])[0] == 0x8000).all()
    small = (grid >= 2.0 ** -125) & (grid <= 2.0 ** -20)
    for sgn in (0, 0x8000):
        hb = (gbits[small] | np.uint16(sgn)).astype(np.uint16)
        half = nearest_bf16_bits(grid[small] / 2 * (-1.0 if sgn else 1.0))
        assert np.array_equal(orc.gelu(hb[None, :])[0], half)


def check_gelu_quantize(orc) -> None:
    """The fused producer step is the quantizer applied to the bf16 GELU
    output: the quantizer's own invariants hold on it (absmax of GELU(h) maps
    to +-127; rows of large negative h give GELU -0 and an all-zero row)."""
    rng = np.random.default_rng(32)
    h = to_bits((rng.standard_normal((16, 256)) * 4).astype(np.float32))
    h[3, :] = to_bits(np.full(256, -20.0, np.float32))
    q, s = orc.gelu_quantize_act(h)
    g = bits_to_float(orc.gelu(h))
    assert s[3] == 0.0 and (q[3] == 0).all()
    for r in range(16):
        if s[r] > 0:
            assert np.abs(q[r]).max() == 127
            k = np.abs(g[r]).argmax()
            assert abs(int(q[r, k])) == 127


ALL_CHECKS += [check_f64_to_bf16, check_gelu_exact, check_gelu_f64_vs_torch, check_gelu_quantize]
