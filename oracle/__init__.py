"""CPU oracle of the W8A8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never links,
loads or calls it, and it imports nothing from the product package.

The arithmetic lives in ``oracle.c`` (plain C, one IEEE binary32 operation
per step, exact int64 dot products); this module only compiles it with gcc
and marshals numpy arrays through ctypes.  What each function computes, and
the readings of the paper it follows ("Realizing Native INT8 Compute for
Diffusion Transformers on Consumer GPUs", abstract: per-token activation
quantization, per-channel weight quantization, int8 x int8 -> int32 GEMM,
per-token x per-channel dequantization and bias folded into the epilogue,
bf16 output), is stated in the C file's header.

Every function is pinned by the CPU tests to something other than itself
(numpy's float32 division and rint, numpy's int64 matmul, torch's bf16
conversion, hand-worked examples, closed forms and invariants; GELU to the
correctly rounded bf16 value of the exact function in 60-digit decimal
arithmetic on every bf16 input).  No function is "parity unpinned".
"""
from __future__ import annotations

import concurrent.futures
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")

# -ffp-contract=off: no fused multiply-add, every op rounds on its own.
# No -ffast-math: IEEE division, subnormals, signed zeros.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile an oracle C source (by default oracle.c) into a shared object (gcc)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def default_threads() -> int:
    return os.cpu_count() or 1


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, libpath: str):
        lib = ctypes.CDLL(libpath)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_bf16_rne.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_quantize_rows_bf16.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.oracle_quantize_rows_f32.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.oracle_gemm_i64.argtypes = [p, p, i64, i64, i64, p, ctypes.c_int]
        lib.oracle_epilogue.argtypes = [p, p, p, p, i64, i64, p]
        lib.oracle_epilogue_f64.argtypes = [p, p, p, p, i64, i64, p]
        lib.oracle_linear.argtypes = [p, p, p, p, i64, i64, i64, p, p, p, p, ctypes.c_int]
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_f32_to_e4m3_rne.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_e4m3_rne.restype = ctypes.c_uint8
        lib.oracle_quantize_rows_bf16_fp8.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.oracle_quantize_rows_f32_fp8.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.oracle_gemm_fp8_f64.argtypes = [p, p, i64, i64, i64, p]
        lib.oracle_epilogue_fp8.argtypes = [p, p, p, p, i64, i64, p]
        lib.oracle_gelu_f64.argtypes = [ctypes.c_double]
        lib.oracle_gelu_f64.restype = ctypes.c_double
        lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_gelu_f64_array.argtypes = [p, i64, p]
        lib.oracle_gelu_f64_array.restype = None
        lib.oracle_f64_to_bf16_array.argtypes = [p, i64, p]
        lib.oracle_f64_to_bf16_array.restype = None
        lib.oracle_gelu_rows.argtypes = [p, i64, i64, i64, p, i64]
        for fn in ("oracle_quantize_rows_bf16", "oracle_quantize_rows_f32", "oracle_gemm_i64",
                   "oracle_epilogue", "oracle_epilogue_f64", "oracle_linear", "oracle_quantize_rows_bf16_fp8",
                   "oracle_quantize_rows_f32_fp8", "oracle_gemm_fp8_f64", "oracle_epilogue_fp8",
                   "oracle_gelu_rows"):
            getattr(lib, fn).restype = ctypes.c_int
        self.lib = lib
        self.path = libpath

    @staticmethod
    def _check(rc: int, what: str) -> None:
        if rc != 0:
            raise RuntimeError(f"oracle {what} failed with code {rc}")

    # ------------------------------------------------------------ bf16

    def bf16_bits_to_f32(self, bits) -> np.ndarray:
        """bf16 bit patterns (uint16) -> float32, exact (element by element in C)."""
        b = _c(bits, np.uint16)
        out = np.empty(b.shape, np.float32)
        fi, fo = b.reshape(-1), out.reshape(-1)
        f = self.lib.oracle_bf16_to_f32
        for i in range(fi.size):
            fo[i] = f(int(fi[i]))
        return out

    def f32_to_bf16_bits(self, x) -> np.ndarray:
        """float32 -> bf16 bit patterns, round to nearest even (element by element in C)."""
        a = _c(x, np.float32)
        out = np.empty(a.shape, np.uint16)
        fi, fo = a.reshape(-1), out.reshape(-1)
        f = self.lib.oracle_f32_to_bf16_rne
        for i in range(fi.size):
            fo[i] = f(float(fi[i]))
        return out

    # ------------------------------------------------------ quantizers

    def quantize_act(self, x_bits) -> tuple[np.ndarray, np.ndarray]:
        """Per-token quantization of bf16 X [M, K] (uint16 bit patterns).

        Returns (xq int8 [M, K], scale_a float32 [M])."""
        x = _c(x_bits, np.uint16)
        M, K = x.shape
        q = np.empty((M, K), np.int8)
        s = np.empty((M,), np.float32)
        self._check(self.lib.oracle_quantize_rows_bf16(_ptr(x), M, K, K, _ptr(q), K, _ptr(s)),
                    "quantize_act")
        return q, s

    def quantize_weight(self, w) -> tuple[np.ndarray, np.ndarray]:
        """Per-output-channel quantization of fp32 W [N, K].

        Returns (wq int8 [N, K], scale_w float32 [N])."""
        a = _c(w, np.float32)
        N, K = a.shape
        q = np.empty((N, K), np.int8)
        s = np.empty((N,), np.float32)
        self._check(self.lib.oracle_quantize_rows_f32(_ptr(a), N, K, K, _ptr(q), K, _ptr(s)),
                    "quantize_weight")
        return q, s

    # ------------------------------------------------ GEMM / epilogue

    def gemm_i64(self, xq, wq, nthreads: int | None = None) -> np.ndarray:
        """Exact acc[m, n] = sum_k xq[m, k] * wq[n, k] as int64 [M, N]."""
        a = _c(xq, np.int8)
        b = _c(wq, np.int8)
        M, K = a.shape
        N, K2 = b.shape
        assert K == K2, "inner dimensions differ"
        acc = np.empty((M, N), np.int64)
        self._check(self.lib.oracle_gemm_i64(_ptr(a), _ptr(b), M, N, K, _ptr(acc),
                                             nthreads or default_threads()), "gemm_i64")
        return acc

    def epilogue(self, acc, scale_a, scale_w, bias_bits=None) -> np.ndarray:
        """bf16 (uint16 bits) [M, N] = bf16_rne((fl32(acc)*s_a[m])*s_w[n] + bias[n])."""
        c = _c(acc, np.int64)
        M, N = c.shape
        sa = _c(scale_a, np.float32)
        sw = _c(scale_w, np.float32)
        bias = None if bias_bits is None else _c(bias_bits, np.uint16)
        out = np.empty((M, N), np.uint16)
        self._check(self.lib.oracle_epilogue(_ptr(c), _ptr(sa), _ptr(sw), _ptr(bias), M, N, _ptr(out)),
                    "epilogue")
        return out

    def epilogue_f64(self, acc, scale_a, scale_w, bias_bits=None) -> np.ndarray:
        """The epilogue in binary64, unrounded: bounds the binary32 oracle's error."""
        c = _c(acc, np.int64)
        M, N = c.shape
        sa = _c(scale_a, np.float32)
        sw = _c(scale_w, np.float32)
        bias = None if bias_bits is None else _c(bias_bits, np.uint16)
        out = np.empty((M, N), np.float64)
        self._check(self.lib.oracle_epilogue_f64(_ptr(c), _ptr(sa), _ptr(sw), _ptr(bias), M, N,
                                                 _ptr(out)), "epilogue_f64")
        return out

    def linear(self, x_bits, wq, scale_w, bias_bits=None, nthreads: int | None = None):
        """The whole layer.

        Returns (out bf16 bits [M,N], xq int8 [M,K], scale_a [M], acc int64 [M,N])."""
        x = _c(x_bits, np.uint16)
        M, K = x.shape
        w = _c(wq, np.int8)
        N = w.shape[0]
        assert w.shape[1] == K
        sw = _c(scale_w, np.float32)
        bias = None if bias_bits is None else _c(bias_bits, np.uint16)
        out = np.empty((M, N), np.uint16)
        xq = np.empty((M, K), np.int8)
        sa = np.empty((M,), np.float32)
        acc = np.empty((M, N), np.int64)
        self._check(self.lib.oracle_linear(_ptr(x), _ptr(w), _ptr(sw), _ptr(bias), M, N, K, _ptr(out),
                                           _ptr(xq), _ptr(sa), _ptr(acc),
                                           nthreads or default_threads()), "linear")
        return out, xq, sa, acc


    # ------------------------------------------------------ fp8 e4m3

    def e4m3_to_f64(self, codes) -> np.ndarray:
        """E4M3 codes (uint8) -> their values (binary64), element by element in C."""
        c = _c(codes, np.uint8)
        out = np.empty(c.shape, np.float64)
        fi, fo = c.reshape(-1), out.reshape(-1)
        f = self.lib.oracle_e4m3_to_f64
        for i in range(fi.size):
            fo[i] = f(int(fi[i]))
        return out

    def f32_to_e4m3(self, x) -> np.ndarray:
        """float32 (|x| <= 448) -> nearest E4M3 code, ties to even (element by element in C)."""
        a = _c(x, np.float32)
        out = np.empty(a.shape, np.uint8)
        fi, fo = a.reshape(-1), out.reshape(-1)
        f = self.lib.oracle_f32_to_e4m3_rne
        for i in range(fi.size):
            fo[i] = f(float(fi[i]))
        return out

    def quantize_act_fp8(self, x_bits) -> tuple[np.ndarray, np.ndarray]:
        """Per-token FP8 quantization of bf16 X [M, K]: (codes uint8 [M, K], scale_a [M])."""
        x = _c(x_bits, np.uint16)
        M, K = x.shape
        q = np.empty((M, K), np.uint8)
        s = np.empty((M,), np.float32)
        self._check(self.lib.oracle_quantize_rows_bf16_fp8(_ptr(x), M, K, K, _ptr(q), K, _ptr(s)),
                    "quantize_act_fp8")
        return q, s

    def quantize_weight_fp8(self, w) -> tuple[np.ndarray, np.ndarray]:
        """Per-channel FP8 quantization of fp32 W [N, K]: (codes uint8 [N, K], scale_w [N])."""
        a = _c(w, np.float32)
        N, K = a.shape
        q = np.empty((N, K), np.uint8)
        s = np.empty((N,), np.float32)
        self._check(self.lib.oracle_quantize_rows_f32_fp8(_ptr(a), N, K, K, _ptr(q), K, _ptr(s)),
                    "quantize_weight_fp8")
        return q, s

    def gemm_fp8(self, aq, bq, nthreads: int | None = None) -> np.ndarray:
        """acc [M, N] = sum_k e4m3(aq[m,k]) * e4m3(bq[n,k]) in binary64.

        Row blocks run on host threads (each element is the same
        single-threaded sum whatever the split)."""
        a = _c(aq, np.uint8)
        b = _c(bq, np.uint8)
        M, K = a.shape
        N, K2 = b.shape
        assert K == K2
        acc = np.empty((M, N), np.float64)
        nt = max(1, min(nthreads or default_threads(), M))
        bounds = [M * t // nt for t in range(nt + 1)]

        def run(t):
            r0, r1 = bounds[t], bounds[t + 1]
            if r1 > r0:
                self._check(self.lib.oracle_gemm_fp8_f64(_ptr(a[r0:r1]), _ptr(b), r1 - r0, N, K,
                                                         _ptr(acc[r0:r1])), "gemm_fp8")

        if nt == 1:
            run(0)
        else:
            with concurrent.futures.ThreadPoolExecutor(nt) as ex:
                list(ex.map(run, range(nt)))
        return acc

    def epilogue_fp8(self, acc, scale_a, scale_w, bias_bits=None) -> np.ndarray:
        """bf16 bits [M, N] = bf16_rne((fl32(acc) * s_a[m]) * s_w[n] + bias[n])."""
        c = _c(acc, np.float64)
        M, N = c.shape
        sa = _c(scale_a, np.float32)
        sw = _c(scale_w, np.float32)
        bias = None if bias_bits is None else _c(bias_bits, np.uint16)
        out = np.empty((M, N), np.uint16)
        self._check(self.lib.oracle_epilogue_fp8(_ptr(c), _ptr(sa), _ptr(sw), _ptr(bias), M, N, _ptr(out)),
                    "epilogue_fp8")
        return out


    # --------------------------------------- GELU (producer of X), fused quantizer

    def gelu_f64(self, x) -> np.ndarray:
        """GELU (tanh form) in binary64, element-wise, before any bf16 rounding."""
        a = _c(x, np.float64)
        y = np.empty_like(a)
        self.lib.oracle_gelu_f64_array(_ptr(a), a.size, _ptr(y))
        return y

    def f64_to_bf16_bits(self, x) -> np.ndarray:
        """float64 -> bf16 bit patterns, rounded once to nearest even."""
        a = _c(x, np.float64)
        y = np.empty(a.shape, np.uint16)
        self.lib.oracle_f64_to_bf16_array(_ptr(a), a.size, _ptr(y))
        return y

    def gelu(self, h_bits) -> np.ndarray:
        """bf16 bits [M, K] -> bf16 bits of bf16_rne(GELU(h))."""
        h = _c(h_bits, np.uint16)
        M, K = h.shape
        g = np.empty((M, K), np.uint16)
        self._check(self.lib.oracle_gelu_rows(_ptr(h), M, K, K, _ptr(g), K), "gelu_rows")
        return g

    def gelu_quantize_act(self, h_bits):
        """The per-token quantizer applied to bf16_rne(GELU(h)): (codes, scales)."""
        return self.quantize_act(self.gelu(h_bits))


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle compiled from oracle.c (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def bf16_bits_to_f32(bits):
    return get().bf16_bits_to_f32(bits)


def f32_to_bf16_bits(x):
    return get().f32_to_bf16_bits(x)


def quantize_act(x_bits):
    return get().quantize_act(x_bits)


def quantize_weight(w):
    return get().quantize_weight(w)


def gemm_i64(xq, wq, nthreads: int | None = None):
    return get().gemm_i64(xq, wq, nthreads)


def epilogue(acc, scale_a, scale_w, bias_bits=None):
    return get().epilogue(acc, scale_a, scale_w, bias_bits)


def epilogue_f64(acc, scale_a, scale_w, bias_bits=None):
    return get().epilogue_f64(acc, scale_a, scale_w, bias_bits)


def linear(x_bits, wq, scale_w, bias_bits=None, nthreads: int | None = None):
    return get().linear(x_bits, wq, scale_w, bias_bits, nthreads)


def e4m3_to_f64(codes):
    return get().e4m3_to_f64(codes)


def f32_to_e4m3(x):
    return get().f32_to_e4m3(x)


def quantize_act_fp8(x_bits):
    return get().quantize_act_fp8(x_bits)


def quantize_weight_fp8(w):
    return get().quantize_weight_fp8(w)


def gemm_fp8(aq, bq):
    return get().gemm_fp8(aq, bq)


def epilogue_fp8(acc, scale_a, scale_w, bias_bits=None):
    return get().epilogue_fp8(acc, scale_a, scale_w, bias_bits)


def gelu_f64(x):
    return get().gelu_f64(x)


def f64_to_bf16_bits(x):
    return get().f64_to_bf16_bits(x)


def gelu(h_bits):
    return get().gelu(h_bits)


def gelu_quantize_act(h_bits):
    return get().gelu_quantize_act(h_bits)
