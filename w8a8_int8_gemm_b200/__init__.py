"""B200-native W8A8 linear layer: Python binding of libw8a8.so.

The functions below have the names of the C entry points in
``include/w8a8.h`` and do argument marshalling only: they check that the
torch tensors have the layout the C ABI expects, allocate outputs the
caller did not pass (torch is used for device memory and streams), and call
the library on the current CUDA stream.  Every step of the computation runs
in the library's CUDA kernels; there is no fallback.  If the shared object
has not been built, importing this package raises ImportError.

Method: "Realizing Native INT8 Compute for Diffusion Transformers on
Consumer GPUs: A Fused INT8 GEMM Kernel for Ideogram 4.0" (arXiv
2606.14598), abstract -- per-token activation quantization, an int8 x int8
-> int32 GEMM against per-channel int8 weights, and the per-token x
per-channel dequantization plus bias folded into the GEMM epilogue, bf16 out.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "W8A8Error", "lib_path", "header_path", "exported_names",
    "w8a8_status_string", "w8a8_abi_version",
    "w8a8_quantize_act", "w8a8_quantize_weight", "w8a8_gemm", "w8a8_gemm_ex",
    "w8a8_gemm_i32", "w8a8_gemm_i32_ex", "w8a8_linear", "w8a8_linear_fused", "w8a8_linear_sync_words",
    "w8a8_linear_noalloc",
    "w8a8_quantize_act_fp8", "w8a8_quantize_weight_fp8", "w8a8_gemm_fp8", "w8a8_gemm_fp8_ex",
    "w8a8_gemm_fp8_f32", "w8a8_gemm_fp8_f32_ex", "w8a8_linear_fp8",
    "w8a8_quantize_act_gelu", "w8a8_gelu", "w8a8_linear_gelu", "ACT_NONE", "ACT_GELU",
    "LinearDesc", "Chain", "linear_layer", "w8a8_chain_create", "w8a8_chain_launch", "w8a8_chain_layers",
    "w8a8_chain_destroy",
    "w8a8_select_config",
    "w8a8_read_device_error", "w8a8_set_wait_timeout_ns", "w8a8_selftest_wait_timeout",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libw8a8.so")
header_path = os.path.join(os.path.dirname(_PKG), "include", "w8a8.h")

W8A8_OK = 0
W8A8_ERR_TIMEOUT = 5
ACT_NONE = 0   # W8A8_ACT_NONE
ACT_GELU = 1   # W8A8_ACT_GELU


class W8A8Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {w8a8_status_string(status)} (status {status})")


class GemmConfig(ctypes.Structure):
    _fields_ = [("block_m", ctypes.c_int32), ("block_n", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("raster_group", ctypes.c_int32), ("reserved", ctypes.c_int32 * 3)]

    def as_dict(self) -> dict:
        return {"block_m": self.block_m, "block_n": self.block_n, "stages": self.stages,
                "grid": self.grid, "raster_group": self.raster_group}


class LinearDesc(ctypes.Structure):
    """w8a8_linear_desc: one layer of a chain (device pointers and sizes)."""
    _fields_ = [("x", ctypes.c_void_p), ("wq", ctypes.c_void_p), ("scale_w", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("out", ctypes.c_void_p), ("ws_xq", ctypes.c_void_p),
                ("ws_scale_a", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("input_act", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(lib_path):
        raise ImportError(
            f"{lib_path} is missing: build the CUDA library first "
            "(python w8a8_int8_gemm_b200/build.py, or __graft_entry__.build())")
    lib = ctypes.CDLL(lib_path)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    sigs = {
        "w8a8_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "w8a8_abi_version": ([], ctypes.c_int),
        "w8a8_quantize_act": ([p, i64, i64, i64, p, i64, p, p], ctypes.c_int),
        "w8a8_quantize_weight": ([p, i64, i64, i64, p, i64, p, p], ctypes.c_int),
        "w8a8_gemm": ([p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_gemm_ex": ([p, p, p, p, p, p, i64, i64, i64, ctypes.POINTER(GemmConfig), p], ctypes.c_int),
        "w8a8_gemm_i32": ([p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_gemm_i32_ex": ([p, p, p, i64, i64, i64, ctypes.POINTER(GemmConfig), p], ctypes.c_int),
        "w8a8_linear": ([p, p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_linear_fused": ([p, p, p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_linear_sync_words": ([i64], i64),
        "w8a8_linear_noalloc": ([p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_quantize_act_fp8": ([p, i64, i64, i64, p, i64, p, p], ctypes.c_int),
        "w8a8_quantize_weight_fp8": ([p, i64, i64, i64, p, i64, p, p], ctypes.c_int),
        "w8a8_gemm_fp8": ([p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_gemm_fp8_ex": ([p, p, p, p, p, p, i64, i64, i64, ctypes.POINTER(GemmConfig), p], ctypes.c_int),
        "w8a8_gemm_fp8_f32": ([p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_gemm_fp8_f32_ex": ([p, p, p, i64, i64, i64, ctypes.POINTER(GemmConfig), p], ctypes.c_int),
        "w8a8_linear_fp8": ([p, p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_quantize_act_gelu": ([p, i64, i64, i64, p, i64, p, p], ctypes.c_int),
        "w8a8_gelu": ([p, i64, i64, i64, p, i64, p], ctypes.c_int),
        "w8a8_linear_gelu": ([p, p, p, p, p, p, p, i64, i64, i64, p], ctypes.c_int),
        "w8a8_chain_create": ([ctypes.POINTER(LinearDesc), i32, ctypes.POINTER(p)], ctypes.c_int),
        "w8a8_chain_launch": ([p, p], ctypes.c_int),
        "w8a8_chain_layers": ([p], i32),
        "w8a8_chain_destroy": ([p], ctypes.c_int),
        "w8a8_select_config": ([i64, i64, i64, ctypes.POINTER(GemmConfig)], ctypes.c_int),
        "w8a8_read_device_error": ([ctypes.POINTER(i32), i32], ctypes.c_int),
        "w8a8_set_wait_timeout_ns": ([i64], ctypes.c_int),
        "w8a8_selftest_wait_timeout": ([i64, p], ctypes.c_int),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def exported_names() -> list[str]:
    """Names of the functions include/w8a8.h declares."""
    with open(header_path) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"W8A8_API\s+[\w\s\*]+?\b(w8a8_\w+)\s*\(", text)))


# ------------------------------------------------------------ helpers


def _check(status: int, what: str) -> None:
    if status != W8A8_OK:
        raise W8A8Error(status, what)


def _stream(stream, device) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    if t.numel() > 0 and t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous in its last dimension")


def _need_contig(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple) -> None:
    _need(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cfg(config) -> GemmConfig | None:
    if config is None:
        return None
    if isinstance(config, GemmConfig):
        return config
    c = GemmConfig()
    for k in ("block_m", "block_n", "stages", "grid", "raster_group"):
        setattr(c, k, int(config[k]))
    return c


# --------------------------------------------------------- entry points


def w8a8_status_string(status: int) -> str:
    return _lib.w8a8_status_string(int(status)).decode()


def w8a8_abi_version() -> int:
    return int(_lib.w8a8_abi_version())


def w8a8_quantize_act(x: torch.Tensor, xq: torch.Tensor | None = None, scale_a: torch.Tensor | None = None,
                      stream=None):
    """Per-token int8 quantization of bf16 x [M, K] -> (xq int8 [M, K], scale_a fp32 [M])."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if scale_a is None:
        scale_a = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need(xq, "xq", torch.int8, 2)
    if tuple(xq.shape) != (M, K):
        raise ValueError("xq must have the shape of x")
    _need_contig(scale_a, "scale_a", torch.float32, (M,))
    _check(_lib.w8a8_quantize_act(_ptr(x), M, K, x.stride(0) if M else K, _ptr(xq),
                                  xq.stride(0) if M else K, _ptr(scale_a), _stream(stream, x.device)),
           "w8a8_quantize_act")
    return xq, scale_a


def w8a8_quantize_weight(w: torch.Tensor, wq: torch.Tensor | None = None, scale_w: torch.Tensor | None = None,
                         stream=None):
    """Per-output-channel int8 quantization of fp32 w [N, K] -> (wq int8 [N, K], scale_w fp32 [N])."""
    _need(w, "w", torch.float32, 2)
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    if scale_w is None:
        scale_w = torch.empty((N,), dtype=torch.float32, device=w.device)
    _need(wq, "wq", torch.int8, 2)
    if tuple(wq.shape) != (N, K):
        raise ValueError("wq must have the shape of w")
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    _check(_lib.w8a8_quantize_weight(_ptr(w), N, K, w.stride(0) if N else K, _ptr(wq),
                                     wq.stride(0) if N else K, _ptr(scale_w), _stream(stream, w.device)),
           "w8a8_quantize_weight")
    return wq, scale_w


def _gemm_operands(xq, wq):
    _need(xq, "xq", torch.int8, 2)
    _need(wq, "wq", torch.int8, 2)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: xq has K={K}, wq has K={K2}")
    _need_contig(xq, "xq", torch.int8, (M, K))
    _need_contig(wq, "wq", torch.int8, (N, K))
    return M, N, K


def w8a8_gemm_ex(xq, wq, scale_a, scale_w, bias=None, out=None, config=None, stream=None):
    """Fused GEMM with an explicit tile configuration (None = selected per shape)."""
    M, N, K = _gemm_operands(xq, wq)
    _need_contig(scale_a, "scale_a", torch.float32, (M,))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    c = _cfg(config)
    st = _lib.w8a8_gemm_ex(_ptr(xq), _ptr(wq), _ptr(scale_a), _ptr(scale_w), _ptr(bias), _ptr(out), M, N, K,
                           ctypes.byref(c) if c is not None else None, _stream(stream, xq.device))
    _check(st, "w8a8_gemm_ex")
    return out


def w8a8_gemm(xq, wq, scale_a, scale_w, bias=None, out=None, stream=None):
    """out bf16 [M, N] = bf16((fl32(xq @ wq^T) * scale_a[:, None]) * scale_w[None, :] + bias)."""
    M, N, K = _gemm_operands(xq, wq)
    _need_contig(scale_a, "scale_a", torch.float32, (M,))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _check(_lib.w8a8_gemm(_ptr(xq), _ptr(wq), _ptr(scale_a), _ptr(scale_w), _ptr(bias), _ptr(out), M, N, K,
                          _stream(stream, xq.device)), "w8a8_gemm")
    return out


def w8a8_gemm_i32(xq, wq, acc=None, stream=None, config=None):
    """Raw int32 accumulators acc [M, N] = xq @ wq^T (exact)."""
    M, N, K = _gemm_operands(xq, wq)
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    _need_contig(acc, "acc", torch.int32, (M, N))
    if config is None:
        st = _lib.w8a8_gemm_i32(_ptr(xq), _ptr(wq), _ptr(acc), M, N, K, _stream(stream, xq.device))
    else:
        c = _cfg(config)
        st = _lib.w8a8_gemm_i32_ex(_ptr(xq), _ptr(wq), _ptr(acc), M, N, K, ctypes.byref(c),
                                   _stream(stream, xq.device))
    _check(st, "w8a8_gemm_i32")
    return acc


def w8a8_gemm_i32_ex(xq, wq, acc=None, config=None, stream=None):
    return w8a8_gemm_i32(xq, wq, acc=acc, stream=stream, config=config)


def w8a8_linear(x, wq, scale_w, bias=None, out=None, ws_xq=None, ws_scale_a=None, stream=None):
    """The W8A8 linear layer: out bf16 [M, N] from bf16 x [M, K] and int8 wq [N, K].

    ws_xq int8 [M, K] and ws_scale_a fp32 [M] receive the quantized
    activations (allocated here if not given)."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _need(wq, "wq", torch.int8, 2)
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"inner dimensions differ: x has K={K}, wq has K={wq.shape[1]}")
    _need_contig(x, "x", torch.bfloat16, (M, K))
    _need_contig(wq, "wq", torch.int8, (N, K))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    dev = x.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if ws_xq is None:
        ws_xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    if ws_scale_a is None:
        ws_scale_a = torch.empty((M,), dtype=torch.float32, device=dev)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _need_contig(ws_xq, "ws_xq", torch.int8, (M, K))
    _need_contig(ws_scale_a, "ws_scale_a", torch.float32, (M,))
    _check(_lib.w8a8_linear(_ptr(x), _ptr(wq), _ptr(scale_w), _ptr(bias), _ptr(out), _ptr(ws_xq),
                            _ptr(ws_scale_a), M, N, K, _stream(stream, dev)), "w8a8_linear")
    return out


def w8a8_linear_sync_words(M: int) -> int:
    return int(_lib.w8a8_linear_sync_words(int(M)))


def w8a8_linear_fused(x, wq, scale_w, bias=None, out=None, ws_xq=None, ws_scale_a=None, ws_sync=None,
                      stream=None):
    """The W8A8 linear layer as one kernel (quantization inside the GEMM).

    ws_sync: int32 tensor of w8a8_linear_sync_words(M) words, zeroed once by
    the caller; each completed call leaves it zeroed (allocated and zeroed
    here if not given)."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _need(wq, "wq", torch.int8, 2)
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"inner dimensions differ: x has K={K}, wq has K={wq.shape[1]}")
    _need_contig(x, "x", torch.bfloat16, (M, K))
    _need_contig(wq, "wq", torch.int8, (N, K))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    dev = x.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if ws_xq is None:
        ws_xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    if ws_scale_a is None:
        ws_scale_a = torch.empty((M,), dtype=torch.float32, device=dev)
    if ws_sync is None:
        ws_sync = torch.zeros((w8a8_linear_sync_words(M),), dtype=torch.int32, device=dev)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _need_contig(ws_xq, "ws_xq", torch.int8, (M, K))
    _need_contig(ws_scale_a, "ws_scale_a", torch.float32, (M,))
    _need_contig(ws_sync, "ws_sync", torch.int32, (w8a8_linear_sync_words(M),))
    _check(_lib.w8a8_linear_fused(_ptr(x), _ptr(wq), _ptr(scale_w), _ptr(bias), _ptr(out), _ptr(ws_xq),
                                  _ptr(ws_scale_a), _ptr(ws_sync), M, N, K, _stream(stream, dev)),
           "w8a8_linear_fused")
    return out


def w8a8_linear_noalloc(x, wq, scale_w, bias=None, out=None, stream=None):
    """w8a8_linear without a workspace, for callers that cannot allocate
    device memory: the quantized activations live in one fixed 32 MiB array
    inside the library (see include/w8a8.h for the limit and for why
    overlapping calls race).  `out` must be given by such callers; if it is
    omitted, this wrapper allocates it with torch for convenience."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _need(wq, "wq", torch.int8, 2)
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"inner dimensions differ: x has K={K}, wq has K={wq.shape[1]}")
    _need_contig(x, "x", torch.bfloat16, (M, K))
    _need_contig(wq, "wq", torch.int8, (N, K))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _check(_lib.w8a8_linear_noalloc(_ptr(x), _ptr(wq), _ptr(scale_w), _ptr(bias), _ptr(out), M, N, K,
                                    _stream(stream, x.device)), "w8a8_linear_noalloc")
    return out


# ------------------------------------------------- FP8 (E4M3) variant
# E4M3 codes travel as torch.uint8 tensors (view them as
# torch.float8_e4m3fn to read their values).


def _quantize_fp8(fn, what, src, dtype, q, scale, stream):
    _need(src, "x" if dtype == torch.bfloat16 else "w", dtype, 2)
    R, K = src.shape
    if q is None:
        q = torch.empty((R, K), dtype=torch.uint8, device=src.device)
    if scale is None:
        scale = torch.empty((R,), dtype=torch.float32, device=src.device)
    _need(q, "codes", torch.uint8, 2)
    if tuple(q.shape) != (R, K):
        raise ValueError("the codes must have the shape of the input")
    _need_contig(scale, "scale", torch.float32, (R,))
    _check(fn(_ptr(src), R, K, src.stride(0) if R else K, _ptr(q), q.stride(0) if R else K, _ptr(scale),
              _stream(stream, src.device)), what)
    return q, scale


def w8a8_quantize_act_fp8(x, xq=None, scale_a=None, stream=None):
    """Per-token E4M3 quantization of bf16 x [M, K] -> (xq uint8 [M, K], scale_a fp32 [M])."""
    return _quantize_fp8(_lib.w8a8_quantize_act_fp8, "w8a8_quantize_act_fp8", x, torch.bfloat16, xq, scale_a,
                         stream)


def w8a8_quantize_weight_fp8(w, wq=None, scale_w=None, stream=None):
    """Per-output-channel E4M3 quantization of fp32 w [N, K] -> (wq uint8 [N, K], scale_w fp32 [N])."""
    return _quantize_fp8(_lib.w8a8_quantize_weight_fp8, "w8a8_quantize_weight_fp8", w, torch.float32, wq,
                         scale_w, stream)


def _fp8_operands(xq, wq):
    _need(xq, "xq", torch.uint8, 2)
    _need(wq, "wq", torch.uint8, 2)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: xq has K={K}, wq has K={K2}")
    _need_contig(xq, "xq", torch.uint8, (M, K))
    _need_contig(wq, "wq", torch.uint8, (N, K))
    return M, N, K


def w8a8_gemm_fp8_ex(xq, wq, scale_a, scale_w, bias=None, out=None, config=None, stream=None):
    """FP8 GEMM + dequant/bias epilogue, bf16 out [M, N]; config None = selected per shape."""
    M, N, K = _fp8_operands(xq, wq)
    _need_contig(scale_a, "scale_a", torch.float32, (M,))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    c = _cfg(config)
    st = _lib.w8a8_gemm_fp8_ex(_ptr(xq), _ptr(wq), _ptr(scale_a), _ptr(scale_w), _ptr(bias), _ptr(out), M, N, K,
                               ctypes.byref(c) if c is not None else None, _stream(stream, xq.device))
    _check(st, "w8a8_gemm_fp8_ex")
    return out


def w8a8_gemm_fp8(xq, wq, scale_a, scale_w, bias=None, out=None, stream=None):
    """out bf16 [M, N] = bf16((acc * scale_a[:, None]) * scale_w[None, :] + bias), acc the fp32 E4M3 product."""
    return w8a8_gemm_fp8_ex(xq, wq, scale_a, scale_w, bias=bias, out=out, config=None, stream=stream)


def w8a8_gemm_fp8_f32(xq, wq, acc=None, stream=None, config=None):
    """Raw fp32 accumulators acc [M, N] of the E4M3 product xq @ wq^T."""
    M, N, K = _fp8_operands(xq, wq)
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.float32, device=xq.device)
    _need_contig(acc, "acc", torch.float32, (M, N))
    c = _cfg(config)
    st = _lib.w8a8_gemm_fp8_f32_ex(_ptr(xq), _ptr(wq), _ptr(acc), M, N, K,
                                   ctypes.byref(c) if c is not None else None, _stream(stream, xq.device))
    _check(st, "w8a8_gemm_fp8_f32")
    return acc


def w8a8_gemm_fp8_f32_ex(xq, wq, acc=None, config=None, stream=None):
    return w8a8_gemm_fp8_f32(xq, wq, acc=acc, stream=stream, config=config)


def w8a8_linear_fp8(x, wq, scale_w, bias=None, out=None, ws_xq=None, ws_scale_a=None, stream=None):
    """The FP8 linear layer: out bf16 [M, N] from bf16 x [M, K] and E4M3 wq uint8 [N, K]."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _need(wq, "wq", torch.uint8, 2)
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"inner dimensions differ: x has K={K}, wq has K={wq.shape[1]}")
    _need_contig(x, "x", torch.bfloat16, (M, K))
    _need_contig(wq, "wq", torch.uint8, (N, K))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    dev = x.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if ws_xq is None:
        ws_xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    if ws_scale_a is None:
        ws_scale_a = torch.empty((M,), dtype=torch.float32, device=dev)
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _need_contig(ws_xq, "ws_xq", torch.uint8, (M, K))
    _need_contig(ws_scale_a, "ws_scale_a", torch.float32, (M,))
    _check(_lib.w8a8_linear_fp8(_ptr(x), _ptr(wq), _ptr(scale_w), _ptr(bias), _ptr(out), _ptr(ws_xq),
                                _ptr(ws_scale_a), M, N, K, _stream(stream, dev)), "w8a8_linear_fp8")
    return out


# ------------------------------------------------- GELU before a linear layer


def w8a8_quantize_act_gelu(h, xq=None, scale_a=None, stream=None):
    """Per-token int8 quantization of bf16_rne(GELU(h)) in one pass -> (xq int8 [M, K], scale_a fp32 [M])."""
    _need(h, "h", torch.bfloat16, 2)
    M, K = h.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=h.device)
    if scale_a is None:
        scale_a = torch.empty((M,), dtype=torch.float32, device=h.device)
    _need(xq, "xq", torch.int8, 2)
    if tuple(xq.shape) != (M, K):
        raise ValueError("xq must have the shape of h")
    _need_contig(scale_a, "scale_a", torch.float32, (M,))
    _check(_lib.w8a8_quantize_act_gelu(_ptr(h), M, K, h.stride(0) if M else K, _ptr(xq), xq.stride(0) if M else K,
                                       _ptr(scale_a), _stream(stream, h.device)), "w8a8_quantize_act_gelu")
    return xq, scale_a


def w8a8_gelu(h, g=None, stream=None):
    """g bf16 [M, K] = bf16_rne(GELU(h)) (the unfused producer)."""
    _need(h, "h", torch.bfloat16, 2)
    M, K = h.shape
    if g is None:
        g = torch.empty((M, K), dtype=torch.bfloat16, device=h.device)
    _need(g, "g", torch.bfloat16, 2)
    if tuple(g.shape) != (M, K):
        raise ValueError("g must have the shape of h")
    _check(_lib.w8a8_gelu(_ptr(h), M, K, h.stride(0) if M else K, _ptr(g), g.stride(0) if M else K,
                          _stream(stream, h.device)), "w8a8_gelu")
    return g


def w8a8_linear_gelu(h, wq, scale_w, bias=None, out=None, ws_xq=None, ws_scale_a=None, stream=None):
    """out bf16 [M, N] = GELU(h) W^T + b: w8a8_quantize_act_gelu then w8a8_gemm."""
    l = linear_layer(h, wq, scale_w, bias, out, ws_xq, ws_scale_a, ACT_GELU)
    _check(_lib.w8a8_linear_gelu(_ptr(l["x"]), _ptr(wq), _ptr(scale_w), _ptr(bias), _ptr(l["out"]),
                                 _ptr(l["ws_xq"]), _ptr(l["ws_scale_a"]), l["M"], l["N"], l["K"],
                                 _stream(stream, h.device)), "w8a8_linear_gelu")
    return l["out"]


# ------------------------------------------------- chains of linear layers


def linear_layer(x, wq, scale_w, bias=None, out=None, ws_xq=None, ws_scale_a=None, input_act: int = ACT_NONE) -> dict:
    """One layer of a chain: the tensors of a w8a8_linear call, with the
    output and workspace allocated here when not given.  x may be an
    earlier layer's ``out``; input_act=ACT_GELU makes the layer compute
    GELU(x) W^T + b (w8a8_linear_gelu)."""
    _need(x, "x", torch.bfloat16, 2)
    M, K = x.shape
    _need(wq, "wq", torch.int8, 2)
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError(f"inner dimensions differ: x has K={K}, wq has K={wq.shape[1]}")
    _need_contig(x, "x", torch.bfloat16, (M, K))
    _need_contig(wq, "wq", torch.int8, (N, K))
    _need_contig(scale_w, "scale_w", torch.float32, (N,))
    if bias is not None:
        _need_contig(bias, "bias", torch.bfloat16, (N,))
    dev = x.device
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if out is None else out
    ws_xq = torch.empty((M, K), dtype=torch.int8, device=dev) if ws_xq is None else ws_xq
    ws_scale_a = torch.empty((M,), dtype=torch.float32, device=dev) if ws_scale_a is None else ws_scale_a
    _need_contig(out, "out", torch.bfloat16, (M, N))
    _need_contig(ws_xq, "ws_xq", torch.int8, (M, K))
    _need_contig(ws_scale_a, "ws_scale_a", torch.float32, (M,))
    return {"x": x, "wq": wq, "scale_w": scale_w, "bias": bias, "out": out, "ws_xq": ws_xq,
            "ws_scale_a": ws_scale_a, "M": M, "N": N, "K": K, "input_act": int(input_act)}


class Chain:
    """A recorded chain of linear layers (w8a8_chain_t).  Keeps the layers'
    tensors alive as long as the chain exists; close() frees the graph."""

    def __init__(self, handle: int, layers: list):
        self._handle = ctypes.c_void_p(handle)
        self.layers = layers

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._handle:
            raise ValueError("the chain has been closed")
        return self._handle

    def launch(self, stream=None) -> None:
        w8a8_chain_launch(self, stream)

    def close(self) -> None:
        if self._handle:
            st = _lib.w8a8_chain_destroy(self._handle)
            self._handle = ctypes.c_void_p(None)
            _check(st, "w8a8_chain_destroy")

    def __del__(self):
        try:
            if self._handle:
                _lib.w8a8_chain_destroy(self._handle)
        except Exception:  # interpreter shutdown
            pass


def w8a8_chain_create(layers: list) -> Chain:
    """Record the layers (dicts from linear_layer) as one CUDA graph on the current device."""
    descs = (LinearDesc * max(1, len(layers)))()
    for i, l in enumerate(layers):
        descs[i] = LinearDesc(_ptr(l["x"]), _ptr(l["wq"]), _ptr(l["scale_w"]), _ptr(l.get("bias")), _ptr(l["out"]),
                              _ptr(l["ws_xq"]), _ptr(l["ws_scale_a"]), l["M"], l["N"], l["K"],
                              int(l.get("input_act", ACT_NONE)), 0)
    h = ctypes.c_void_p(None)
    _check(_lib.w8a8_chain_create(descs, len(layers), ctypes.byref(h)), "w8a8_chain_create")
    return Chain(h.value, list(layers))


def w8a8_chain_launch(chain: Chain, stream=None) -> None:
    dev = chain.layers[0]["x"].device if chain.layers else torch.device("cuda")
    _check(_lib.w8a8_chain_launch(chain.handle, _stream(stream, dev)), "w8a8_chain_launch")


def w8a8_chain_layers(chain: Chain) -> int:
    return int(_lib.w8a8_chain_layers(chain.handle))


def w8a8_chain_destroy(chain: Chain) -> None:
    chain.close()


def w8a8_select_config(M: int, N: int, K: int) -> dict:
    c = GemmConfig()
    _check(_lib.w8a8_select_config(M, N, K, ctypes.byref(c)), "w8a8_select_config")
    return c.as_dict()


def w8a8_read_device_error(clear: bool = True) -> int:
    """Synchronize the device and return (and clear) the kernels' timeout code (0 = none)."""
    code = ctypes.c_int32(0)
    st = _lib.w8a8_read_device_error(ctypes.byref(code), 1 if clear else 0)
    if st not in (W8A8_OK, W8A8_ERR_TIMEOUT):
        raise W8A8Error(st, "w8a8_read_device_error")
    return int(code.value)


def w8a8_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.w8a8_set_wait_timeout_ns(int(ns)), "w8a8_set_wait_timeout_ns")


def w8a8_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(_lib.w8a8_selftest_wait_timeout(int(timeout_ns), _stream(stream, torch.device("cuda"))),
           "w8a8_selftest_wait_timeout")


def raw_lib() -> ctypes.CDLL:
    """The loaded shared object (for tests that call the C ABI with raw pointers)."""
    return _lib
