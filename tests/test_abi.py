"""The C ABI on the host (no GPU needed): the shared object loads, exports
every function include/w8a8.h declares and nothing else, and rejects bad
arguments before touching any device."""
import ctypes
import subprocess

import pytest

import __graft_entry__


@pytest.fixture(scope="module")
def w8():
    __graft_entry__.build()
    import w8a8_int8_gemm_b200 as mod
    return mod


def test_exports_match_header(w8):
    declared = set(w8.exported_names())
    assert {"w8a8_quantize_act", "w8a8_gemm", "w8a8_linear", "w8a8_gemm_i32"} <= declared
    lib = w8.raw_lib()
    for name in declared:
        assert hasattr(lib, name), f"{name} declared but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", w8.lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    ours = {n for n in exported if n.startswith("w8a8_")}
    assert ours == declared, f"exported {sorted(ours ^ declared)} differ from the header"


def test_status_strings(w8):
    assert w8.w8a8_status_string(0) == "ok"
    for s in range(1, 8):
        assert w8.w8a8_status_string(s) not in ("ok", "unknown status")
    assert w8.w8a8_status_string(99) == "unknown status"
    assert w8.w8a8_abi_version() == 101


def _gemm_i32(lib, xq, wq, acc, M, N, K):
    return lib.w8a8_gemm_i32(xq, wq, acc, M, N, K, None)


def test_host_validation_without_device(w8):
    lib = w8.raw_lib()
    A = 0x10000  # fake 16-byte-aligned addresses: never dereferenced on these paths
    # shapes
    assert _gemm_i32(lib, A, A, A, 4, 8, 24) == 1          # K % 16
    assert _gemm_i32(lib, A, A, A, 4, 8, 0) == 1           # K == 0
    assert _gemm_i32(lib, A, A, A, 4, 12, 32) == 1         # N % 8
    assert _gemm_i32(lib, A, A, A, -1, 8, 32) == 1         # negative M
    assert _gemm_i32(lib, A, A, A, 4, 8, 133152) == 1      # K * 127^2 >= 2^31
    # empty problems succeed without launching
    assert _gemm_i32(lib, A, A, A, 0, 8, 32) == 0
    assert _gemm_i32(lib, A, A, A, 4, 0, 32) == 0
    # null and misaligned pointers
    assert _gemm_i32(lib, None, A, A, 4, 8, 32) == 1
    assert _gemm_i32(lib, A + 8, A, A, 4, 8, 32) == 2
    assert _gemm_i32(lib, A, A, A + 4, 4, 8, 32) == 2
    assert lib.w8a8_gemm(A, A, A, A, A + 2, A, 4, 8, 32, None) == 2   # misaligned bias
    assert lib.w8a8_gemm(A, A, None, A, None, A, 4, 8, 32, None) == 1  # missing scale_a
    # quantizers
    assert lib.w8a8_quantize_act(A, 4, 32, 16, A, 32, A, None) == 1    # ldx < K
    assert lib.w8a8_quantize_act(A, 4, 32, 36, A, 32, A, None) == 2    # ldx * 2 not 16-byte
    assert lib.w8a8_quantize_act(A, 4, 32, 32, A, 40, A, None) == 2    # ldxq not 16-byte
    assert lib.w8a8_quantize_act(A, 0, 32, 32, A, 32, A, None) == 0
    assert lib.w8a8_quantize_weight(A, 4, 32, 34, A, 32, A, None) == 2  # ldw * 4 not 16-byte
    # linear validates the whole call first
    assert lib.w8a8_linear(A, A, A, None, A, A, A, 4, 12, 32, None) == 1
    assert lib.w8a8_linear(A, A, A, None, A, A + 1, A, 4, 8, 32, None) == 2
    assert lib.w8a8_linear(A, A, A, None, A, A, A, 0, 8, 32, None) == 0
    # the fused layer: same checks, plus its counter workspace
    assert lib.w8a8_linear_fused(A, A, A, None, A, A, A, None, 4, 8, 32, None) == 1   # no ws_sync
    assert lib.w8a8_linear_fused(A, A, A, None, A, A, A, A + 4, 4, 8, 32, None) == 2  # misaligned ws_sync
    assert lib.w8a8_linear_fused(A, A, A, None, A, A, A, A, 4, 12, 32, None) == 1     # N % 8
    assert lib.w8a8_linear_fused(A, A, A, None, A, A, A, A, 0, 8, 32, None) == 0      # empty
    assert lib.w8a8_linear_sync_words(0) == 1
    assert lib.w8a8_linear_sync_words(128) == 2
    assert lib.w8a8_linear_sync_words(129) == 3
    assert lib.w8a8_linear_sync_words(4096) == 33
    # the FP8 (E4M3) variant: the same checks
    assert lib.w8a8_quantize_act_fp8(A, 4, 32, 16, A, 32, A, None) == 1      # ldx < K
    assert lib.w8a8_quantize_act_fp8(A, 4, 32, 32, A, 40, A, None) == 2      # ldxq not 16-byte
    assert lib.w8a8_quantize_weight_fp8(A, 4, 24, 24, A, 32, A, None) == 1   # K % 16
    assert lib.w8a8_quantize_weight_fp8(A, 0, 32, 32, A, 32, A, None) == 0   # empty
    assert lib.w8a8_gemm_fp8(A, A, A, A, A + 2, A, 4, 8, 32, None) == 2      # misaligned bias
    assert lib.w8a8_gemm_fp8(A, A, None, A, None, A, 4, 8, 32, None) == 1    # missing scale_a
    assert lib.w8a8_gemm_fp8_f32(A, A, A, 4, 12, 32, None) == 1             # N % 8
    assert lib.w8a8_gemm_fp8_f32(A, A, A, 0, 8, 32, None) == 0              # empty
    assert lib.w8a8_linear_fp8(A, A, A, None, A, A, A, 4, 8, 133152, None) == 1   # K too large
    assert lib.w8a8_linear_fp8(A, A, A, None, A, A + 4, A, 4, 8, 32, None) == 2   # misaligned ws_xq
    assert lib.w8a8_linear_fp8(A, A, A, None, A, A, None, 4, 8, 32, None) == 1    # no ws_scale_a
    cfg = w8.GemmConfig(block_m=256, block_n=256, stages=7, grid=2, raster_group=1)
    assert lib.w8a8_gemm_fp8_f32_ex(A, A, A, 4, 8, 32, ctypes.byref(cfg), None) == 1  # too many stages
    # GELU before a linear layer
    assert lib.w8a8_quantize_act_gelu(A, 4, 32, 16, A, 32, A, None) == 1    # ldx < K
    assert lib.w8a8_quantize_act_gelu(A, 0, 32, 32, A, 32, A, None) == 0    # empty
    assert lib.w8a8_gelu(A, 4, 12, 12, A, 12, None) == 1                    # K % 8
    assert lib.w8a8_gelu(A, 4, 16, 20, A, 16, None) == 2                    # ldh % 8
    assert lib.w8a8_gelu(A + 2, 4, 16, 16, A, 16, None) == 2                # misaligned h
    assert lib.w8a8_gelu(A, 0, 16, 16, A, 16, None) == 0                    # empty
    assert lib.w8a8_linear_gelu(A, A, A, None, A, A, A, 4, 12, 32, None) == 1
    assert lib.w8a8_linear_gelu(A, A, A, None, A, A + 1, A, 4, 8, 32, None) == 2
    # the no-allocation layer: w8a8_linear's checks, in its order, before the
    # device check, which comes before the scratch capacity (so an invalid call
    # that is also too large is an argument error, not a capacity error)
    assert lib.w8a8_linear_noalloc(A, A, A, None, A, 4, 12, 32, None) == 1         # N % 8
    assert lib.w8a8_linear_noalloc(A, A, A, None, A, 9000, 8, 24, None) == 1       # K % 16
    assert lib.w8a8_linear_noalloc(None, A, A, None, A, 4, 8, 32, None) == 1       # no x
    assert lib.w8a8_linear_noalloc(A, A, A, None, None, 4, 8, 32, None) == 1       # no out
    assert lib.w8a8_linear_noalloc(A + 8, A, A, None, A, 4, 8, 32, None) == 2      # misaligned x
    assert lib.w8a8_linear_noalloc(A, A, A, A + 2, A, 4, 8, 32, None) == 2         # misaligned bias
    assert lib.w8a8_linear_noalloc(A, A, A, None, A, 0, 8, 32, None) == 0          # empty
    big = lib.w8a8_linear_noalloc(A, A, A, None, A, 1 << 16, 8, 4096, None)        # valid, 256 MiB of codes
    import torch
    assert big == 7 if torch.cuda.is_available() else big in (3, 6), big  # no device here: not a capacity error
    # chains of linear layers: every layer is validated before any CUDA call
    h = ctypes.c_void_p(None)
    assert lib.w8a8_chain_create(None, 1, ctypes.byref(h)) == 1
    d = (w8.LinearDesc * 2)()
    d[0] = w8.LinearDesc(A, A, A, None, A, A, A, 4, 8, 32)
    d[1] = w8.LinearDesc(A, A, A, None, A, A, A, 4, 12, 32)                  # N % 8
    assert lib.w8a8_chain_create(d, 2, ctypes.byref(h)) == 1 and not h.value
    d[1] = w8.LinearDesc(A, A, A, None, A, A + 4, A, 4, 8, 32)               # misaligned ws_xq
    assert lib.w8a8_chain_create(d, 2, ctypes.byref(h)) == 2 and not h.value
    assert lib.w8a8_chain_create(d, 0, ctypes.byref(h)) == 1
    d[1] = w8.LinearDesc(A, A, A, None, A, A, A, 4, 8, 32, 7, 0)             # unknown input_act
    assert lib.w8a8_chain_create(d, 2, ctypes.byref(h)) == 1
    assert lib.w8a8_chain_create(d, 1, None) == 1
    assert lib.w8a8_chain_launch(None, None) == 1
    assert lib.w8a8_chain_layers(None) == 0 and lib.w8a8_chain_destroy(None) == 0
    # explicit configurations
    cfg = w8.GemmConfig(block_m=128, block_n=200, stages=4, grid=1, raster_group=1)
    assert lib.w8a8_gemm_i32_ex(A, A, A, 4, 8, 32, ctypes.byref(cfg), None) == 1
    cfg = w8.GemmConfig(block_m=128, block_n=256, stages=5, grid=1, raster_group=1)
    assert lib.w8a8_gemm_i32_ex(A, A, A, 4, 8, 32, ctypes.byref(cfg), None) == 1
    assert lib.w8a8_select_config(4, 8, 32, None) == 1
    assert lib.w8a8_selftest_wait_timeout(10, None) == 1


def test_binding_without_the_library_fails_loudly(tmp_path):
    """The Python binding has no fallback: a copy of the package without
    libw8a8.so raises ImportError on import (naming the missing library)."""
    import os
    import shutil
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = tmp_path / "w8a8_int8_gemm_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(root, "w8a8_int8_gemm_b200", "__init__.py"), pkg / "__init__.py")
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n    import w8a8_int8_gemm_b200\nexcept ImportError as e:\n    print('ImportError:', e); sys.exit(3)\n"
            "sys.exit(0)\n")
    out = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 3, out.stdout + out.stderr
    assert "libw8a8.so is missing" in out.stdout
