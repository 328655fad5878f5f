"""Failure detection on the GPU without any fault.

* bad arguments are rejected on the host before any launch;
* every wait inside the kernels is bounded: the self-test kernel waits on a
  barrier nothing completes, the wait runs out after its (short) limit, the
  kernel records its site in the device error word and returns, and the
  CUDA context stays usable (a GEMM right after still matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def test_rejects_bad_shapes(w8):
    dev = torch.device("cuda")
    xq = torch.zeros((4, 24), dtype=torch.int8, device=dev)
    wq = torch.zeros((8, 24), dtype=torch.int8, device=dev)
    with pytest.raises(w8.W8A8Error) as e:
        w8.w8a8_gemm_i32(xq, wq)  # K % 16 != 0
    assert e.value.status == 1
    xq = torch.zeros((4, 32), dtype=torch.int8, device=dev)
    wq = torch.zeros((12, 32), dtype=torch.int8, device=dev)
    with pytest.raises(w8.W8A8Error) as e:
        w8.w8a8_gemm_i32(xq, wq)  # N % 8 != 0
    assert e.value.status == 1


def test_rejects_misaligned(w8):
    dev = torch.device("cuda")
    buf = torch.zeros(4 * 32 + 8, dtype=torch.int8, device=dev)
    xq = buf[8:].view(4, 32)  # 8-byte offset
    wq = torch.zeros((8, 32), dtype=torch.int8, device=dev)
    with pytest.raises(w8.W8A8Error) as e:
        w8.w8a8_gemm_i32(xq, wq)
    assert e.value.status == 2


def test_rejects_bad_config(w8):
    dev = torch.device("cuda")
    xq = torch.zeros((4, 32), dtype=torch.int8, device=dev)
    wq = torch.zeros((8, 32), dtype=torch.int8, device=dev)
    for cfg in [dict(block_m=64, block_n=256, stages=4, grid=1, raster_group=1),
                dict(block_m=128, block_n=192, stages=4, grid=1, raster_group=1),
                dict(block_m=128, block_n=256, stages=5, grid=1, raster_group=1),
                dict(block_m=128, block_n=128, stages=1, grid=1, raster_group=1),
                dict(block_m=128, block_n=128, stages=2, grid=0, raster_group=1),
                dict(block_m=256, block_n=256, stages=7, grid=2, raster_group=1),
                dict(block_m=256, block_n=256, stages=4, grid=1, raster_group=1)]:
        with pytest.raises(w8.W8A8Error):
            w8.w8a8_gemm_i32(xq, wq, config=cfg)


def test_bounded_wait_times_out_and_context_survives(w8):
    assert w8.w8a8_read_device_error() == 0
    w8.w8a8_selftest_wait_timeout(2_000_000)  # 2 ms
    code = w8.w8a8_read_device_error(clear=True)
    assert code == 6, f"expected the self-test site code, got {code}"
    assert w8.w8a8_read_device_error() == 0
    # the context is still usable
    rng = np.random.default_rng(0)
    a = rng.integers(-127, 128, (130, 96), dtype=np.int8)
    b = rng.integers(-127, 128, (40, 96), dtype=np.int8)
    acc = w8.w8a8_gemm_i32(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemm_i64(a, b))
