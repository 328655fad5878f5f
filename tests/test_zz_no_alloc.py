"""w8a8_linear_noalloc: the W8A8 linear layer for callers that cannot
allocate device memory (a runtime whose device memory is all pre-reserved,
a latency-critical path where cudaMalloc / cudaFree would synchronize the
device, a plugin interface that passes only inputs and outputs).

The entry point keeps the quantized activations in one fixed array inside
the library.  These tests call it through the C ABI and check that its
output equals w8a8_linear's (within the 1-ulp bf16 tolerance of the other
tests; in practice bit-identical, the kernels are the same) on two calls in
a row -- the second call finds the first call's leftovers in the shared
array --, at the size the header advertises (also against the CPU oracle)
and at the largest size that fits, and that a problem larger than the
array, by 4 bytes or by far, is refused without touching the output.  This
file is collected last on purpose."""
import numpy as np
import pytest
import torch

from tests.util import bf16_ulp_diff, is_nan_bits, torch_bf16_to_bits

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 7  # W8A8_ERR_SCRATCH_LIMIT


def _inputs(M, N, K, seed, dev):
    rng = np.random.default_rng(seed)
    x = (torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)) * 2).to(torch.bfloat16).to(dev)
    wq = torch.from_numpy(rng.integers(-127, 128, (N, K), dtype=np.int8)).to(dev)
    sw = torch.from_numpy(np.exp(rng.uniform(-9, -3, N)).astype(np.float32)).to(dev)
    bias = (torch.from_numpy(rng.standard_normal(N).astype(np.float32)) * 0.1).to(torch.bfloat16).to(dev)
    return x, wq, sw, bias


def _noalloc_raw(w8, x, wq, sw, bias, out):
    """Call the C entry point directly with device pointers."""
    M, K = x.shape
    N = wq.shape[0]
    stream = torch.cuda.current_stream(x.device).cuda_stream
    return w8.raw_lib().w8a8_linear_noalloc(x.data_ptr(), wq.data_ptr(), sw.data_ptr(), bias.data_ptr(),
                                            out.data_ptr(), M, N, K, stream)


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    import w8a8_int8_gemm_b200 as w8
    assert torch.cuda.is_available()
    dev = torch.device("cuda")
    # two different problems back to back; the second is smaller than the first,
    # so stale codes of the first call remain in the shared array around it
    for (M, N, K, seed) in [(4096, 3072, 3072, 1), (777, 1032, 2064, 2)]:
        x, wq, sw, bias = _inputs(M, N, K, seed, dev)
        ref = w8.w8a8_linear(x, wq, sw, bias)
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        assert _noalloc_raw(w8, x, wq, sw, bias, out) == 0
        torch.cuda.synchronize()
        assert w8.w8a8_read_device_error() == 0
        got = torch_bf16_to_bits(out)
        assert not is_nan_bits(got).any()
        assert bf16_ulp_diff(got, torch_bf16_to_bits(ref)).max() <= 1


def test_noalloc_at_the_advertised_size_matches_the_oracle():
    """9216 tokens x K = 3072 (the size the header gives as fitting) against
    w8a8_linear and against the CPU oracle on every row."""
    import oracle
    import w8a8_int8_gemm_b200 as w8
    from tests.util import bf16_bits_to_torch
    import workloads
    dev = torch.device("cuda")
    M, N, K = 9216, 1032, 3072
    x_bits = workloads.gen_activations(M, K, seed=91)
    w = workloads.gen_weight(N, K, 92)
    b_bits = workloads.gen_bias(N, 93)
    x = bf16_bits_to_torch(x_bits, dev)
    bias = bf16_bits_to_torch(b_bits, dev)
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).to(dev))
    ref = w8.w8a8_linear(x, wq, sw, bias)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    assert _noalloc_raw(w8, x, wq, sw, bias, out) == 0
    torch.cuda.synchronize()
    assert w8.w8a8_read_device_error() == 0
    got = torch_bf16_to_bits(out)
    assert np.array_equal(got, torch_bf16_to_bits(ref))
    wq_o, sw_o = oracle.quantize_weight(w)
    want, *_ = oracle.linear(x_bits, wq_o, sw_o, b_bits)
    assert bf16_ulp_diff(got, want).max() <= 1


# The scratch holds M*K codes rounded up to 256 bytes, then 4*M bytes of
# scales, in 32 MiB: at K = 864, 38656 tokens leave 1024 bytes free and
# 38657 need 4 bytes more than there are.
EDGE_K, EDGE_M_FITS = 864, 38656


def test_noalloc_at_the_edge_of_its_scratch():
    import w8a8_int8_gemm_b200 as w8
    dev = torch.device("cuda")
    M, N, K = EDGE_M_FITS, 136, EDGE_K
    assert (M * K + 255) // 256 * 256 + 4 * M == (32 << 20) - 1024
    x, wq, sw, bias = _inputs(M, N, K, 5, dev)
    ref = w8.w8a8_linear(x, wq, sw, bias)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    assert _noalloc_raw(w8, x, wq, sw, bias, out) == 0
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_refuses_problems_beyond_its_scratch():
    import w8a8_int8_gemm_b200 as w8
    dev = torch.device("cuda")
    M, N, K = 8192, 16, 8192  # 64 MiB of codes > 32 MiB of scratch
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    sw = torch.ones(N, device=dev)
    bias = torch.zeros(N, dtype=torch.bfloat16, device=dev)
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device=dev)
    assert _noalloc_raw(w8, x, wq, sw, bias, out) == SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((out == 3.0).all()), "a refused call must not write the output"
    assert "scratch" in w8.w8a8_status_string(SCRATCH_LIMIT)
    # 4 bytes beyond the scratch
    M, K = EDGE_M_FITS + 1, EDGE_K
    assert (M * K + 255) // 256 * 256 + 4 * M == (32 << 20) + 4
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device=dev)
    assert _noalloc_raw(w8, x, wq, sw, bias, out) == SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
