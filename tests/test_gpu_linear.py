"""GPU parity of the whole W8A8 linear layer (w8a8_linear, and the
one-kernel w8a8_linear_fused) against the CPU oracle, on every DiT workload
at full size in the launch configuration the benchmark uses (the selected
tile configuration, all tokens in one call), on EVERY row:

* the weight is quantized on both sides from the same seeded fp32 weight
  (codes and scales must agree bit for bit first);
* per-token codes and scales are bit-exact;
* the int32 accumulators of w8a8_gemm_i32 on those codes are bit-exact to
  the oracle's exact integer GEMM;
* the bf16 output of both entry points is within 1 ulp of the oracle and
  has no NaN;
* cosine similarity (the paper's accuracy metric): against the fp64 product
  of the dequantized operands it is 1 up to bf16 output rounding; against
  the unquantized fp64 product it must stay high.

The oracle runs once per workload (its exact GEMM threaded over the host's
cores, in row chunks), and both entry points are compared with it.

Paper: "Realizing Native INT8 Compute for Diffusion Transformers on Consumer
GPUs" (arXiv 2606.14598), abstract: the int32 accumulation is "bit-exact",
the outputs match "at cosine similarity 1.0 with no NaNs"."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.util import bf16_bits_to_torch, bf16_ulp_diff, is_nan_bits, row_chunks, torch_bf16_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


ENTRY_POINTS = ["w8a8_linear", "w8a8_linear_fused"]


def _call(w8, entry, x, wq, sw, bias, xq, sa):
    if entry == "w8a8_linear":
        return w8.w8a8_linear(x, wq, sw, bias, ws_xq=xq, ws_scale_a=sa)
    sync = torch.zeros((w8.w8a8_linear_sync_words(x.shape[0]),), dtype=torch.int32, device=x.device)
    out = w8.w8a8_linear_fused(x, wq, sw, bias, ws_xq=xq, ws_scale_a=sa, ws_sync=sync)
    torch.cuda.synchronize()
    assert int(sync.abs().sum()) == 0, "the fused call must leave its counters zeroed"
    return out


def _cosines(got_rows, xq_o, sa_o, wq_o, sw_o, x_rows, w, bias_bits):
    """The paper's accuracy metric (cosine similarity) on a few rows.  Against
    the product of the dequantized operands (xq*s_a)(wq*s_w)^T + bias in fp64
    only the bf16 output rounding separates the two: cosine >= 1 - 2^-15.
    Against the unquantized fp64 product the int8 quantization error enters
    too; for the outlier workload (per-token step ~ 20*max|N(0,1)|/127) it is
    about 1e-3, so that check only guards against gross errors."""
    y = torch.from_numpy(got_rows.view(np.int16)).view(torch.bfloat16).double().numpy()
    b64 = oracle.bf16_bits_to_f32(bias_bits).astype(np.float64)
    deq = (xq_o.astype(np.float64) * sa_o[:, None]) @ (wq_o.astype(np.float64) * sw_o[:, None]).T + b64
    ref = oracle.bf16_bits_to_f32(x_rows).astype(np.float64) @ w.astype(np.float64).T + b64

    def cos(a, b):
        return float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))

    assert cos(deq, y) >= 1 - 2.0 ** -15, cos(deq, y)
    assert cos(ref, y) >= 0.99, cos(ref, y)


def _run(w8, name, entries=ENTRY_POINTS):
    wl = workloads.WORKLOADS[name]
    d = workloads.make(wl)
    dev = torch.device("cuda")
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(d["w"]).to(dev))
    x = bf16_bits_to_torch(d["x"], dev)
    bias = bf16_bits_to_torch(d["bias"], dev)
    wq_o, sw_o = oracle.quantize_weight(d["w"])
    torch.cuda.synchronize()
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), sw_o.view(np.uint32)), "weight scales differ"
    assert np.array_equal(wq.cpu().numpy(), wq_o), "weight codes differ"

    outs = {}
    for entry in entries:
        xq = torch.empty((wl.M, wl.K), dtype=torch.int8, device=dev)
        sa = torch.empty((wl.M,), dtype=torch.float32, device=dev)
        out = _call(w8, entry, x, wq, sw, bias, xq, sa)
        torch.cuda.synchronize()
        assert w8.w8a8_read_device_error() == 0
        outs[entry] = (torch_bf16_to_bits(out), xq.cpu().numpy(), sa.cpu().numpy())
        del out
    acc = w8.w8a8_gemm_i32(torch.from_numpy(outs[entries[0]][1]).to(dev), wq)
    torch.cuda.synchronize()
    acc = acc.cpu().numpy()

    worst = 0
    for rows in row_chunks(wl.M):
        out_o, xq_o, sa_o, acc_o = oracle.linear(d["x"][rows], wq_o, sw_o, d["bias"])
        assert np.array_equal(acc[rows], acc_o), f"int32 accumulators differ in rows {rows}"
        for entry, (got, xq_g, sa_g) in outs.items():
            assert np.array_equal(sa_g[rows].view(np.uint32), sa_o.view(np.uint32)), f"{entry}: token scales"
            assert np.array_equal(xq_g[rows], xq_o), f"{entry}: token codes differ in rows {rows}"
            assert not is_nan_bits(got[rows]).any(), f"{entry}: NaN in the output"
            ulp = bf16_ulp_diff(got[rows], out_o)
            assert ulp.max() <= 1, f"{entry}: {ulp.max()} ulp at {np.argwhere(ulp > 1)[:3].tolist()} + {rows.start}"
            worst = max(worst, int(ulp.max()))
        if rows.start == 0:
            r8 = slice(0, min(8, wl.M))
            _cosines(outs[entries[0]][0][r8], xq_o[r8], sa_o[r8], wq_o, sw_o, d["x"][r8], d["w"], d["bias"])
    return worst


def test_linear_tiny_all_rows(w8):
    assert _run(w8, "tiny") <= 1


@pytest.mark.parametrize("name", ["qkv_768", "mlp_up_1024"])
def test_linear_dit_workloads_every_row(w8, name):
    _run(w8, name)


@pytest.mark.parametrize("name", ["sweep_qkv", "sweep_out", "sweep_up", "sweep_down"])
def test_linear_block_sweep_every_row(w8, name):
    _run(w8, name)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (130, 392, 1040), (333, 520, 3088), (4096, 12288, 3072)])
def test_fused_equals_two_kernel_path(w8, M, N, K):
    """The fused layer gives bit-identical outputs, codes and scales, call
    after call on the same counter workspace (which it leaves zeroed)."""
    rng = np.random.default_rng(M + N + K)
    dev = torch.device("cuda")
    x = (torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)) * 3).to(torch.bfloat16).to(dev)
    wq = torch.from_numpy(rng.integers(-127, 128, (N, K), dtype=np.int8)).to(dev)
    sw = torch.from_numpy(np.exp(rng.uniform(-9, -3, N)).astype(np.float32)).to(dev)
    bias = (torch.from_numpy(rng.standard_normal(N).astype(np.float32)) * 0.1).to(torch.bfloat16).to(dev)
    xq1 = torch.empty((M, K), dtype=torch.int8, device=dev)
    sa1 = torch.empty((M,), dtype=torch.float32, device=dev)
    ref = w8.w8a8_linear(x, wq, sw, bias, ws_xq=xq1, ws_scale_a=sa1)
    sync = torch.zeros((w8.w8a8_linear_sync_words(M),), dtype=torch.int32, device=dev)
    for _ in range(3):
        xq2 = torch.full((M, K), 7, dtype=torch.int8, device=dev)
        sa2 = torch.full((M,), -1.0, dtype=torch.float32, device=dev)
        out = w8.w8a8_linear_fused(x, wq, sw, bias, ws_xq=xq2, ws_scale_a=sa2, ws_sync=sync)
        torch.cuda.synchronize()
        assert w8.w8a8_read_device_error() == 0
        assert int(sync.abs().sum()) == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert torch.equal(xq2, xq1) and torch.equal(sa2.view(torch.int32), sa1.view(torch.int32))


@pytest.mark.parametrize("entry", ENTRY_POINTS)
def test_linear_ragged(w8, entry):
    """Token counts that are not multiples of the tile, N not a multiple of 256."""
    rng = np.random.default_rng(5)
    dev = torch.device("cuda")
    for M, N, K in [(1, 8, 16), (77, 136, 144), (130, 392, 1040)]:
        x_bits = workloads._to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        bias_bits = workloads.gen_bias(N, M)
        wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).to(dev))
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sa = torch.empty((M,), dtype=torch.float32, device=dev)
        out = _call(w8, entry, bf16_bits_to_torch(x_bits, dev), wq, sw, bf16_bits_to_torch(bias_bits, dev), xq, sa)
        torch.cuda.synchronize()
        wq_o, sw_o = oracle.quantize_weight(w)
        out_o, *_ = oracle.linear(x_bits, wq_o, sw_o, bias_bits)
        assert bf16_ulp_diff(torch_bf16_to_bits(out), out_o).max() <= 1, (M, N, K)


def test_linear_zero_tokens_give_bias(w8):
    dev = torch.device("cuda")
    M, N, K = 40, 264, 96
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    x[3, 5] = 2.0
    wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev)
    sw = torch.rand(N, device=dev) * 0.01
    bias = (torch.randn(N, device=dev) * 0.1).to(torch.bfloat16)
    out = w8.w8a8_linear(x, wq, sw, bias)
    torch.cuda.synchronize()
    rows = [r for r in range(M) if r != 3]
    assert torch.equal(out[rows], bias.expand(M - 1, N))
