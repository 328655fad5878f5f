"""GPU parity of GELU before a linear layer (the producer of X fused with the
per-token quantizer) against the CPU oracle.

* w8a8_gelu: bit-exact bf16_rne(GELU(h)) on every bf16 bit pattern that is
  not a NaN (both infinities included: +inf -> +inf, -inf -> NaN on both
  sides, -inf / inf);
* w8a8_quantize_act_gelu: codes and scales bit-exact to the oracle's
  quantizer applied to the oracle's GELU, on the warp-per-row (K <= 4096),
  block-per-row (K <= 32768) and two-pass paths; and bit-identical to
  w8a8_gelu followed by w8a8_quantize_act on the GPU;
* w8a8_linear_gelu and a chain layer with input_act = GELU: outputs equal to
  the oracle's GELU -> linear layer.

GELU is the library's definition (the tanh form evaluated in binary64 and
rounded once to bf16; see include/w8a8.h): the pages name no activation
function.  The oracle it is compared with equals the correctly rounded bf16
value of the exact function on every bf16 input but 256 documented
near-ties (its CPU pins), so the exhaustive test below also shows that
CUDA's binary64 exp and the C library's never round to different bf16
values."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.util import bf16_bits_to_torch, torch_bf16_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w8():
    import w8a8_int8_gemm_b200 as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _is_nan(bits):
    return ((bits & 0x7F80) == 0x7F80) & ((bits & 0x7F) != 0)


def test_gelu_every_bf16_pattern(w8):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    pats = pats[~_is_nan(pats)]
    pats = np.concatenate([pats, np.zeros((-len(pats)) % 64, np.uint16)]).reshape(-1, 64)
    got = torch_bf16_to_bits(w8.w8a8_gelu(bf16_bits_to_torch(pats, "cuda")))
    torch.cuda.synchronize()
    want = oracle.gelu(pats)
    nan_g, nan_w = _is_nan(got), _is_nan(want)
    assert np.array_equal(nan_g, nan_w)
    bad = np.argwhere((got != want) & ~nan_w)
    assert bad.size == 0, [(hex(pats[tuple(b)]), hex(got[tuple(b)]), hex(want[tuple(b)])) for b in bad[:5]]


def _act(M, K, seed, scale=4.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    x[0, :] = -20.0                          # GELU -0 everywhere: a zero row
    if M > 2:
        x[1, : K // 2] = 0.0
        x[2, :] = np.linspace(-13, 11, K)      # both tails: GELU -0 below -11, h above 4
    return oracle.f32_to_bf16_bits(x)


# The table kernel at 2, 4, 6 and 8 vectors per thread (K up to 4096, 8192,
# 12288, 16384; ragged and full), with more rows than row groups in the grid
# (the persistent loop and its prefetch of the next row: 1500 x 3072,
# 700 x 12288), and the per-element kernels beyond 16384.
@pytest.mark.parametrize("M,K", [(37, 272), (130, 3072), (17, 4096), (11, 8192), (7, 6160), (9, 12288),
                                 (5, 16384), (3, 14352), (1500, 3072), (700, 12288), (3, 24592), (2, 40000)])
def test_quantize_act_gelu(w8, M, K):
    h = _act(M, K, M + K)
    ht = bf16_bits_to_torch(h, "cuda")
    q, s = w8.w8a8_quantize_act_gelu(ht)
    g = w8.w8a8_gelu(ht)
    q2, s2 = w8.w8a8_quantize_act(g)
    torch.cuda.synchronize()
    q_want, s_want = oracle.gelu_quantize_act(h)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_want.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_want)
    assert torch.equal(q, q2) and torch.equal(s, s2), "fused and unfused differ"


def test_linear_gelu(w8):
    M, N, K = 300, 520, 3072
    h = _act(M, K, 5)
    w = workloads.gen_weight(N, K, 6)
    b = workloads.gen_bias(N, 7)
    dev = torch.device("cuda")
    wq, sw = w8.w8a8_quantize_weight(torch.from_numpy(w).to(dev))
    out = w8.w8a8_linear_gelu(bf16_bits_to_torch(h, dev), wq, sw, bf16_bits_to_torch(b, dev))
    torch.cuda.synchronize()
    wq_o, sw_o = oracle.quantize_weight(w)
    out_o, _, _, _ = oracle.linear(oracle.gelu(h), wq_o, sw_o, b)
    assert np.array_equal(torch_bf16_to_bits(out), out_o)


def test_chain_layer_with_gelu_input(w8):
    M = 200
    x = _act(M, 512, 9, scale=1.0)
    w1, w2 = workloads.gen_weight(1024, 512, 10), workloads.gen_weight(256, 1024, 11)
    dev = torch.device("cuda")
    wq1, sw1 = w8.w8a8_quantize_weight(torch.from_numpy(w1).to(dev))
    wq2, sw2 = w8.w8a8_quantize_weight(torch.from_numpy(w2).to(dev))
    l1 = w8.linear_layer(bf16_bits_to_torch(x, dev), wq1, sw1)
    l2 = w8.linear_layer(l1["out"], wq2, sw2, input_act=w8.ACT_GELU)
    chain = w8.w8a8_chain_create([l1, l2])
    chain.launch()
    torch.cuda.synchronize()
    h_o, _, _, _ = oracle.linear(x, *oracle.quantize_weight(w1))
    y_o, xq_o, sa_o, _ = oracle.linear(oracle.gelu(h_o), *oracle.quantize_weight(w2))
    assert np.array_equal(torch_bf16_to_bits(l1["out"]), h_o)
    assert np.array_equal(l2["ws_xq"].cpu().numpy(), xq_o)
    assert np.array_equal(torch_bf16_to_bits(l2["out"]), y_o)
    chain.close()


_CAPTURE_FIRST = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import oracle
import w8a8_int8_gemm_b200 as w8
from tests.test_gpu_gelu import _act
from tests.util import bf16_bits_to_torch
h = _act(600, 12288, 21)
x = bf16_bits_to_torch(h, "cuda")
q = torch.empty((600, 12288), dtype=torch.int8, device="cuda")
s = torch.empty((600,), dtype=torch.float32, device="cuda")
g = torch.cuda.CUDAGraph()
stream = torch.cuda.Stream()
with torch.cuda.stream(stream):
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        w8.w8a8_quantize_act_gelu(x, q, s, stream=stream)
g.replay()
torch.cuda.synchronize()
q_want, s_want = oracle.gelu_quantize_act(h)
assert np.array_equal(s.cpu().numpy().view(np.uint32), s_want.view(np.uint32)), "scales differ"
assert np.array_equal(q.cpu().numpy(), q_want), "codes differ"
print("ok")
"""


def test_quantize_act_gelu_first_call_captured(w8, tmp_path):
    """A process whose first GELU quantizer call is recorded into a CUDA graph
    (the table kernel's launch geometry is then the one chosen without the
    occupancy query, clusters of two) gives the oracle's codes."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "capture_first.py"
    script.write_text(_CAPTURE_FIRST)
    out = subprocess.run([sys.executable, str(script), root], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0 and "ok" in out.stdout, out.stdout[-2000:] + out.stderr[-2000:]
